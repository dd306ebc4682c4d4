// fa_fwd_short_sm100.cu -- attention forward for short key sets (Sk <= 128,
// D = 64 or 128) on sm_100a: text-to-image cross-attention over a few dozen
// text tokens, short self-attention heads.
//
// With every key of a head inside one tile, the online-softmax recurrence of
// the streaming kernel ("FlashAttention-2 在昇腾 NPU 上如何做到 3 倍加速？深度拆解
// ops-transformer 的实现", sections 2.1-2.2) has a single step: the row max is
// exact, no rescale of O is ever needed, and the work of a 128-row query tile is
// one S = Q K^T, one softmax and one P.V.  What bounds such a launch is moving
// Q in and O out (the keys and values of a head are a few KiB), so this kernel
// keeps many query tiles of a CTA in flight instead of streaming keys:
//
//  * work: the B*H*ceil(Sq/128) query tiles in (b, h, tile) order, split into
//    one contiguous range per CTA (one persistent CTA per SM); K and V of a
//    head are loaded once per range segment into one of two slots, so the next
//    head's keys load while the last tiles of the current head finish;
//  * warp 12 (TMA): Q tiles into a ring of stages, K/V on head changes;
//  * warp 13 (issued by lane 0): S_i = Q_i K^T into TMEM slot i mod NS (three
//    slots for D = 64, two for D = 128) once the P.V of tile i - NS has read
//    the slot, so a softmax warpgroup finds its next tile's scores ready;
//  * warp 15 (issued by lane 0): O_i = P_i V into O slot i mod 2 with P_i read
//    from TMEM (two issuing warps: the waits of one do not hold the other);
//  * warpgroups 0 and 1 (softmax): warpgroup i mod 2 takes tile i, one query
//    row per thread: reads the row's 16-key chunks that hold keys with one
//    TMEM wait (the chunk count is a template parameter chosen per launch),
//    masks keys past Sk (and past the diagonal when causal), takes the row
//    max, writes P as
//    packed 16-bit pairs over S, and leaves 1/l and the LSE of its row in the
//    row's first bytes of the tile's Q stage (Q is dead once S is formed);
//  * warpgroup 2 (epilogue): scales O by 1/l, converts it and writes it over
//    the same Q stage in the 128-byte-swizzled layout of the output tensor
//    map, the LSE straight to global memory; then O's TMEM slot is free;
//  * warp 14 (store, issued by lane 0): one TMA tensor store per staged O
//    tile (rows past Sq are clipped); a stage is released for the next Q load
//    once its store has read it.
//
// Numerics follow the streaming kernel: exp2 with the scale folded into one
// FMA, fp32 sums, P rounded to the input type; bf16 normalises O by the sum of
// the rounded weights, fp16 by the fp32 sum; LSE = (m + log2 l) ln 2.
//
// Every mbarrier wait is bounded: after WAIT_TIMEOUT_CYCLES the waiting thread
// raises the CTA's abort flag and this unit's status word, every role leaves,
// in-flight copies, stores and MMAs are waited for (bounded), TMEM is freed.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa_internal.h"

namespace fa {
namespace {

// Status words of this translation unit (see read_and_clear_status_short).
__device__ int g_status = 0;
__device__ int g_status_site = 0;

#include "sm100_helpers.cuh"

constexpr int BM = 128;              // query rows per tile
constexpr int THREADS = 512;         // 16 warps
constexpr int W_TMA = 12;
constexpr int W_MMA = 13;
constexpr int W_STORE = 14;
constexpr int W_PV = 15;
constexpr int REG_LAUNCH = 128;      // 65536 / 512
constexpr int REG_SOFTMAX = 184;
constexpr int REG_EPI = 80;
constexpr int REG_CTRL = 64;
// setmaxnreg.inc waits until the registers are free: the split must fit the
// launch allocation and each SM sub-partition (one warp of every warpgroup)
static_assert(2 * 128 * REG_SOFTMAX + 128 * REG_EPI + 128 * REG_CTRL <= THREADS * REG_LAUNCH,
              "register split exceeds the launch allocation");
static_assert(2 * REG_SOFTMAX + REG_EPI + REG_CTRL <= 512, "register split exceeds a sub-partition");
constexpr uint32_t TMEM_COLS = 512;

template <int D>
struct SLayout {
    // TMEM: NS score slots of 128 columns (S, then P over its first columns),
    // then two O slots of D columns
    static constexpr int NS = (D == 64) ? 3 : 2;
    static constexpr uint32_t COL_O = 128u * NS;
    static_assert(COL_O + 2 * D <= TMEM_COLS, "TMEM budget exceeded");
    static constexpr int CHUNKS = D / 64;                   // 128-byte swizzle atoms along D
    static constexpr int CHUNK_BYTES = BM * 128;            // 128 rows x 128 bytes
    static constexpr int TILE_BYTES = CHUNKS * CHUNK_BYTES; // a Q (or staged O) tile; room for K or V
    static constexpr int NQ = (D == 64) ? 6 : 3;            // Q stages
    static constexpr int KV_SLOT = 2 * TILE_BYTES;          // K at 0, V at TILE_BYTES
    static constexpr int Q_OFF = 0;
    static constexpr int KV_OFF = Q_OFF + NQ * TILE_BYTES;
    static constexpr int BAR_OFF = KV_OFF + 2 * KV_SLOT;
    static constexpr int B_QFULL = 0;                       // [NQ] TMA -> MMA
    static constexpr int B_QEMPTY = B_QFULL + NQ;           // [NQ] store -> TMA: O of the stage stored
    static constexpr int B_KVFULL = B_QEMPTY + NQ;          // [2] TMA -> MMA
    static constexpr int B_KVEMPTY = B_KVFULL + 2;          // [2] MMA -> TMA: last P.V of the head done
    // Each barrier below is indexed so that the arrivals of a later phase
    // depend on a wait for the earlier one: no phase is passed unobserved.
    static constexpr int B_SFULL = B_KVEMPTY + 2;           // [NS] MMA -> softmax, by S slot
    static constexpr int B_PFULL = B_SFULL + NS;            // [NS] softmax -> MMA: P written (128 arrivals)
    static constexpr int B_OEMPTY = B_PFULL + NS;           // [2] epilogue -> MMA: O slot read out (128)
    static constexpr int B_OFULL = B_OEMPTY + 2;            // [2] MMA -> epilogue, by O slot
    // [8] softmax -> epilogue: 1/l and LSE of tile i in its stage, at i mod 8
    // (tile i + 8's softmax needs the S issued after the P.V of tile i + 5,
    // which waits for the epilogue of tile i + 3)
    static constexpr int B_STATS = B_OFULL + 2;
    static constexpr int B_OSTAGED = B_STATS + 8;           // [NQ] epilogue -> store, by stage (128)
    static constexpr int B_PDONE = B_OSTAGED + NQ;          // [NS] P.V warp -> S warp: the slot's P read
    static constexpr int B_FIN = B_PDONE + NS;              // both MMA warps: all their MMAs complete (2 commits)
    static constexpr int NBAR = B_FIN + 1;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;     // tmem base, abort flag
    static constexpr int BYTES = MISC_OFF + 16;
    static constexpr int ALLOC = BYTES + 1024;              // slack for 1 KiB alignment
};

struct SParams {
    CUtensorMap tmap_q;   // box {64, 128} over [B][H][Sq][D]
    CUtensorMap tmap_k;   // box {64, skp} over [B][H][Sk][D]
    CUtensorMap tmap_v;
    CUtensorMap tmap_o;   // box {64, 128} over [B][H][Sq][D] (the output)
    float* lse;           // [B, H, Sq] contiguous
    int BH, H, Sq, Sk;
    int skp;              // Sk rounded up to 16: the N of S = Q K^T and the K of P.V
    int n_mt;             // query tiles per head
    int n_tiles;
    int tiles_q, tiles_r; // n_tiles = tiles_q * grid + tiles_r: CTA c takes tiles_q + (c < tiles_r) tiles
    int causal;
    int causal_off;       // Sk - Sq: query i sees keys j <= i + causal_off under the mask
    float scale_log2;
};

// Instruction descriptor for kind::f16 with fp32 accumulate, M = 128.
__host__ __device__ constexpr uint32_t idesc_f16(bool bf16, int N, bool b_mn_major) {
    return (1u << 4)                                   // D format: f32
           | ((bf16 ? 1u : 0u) << 7)                   // A format
           | ((bf16 ? 1u : 0u) << 10)                  // B format
           | ((b_mn_major ? 1u : 0u) << 16)            // B major (A is K-major)
           | ((uint32_t)(N >> 3) << 17)                // N / 8
           | ((uint32_t)(BM >> 4) << 24);              // M / 16
}

// The CTA's tiles: a contiguous range of the tile order, the ranges of all CTAs
// differing in length by at most one.
__device__ __forceinline__ void tile_range(const SParams& p, int& t0, int& n) {
    const int c = (int)blockIdx.x;
    t0 = c * p.tiles_q + min(c, p.tiles_r);
    n = p.tiles_q + (c < p.tiles_r ? 1 : 0);
}

// Position of a tile in (head, query tile) order, stepped without divisions
// (a division by a runtime value costs the single-thread roles ~100 cycles).
struct TilePos {
    int bh, mt;  // head (b * H + h) and query tile within it
    int ub, uh;  // batch and head
    __device__ __forceinline__ void init(const SParams& p, int t) {
        bh = t / p.n_mt;
        mt = t - bh * p.n_mt;
        ub = bh / p.H;
        uh = bh - ub * p.H;
    }
    __device__ __forceinline__ void next(const SParams& p) {
        if (++mt == p.n_mt) {
            mt = 0;
            ++bh;
            if (++uh == p.H) { uh = 0; ++ub; }
        }
    }
};

// 32 lanes x 8 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}

__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}

// ------------------------------------------------------------------ roles
//
// The TMA, MMA and store roles run on whole warps with warp-uniform control
// flow: every lane waits, lane 0 alone issues copies, MMAs, commits and
// arrivals.

// Bounded wait whose result is the same in every lane of the warp.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile uint32_t* abort_flag, int site) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, site));
}

template <int D>
__device__ void producer_role(const SParams& p, uint8_t* smem, volatile uint32_t* abort_flag) {
    using L = SLayout<D>;
    const uint32_t base = smem_u32(smem);
    auto bar = [&](int i) { return base + L::BAR_OFF + 8u * (uint32_t)i; };
    int t0, n;
    tile_range(p, t0, n);
    const uint32_t kv_bytes = 2u * (uint32_t)p.skp * (uint32_t)D * 2u;  // K and V boxes of skp rows
    const bool leader = (threadIdx.x & 31) == 0;
    int kv = -1;
    bool ok = true;
    uint32_t q_mask = 0, q_par = 0, kv_mask = 0, kv_par = 0;  // fills issued and their phase parities
    TilePos pos;
    pos.init(p, t0);
    for (int i = 0; i < n; ++i, pos.next(p)) {
        const int mt = pos.mt, ub = pos.ub, uh = pos.uh;
        if (i == 0 || mt == 0) {  // a new head: its K/V into the next slot
            ++kv;
            const int ks = kv & 1;
            const uint32_t ph = (uint32_t)(kv >> 1) & 1u;
            if (!warp_wait(bar(L::B_KVEMPTY + ks), ph ^ 1u, abort_flag, 140)) { ok = false; break; }
            kv_mask |= 1u << ks;
            kv_par = (kv_par & ~(1u << ks)) | (ph << ks);
            if (leader) {
                mbar_expect_tx(bar(L::B_KVFULL + ks), kv_bytes);
                const uint32_t dst = base + L::KV_OFF + (uint32_t)ks * L::KV_SLOT;
#pragma unroll
                for (int c = 0; c < L::CHUNKS; ++c)
                    tma_load_4d(dst + c * L::CHUNK_BYTES, &p.tmap_k, bar(L::B_KVFULL + ks), c * 64, 0, uh, ub);
#pragma unroll
                for (int c = 0; c < L::CHUNKS; ++c)
                    tma_load_4d(dst + L::TILE_BYTES + c * L::CHUNK_BYTES, &p.tmap_v, bar(L::B_KVFULL + ks), c * 64,
                                0, uh, ub);
            }
            __syncwarp();
        }
        const int s = i % L::NQ;
        const uint32_t ph = (uint32_t)(i / L::NQ) & 1u;
        if (!warp_wait(bar(L::B_QEMPTY + s), ph ^ 1u, abort_flag, 141)) { ok = false; break; }
        q_mask |= 1u << s;
        q_par = (q_par & ~(1u << s)) | (ph << s);
        if (leader) {
            mbar_expect_tx(bar(L::B_QFULL + s), L::TILE_BYTES);
            const uint32_t dst = base + L::Q_OFF + (uint32_t)s * L::TILE_BYTES;
#pragma unroll
            for (int c = 0; c < L::CHUNKS; ++c)
                tma_load_4d(dst + c * L::CHUNK_BYTES, &p.tmap_q, bar(L::B_QFULL + s), c * 64, mt * BM, uh, ub);
        }
        __syncwarp();
    }
    if (!ok) {
        // drain the copies this warp issued before leaving
        for (int s = 0; s < L::NQ; ++s)
            if (q_mask & (1u << s)) mbar_drain(bar(L::B_QFULL + s), (q_par >> s) & 1u);
        for (int s = 0; s < 2; ++s)
            if (kv_mask & (1u << s)) mbar_drain(bar(L::B_KVFULL + s), (kv_par >> s) & 1u);
    }
}

template <int D, bool BF16>
__device__ void mma_role(const SParams& p, uint8_t* smem, uint32_t tmem, bool is_pv_warp,
                         volatile uint32_t* abort_flag) {
    using L = SLayout<D>;
    const uint32_t base = smem_u32(smem);
    auto bar = [&](int i) { return base + L::BAR_OFF + 8u * (uint32_t)i; };
    int t0, n;
    tile_range(p, t0, n);
    const uint32_t idesc_s = idesc_f16(BF16, p.skp, false);
    constexpr uint32_t IDESC_PV = idesc_f16(BF16, D, true);
    const int ksteps_pv = p.skp / 16;
    // S = Q K^T: A = Q (K-major), B = K (K-major), 128-byte swizzle, 8-row groups
    // 1024 bytes apart; K steps of 16 elements advance 32 bytes inside an atom and
    // a whole chunk across the 64-column chunks.
    // O = P V: A = P in TMEM (16 keys per 8 columns), B = V read MN-major (D
    // contiguous): 64-element chunks a chunk apart (leading byte offset; unused
    // with one chunk), 8-key groups 1024 bytes apart; K steps of 16 keys advance
    // 2 KiB.
    constexpr uint32_t V_LBO = (D == 128) ? (uint32_t)L::CHUNK_BYTES : 1024u;
    const uint64_t dq = sw128_desc(base + L::Q_OFF, 16, 1024);
    const uint64_t dk = sw128_desc(base + L::KV_OFF, 16, 1024);
    const uint64_t dv = sw128_desc(base + L::KV_OFF + L::TILE_BYTES, V_LBO, 1024);
    const uint32_t dq_lo = (uint32_t)dq, dq_hi = (uint32_t)(dq >> 32);
    const uint32_t dk_lo = (uint32_t)dk, dk_hi = (uint32_t)(dk >> 32);
    const uint32_t dv_lo = (uint32_t)dv, dv_hi = (uint32_t)(dv >> 32);

    // Positions of the next tile whose S is to be issued (ps) and of the next
    // tile whose P.V is (pp), with their K/V indices within the range (heads are
    // contiguous in the tile order: the index counts head changes)
    TilePos ps, pp;
    ps.init(p, t0);
    pp = ps;
    int kv_s = 0, kv_p = 0;
    const bool leader = (threadIdx.x & 31) == 0;
    bool ok = true;

    auto issue_s = [&](int i) -> bool {
        const int s = i % L::NQ;
        if (!warp_wait(bar(L::B_QFULL + s), (uint32_t)(i / L::NQ) & 1u, abort_flag, 142)) return false;
        const int kv = kv_s;
        if (i == 0 || ps.mt == 0) {  // the first tile of its K/V
            if (!warp_wait(bar(L::B_KVFULL + (kv & 1)), (uint32_t)(kv >> 1) & 1u, abort_flag, 143)) return false;
        }
        const int slot = i % L::NS;
        const uint32_t a_lo = dq_lo + (uint32_t)s * ((uint32_t)L::TILE_BYTES >> 4);
        const uint32_t b_lo = dk_lo + (uint32_t)(kv & 1) * ((uint32_t)L::KV_SLOT >> 4);
        const uint32_t d_tmem = tmem + 128u * (uint32_t)slot;
        if (leader) {
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t off = (uint32_t)(((ks & 3) * 32 + (ks >> 2) * L::CHUNK_BYTES) >> 4);
                tc_mma_ss2(d_tmem, a_lo + off, dq_hi, b_lo + off, dk_hi, idesc_s, ks > 0 ? 1u : 0u);
            }
            tc_commit(bar(L::B_SFULL + slot));
        }
        __syncwarp();
        ps.next(p);
        if (ps.mt == 0) ++kv_s;
        return true;
    };
    auto issue_pv = [&](int i) -> bool {
        const int slot = i % L::NS, b = i & 1;
        if (!warp_wait(bar(L::B_PFULL + slot), (uint32_t)(i / L::NS) & 1u, abort_flag, 144)) return false;
        if (!warp_wait(bar(L::B_OEMPTY + b), (uint32_t)(i >> 1) & 1u, abort_flag, 150)) return false;
        tc_fence_after();  // P was written, O read, by tcgen05.st / ld of other threads
        const int kv = kv_p;
        const uint32_t b_lo = dv_lo + (uint32_t)(kv & 1) * ((uint32_t)L::KV_SLOT >> 4);
        const uint32_t a_tmem = tmem + 128u * (uint32_t)slot;
        const uint32_t d_tmem = tmem + L::COL_O + (uint32_t)(D * b);
        if (leader) {
#pragma unroll 1
            for (int ks = 0; ks < ksteps_pv; ++ks)
                tc_mma_ts2(d_tmem, a_tmem + (uint32_t)(ks * 8), b_lo + (uint32_t)(ks * (2048 >> 4)), dv_hi, IDESC_PV,
                           ks > 0 ? 1u : 0u);
            tc_commit(bar(L::B_OFULL + b));
            // the last P.V of its K/V: the slot may be refilled once this completes
            if (i == n - 1 || pp.mt == p.n_mt - 1) tc_commit(bar(L::B_KVEMPTY + (kv & 1)));
        }
        __syncwarp();
        pp.next(p);
        if (pp.mt == 0) ++kv_p;
        return true;
    };
    // Two issuing warps: this warp (S_j into slot j mod NS once the P.V of tile
    // j - NS has completed: that slot held its P) and the P.V warp.  A new
    // K/V slot's first S waits for the slot's fill, which follows the last P.V
    // of the index two before (issued by the other warp, whose P and therefore
    // S came earlier): no wait cycle.
    if (is_pv_warp) {
        for (int i = 0; ok && i < n; ++i) {
            ok = issue_pv(i);
            if (ok && leader) tc_commit(bar(L::B_PDONE + i % L::NS));
            __syncwarp();
        }
    } else {
        for (int j = 0; ok && j < n; ++j) {
            if (j >= L::NS) {
                ok = warp_wait(bar(L::B_PDONE + j % L::NS), (uint32_t)(j / L::NS - 1) & 1u, abort_flag, 151);
                if (!ok) break;
            }
            ok = issue_s(j);
        }
    }
    if (leader) tc_commit(bar(L::B_FIN));
    __syncwarp();
    mbar_drain(bar(L::B_FIN), 0u);
}

// NC 16-key chunks of a row (32 lanes x 16 columns each) loaded with one
// wait; the empty statements after the wait tie each register to it, so no
// use of a value can be scheduled before the load has completed.
template <int NC>
__device__ __forceinline__ void tmem_ld_chunks(uint32_t taddr, uint32_t (&r)[NC * 16]) {
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        uint32_t* x = r + 16 * c;
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(x[0]), "=r"(x[1]), "=r"(x[2]), "=r"(x[3]), "=r"(x[4]), "=r"(x[5]), "=r"(x[6]), "=r"(x[7]),
              "=r"(x[8]), "=r"(x[9]), "=r"(x[10]), "=r"(x[11]), "=r"(x[12]), "=r"(x[13]), "=r"(x[14]), "=r"(x[15])
            : "r"(taddr + 16u * (uint32_t)c));
    }
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        uint32_t* x = r + 16 * c;
        asm volatile("" : "+r"(x[0]), "+r"(x[1]), "+r"(x[2]), "+r"(x[3]), "+r"(x[4]), "+r"(x[5]), "+r"(x[6]),
                     "+r"(x[7]), "+r"(x[8]), "+r"(x[9]), "+r"(x[10]), "+r"(x[11]), "+r"(x[12]), "+r"(x[13]),
                     "+r"(x[14]), "+r"(x[15]));
    }
}

// The softmax of the tiles of warpgroup b for rows whose keys fill NC 16-key
// chunks (NC = skp / 16, a compile-time count: the row is read from TMEM with
// one wait and kept in registers for the max and the weights).
template <int D, bool BF16, int NC>
__device__ void softmax_tiles(const SParams& p, uint8_t* smem, uint32_t tmem, int b, int warp_in_group,
                              volatile uint32_t* abort_flag) {
    using L = SLayout<D>;
    const uint32_t base = smem_u32(smem);
    auto bar = [&](int i) { return base + L::BAR_OFF + 8u * (uint32_t)i; };
    const int lane = threadIdx.x & 31;
    const int r = warp_in_group * 32 + lane;  // row in the tile = TMEM lane
    const uint32_t lane_sel = (uint32_t)(warp_in_group * 32) << 16;
    const float sl2 = p.scale_log2;
    const float2 sl2x2 = make_float2(sl2, sl2);
    int t0, n;
    tile_range(p, t0, n);
    TilePos pos;
    pos.init(p, t0 + b);
    for (int i = b; i < n; i += 2, pos.next(p), pos.next(p)) {
        const int row = pos.mt * BM + r;
        const int key_limit = p.causal ? min(row + p.causal_off, p.Sk - 1) : p.Sk - 1;  // last visible key
        const int slot = i % L::NS;
        const uint32_t ts = tmem + lane_sel + 128u * (uint32_t)slot;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_SFULL + slot), (uint32_t)(i / L::NS) & 1u, abort_flag, 145 + b)))
            return;
        tc_fence_after();
        uint32_t u[NC * 16];
        tmem_ld_chunks<NC>(ts, u);
        float x[NC * 16];
        // keys past the row's last visible key drop out
#pragma unroll
        for (int c = 0; c < NC * 16; ++c) x[c] = (c > key_limit) ? -INFINITY : __uint_as_float(u[c]);
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const float* y = x + 16 * c;
            mx0 = max3(mx0, max3(y[0], y[1], y[2]), max3(y[3], y[4], y[5]));
            mx1 = max3(mx1, max3(y[6], y[7], y[8]), max3(y[9], y[10], y[11]));
            mx0 = max3(mx0, y[12], y[13]);
            mx1 = max3(mx1, y[14], y[15]);
        }
        // every row sees key 0, so the max is finite
        const float m = fmaxf(mx0, mx1) * sl2;
        const float2 negm2 = make_float2(-m, -m);
        float2 lsum0 = make_float2(0.f, 0.f), lsum1 = make_float2(0.f, 0.f);
        float2 rsum0 = make_float2(0.f, 0.f), rsum1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            uint32_t pk[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float2 y = __ffma2_rn(make_float2(x[16 * c + 2 * j], x[16 * c + 2 * j + 1]), sl2x2, negm2);
                const float2 e = make_float2(ex2(y.x), ex2(y.y));
                pk[j] = pack2<BF16>(e.x, e.y);
                if (j & 1) lsum1 = __fadd2_rn(lsum1, e); else lsum0 = __fadd2_rn(lsum0, e);
                if constexpr (BF16) {
                    if (j & 1) rsum1 = add_bf16x2(rsum1, pk[j]); else rsum0 = add_bf16x2(rsum0, pk[j]);
                }
            }
            // P (16-bit, two keys per column) over the first columns of S
            tmem_st8(ts + 8u * (uint32_t)c, pk);
        }
        const float2 ls = __fadd2_rn(lsum0, lsum1);
        const float l = ls.x + ls.y;
        const float2 rs = __fadd2_rn(rsum0, rsum1);
        const float norm = BF16 ? (rs.x + rs.y) : l;
        // 1/norm and the LSE for the epilogue, in this row's first bytes of the
        // tile's stage (the epilogue thread of this row reads them before it
        // writes the row's output there)
        *reinterpret_cast<float2*>(smem + L::Q_OFF + (i % L::NQ) * L::TILE_BYTES + r * 128) =
            make_float2(1.f / norm, (m + __log2f(l)) * 0.69314718055994530942f);
        mbar_arrive(bar(L::B_STATS + (i & 7)));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(L::B_PFULL + slot));
    }
}

template <int D, bool BF16>
__device__ void softmax_role(const SParams& p, uint8_t* smem, uint32_t tmem, int b, int warp_in_group,
                             volatile uint32_t* abort_flag) {
    switch (p.skp / 16) {
        case 1: softmax_tiles<D, BF16, 1>(p, smem, tmem, b, warp_in_group, abort_flag); break;
        case 2: softmax_tiles<D, BF16, 2>(p, smem, tmem, b, warp_in_group, abort_flag); break;
        case 3: softmax_tiles<D, BF16, 3>(p, smem, tmem, b, warp_in_group, abort_flag); break;
        case 4: softmax_tiles<D, BF16, 4>(p, smem, tmem, b, warp_in_group, abort_flag); break;
        case 5: softmax_tiles<D, BF16, 5>(p, smem, tmem, b, warp_in_group, abort_flag); break;
        case 6: softmax_tiles<D, BF16, 6>(p, smem, tmem, b, warp_in_group, abort_flag); break;
        case 7: softmax_tiles<D, BF16, 7>(p, smem, tmem, b, warp_in_group, abort_flag); break;
        default: softmax_tiles<D, BF16, 8>(p, smem, tmem, b, warp_in_group, abort_flag); break;
    }
}

template <int D, bool BF16>
__device__ void epilogue_role(const SParams& p, uint8_t* smem, uint32_t tmem, int warp_in_group,
                              volatile uint32_t* abort_flag) {
    using L = SLayout<D>;
    const uint32_t base = smem_u32(smem);
    auto bar = [&](int i) { return base + L::BAR_OFF + 8u * (uint32_t)i; };
    const int lane = threadIdx.x & 31;
    const int r = warp_in_group * 32 + lane;
    const uint32_t lane_sel = (uint32_t)(warp_in_group * 32) << 16;
    int t0, n;
    tile_range(p, t0, n);
    // both O slots start free
    mbar_arrive(bar(L::B_OEMPTY + 0));
    mbar_arrive(bar(L::B_OEMPTY + 1));
    TilePos pos;
    pos.init(p, t0);
    for (int i = 0; i < n; ++i, pos.next(p)) {
        const int b = i & 1;
        const int bh = pos.bh;
        const int row = pos.mt * BM + r;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_OFULL + b), (uint32_t)(i >> 1) & 1u, abort_flag, 147)))
            return;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_STATS + (i & 7)), (uint32_t)(i >> 3) & 1u, abort_flag, 148)))
            return;
        tc_fence_after();
        uint8_t* stg = smem + L::Q_OFF + (i % L::NQ) * L::TILE_BYTES + r * 128;
        const float2 fin = *reinterpret_cast<const float2*>(stg);  // (1/norm, LSE)
        const float2 inv2 = make_float2(fin.x, fin.x);
        const uint32_t to = tmem + lane_sel + L::COL_O + (uint32_t)(D * b);
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32u(to + 32u * (uint32_t)c, o);
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float2 v = __fmul2_rn(make_float2(__uint_as_float(o[2 * j]), __uint_as_float(o[2 * j + 1])), inv2);
                w[j] = pack2<BF16>(v.x, v.y);
            }
            uint8_t* chunk = stg + (c >> 1) * L::CHUNK_BYTES;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int unit = (c & 1) * 4 + q;  // 16-byte unit of the 128-byte row
                *reinterpret_cast<uint4*>(chunk + ((unit ^ (r & 7)) << 4)) =
                    make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
            }
        }
        // the staged tile is read by the TMA engine (async proxy)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (row < p.Sq) p.lse[(size_t)bh * (size_t)p.Sq + row] = fin.y;
        tc_fence_before();  // O slot b read out: the P.V of tile i + 2 may overwrite it
        mbar_arrive(bar(L::B_OEMPTY + b));
        mbar_arrive(bar(L::B_OSTAGED + i % L::NQ));
    }
}

template <int D>
__device__ void store_role(const SParams& p, uint8_t* smem, volatile uint32_t* abort_flag) {
    using L = SLayout<D>;
    const uint32_t base = smem_u32(smem);
    auto bar = [&](int i) { return base + L::BAR_OFF + 8u * (uint32_t)i; };
    int t0, n;
    tile_range(p, t0, n);
    const bool leader = (threadIdx.x & 31) == 0;
    TilePos pos;
    pos.init(p, t0);
    int i = 0;
    for (; i < n; ++i, pos.next(p)) {
        if (!warp_wait(bar(L::B_OSTAGED + i % L::NQ), (uint32_t)(i / L::NQ) & 1u, abort_flag, 149)) break;
        if (leader) {
            const uint32_t src = base + L::Q_OFF + (uint32_t)(i % L::NQ) * L::TILE_BYTES;
#pragma unroll
            for (int c = 0; c < L::CHUNKS; ++c)
                tma_store_4d(&p.tmap_o, src + c * L::CHUNK_BYTES, c * 64, pos.mt * BM, pos.uh, pos.ub);
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            // a stage may take the next Q tile once its store has read it: the
            // previous tile's store (all groups but the newest) is waited for here
            if (i > 0) {
                asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                mbar_arrive(bar(L::B_QEMPTY + (i - 1) % L::NQ));
            }
        }
        __syncwarp();
    }
    if (leader) {
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        if (i > 0) mbar_arrive(bar(L::B_QEMPTY + (i - 1) % L::NQ));
        asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    }
    __syncwarp();
}

template <int D, bool BF16>
__global__ void __launch_bounds__(THREADS, 1) fa_fwd_kernel_short(const __grid_constant__ SParams p) {
    using L = SLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t base = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int wg = warp >> 2;
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    volatile uint32_t* abort_flag = misc + 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < L::NBAR; ++i) {
            uint32_t count = 1;  // TMA transaction or tcgen05.commit arrivals, or the store thread
            if ((i >= L::B_PFULL && i < L::B_OFULL) || (i >= L::B_STATS && i < L::B_PDONE))
                count = BM;      // one arrival per thread of a warpgroup (P, O read out, stats, staged O)
            if (i == L::B_FIN) count = 2;  // one commit from each MMA warp
            mbar_init(base + L::BAR_OFF + 8 * i, count);
        }
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == W_TMA && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmap_q)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmap_k)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmap_v)) : "memory");
        // the first tile's Q and its head's K and V into L2 while the previous
        // kernel in the stream may still run: a prefetch only warms L2, the
        // point of coherence, so the loads after the dependency wait still see
        // that kernel's writes
        int t0, n;
        tile_range(p, t0, n);
        if (n > 0) {
            TilePos pos;
            pos.init(p, t0);
#pragma unroll
            for (int c = 0; c < L::CHUNKS; ++c) {
                l2_prefetch_4d(&p.tmap_q, c * 64, pos.mt * BM, pos.uh, pos.ub);
                l2_prefetch_4d(&p.tmap_k, c * 64, 0, pos.uh, pos.ub);
                l2_prefetch_4d(&p.tmap_v, c * 64, 0, pos.uh, pos.ub);
            }
        }
    }
    if (warp == W_STORE && lane == 0)
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmap_o)) : "memory");
    if (warp == W_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(misc)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    grid_dependency_sync();  // the previous kernel in the stream has completed

    if (wg < 2) {
        setmaxnreg_inc<REG_SOFTMAX>();
        softmax_role<D, BF16>(p, smem, tmem, wg, warp & 3, abort_flag);
    } else if (wg == 2) {
        setmaxnreg_dec<REG_EPI>();
        epilogue_role<D, BF16>(p, smem, tmem, warp & 3, abort_flag);
    } else {
        setmaxnreg_dec<REG_CTRL>();
        if (warp == W_TMA) producer_role<D>(p, smem, abort_flag);
        else if (warp == W_MMA || warp == W_PV) mma_role<D, BF16>(p, smem, tmem, warp == W_PV, abort_flag);
        else if (warp == W_STORE) store_role<D>(p, smem, abort_flag);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == W_MMA) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

template <int D, bool BF16>
cudaError_t launch_short(const LaunchArgs& a, cudaStream_t stream) {
    using L = SLayout<D>;
    static_assert(L::ALLOC <= 232448, "shared memory budget exceeded");
    auto kern = fa_fwd_kernel_short<D, BF16>;
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), L::ALLOC);
    if (e != cudaSuccess) return e;
    SParams p;
    p.tmap_q = a.tmap_q;
    p.tmap_k = a.tmap_k;
    p.tmap_v = a.tmap_v;
    p.tmap_o = a.tmap_o;
    p.lse = a.lse;
    p.BH = a.B * a.H;
    p.H = a.H;
    p.Sq = a.Sq;
    p.Sk = a.Sk;
    p.skp = (a.Sk + 15) / 16 * 16;
    p.n_mt = (a.Sq + BM - 1) / BM;
    p.n_tiles = p.BH * p.n_mt;
    p.tiles_q = p.n_tiles / a.grid;
    p.tiles_r = p.n_tiles - p.tiles_q * a.grid;
    p.causal = a.causal;
    p.causal_off = a.Sk - a.Sq;
    p.scale_log2 = a.scale_log2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.grid, 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = L::ALLOC;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    set_programmatic_launch(cfg, attr);
    return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

cudaError_t launch_fwd_short_sm100(const LaunchArgs& a, cudaStream_t stream) {
    if (a.Sk < 1 || a.Sk > SHORT_SK_MAX || a.mask || a.drop.enabled) return cudaErrorInvalidValue;
    if (a.D == 128) return a.dtype == 1 ? launch_short<128, true>(a, stream) : launch_short<128, false>(a, stream);
    if (a.D == 64) return a.dtype == 1 ? launch_short<64, true>(a, stream) : launch_short<64, false>(a, stream);
    return cudaErrorInvalidValue;
}

cudaError_t read_and_clear_status_short(cudaStream_t stream, int* status, int* site) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    int st = 0, si = 0;
    e = cudaMemcpyFromSymbolAsync(&st, g_status, sizeof(int), 0, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess)
        e = cudaMemcpyFromSymbolAsync(&si, g_status_site, sizeof(int), 0, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    if (st != 0) {
        const int zero = 0;
        e = cudaMemcpyToSymbolAsync(g_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream);
        if (e == cudaSuccess)
            e = cudaMemcpyToSymbolAsync(g_status_site, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    }
    *status = st;
    *site = si;
    return e;
}

}  // namespace fa
