// fa_bwd_sm100.cu -- attention backward pass (dQ, dK, dV) for B200 (sm_100a).
//
// Gradients of O = softmax(scale * Q K^T [+ causal]) V for an upstream
// gradient dO, by the FlashAttention-2 recomputation scheme: the forward pass
// keeps only O and the per-row log-sum-exp; the backward pass recomputes the
// scores and weights tile by tile instead of storing the S x S matrix
// ("FlashAttention-2 在昇腾 NPU 上如何做到 3 倍加速？深度拆解 ops-transformer 的实现",
// the recomputation row of the core-optimisation table and section 6.2; the
// backward configuration of the gsyq.cn catlass FlashAttention page,
// "反向传播的特殊处理", whose non-deterministic mode accumulates with atomic
// adds, as dQ does here).
//
// With P_ij = exp(scale * q_i.k_j - LSE_i), dP_ij = dO_i.v_j and
// Delta_i = sum_d dO_id O_id (= sum_j P_ij dP_ij):
//   dV_j = sum_i P_ij dO_i
//   dS_ij = P_ij (dP_ij - Delta_i)
//   dK_j = scale * sum_i dS_ij q_i
//   dQ_i = scale * sum_j dS_ij k_j
//
// Three launches on the caller's stream:
//   1. bwd_prep_kernel: Delta_i, LSE_i * log2(e) (rows padded to a multiple of
//      128: +inf, so that their weights are 0) and a zeroed fp32 dQ accumulator;
//   2. fa_bwd_kernel_wide: one persistent CTA per SM; a work unit is (b, h,
//      128-key tile[, half of D at D = 256][, chunk of the query range]).  The
//      CTA keeps K_n, V_n in shared memory and dK, dV in tensor memory and
//      walks the query rows that see its keys in 64-row steps with
//      double-buffered scores (see below):
//        S^T = K Q_m^T, dP^T = V dO_m^T   (tcgen05.mma, fp32 in TMEM)
//        P^T, dS^T                          (one key row per thread, packed to
//                                            16 bits in TMEM; dS^T also to SMEM)
//        dV += P^T dO_m, dK += dS^T Q_m     (A operand from TMEM)
//        dQ_m^T = K^T dS^T                  (into the step's dP^T columns)
//      (D = 64: dQ_m^T first, and dK takes dS^T from SMEM, not TMEM)
//      dQ_m is added to the fp32 accumulator (a TMA bulk reduce-add, or
//      per-element atomics, or in key-tile order in deterministic mode); dK,
//      dV are written once per unit.  D = 64 runs the D = 128 instantiation
//      on the first 64-column chunk of Q, K, V and dO: the scores reduce over
//      it alone, and the lanes of dQ^T and the columns of dK, dV past 64 that
//      the other chunk feeds are never written out;
//   3. bwd_post_kernel: dQ = scale * accumulator, rounded to the 16-bit dtype
//      (and, after a split query range, bwd_post_kv_kernel for dK and dV).
//
// Every mbarrier wait is bounded like the forward kernel's (abort flag, status
// word read by fa_check_status, drained copies, TMEM freed).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa_internal.h"

namespace fa {
namespace {

// Status words of this translation unit (see read_and_clear_status_bwd).
__device__ int g_status = 0;
__device__ int g_status_site = 0;

#include "sm100_helpers.cuh"

constexpr int BW_TMA = 0;          // warp 0 lane 0: TMA loads and unit claims
constexpr int BW_MMA = 1;          // warp 1 lane 0: every tcgen05.mma; TMEM owner
constexpr int TILE = 128;          // keys per unit and query rows per step
constexpr uint32_t BWD_TMEM_COLS = 512;

struct Strides3 {
    long long s[3];  // element strides over b, h and the row
};

struct BwdParams {
    CUtensorMap tmap_q;
    CUtensorMap tmap_k;
    CUtensorMap tmap_v;
    CUtensorMap tmap_do;
    CUtensorMap tmap_dq;  // fp32 dQ accumulator [BH][Sq][D], box {128, 64, 1} (bulk reduce-add)
    const float* lse2;    // [BH][Sq_pad] LSE * log2(e), +inf on padded rows
    const float* delta;   // [BH][Sq_pad] rowsum(dO * O), 0 on padded rows
    float* dq_acc;        // [BH][Sq][D] fp32, zeroed by the prep kernel
    uint8_t* dk;          // [B][H][Sk][D] 16-bit at byte strides dk_s (over b, h, key row)
    uint8_t* dv;          // the same at dv_s
    long long dk_s[3], dv_s[3];
    // Split query range (key sets of at most KV_ACC_ROWS keys, few units): a
    // unit takes chunk c of its key tile's query steps, q_chunk steps long, and
    // adds its dK (scaled) and dV in fp32 to dk_acc / dv_acc [BH][KV_ACC_ROWS][D]
    // instead of writing them; q_split = 1: off.  With one key tile per head a
    // step's dQ rows are complete in the unit that forms them: the split
    // instantiation of the D = 128 kernel (which has the dQ staging tile)
    // writes them to dq (16-bit, byte strides dq_s) directly.
    int q_split, q_chunk;
    float* dk_acc;
    float* dv_acc;
    uint8_t* dq;
    long long dq_s[3];
    int BH, H, Sq, Sk, Sq_pad, n_mtiles, n_ktiles, n_units, causal, causal_off;
    int dh;               // head dimension of the tensors (64: run by the D = 128 kernel on its first column chunk)
    int head_group;       // causal claim order: heads per group (their Q, dO, dQ fit in L2)
    int* dq_flags;        // deterministic mode: [BH][flag_steps][4] key tiles added so far per
                          // (head, query step, warp); null: dQ is added with atomics
    int flag_steps;
    const uint8_t* mask;         // explicit boolean mask (nonzero = attend), or null
    long long m_sb, m_sh, m_ss;  // its element strides over b, h and the query row
    float scale_log2;     // scale * log2(e)
    float scale;
    unsigned int* sched;  // zeroed unit counter (causal), or null
    // dropout: on/off, threshold in every byte, generator key, counter word 3, 1 / (1 - p)
    int drop;
    uint32_t drop_p8x4, seed_lo, seed_hi, drop_offset;
    float keep_scale;
};

struct BUnit {
    int bh;
    int n;      // key tile
    int m_lo;   // first query tile that sees a key of the tile
    int T;      // query tiles visited
    int half;   // D = 256: the 128-wide half of the head dimension whose dK, dV, dQ this unit forms
};

// Units: with the causal mask the number of query tiles falls with the key
// tile index, so units are claimed in key-tile order (longest first), heads
// innermost, within groups of head_group heads whose Q, dO and dQ accumulator
// stay in L2 together; without the mask, heads outermost (CTAs running
// together share one head's Q, dO and dQ in L2).
__device__ __forceinline__ void causal_unit_order(const BwdParams& p, int u, int* bh, int* n) {
    const int per_group = p.head_group * p.n_ktiles;
    const int g = u / per_group;
    const int within = u - g * per_group;
    const int gh = min(p.head_group, p.BH - g * p.head_group);  // heads in this group
    *n = within / gh;
    *bh = g * p.head_group + (within - *n * gh);
}

// Split query range: chunk c of the unit's steps [m_lo, n_mtiles).  The host
// picks q_chunk so that no chunk is empty (one key tile: m_lo = 0).
__device__ __forceinline__ void split_query_range(const BwdParams& p, int c, BUnit& U) {
    const int lo = max(U.m_lo, c * p.q_chunk);
    const int hi = min(U.m_lo + U.T, (c + 1) * p.q_chunk);
    U.m_lo = lo;
    U.T = hi - lo;
}

__host__ __device__ constexpr uint32_t make_idesc_bwd(bool bf16, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4)                                   // D format: f32
           | ((bf16 ? 1u : 0u) << 7)                   // A format
           | ((bf16 ? 1u : 0u) << 10)                  // B format
           | ((a_mn_major ? 1u : 0u) << 15)            // A major
           | ((b_mn_major ? 1u : 0u) << 16)            // B major
           | ((uint32_t)(N >> 3) << 17)                // N / 8
           | ((uint32_t)(TILE >> 4) << 24);            // M / 16 (M = 128)
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// TMA bulk reduce-add of a shared-memory box into a 3-D fp32 tensor (rows past
// the tensor's extent are clipped), tracked by this thread's bulk groups.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2) {
    asm volatile(
        "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(src), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until this thread's bulk groups have read their shared-memory sources
// (`read`) or completed.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// Split query range: one thread's key row of dV and dK (W columns of fp32 in
// TMEM from dv_col / dk_col) added to the fp32 accumulator rows, dK scaled.
// The TMEM loads are warp-collective: every lane loads, valid lanes add.
__device__ __noinline__ void kv_partial_add(uint32_t dv_col, uint32_t dk_col, float* dva, float* dka,
                                            float scale, bool valid, int width) {
#pragma unroll 1
    for (int c = 0; c < width / 32; ++c) {
        uint32_t r[32];
        tmem_ld32u(dv_col + 32 * c, r);
        if (valid) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                red_add_v4(dva + 32 * c + 4 * i, __uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                           __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
        }
        tmem_ld32u(dk_col + 32 * c, r);
        if (valid) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                red_add_v4(dka + 32 * c + 4 * i, __uint_as_float(r[4 * i]) * scale, __uint_as_float(r[4 * i + 1]) * scale,
                           __uint_as_float(r[4 * i + 2]) * scale, __uint_as_float(r[4 * i + 3]) * scale);
        }
    }
}

// Deterministic dQ: the key tiles of one head add their dQ contributions to
// each query step in key-tile order.  A warp waits (bounded) until the step's
// counter for it equals its key tile, adds with plain loads and stores that
// bypass L1, and passes the turn on with a release store.  Units are claimed
// from the counter in key-tile order, so the tile a warp waits for belongs to a
// CTA that is already running.
__device__ __forceinline__ bool wait_turn(const int* flag, int target, volatile uint32_t* abort_flag, int site) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) {
        const long long t0 = clock64();
        for (uint32_t it = 0;; ++it) {
            int v;
            asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
            if (v == target) break;
            if ((it & 15u) == 15u) {
                if (*abort_flag) { ok = 0; break; }
                if (clock64() - t0 > WAIT_TIMEOUT_CYCLES) {
                    *abort_flag = 1u;
                    record_failure(site);
                    ok = 0;
                    break;
                }
            }
            __nanosleep(32);
        }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

__device__ __forceinline__ void pass_turn(int* flag, int next) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) {
        __threadfence();
        asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(flag), "r"(next) : "memory");
    }
}

// Explicit mask, transposed for a warp that owns keys key0 .. key0 + 31 (one
// per lane): returns for this lane's key the bits of queries q0 .. q0 + 31
// (bit i set = query q0 + i may attend).  Lane i reads query row q0 + i's 32
// mask bytes (two 16-byte loads; byte loads on the ragged last keys; rows past
// Sq read the last row), folds them into 32 bits, and 32 ballots transpose the
// warp's 32 x 32 bit block.
__device__ __forceinline__ uint32_t mask_col_bits(const uint8_t* mhead, long long ss, int Sq, int Sk, int q0,
                                                  int key0) {
    const int lane = threadIdx.x & 31;
    const uint8_t* r = mhead + (long long)min(q0 + lane, Sq - 1) * ss + key0;
    uint32_t rowbits = 0u;
    if (key0 + 32 <= Sk) {
        const uint4 a = __ldg(reinterpret_cast<const uint4*>(r));
        const uint4 b = __ldg(reinterpret_cast<const uint4*>(r + 16));
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            // one bit per nonzero byte, gathered into a nibble (byte i -> bit i)
            const uint32_t t = __vcmpne4(w[e], 0u) & 0x01010101u;
            rowbits |= ((t * 0x01020408u) >> 24 & 0xFu) << (4 * e);
        }
    } else {
        for (int c = 0; c < Sk - key0; ++c)
            if (r[c]) rowbits |= 1u << c;
    }
    uint32_t col = 0u;
#pragma unroll
    for (int kk = 0; kk < 32; ++kk) {
        const uint32_t bal = __ballot_sync(0xffffffffu, (rowbits >> kk) & 1u);
        if (lane == kk) col = bal;
    }
    return col;
}

// Dropout keep decisions in the same transposed form: for this lane's key
// (key0 + lane) the bits of queries q0 .. q0 + 31 (bit i set = the weight of
// query q0 + i is kept).  Lane i draws the two generator blocks of query
// q0 + i over keys key0 .. key0 + 31 (key0 a multiple of 16), folds their
// keep bytes into 32 bits, and 32 ballots transpose the warp's block.
__device__ __forceinline__ uint32_t dropout_col_bits(const BwdParams& p, int bh, int q0, int key0) {
    const int lane = threadIdx.x & 31;
    const uint32_t q = (uint32_t)(q0 + lane), g = (uint32_t)key0 >> 4;
    const uint4 a = dropout_keep_bytes(g, q, (uint32_t)bh, p.drop_offset, p.seed_lo, p.seed_hi, p.drop_p8x4);
    const uint4 b = dropout_keep_bytes(g + 1u, q, (uint32_t)bh, p.drop_offset, p.seed_lo, p.seed_hi, p.drop_p8x4);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t rowbits = 0u;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const uint32_t t = w[e] & 0x01010101u;  // one byte per key: 1 kept, 0 dropped
        rowbits |= ((t * 0x01020408u) >> 24 & 0xFu) << (4 * e);
    }
    uint32_t col = 0u;
#pragma unroll
    for (int kk = 0; kk < 32; ++kk) {
        const uint32_t bal = __ballot_sync(0xffffffffu, (rowbits >> kk) & 1u);
        if (lane == kk) col = bal;
    }
    return col;
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Reads the work-unit indices published by the TMA lane (same protocol as the
// forward kernel's ring): -1 when the CTA has no more work, -2 on abort.
// ------------------------------------------------------------------------
// 64-row query steps with double-buffered S^T / dP^T (D = 64 on the D = 128
// instantiation with its second column chunk unused, D = 128, D = 256).
//
// Tensor memory: S0 [0,64) dP0 [64,128) S1 [128,192) dP1 [192,256), dV
// [256,384), dK [384,512).  While the dS warpgroup turns step g's S^T, dP^T
// (buffer g&1) into P^T, dS^T, the MMA lane already computes step g+1's into
// the other buffer; then dV += P^T dO, dK += dS^T Q and dQ^T = K^T dS^T (M = D
// = 128 lanes, N = 64 queries) into step g's dP columns (after dK has read
// dS^T there), which the output warpgroup reads out (one head-dimension lane
// per thread) into the fp32 dQ accumulator.  The next S^T into a buffer needs
// no wait; only its dP^T waits for that buffer's dQ^T read-out, and the S^T
// MMAs issued before it cover that latency.  Q and dO stream through three 32 KiB stages.  Every role
// derives buffer, stage and barrier parities from the global step count g.
//
// D = 256: dK and dV of a 128-key tile would fill the 512 tensor-memory columns
// by themselves, so a work unit is (head, key tile, half of D): it computes
// the full-D scores S^T = K Q^T and dP^T = V dO^T (16 K steps), then dK, dV and
// dQ for its 128-wide half only, in the same column layout as D = 128; the
// two halves of a key tile are two units (S^T and dP^T are formed twice: 1.4x
// the MMA work of one pass).  K and V (64 KiB each) stay in shared memory, so
// one 64 KiB Q/dO stage is all that fits.
constexpr int QM = 64;  // query rows per step
// 16 warps: warpgroup 0 = TMA lane (warp 0) and MMA lane (warp 1); warpgroups 1
// and 3 = the dS work of query columns [0, 32) and [32, 64) of each step (two
// warps per SM sub-partition hide each other's latencies); warpgroup 2 = dQ^T
// read-out and the dK/dV epilogue.
constexpr int BWD2_THREADS = 512;
constexpr uint32_t UNIT_READERS_BWD2 = 1 + 3 * TILE;
// Register split (launch: 128 per thread): control 64, dS 176 each, output 96;
// per SM sub-partition one warp of each warpgroup: 64 + 176 + 96 + 176 = 512.
// D = 256 moves 8 registers from each dS warp to the output warp (its dQ and
// dK/dV addresses depend on the unit's half of the head dimension).
template <int D>
struct Reg2 {
    static constexpr int CTRL = 64;
    static constexpr int DS = (D == 128) ? 176 : 168;
    static constexpr int OUT = (D == 128) ? 96 : 112;
    static_assert(CTRL + 2 * DS + OUT <= 4 * 128, "register split exceeds the launch budget");
};

template <int D>
struct Bwd2Smem {
    static constexpr int CHUNKS = D / 64;            // 64-column chunks of a row
    static constexpr int HALVES = D / 128;           // passes over the head dimension per key tile
    static constexpr int KCHUNK = TILE * 128;        // K/V: [128 rows][64 cols] per chunk
    static constexpr int QCHUNK = QM * 128;          // Q/dO: [64 rows][64 cols] per chunk
    static constexpr int KV_TILE = TILE * D * 2;     // 32 KiB (D = 128), 64 KiB (D = 256)
    static constexpr int Q_TILE = QM * D * 2;        // 16 KiB, 32 KiB
    static constexpr int NSTAGE = (D == 128) ? 3 : 1;
    static constexpr int K_OFF = 0;
    static constexpr int V_OFF = KV_TILE;
    static constexpr int STAGE_OFF = 2 * KV_TILE;    // stage: Q_m, dO_m
    static constexpr int STAGE_BYTES = 2 * Q_TILE;
    static constexpr int DS_OFF = STAGE_OFF + NSTAGE * STAGE_BYTES;  // dS^T [2][128 keys][64 queries]
    static constexpr int DS_BYTES = TILE * QM * 2;                 // 16 KiB
    static constexpr int STATS_OFF = DS_OFF + 2 * DS_BYTES;          // per stage: lse2[64], delta[64]
    static constexpr int STATS_BYTES = 2 * QM * 4;
    // D = 128, atomic mode: a step's dQ (64 queries x 128 fp32, row-major) staged
    // for one bulk reduce-add by the TMA engine; it does not fit beside D = 256's
    // K and V, which keep per-element atomics
    static constexpr bool DQ_BULK = (D == 128);
    static constexpr int DQS_OFF = STATS_OFF + NSTAGE * STATS_BYTES;  // 128-byte aligned
    static constexpr int DQS_BYTES = DQ_BULK ? QM * 128 * 4 : 0;
    static constexpr int BAR_OFF = DQS_OFF + DQS_BYTES;
    enum {
        B_KVFULL = 0,
        B_KVEMPTY,
        B_DKVFULL,
        B_DKVEMPTY,
        B_FIN,
        B_UFULL,                    // [2]
        B_UEMPTY = B_UFULL + 2,     // [2]
        B_SFULL = B_UEMPTY + 2,     // [2] per buffer
        B_PFULL = B_SFULL + 2,      // [2]
        B_DQFULL = B_PFULL + 2,     // [2]
        B_DQEMPTY = B_DQFULL + 2,   // [2]
        B_DSEMPTY = B_DQEMPTY + 2,  // [2]
        B_QFULL = B_DSEMPTY + 2,    // [NSTAGE]
        B_QEMPTY = B_QFULL + NSTAGE,
        B_DQSYNC = B_QEMPTY + NSTAGE,  // the output warpgroup's own barrier (dQ staging)
        NBAR = B_DQSYNC + 1
    };
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    static constexpr int UNIT_OFF = MISC_OFF + 16;
    static constexpr int BYTES = UNIT_OFF + 8;
    static constexpr int ALLOC = BYTES + 1024;
};

constexpr uint32_t COL2_DV = 256;
constexpr uint32_t COL2_DK = 384;
__device__ __forceinline__ uint32_t col2_s(uint32_t b) { return 128u * b; }
__device__ __forceinline__ uint32_t col2_dp(uint32_t b) { return 128u * b + 64u; }

// Units for 64-row steps: m_lo counts steps; with D = 256 the two halves of a
// key tile are consecutive units.
template <int D>
__device__ __forceinline__ BUnit decode_bwd2_unit(const BwdParams& p, int u) {
    BUnit U;
    constexpr int HALVES = Bwd2Smem<D>::HALVES;
    int c = 0;
    if (p.q_split > 1) {
        c = u % p.q_split;
        u /= p.q_split;
    }
    U.half = u % HALVES;
    u /= HALVES;
    if (p.causal) {
        causal_unit_order(p, u, &U.bh, &U.n);
        const int q_first = U.n * TILE - p.causal_off;
        U.m_lo = q_first > 0 ? q_first / QM : 0;
    } else {
        U.bh = u / p.n_ktiles;
        U.n = u - U.bh * p.n_ktiles;
        U.m_lo = 0;
    }
    U.T = p.n_mtiles - U.m_lo;  // n_mtiles counts 64-row steps here
    if (p.q_split > 1) split_query_range(p, c, U);
    return U;
}

template <int D>
struct Bwd2UnitReader {
    int slot = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ int next(uint8_t* smem, volatile uint32_t* abort_flag, int site) {
        using L = Bwd2Smem<D>;
        const uint32_t bar0 = smem_u32(smem) + L::BAR_OFF;
        if (!mbar_wait(bar0 + 8u * (uint32_t)(L::B_UFULL + slot), phase, abort_flag, site)) return -2;
        const int u = reinterpret_cast<volatile int*>(smem + L::UNIT_OFF)[slot];
        mbar_arrive(bar0 + 8u * (uint32_t)(L::B_UEMPTY + slot));
        if (++slot == 2) { slot = 0; phase ^= 1u; }
        return u;
    }
};

// DH < D (the D = 128 kernel on D = 64 tensors): only the first DH / 64
// column chunks of K, V, Q and dO are loaded.  The scores reduce over those
// chunks only; the products that read the other chunks (dQ^T's rows, dK's and
// dV's columns past DH) are never written out, so those chunks may hold any
// data.
template <int D, int DH>
__device__ void bwd2_producer(const BwdParams& p, uint8_t* smem, volatile uint32_t* abort_flag) {
    using L = Bwd2Smem<D>;
    constexpr int CH = (DH < D) ? DH / 64 : L::CHUNKS;  // column chunks loaded
    const uint32_t base = smem_u32(smem);
    const uint32_t bar0 = base + L::BAR_OFF;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    volatile int* ring = reinterpret_cast<volatile int*>(smem + L::UNIT_OFF);
    int uslot = 0;
    uint32_t uphase = 0;
    bool ok = true;
    int kv_fill = -1;
    uint32_t fill_mask = 0, fill_parity = 0;
    uint32_t g = 0;  // global step count
    int nunit = 0;
    for (int k = 0;; ++k) {
        int u = p.sched ? (int)atomicAdd(p.sched, 1u) : (int)blockIdx.x + k * (int)gridDim.x;
        if (u >= p.n_units) u = -1;
        if (!mbar_wait(bar(L::B_UEMPTY + uslot), uphase ^ 1u, abort_flag, 60)) { ok = false; break; }
        ring[uslot] = u;
        mbar_arrive(bar(L::B_UFULL + uslot));
        if (++uslot == 2) { uslot = 0; uphase ^= 1u; }
        if (u < 0) break;
        const BUnit U = decode_bwd2_unit<D>(p, u);
        const int b = U.bh / p.H, h = U.bh - b * p.H;
        const uint32_t kvp = (uint32_t)nunit & 1u;
        if (!mbar_wait(bar(L::B_KVEMPTY), kvp ^ 1u, abort_flag, 61)) { ok = false; break; }
        mbar_expect_tx(bar(L::B_KVFULL), 2 * CH * L::KCHUNK);
        kv_fill = (int)kvp;
        ++nunit;
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            tma_load_4d(base + L::K_OFF + c * L::KCHUNK, &p.tmap_k, bar(L::B_KVFULL), c * 64, U.n * TILE, h, b);
            tma_load_4d(base + L::V_OFF + c * L::KCHUNK, &p.tmap_v, bar(L::B_KVFULL), c * 64, U.n * TILE, h, b);
        }
        for (int t = 0; t < U.T; ++t, ++g) {
            const int m = U.m_lo + t;
            const int st = (int)(g % L::NSTAGE);
            const uint32_t sp = (g / L::NSTAGE) & 1u;
            if (!mbar_wait(bar(L::B_QEMPTY + st), sp ^ 1u, abort_flag, 62)) { ok = false; break; }
            mbar_expect_tx(bar(L::B_QFULL + st), 2 * CH * L::QCHUNK + L::STATS_BYTES);
            fill_mask |= 1u << st;
            fill_parity = (fill_parity & ~(1u << st)) | (sp << st);
            const uint32_t dst = base + L::STAGE_OFF + st * L::STAGE_BYTES;
#pragma unroll
            for (int c = 0; c < CH; ++c) {
                tma_load_4d(dst + c * L::QCHUNK, &p.tmap_q, bar(L::B_QFULL + st), c * 64, m * QM, h, b);
                tma_load_4d(dst + L::Q_TILE + c * L::QCHUNK, &p.tmap_do, bar(L::B_QFULL + st), c * 64, m * QM, h, b);
            }
            const size_t srow = (size_t)U.bh * (size_t)p.Sq_pad + (size_t)m * QM;
            const uint32_t sdst = base + L::STATS_OFF + st * L::STATS_BYTES;
            bulk_load(sdst, p.lse2 + srow, QM * 4, bar(L::B_QFULL + st));
            bulk_load(sdst + QM * 4, p.delta + srow, QM * 4, bar(L::B_QFULL + st));
        }
        if (!ok) break;
    }
    if (!ok) {
        for (int i = 0; i < L::NSTAGE; ++i)
            if (fill_mask & (1u << i)) mbar_drain(bar(L::B_QFULL + i), (fill_parity >> i) & 1u);
        if (kv_fill >= 0) mbar_drain(bar(L::B_KVFULL), (uint32_t)kv_fill);
    }
}

template <int D, bool BF16, int DH>
__device__ void bwd2_mma(const BwdParams& p, uint8_t* smem, uint32_t tmem, volatile uint32_t* abort_flag) {
    using L = Bwd2Smem<D>;
    const uint32_t base = smem_u32(smem);
    const uint32_t bar0 = base + L::BAR_OFF;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    constexpr uint32_t IDESC_S = make_idesc_bwd(BF16, QM, false, false);   // S^T, dP^T: N = 64 queries
    constexpr uint32_t IDESC_KV = make_idesc_bwd(BF16, 128, false, true);  // dV, dK: A in TMEM, B MN-major
    constexpr uint32_t IDESC_DQ = make_idesc_bwd(BF16, QM, true, true);    // dQ^T: A = K^T, B = dS^T
    // K-major: K, V ([128 rows][128], chunks 16 KiB apart), Q, dO ([64 rows][128],
    // chunks 8 KiB apart); a K step of 16 elements is +32 bytes in a chunk.
    // MN-major: Q, dO along D (2 chunks 8 KiB apart), K along D (2 chunks 16 KiB
    // apart), dS^T along the queries (one 64-wide chunk); 8-row groups 1 KiB
    // apart and a K step of 16 rows +2 KiB throughout.
    const uint64_t a_k = sw128_desc(base + L::K_OFF, 16, 1024);
    const uint64_t a_v = sw128_desc(base + L::V_OFF, 16, 1024);
    const uint64_t b_stage_k = sw128_desc(base + L::STAGE_OFF, 16, 1024);
    const uint64_t b_stage_mn = sw128_desc(base + L::STAGE_OFF, (uint32_t)L::QCHUNK, 1024);
    const uint64_t a_kt = sw128_desc(base + L::K_OFF, (uint32_t)L::KCHUNK, 1024);
    const uint64_t b_ds = sw128_desc(base + L::DS_OFF, 1024, 1024);
    const uint64_t a_ds = sw128_desc(base + L::DS_OFF, 16, 1024);  // dS^T as a K-major A (K = 64 queries)
    // DH < D (D = 64 tensors): dQ^T is issued before dV and dK, and dK takes
    // dS^T from shared memory, so dQ^T's read-out (which the step after next's
    // dP^T waits for) starts one product pair earlier.  At the full head
    // dimension the extra shared-memory operand of dK costs more than it saves.
    constexpr bool DQ_FIRST = DH < D;
    constexpr uint32_t STAGE16 = (uint32_t)L::STAGE_BYTES >> 4;
    constexpr uint32_t QTILE16 = (uint32_t)L::Q_TILE >> 4;
    constexpr uint32_t DS16 = (uint32_t)L::DS_BYTES >> 4;
    auto lo = [](uint64_t d) { return (uint32_t)d; };
    auto hi = [](uint64_t d) { return (uint32_t)(d >> 32); };

    // S^T or dP^T of one step: A = K or V (128 keys), B = Q or dO (64 queries),
    // K = the tensors' head dimension (the loaded chunks)
    auto issue_sp = [&](uint32_t d_tmem, uint64_t a, uint32_t b_off16) {
#pragma unroll
        for (int ks = 0; ks < (DH < D ? DH : D) / 16; ++ks) {
            const uint32_t in_chunk = (uint32_t)((ks & 3) * 32) >> 4;
            const uint32_t a_off = in_chunk + (uint32_t)(((ks >> 2) * L::KCHUNK) >> 4);
            const uint32_t b_off = in_chunk + (uint32_t)(((ks >> 2) * L::QCHUNK) >> 4);
            tc_mma_ss2(d_tmem, lo(a) + a_off, hi(a), lo(b_stage_k) + b_off16 + b_off, hi(b_stage_k), IDESC_S,
                       ks > 0 ? 1u : 0u);
        }
    };
    // dV or dK += A(tmem, 64 queries packed) B(smem MN-major, 64 rows x 128).  The
    // packed pairs of queries [32c, 32c + 32) sit in columns 32c .. 32c + 15 of
    // the buffer (each dS warpgroup packs into its own columns), so the K step
    // of queries 16 ks .. 16 ks + 15 reads columns 32 (ks / 2) + 8 (ks % 2).
    // (D = 256: B is the unit's 128-wide half of dO or Q, chunks 2 half and 2 half + 1)
    constexpr bool SPLIT = L::HALVES > 1;
    uint32_t half_q16 = 0, half_k16 = 0;
    auto issue_kv = [&](uint32_t d_tmem, uint32_t a_tmem, uint32_t b_off16, bool accumulate) {
#pragma unroll
        for (int ks = 0; ks < QM / 16; ++ks)
            tc_mma_ts2(d_tmem, a_tmem + (uint32_t)((ks >> 1) * 32 + (ks & 1) * 8),
                       lo(b_stage_mn) + (SPLIT ? half_q16 : 0u) + b_off16 + (uint32_t)(ks * (2048 >> 4)), hi(b_stage_mn),
                       IDESC_KV,
                       (accumulate || ks > 0) ? 1u : 0u);
    };
    auto wait_p = [&](uint32_t bar_idx, uint32_t parity, int site) -> bool {
        return mbar_wait(bar(bar_idx), parity, abort_flag, site);
    };

    uint32_t g = 0;
    int nunit = 0;
    bool ok = true;
    Bwd2UnitReader<D> units;
    for (;;) {
        const int u = units.next(smem, abort_flag, 63);
        if (u < 0) break;
        const BUnit U = decode_bwd2_unit<D>(p, u);
        const uint32_t kvp = (uint32_t)nunit & 1u;
        ++nunit;
        if constexpr (SPLIT) {
            half_q16 = (uint32_t)(U.half * 2 * L::QCHUNK) >> 4;
            half_k16 = (uint32_t)(U.half * 2 * L::KCHUNK) >> 4;
        }
        if (!wait_p(L::B_KVFULL, kvp, 64)) { ok = false; break; }
        // step g's S^T and dP^T into buffer g & 1
        auto issue_step = [&](uint32_t gs) -> bool {
            const uint32_t b = gs & 1u;
            const int st = (int)(gs % L::NSTAGE);
            if (!wait_p(L::B_QFULL + st, (gs / L::NSTAGE) & 1u, 65)) return false;
            const uint32_t q16 = (uint32_t)st * STAGE16;
            issue_sp(tmem + col2_s(b), a_k, q16);
            // the buffer's previous dQ^T (step gs - 2, in its dP columns) has been read out
            if (!wait_p(L::B_DQEMPTY + b, ((gs >> 1) & 1u) ^ 1u, 66)) return false;
            tc_fence_after();
            issue_sp(tmem + col2_dp(b), a_v, q16 + QTILE16);
            tc_commit(bar(L::B_SFULL + b));
            return true;
        };
        if (!issue_step(g)) { ok = false; break; }
        for (int t = 0; t < U.T; ++t, ++g) {
            const uint32_t b = g & 1u;
            const int st = (int)(g % L::NSTAGE);
            // the next step's scores run while this step's dS is formed; with a single
            // Q/dO stage (D = 256) the next step's Q and dO can only load once this
            // step's dK and dV products have released the stage, so they come later
            if (L::NSTAGE > 1 && t + 1 < U.T && !issue_step(g + 1)) { ok = false; break; }
            if (!wait_p(L::B_PFULL + b, (g >> 1) & 1u, 67)) { ok = false; break; }
            tc_fence_after();
            if (t == 0) {
                if (!wait_p(L::B_DKVEMPTY, kvp ^ 1u, 68)) { ok = false; break; }
                tc_fence_after();
            }
            const uint32_t q16 = (uint32_t)st * STAGE16;
            // dQ^T = K^T dS^T into this step's dP columns
            auto issue_dq = [&]() {
#pragma unroll
                for (int ks = 0; ks < TILE / 16; ++ks) {
                    const uint32_t off = (uint32_t)(ks * (2048 >> 4));
                    tc_mma_ss2(tmem + col2_dp(b), lo(a_kt) + (SPLIT ? half_k16 : 0u) + off, hi(a_kt),
                               lo(b_ds) + b * DS16 + off, hi(b_ds), IDESC_DQ, ks > 0 ? 1u : 0u);
                }
                tc_commit(bar(L::B_DQFULL + b));
            };
            if constexpr (DQ_FIRST) {
                issue_dq();
                issue_kv(tmem + COL2_DV, tmem + col2_s(b), q16 + QTILE16, t > 0);  // dV += P^T dO_m
                // dK += dS^T Q_m, A = dS^T from shared memory (16 queries = 32 bytes per K step)
#pragma unroll
                for (int ks = 0; ks < QM / 16; ++ks)
                    tc_mma_ss2(tmem + COL2_DK, lo(a_ds) + b * DS16 + (uint32_t)((ks * 32) >> 4), hi(a_ds),
                               lo(b_stage_mn) + (SPLIT ? half_q16 : 0u) + q16 + (uint32_t)(ks * (2048 >> 4)),
                               hi(b_stage_mn), IDESC_KV, (t > 0 || ks > 0) ? 1u : 0u);
                tc_commit(bar(L::B_QEMPTY + st));
            } else {
                issue_kv(tmem + COL2_DV, tmem + col2_s(b), q16 + QTILE16, t > 0);  // dV += P^T dO_m
                issue_kv(tmem + COL2_DK, tmem + col2_dp(b), q16, t > 0);          // dK += dS^T Q_m
                tc_commit(bar(L::B_QEMPTY + st));
                issue_dq();
            }
            tc_commit(bar(L::B_DSEMPTY + b));
            if (L::NSTAGE == 1 && t + 1 < U.T && !issue_step(g + 1)) { ok = false; break; }
        }
        if (!ok) break;
        tc_commit(bar(L::B_DKVFULL));
        tc_commit(bar(L::B_KVEMPTY));
    }
    (void)ok;
    tc_commit(bar(L::B_FIN));
    mbar_drain(bar(L::B_FIN), 0u);
}

// DH < D: dK reads dS^T from shared memory, so it is not stored to TMEM.
template <int D, bool BF16, bool MASK, bool DROP, int DH>
__device__ void bwd2_ds_role(const BwdParams& p, uint8_t* smem, uint32_t tmem, int warp_in_group, int c,
                             volatile uint32_t* abort_flag) {
    using L = Bwd2Smem<D>;
    const uint32_t base = smem_u32(smem);
    const uint32_t bar0 = base + L::BAR_OFF;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    const int lane = threadIdx.x & 31;
    const int row = warp_in_group * 32 + lane;  // key row
    const uint32_t lane_sel = (uint32_t)(warp_in_group * 32) << 16;
    const float sl2 = p.scale_log2;
    const int sw = row & 7;
    uint32_t g = 0;
    Bwd2UnitReader<D> units;
    for (;;) {
        const int u = units.next(smem, abort_flag, 69);
        if (!__all_sync(0xffffffffu, u != -2)) return;
        if (u < 0) break;
        const BUnit U = decode_bwd2_unit<D>(p, u);
        const int key = U.n * TILE + row;
        const bool key_ok = key < p.Sk;
        const int q_min = p.causal ? key - p.causal_off : 0;
        const uint8_t* mhead =
            MASK ? p.mask + (long long)(U.bh / p.H) * p.m_sb + (long long)(U.bh % p.H) * p.m_sh : nullptr;
        for (int t = 0; t < U.T; ++t, ++g) {
            const int m = U.m_lo + t;
            const uint32_t b = g & 1u;
            const int st = (int)(g % L::NSTAGE);
            // the stage's statistics and the free dS^T buffer are normally ready long
            // before the scores: take those waits first
            if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_QFULL + st), (g / L::NSTAGE) & 1u, abort_flag, 71)))
                return;
            if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_DSEMPTY + b), ((g >> 1) & 1u) ^ 1u, abort_flag, 72)))
                return;
            if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_SFULL + b), (g >> 1) & 1u, abort_flag, 70))) return;
            tc_fence_after();
            const float* lse2s = reinterpret_cast<const float*>(smem + L::STATS_OFF + st * L::STATS_BYTES);
            const float* dls = lse2s + QM;
            const bool need_mask = !key_ok || (m * QM + 32 * c < q_min) || MASK;
            // explicit mask: this key's bits over the 32 queries of this warpgroup
            uint32_t mbits = 0xffffffffu;
            if constexpr (MASK)
                mbits = mask_col_bits(mhead, p.m_ss, p.Sq, p.Sk, m * QM + 32 * c, U.n * TILE + warp_in_group * 32);
            // dropout: this key's keep bits over the same 32 queries
            uint32_t zbits = 0xffffffffu;
            if constexpr (DROP) zbits = dropout_col_bits(p, U.bh, m * QM + 32 * c, U.n * TILE + warp_in_group * 32);
            uint8_t* ds_row = smem + L::DS_OFF + b * L::DS_BYTES + (row >> 3) * 1024 + (row & 7) * 128;
            {
                uint32_t sr[32], dr[32];
                tmem_ld32u(tmem + lane_sel + col2_s(b) + 32 * c, sr);
                tmem_ld32u(tmem + lane_sel + col2_dp(b) + 32 * c, dr);
                uint32_t pk[16], dk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int j = 32 * c + 2 * i;
                    const float2 l2 = *reinterpret_cast<const float2*>(lse2s + j);
                    const float2 dl = *reinterpret_cast<const float2*>(dls + j);
                    float p0 = ex2(fmaf(__uint_as_float(sr[2 * i]), sl2, -l2.x));
                    float p1 = ex2(fmaf(__uint_as_float(sr[2 * i + 1]), sl2, -l2.y));
                    if (need_mask) {
                        const int q = m * QM + j;
                        if (!key_ok || q < q_min || !((mbits >> (2 * i)) & 1u)) p0 = 0.f;
                        if (!key_ok || q + 1 < q_min || !((mbits >> (2 * i + 1)) & 1u)) p1 = 0.f;
                    }
                    // dropout factors: 1 / (1 - p) for a kept weight, 0 for a dropped one
                    float z0 = 1.f, z1 = 1.f;
                    if constexpr (DROP) {
                        z0 = ((zbits >> (2 * i)) & 1u) ? p.keep_scale : 0.f;
                        z1 = ((zbits >> (2 * i + 1)) & 1u) ? p.keep_scale : 0.f;
                    }
                    pk[i] = pack2<BF16>(p0 * z0, p1 * z1);
                    dk[i] = pack2<BF16>(p0 * (__uint_as_float(dr[2 * i]) * z0 - dl.x),
                                        p1 * (__uint_as_float(dr[2 * i + 1]) * z1 - dl.y));
                }
                // packed into the first 16 of this warpgroup's own 32 columns: the other
                // dS warpgroup may still be reading its raw scores from the rest
                tmem_st16(tmem + lane_sel + col2_s(b) + 32 * c, pk);
                if constexpr (!(DH < D)) tmem_st16(tmem + lane_sel + col2_dp(b) + 32 * c, dk);
#pragma unroll
                for (int gi = 0; gi < 4; ++gi) {
                    const int gr = (c * 4 + gi) ^ sw;
                    *reinterpret_cast<uint4*>(ds_row + gr * 16) =
                        make_uint4(dk[4 * gi], dk[4 * gi + 1], dk[4 * gi + 2], dk[4 * gi + 3]);
                }
            }
            tmem_wait_st();
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(bar(L::B_PFULL + b));
        }
    }
}

// SPLIT: the unit's dK, dV are partial sums over a split query range, added in
// fp32 (a separate instantiation: the branch alone costs the role registers)
template <int D, bool BF16, bool SPLIT, int DH>
__device__ void bwd2_out_role(const BwdParams& p, uint8_t* smem, uint32_t tmem, int warp_in_group,
                              volatile uint32_t* abort_flag) {
    using L = Bwd2Smem<D>;
    const uint32_t base = smem_u32(smem);
    const uint32_t bar0 = base + L::BAR_OFF;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    const int lane = threadIdx.x & 31;
    const int row = warp_in_group * 32 + lane;  // head-dimension index for dQ^T, key row for dK/dV
    const uint32_t lane_sel = (uint32_t)(warp_in_group * 32) << 16;
    // barrier of the 128 output threads around the dQ staging (bounded waits)
    uint32_t sync_phase = 0;
    auto group_sync = [&](int site) -> bool {
        mbar_arrive(bar(L::B_DQSYNC));
        const bool ok = mbar_wait(bar(L::B_DQSYNC), sync_phase, abort_flag, site);
        sync_phase ^= 1u;
        return ok;
    };
    uint32_t g = 0;
    int nunit = 0;
    Bwd2UnitReader<D> units;
    for (;;) {
        const int u = units.next(smem, abort_flag, 73);
        if (!__all_sync(0xffffffffu, u != -2)) return;
        if (u < 0) break;
        const BUnit U = decode_bwd2_unit<D>(p, u);
        const int half = (L::HALVES > 1) ? U.half : 0;  // a constant 0 with one pass
        const uint32_t kvp = (uint32_t)nunit & 1u;
        ++nunit;
        for (int t = 0; t < U.T; ++t, ++g) {
            const int m = U.m_lo + t;
            const uint32_t b = g & 1u;
            if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_DQFULL + b), (g >> 1) & 1u, abort_flag, 74))) return;
            tc_fence_after();
            // dQ[q][d] += dQ^T[d][q]: consecutive threads take consecutive d (coalesced)
            constexpr int dh = DH;
            const bool d_ok = DH >= 128 || row < DH;  // lanes past a 64-wide head dimension hold zeros
            float* dst = p.dq_acc + ((size_t)U.bh * (size_t)p.Sq + (size_t)m * QM) * dh + (size_t)half * 128 + row;
            const int nq = min(QM, p.Sq - m * QM);
            if constexpr (SPLIT && L::DQ_BULK) {
                // one key tile per head: copy dQ^T out of TMEM as dQ[q][d] into the
                // staging tile (once every thread has read the previous step's),
                // free the columns, then write the rows scaled and rounded to dQ,
                // four values per thread and access (rows past Sq skipped)
                if (!__all_sync(0xffffffffu, group_sync(76))) return;
                constexpr int sstride = dh < 128 ? dh : 128;
                float* stg = reinterpret_cast<float*>(smem + L::DQS_OFF) + row;
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t r[32];
                    tmem_ld32u(tmem + lane_sel + col2_dp(b) + 32 * hh, r);
                    if (d_ok) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) stg[(32 * hh + j) * sstride] = __uint_as_float(r[j]);
                    }
                }
                tc_fence_before();
                mbar_arrive(bar(L::B_DQEMPTY + b));
                if (!__all_sync(0xffffffffu, group_sync(77))) return;
                // thread `row` takes chunk j = row mod CPR of rows row / CPR + k * QSTEP
                constexpr int CPR = sstride / 4;  // 4-value chunks per staged row
                constexpr int QSTEP = 128 / CPR;
                const int j = row % CPR;
                const int ub = U.bh / p.H, uh = U.bh - ub * p.H;
                const long long rs = p.dq_s[2];
                uint8_t* dp = p.dq + ub * p.dq_s[0] + uh * p.dq_s[1] + ((long long)m * QM + row / CPR) * rs +
                              half * 256 + j * 8;
                const float4* sp = reinterpret_cast<const float4*>(smem + L::DQS_OFF) + row;
#pragma unroll 1
                for (int q = row / CPR; q < nq; q += QSTEP, dp += QSTEP * rs, sp += 128) {
                    const float4 v = *sp;
                    *reinterpret_cast<uint2*>(dp) = make_uint2(pack2<BF16>(v.x * p.scale, v.y * p.scale),
                                                               pack2<BF16>(v.z * p.scale, v.w * p.scale));
                }
            } else if (!p.dq_flags && L::DQ_BULK) {
                // once the previous step's reduce has read the staging, copy dQ^T
                // out of TMEM as dQ[q][d] (each lane holds one d over the 64
                // queries: a warp writes 32 consecutive floats per query), free
                // the columns, and let one thread hand the box to the TMA engine as
                // a bulk reduce-add (rows past Sq are clipped)
                const bool issuer = threadIdx.x == 2 * 128;  // first thread of the output warpgroup
                if (issuer) bulk_wait_read();
                if (!__all_sync(0xffffffffu, group_sync(76))) return;
                // staging rows of min(dh, 128) values: the box of the dQ accumulator's map
                constexpr int sstride = dh < 128 ? dh : 128;
                float* stg = reinterpret_cast<float*>(smem + L::DQS_OFF) + row;
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t r[32];
                    tmem_ld32u(tmem + lane_sel + col2_dp(b) + 32 * hh, r);
                    if (d_ok) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) stg[(32 * hh + j) * sstride] = __uint_as_float(r[j]);
                    }
                }
                tc_fence_before();
                mbar_arrive(bar(L::B_DQEMPTY + b));
                fence_async_smem();
                if (!__all_sync(0xffffffffu, group_sync(77))) return;
                if (issuer) tma_reduce_add_3d(&p.tmap_dq, base + L::DQS_OFF, half * 128, m * QM, U.bh);
            } else if (!p.dq_flags) {
                // read the whole step, free the columns, then add with atomics
                uint32_t r0[32], r1[32];
                tmem_ld32u(tmem + lane_sel + col2_dp(b), r0);
                tmem_ld32u(tmem + lane_sel + col2_dp(b) + 32, r1);
                tc_fence_before();
                mbar_arrive(bar(L::B_DQEMPTY + b));
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (d_ok && j < nq) atomicAdd(dst + (size_t)j * dh, __uint_as_float(r0[j]));
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (d_ok && 32 + j < nq) atomicAdd(dst + (size_t)(32 + j) * dh, __uint_as_float(r1[j]));
            } else {
                // this key tile's turn for the step, then 32 queries at a time:
                // read-modify-write in batches of 16 (loads in flight together)
                int* flag = p.dq_flags + (((size_t)U.bh * p.flag_steps + m) * L::HALVES + half) * 4 + warp_in_group;
                if (!wait_turn(flag, U.n, abort_flag, 57)) return;
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t r[32];
                    tmem_ld32u(tmem + lane_sel + col2_dp(b) + 32 * hh, r);
                    if (hh == 1) {
                        tc_fence_before();
                        mbar_arrive(bar(L::B_DQEMPTY + b));
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float v[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int jq = 32 * hh + 16 * h + j;
                            v[j] = (d_ok && jq < nq) ? __ldcg(dst + (size_t)jq * dh) : 0.f;
                        }
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int jq = 32 * hh + 16 * h + j;
                            if (d_ok && jq < nq) __stcg(dst + (size_t)jq * dh, v[j] + __uint_as_float(r[16 * h + j]));
                        }
                    }
                }
                pass_turn(flag, U.n + 1);
            }
        }
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_DKVFULL), kvp, abort_flag, 75))) return;
        tc_fence_after();
        const int key = U.n * TILE + row;
        const bool valid = key < p.Sk;
        const int ub = U.bh / p.H, uh = U.bh - ub * p.H;
        const long long kr = valid ? key : 0;
        // this unit's 128 columns of the dK and dV rows (its half of D at D = 256)
        uint8_t* dv_row = p.dv + ub * p.dv_s[0] + uh * p.dv_s[1] + kr * p.dv_s[2] + half * 256;
        uint8_t* dk_row = p.dk + ub * p.dk_s[0] + uh * p.dk_s[1] + kr * p.dk_s[2] + half * 256;
        constexpr int ncol = DH < 128 ? DH : 128;  // this unit's columns of the rows
        if constexpr (SPLIT) {
            // this unit's share of the key row's sums (its half of D), added in fp32
            const size_t acc_row = ((size_t)U.bh * KV_ACC_ROWS + (size_t)kr) * DH + (size_t)half * 128;
            kv_partial_add(tmem + lane_sel + COL2_DV, tmem + lane_sel + COL2_DK, p.dv_acc + acc_row,
                           p.dk_acc + acc_row, p.scale, valid, ncol);
        } else {
#pragma unroll 1
            for (int c = 0; c < ncol / 32; ++c) {
                uint32_t r[32];
                uint32_t w[16];
                tmem_ld32u(tmem + lane_sel + COL2_DV + 32 * c, r);
#pragma unroll
                for (int i = 0; i < 16; ++i) w[i] = pack2<BF16>(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                if (valid) {
                    uint4* d = reinterpret_cast<uint4*>(dv_row + c * 64);
#pragma unroll
                    for (int i = 0; i < 4; ++i) d[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                }
                tmem_ld32u(tmem + lane_sel + COL2_DK + 32 * c, r);
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[i] = pack2<BF16>(__uint_as_float(r[2 * i]) * p.scale, __uint_as_float(r[2 * i + 1]) * p.scale);
                if (valid) {
                    uint4* d = reinterpret_cast<uint4*>(dk_row + c * 64);
#pragma unroll
                    for (int i = 0; i < 4; ++i) d[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                }
            }
        }
        tc_fence_before();
        mbar_arrive(bar(L::B_DKVEMPTY));
    }
}

// DH: the tensors' head dimension (64: this D = 128 kernel on its first column chunk)
template <int D, bool BF16, bool MASK, bool DROP, bool SPLIT = false, int DH = D>
__global__ void __launch_bounds__(BWD2_THREADS, 1) fa_bwd_kernel_wide(const __grid_constant__ BwdParams p) {
    using L = Bwd2Smem<D>;
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
            uint32_t count = 1;
            if ((i >= L::B_DQEMPTY && i < L::B_DQEMPTY + 2) || i == L::B_DKVEMPTY || i == L::B_DQSYNC)
                count = TILE;  // one warpgroup
            if (i >= L::B_PFULL && i < L::B_PFULL + 2) count = 2 * TILE;  // both dS warpgroups
            if (i >= L::B_UEMPTY && i < L::B_UEMPTY + 2) count = UNIT_READERS_BWD2;
            mbar_init(base + L::BAR_OFF + 8 * i, count);
        }
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == BW_TMA && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmap_q)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmap_k)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmap_v)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmap_do)) : "memory");
    }
    if (warp == BW_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(misc)),
                     "r"(BWD_TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    grid_dependency_sync();  // the previous kernel in the stream has completed
    if (wg == 0) {
        setmaxnreg_dec<Reg2<D>::CTRL>();
        if (warp == BW_TMA && lane == 0) bwd2_producer<D, DH>(p, smem, abort_flag);
        if (warp == BW_MMA && lane == 0) bwd2_mma<D, BF16, DH>(p, smem, tmem, abort_flag);
    } else if (wg == 1 || wg == 3) {
        setmaxnreg_inc<Reg2<D>::DS>();
        bwd2_ds_role<D, BF16, MASK, DROP, DH>(p, smem, tmem, warp & 3, wg == 1 ? 0 : 1, abort_flag);
    } else {
        setmaxnreg_dec<Reg2<D>::OUT>();
        bwd2_out_role<D, BF16, SPLIT, DH>(p, smem, tmem, warp & 3, abort_flag);
        // the bulk dQ reductions this thread issued finish before the CTA exits
        if (threadIdx.x == 2 * 128) bulk_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == BW_MMA) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(BWD_TMEM_COLS)
                     : "memory");
    }
}


// Per (bh, query row) of the padded row range: Delta = sum_d dO O in fp32,
// LSE * log2(e), and the row of the dQ accumulator cleared (unless dq_acc is
// null: the split mode writes dQ directly).  A row is taken by D / 8 lanes,
// each with one 16-byte load of O and of dO (several rows per warp when
// D < 256: more loads in flight per warp).  Padded rows get +inf (weight 0)
// and Delta = 0.  Block (0, 0) also clears the scheduler counter, which the
// main kernel (next on the stream) reads, and all blocks together clear
// kv_n4 float4s at kv_zero (the split mode's dK/dV partial sums), if given.
template <int D>
struct PrepShape {
    static constexpr int LANES = D / 8;                      // lanes per row
    static constexpr int ROWS_PER_WARP = 32 / LANES;
    static constexpr int ROWS_PER_BLOCK = 8 * ROWS_PER_WARP;  // 256 threads
};

__device__ __forceinline__ float dot8(uint4 a, uint4 b, bool bf16) {
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 fa, fb;
        if (bf16) {
            fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wa[i]));
            fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wb[i]));
        } else {
            fa = __half22float2(*reinterpret_cast<const __half2*>(&wa[i]));
            fb = __half22float2(*reinterpret_cast<const __half2*>(&wb[i]));
        }
        acc = fmaf(fa.x, fb.x, acc);
        acc = fmaf(fa.y, fb.y, acc);
    }
    return acc;
}

template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout,
                                                       const float* __restrict__ lse, float* __restrict__ lse2,
                                                       float* __restrict__ delta, float* __restrict__ dq_acc, int Sq,
                                                       int Sq_pad, unsigned int* sched, int H, Strides3 os,
                                                       Strides3 dos, float4* __restrict__ kv_zero, size_t kv_n4,
                                                       int* __restrict__ flags_zero, size_t n_flags) {
    grid_dependency_sync();
    // buffers cleared here rather than by a memset between the kernels, spread
    // over all blocks: the split mode's fp32 dK/dV partial sums, and the
    // deterministic mode's turn counters
    const size_t blk = (size_t)blockIdx.y * gridDim.x + blockIdx.x, nthr = (size_t)gridDim.x * gridDim.y * 256;
    if (kv_zero)
        for (size_t i = blk * 256 + threadIdx.x; i < kv_n4; i += nthr) kv_zero[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (flags_zero)
        for (size_t i = blk * 256 + threadIdx.x; i < n_flags; i += nthr) flags_zero[i] = 0;
    using PS = PrepShape<D>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / PS::LANES, part = lane - sub * PS::LANES;  // row within the warp, 8-element part
    const int row = blockIdx.x * PS::ROWS_PER_BLOCK + warp * PS::ROWS_PER_WARP + sub;
    const size_t bh = blockIdx.y;
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0 && sched) *sched = 0u;
    float acc = 0.f;
    const bool real = row < Sq;
    if (real) {
        const long long ub = (long long)(bh / H), uh = (long long)(bh % H);
        const long long eo = ub * os.s[0] + uh * os.s[1] + row * os.s[2] + part * 8;
        const long long ed = ub * dos.s[0] + uh * dos.s[1] + row * dos.s[2] + part * 8;
        const uint4 ov = *reinterpret_cast<const uint4*>(o + eo);
        const uint4 dv = *reinterpret_cast<const uint4*>(dout + ed);
        acc = dot8(ov, dv, BF16);
        if (dq_acc) {  // null when the main kernel writes dQ directly
            float4* z = reinterpret_cast<float4*>(dq_acc + (bh * (size_t)Sq + (size_t)row) * D + (size_t)part * 8);
            z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
            z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    // sum over the row's lanes (aligned groups of LANES lanes)
#pragma unroll
    for (int s = PS::LANES / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if (part == 0 && row < Sq_pad) {
        if (real) {
            // a row that saw no key (LSE = -inf) gets +inf, i.e. weights 0
            const float lv = lse[bh * (size_t)Sq + row];
            lse2[bh * Sq_pad + row] = (lv == -INFINITY) ? __int_as_float(0x7f800000) : lv * 1.4426950408889634f;
            delta[bh * Sq_pad + row] = acc;
        } else {
            lse2[bh * Sq_pad + row] = __int_as_float(0x7f800000);  // +inf
            delta[bh * Sq_pad + row] = 0.f;
        }
    }
}

// dQ = scale * accumulator, rounded to the 16-bit dtype (4 elements per
// thread), written at dQ's element strides over b, h and the query row.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_post_kernel(const float4* __restrict__ acc, uint16_t* __restrict__ dq,
                                                       size_t n4, float scale, int H, int Sq, Strides3 qs) {
    grid_dependency_sync();
    constexpr int G = D / 4;  // 4-element groups per row
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
        const float4 a = acc[i];
        const size_t rowi = i / G;  // (bh, query row), rows of the contiguous accumulator
        const int d = (int)(i - rowi * G) * 4;
        const long long bh = (long long)(rowi / (size_t)Sq), row = (long long)(rowi - (size_t)bh * Sq);
        const long long e = (bh / H) * qs.s[0] + (bh % H) * qs.s[1] + row * qs.s[2] + d;
        *reinterpret_cast<uint2*>(dq + e) =
            make_uint2(pack2<BF16>(a.x * scale, a.y * scale), pack2<BF16>(a.z * scale, a.w * scale));
    }
}

// Split query range: dK, dV = the fp32 partial sums (dK already scaled),
// rounded to the 16-bit dtype, written at their element strides over b, h and
// the key row (4 elements per thread).
template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_post_kv_kernel(const float4* __restrict__ dk_acc,
                                                          const float4* __restrict__ dv_acc, uint16_t* __restrict__ dk,
                                                          uint16_t* __restrict__ dv, size_t n4, int H, int Sk,
                                                          Strides3 ks, Strides3 vs) {
    grid_dependency_sync();
    constexpr int G = D / 4;  // 4-element groups per row
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
        const size_t rowi = i / G;  // (bh, key)
        const int d = (int)(i - rowi * G) * 4;
        const long long bh = (long long)(rowi / (size_t)Sk), key = (long long)(rowi - (size_t)bh * Sk);
        const size_t src = ((size_t)bh * KV_ACC_ROWS + (size_t)key) * G + (size_t)(d / 4);
        const float4 a = dk_acc[src], b = dv_acc[src];
        const long long ub = bh / H, uh = bh % H;
        *reinterpret_cast<uint2*>(dk + ub * ks.s[0] + uh * ks.s[1] + key * ks.s[2] + d) =
            make_uint2(pack2<BF16>(a.x, a.y), pack2<BF16>(a.z, a.w));
        *reinterpret_cast<uint2*>(dv + ub * vs.s[0] + uh * vs.s[1] + key * vs.s[2] + d) =
            make_uint2(pack2<BF16>(b.x, b.y), pack2<BF16>(b.z, b.w));
    }
}

template <int D, bool BF16>
cudaError_t launch_bwd_impl(const BwdLaunchArgs& a, cudaStream_t stream) {
    static_assert(Bwd2Smem<128>::ALLOC <= 232448, "shared memory budget exceeded");
    static_assert(Bwd2Smem<256>::ALLOC <= 232448, "shared memory budget exceeded");
    const int BH = a.B * a.H;
    const int n_mtiles = (a.Sq + TILE - 1) / TILE;
    const int Sq_pad = n_mtiles * TILE;
    constexpr int DW = D >= 128 ? D : 128;
    // Split query range: a key set of at most KV_ACC_ROWS keys (one key tile)
    // whose units leave SMs idle takes chunks of q_chunk steps per unit, about
    // two units per SM; not in deterministic mode (the fp32 adds of the
    // partial sums come in any order), nor with an explicit mask or dropout
    // (the split instantiation has neither)
    const int n_steps = (a.Sq + QM - 1) / QM;  // 64-row steps
    const int n_units1 = BH * ((a.Sk + TILE - 1) / TILE) * Bwd2Smem<DW>::HALVES;
    int q_chunk = n_steps, q_split = 1;
    if (!a.mask && !a.drop.enabled && a.dk_acc && a.dv_acc && !a.dq_flags && a.Sk <= KV_ACC_ROWS && a.sms > 0 &&
        n_units1 < a.sms && n_steps > 1) {
        const int want = (2 * a.sms + n_units1 - 1) / n_units1;  // chunks per key tile
        q_chunk = (n_steps + want - 1) / want;
        q_split = (n_steps + q_chunk - 1) / q_chunk;  // no chunk is empty
        if (q_split == 1) q_chunk = n_steps;
    }
    const bool split = q_split > 1;
    // the split D = 64/128 kernel writes dQ itself (through its dQ staging
    // tile): no accumulator to clear and no dQ post kernel
    const bool dq_direct = split && Bwd2Smem<DW>::DQ_BULK;
    {
        dim3 grid((unsigned)((Sq_pad + PrepShape<D>::ROWS_PER_BLOCK - 1) / PrepShape<D>::ROWS_PER_BLOCK),
                  (unsigned)BH, 1);
        // split: the dK/dV partial sums (contiguous) cleared too; deterministic:
        // the turn counters, [BH][64-row steps][passes over D][4 warps]
        cudaError_t e = launch_kernel(
            bwd_prep_kernel<D, BF16>, grid, dim3(256), 0, stream, static_cast<const uint16_t*>(a.o),
            static_cast<const uint16_t*>(a.dout), a.lse, a.lse2, a.delta, dq_direct ? nullptr : a.dq_acc, a.Sq, Sq_pad,
            a.sched, a.H, Strides3{{a.o_stride[0], a.o_stride[1], a.o_stride[2]}},
            Strides3{{a.do_stride[0], a.do_stride[1], a.do_stride[2]}},
            split ? reinterpret_cast<float4*>(a.dk_acc) : nullptr,
            split ? (size_t)2 * BH * KV_ACC_ROWS * D / 4 : (size_t)0, a.dq_flags,
            a.dq_flags ? (size_t)BH * (size_t)n_steps * Bwd2Smem<DW>::HALVES * 4 : (size_t)0);
        if (e != cudaSuccess) return e;
    }
    {
        // every head dimension runs the 64-row-step kernel (its Q/dO maps have
        // 64-row boxes); D = 64 runs its D = 128 instantiation on the first
        // 64-column chunk of every operand (the scores reduce over it alone;
        // what the unused chunk would feed is never written out).  The split mode
        // has its own instantiation (partial sums added; dQ written directly
        // at D = 64/128).
        void (*kern)(const BwdParams) =
            split ? fa_bwd_kernel_wide<DW, BF16, false, false, true, D>
            : a.drop.enabled
                ? (a.mask ? fa_bwd_kernel_wide<DW, BF16, true, true, false, D>
                          : fa_bwd_kernel_wide<DW, BF16, false, true, false, D>)
                : (a.mask ? fa_bwd_kernel_wide<DW, BF16, true, false, false, D>
                          : fa_bwd_kernel_wide<DW, BF16, false, false, false, D>);
        const int alloc = Bwd2Smem<DW>::ALLOC;
        cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), alloc);
        if (e != cudaSuccess) return e;
        BwdParams p;
        p.tmap_q = a.tmap_q;
        p.tmap_k = a.tmap_k;
        p.tmap_v = a.tmap_v;
        p.tmap_do = a.tmap_do;
        p.tmap_dq = a.tmap_dq;
        p.lse2 = a.lse2;
        p.delta = a.delta;
        p.dq_acc = a.dq_acc;
        p.dk = static_cast<uint8_t*>(a.dk);
        p.dv = static_cast<uint8_t*>(a.dv);
        p.dq = static_cast<uint8_t*>(a.dq);
        for (int i = 0; i < 3; ++i) {
            p.dk_s[i] = a.dk_stride[i] * 2;
            p.dv_s[i] = a.dv_stride[i] * 2;
            p.dq_s[i] = a.dq_stride[i] * 2;
        }
        p.BH = BH;
        p.H = a.H;
        p.Sq = a.Sq;
        p.Sk = a.Sk;
        p.Sq_pad = Sq_pad;
        p.n_mtiles = n_steps;
        p.n_ktiles = (a.Sk + TILE - 1) / TILE;
        p.n_units = BH * p.n_ktiles * Bwd2Smem<DW>::HALVES;
        p.causal = a.causal;
        p.causal_off = a.Sk - a.Sq;
        p.dh = D;
        {
            // heads whose Q, dO (16-bit) and dQ accumulator (fp32) take <= 48 MiB
            const long long per_head = (long long)a.Sq * D * 8;
            const long long g = (48ll << 20) / (per_head > 0 ? per_head : 1);
            p.head_group = (int)(g < 1 ? 1 : (g > BH ? BH : g));
        }
        p.scale_log2 = a.scale * 1.4426950408889634f;
        p.scale = a.scale;
        // units are claimed from the counter with the mask (they differ in length)
        // and in deterministic mode (the order of dQ additions follows the claims)
        p.sched = (a.causal || a.dq_flags) ? a.sched : nullptr;
        p.dq_flags = a.dq_flags;
        p.mask = a.mask;
        p.m_sb = a.mask_stride[0];
        p.m_sh = a.mask_stride[1];
        p.m_ss = a.mask_stride[2];
        p.drop = a.drop.enabled;
        p.drop_p8x4 = a.drop.p8 * 0x01010101u;
        p.seed_lo = a.drop.seed_lo;
        p.seed_hi = a.drop.seed_hi;
        p.drop_offset = a.drop.offset;
        p.keep_scale = a.drop.enabled ? a.drop.keep_scale : 1.f;
        p.flag_steps = (a.Sq + QM - 1) / QM;
        p.q_split = q_split;
        p.q_chunk = q_chunk;
        p.dk_acc = a.dk_acc;
        p.dv_acc = a.dv_acc;
        p.n_units *= q_split;
        const int grid = split ? (p.n_units < a.sms ? p.n_units : a.sms) : a.grid;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)grid, 1, 1);
        cfg.blockDim = dim3(BWD2_THREADS, 1, 1);
        cfg.dynamicSmemBytes = alloc;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        set_programmatic_launch(cfg, attr);
        e = cudaLaunchKernelEx(&cfg, kern, p);
        if (e != cudaSuccess) return e;
        if (split) {
            const size_t n4 = (size_t)BH * (size_t)a.Sk * D / 4;
            const unsigned blocks = (unsigned)((n4 + 255) / 256 < 148u * 16u ? (n4 + 255) / 256 : 148u * 16u);
            e = launch_kernel(bwd_post_kv_kernel<D, BF16>, dim3(blocks), dim3(256), 0, stream,
                              reinterpret_cast<const float4*>(a.dk_acc), reinterpret_cast<const float4*>(a.dv_acc),
                              static_cast<uint16_t*>(a.dk), static_cast<uint16_t*>(a.dv), n4, a.H, a.Sk,
                              Strides3{{a.dk_stride[0], a.dk_stride[1], a.dk_stride[2]}},
                              Strides3{{a.dv_stride[0], a.dv_stride[1], a.dv_stride[2]}});
            if (e != cudaSuccess || dq_direct) return e;  // dQ was written by the main kernel
        }
    }
    {
        const size_t n4 = (size_t)BH * (size_t)a.Sq * D / 4;
        const unsigned blocks = (unsigned)((n4 + 255) / 256 < 148u * 16u ? (n4 + 255) / 256 : 148u * 16u);
        return launch_kernel(bwd_post_kernel<D, BF16>, dim3(blocks), dim3(256), 0, stream,
                             reinterpret_cast<const float4*>(a.dq_acc), static_cast<uint16_t*>(a.dq), n4, a.scale,
                             a.H, a.Sq, Strides3{{a.dq_stride[0], a.dq_stride[1], a.dq_stride[2]}});
    }
}

}  // namespace

cudaError_t launch_bwd_sm100(const BwdLaunchArgs& a, cudaStream_t stream) {
    if (a.D == 256) {
        return a.dtype == 1 ? launch_bwd_impl<256, true>(a, stream) : launch_bwd_impl<256, false>(a, stream);
    }
    if (a.D == 128) {
        return a.dtype == 1 ? launch_bwd_impl<128, true>(a, stream) : launch_bwd_impl<128, false>(a, stream);
    }
    return a.dtype == 1 ? launch_bwd_impl<64, true>(a, stream) : launch_bwd_impl<64, false>(a, stream);
}

cudaError_t read_and_clear_status_bwd(cudaStream_t stream, int* status, int* site) {
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
