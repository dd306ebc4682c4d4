// fa_fwd_sm100.cu -- fused attention forward for sm_100a (B200).
//
// Computes, per (b, h) and query row i,
//   O_i   = sum_j softmax_j(scale * q_i . k_j) v_j      (j <= i when causal)
//   LSE_i = log sum_j exp(scale * q_i . k_j)
// tile by tile with the online-softmax recurrence (running max m, running
// sum l), so the score matrix never reaches HBM.
//
// Method sources (page title, section):
//  - tiling of Q into row blocks and K/V into column blocks, outer loop over
//    Q tiles and inner loop over K/V tiles: "FlashAttention-2 在昇腾 NPU 上如何
//    做到 3 倍加速？深度拆解 ops-transformer 的实现", section 2.1;
//  - online softmax with running max and running exponential sum, and the
//    e^{m_old - m_new} rescale of the output: same page, section 2.2;
//  - fusion of QK^T, softmax and PV in one kernel with only O written back:
//    same page, sections 2.3 and 3.4;
//  - the matrix unit and the vector unit working on different blocks at the
//    same time (Cube/Vector pipelining): same page, sections 3.4 and 7.1;
//  - causal masking by skipping key tiles above the diagonal inside the
//    kernel (mode 2): the gsyq.cn catlass page, "Causal Mask的实现差异";
//  - double-buffered loads overlapping compute: "ops-transformer
//    FlashAttention 算子实战：让昇腾NPU算力彻底释放", section 5.
// The pages target Ascend Cube/Vector units; this kernel is a B200 design.
// One persistent CTA per SM, 16 warps in four warpgroups:
//
//  * warpgroups 0 and 1 (softmax): one per 128-row query tile of the unit;
//    each thread owns one query row (one TMEM lane). It reads its 128 scores,
//    applies the diagonal/tail mask, updates the running max in the log2
//    domain, hands the rescale factor of its O row to the correction
//    warpgroup, computes the weights with the scale folded into one packed
//    FMA before ex2, writes P as packed 16-bit pairs back over the scores in
//    TMEM, and keeps the row sums.
//  * warpgroup 2 (correction): rescales O rows in TMEM when a row's reference
//    max moved (off the softmax's path), and runs the epilogue: O / l to
//    16 bits, O and LSE stores.
//  * warpgroup 3: warp 12 issues tcgen05.mma from one thread (S_t = Q_t K_j^T
//    into TMEM; O_t += P_t V_j with P_t read from TMEM), warp 13 is the TMA
//    producer (Q tiles once per unit, K_j and V_j through a ring of
//    shared-memory stages with full/empty mbarriers; it also takes the work
//    units, from a counter when causal, and publishes them), warps 14-15 idle.
//    The two query tiles ping-pong: the tensor pipe works on one tile while
//    the other tile's softmax runs.
//  Registers are rebalanced with setmaxnreg: 184 for the softmax
//  warpgroups, 72 for correction, 72 for warpgroup 3.
//
// Every mbarrier wait is bounded: after WAIT_TIMEOUT_CYCLES the waiting thread
// raises the CTA's abort flag and the device status word, every role leaves
// its loop, outstanding TMA copies and MMAs are waited for (bounded), TMEM
// is freed and the kernel returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <map>
#include <mutex>

#include "fa_internal.h"

namespace fa {

__device__ int g_status = 0;       // first error code, 0 if none
__device__ int g_status_site = 0;  // (site) | (block << 8) of the first failing wait

// Scratch of fa_fwd_noalloc, for callers that cannot allocate device memory:
// a fixed 256-byte array in the library's own device memory (every GPU that
// loads the library holds it until the process exits).  Word 0 is the causal
// work-unit counter.  All fa_fwd_noalloc calls share it.
static __device__ __align__(256) unsigned int g_noalloc_scratch[NOALLOC_SCRATCH_WORDS];

// Work-unit counters of the causal launches of the other forward entries: one
// 32-byte slot per (context, stream) that has launched a causal forward, handed
// out by the host layer; part of the module's static data, so no call allocates.
static __device__ __align__(256) unsigned int g_sched_pool[SCHED_POOL_SLOTS * SCHED_SLOT_WORDS];

namespace {

constexpr int NUM_THREADS = 512;   // 16 warps
constexpr int WARP_MMA = 12;
constexpr int WARP_TMA = 13;
constexpr int REG_LAUNCH = 128;    // 65536 registers / 512 threads
constexpr int REG_SOFTMAX = 184;
constexpr int REG_CORR = 72;
constexpr int REG_CTRL = 72;
// setmaxnreg.inc waits until the registers are free: the split must fit the
// launch allocation, and each SM sub-partition (one warp of every warpgroup).
static_assert(2 * 128 * REG_SOFTMAX + 128 * REG_CORR + 128 * REG_CTRL <= NUM_THREADS * REG_LAUNCH,
              "register split exceeds the launch allocation");
static_assert(2 * REG_SOFTMAX + REG_CORR + REG_CTRL <= 512, "register split exceeds a sub-partition");

constexpr uint32_t TMEM_COLS = 512;
// When the softmax moves a row's reference max m (log2 units) to the block max:
//  - always when the block max exceeds m by more than TAU = 8 (weights stay
//    <= 2^8, lazy rescale);
//  - bf16 only: also when the block's largest weight 2^(max - m) exceeds
//    KAPPA * l (l = the row sum so far; KAPPA = RESCALE_KAPPA).  Weights are rounded to bf16 (8-bit
//    precision) before P.V, and the rounding of a row's largest weight
//    2^d (0 < d <= 8) is what dominates the error of O when a few keys carry
//    the row (a sharp softmax).  Moving m makes that weight exactly 1.0; when
//    it is skipped, the weight is at most KAPPA/(1+KAPPA) of the row, so its
//    rounding moves O by at most ~2^-9 * KAPPA * |v|.  Soft rows (large l)
//    thus keep the lazy rescale, sharp rows the exact one.
//  fp16 (11-bit precision) uses the lazy rule only.
constexpr float RESCALE_KAPPA = 0.125f;
template <bool BF16>
struct Policy {
    static constexpr float TAU = 8.0f;
    // bf16: O is normalised by the sum of the rounded weights that the P.V
    // product uses (a second sum, lr), so O is a convex combination of V rows
    // (exact in the one-key limit); the LSE keeps the fp32 sum l, whose
    // rounding-free value the log needs on rows with few keys.
    static constexpr bool NORM_BY_ROUNDED_P = BF16;
};

// TMEM column map: S/P of tile 0 and 1, then O of tile 0 and 1.
constexpr uint32_t COL_S0 = 0;
constexpr uint32_t COL_S1 = 128;
constexpr uint32_t COL_O0 = 256;
constexpr uint32_t COL_O1 = 384;

// Shared-memory layout for head dimension D, key tiles of BN rows, QT query
// tiles of BLOCK_M rows per work unit and NQB_ Q buffers.
template <int D, int BN = BLOCK_N, int QT = Q_TILES_PER_CTA, int NQB_ = 1>
struct Smem {
    static constexpr int CHUNKS = D / 64;                  // 128-byte swizzle atoms along D
    static constexpr int Q_CHUNK_BYTES = BLOCK_M * 128;    // 128 rows x 128 bytes
    static constexpr int KV_CHUNK_BYTES = BN * 128;        // BN rows x 128 bytes
    static constexpr int Q_TILE_BYTES = BLOCK_M * D * 2;   // one Q tile
    static constexpr int KV_TILE_BYTES = BN * D * 2;       // one K or V tile
    // K/V ring: a stage holds V_{s-1} and K_s, the two tiles that are first
    // needed together (O0 += P0 V_{s-1}; S0 = Q0 K_s^T) and last used
    // together (O1 += P1 V_{s-1}; S1 = Q1 K_s^T), so one wait and one release
    // cover both.  A unit streams N + 1 stages (the first without V, the last
    // without K).  The ring holds 128 KiB whatever the tile shape.
    static constexpr int STAGE_BYTES = 2 * KV_TILE_BYTES;
    static constexpr int NSTAGE = (128 * 1024) / STAGE_BYTES;
    static constexpr int STAGE_K = 0;                      // offset of K_s in a stage
    static constexpr int STAGE_V = KV_TILE_BYTES;          // offset of V_{s-1}
    // Q buffers: with two (D = 64 only: at D = 128 the K/V ring needs the
    // bytes) the next unit's Q loads while this unit's last key tiles run, and
    // the next unit's first S is issued before this unit's last P.V
    static constexpr int NQB = NQB_;
    static_assert(NQB == 1 || (NQB == 2 && D == 64), "two Q buffers fit at D = 64 only");
    static constexpr int QBUF_BYTES = QT * Q_TILE_BYTES;
    static constexpr int Q_OFF = 0;
    static constexpr int KV_OFF = Q_OFF + NQB * QBUF_BYTES;
    // per-row values handed from the softmax to the correction warpgroup
    static constexpr int ALPHA_OFF = KV_OFF + NSTAGE * STAGE_BYTES;   // float [2][128]
    // float2 [unit parity][tile][row] = (1/l, lse); double-buffered because a
    // softmax warpgroup can finish the next unit before the epilogue of this
    // one has read its values (never two units ahead: the unit after next
    // needs this epilogue's O_t to have been read out)
    static constexpr int FIN_OFF = ALPHA_OFF + 2 * BLOCK_M * 4;
    static constexpr int BAR_OFF = FIN_OFF + 2 * 2 * BLOCK_M * 8;
    // barrier indices
    static constexpr int B_QFULL = 0;                      // [NQB] TMA -> MMA
    static constexpr int B_QEMPTY = NQB;                   // [NQB] MMA -> TMA: the unit's last S issued
    static constexpr int B_STFULL = 2 * NQB;               // [NSTAGE] TMA -> MMA
    static constexpr int B_STEMPTY = B_STFULL + NSTAGE;    // [NSTAGE] MMA -> TMA
    static constexpr int B_SFULL = B_STEMPTY + NSTAGE;     // [2] MMA -> softmax: S_t ready
    // [2] softmax + correction -> MMA: P_t written and O_t ready for it (rescaled,
    // or read out by the previous unit's epilogue); 256 arrivals per phase
    static constexpr int B_PFULL = B_SFULL + 2;
    static constexpr int B_OFULL = B_PFULL + 2;            // [2] MMA -> correction: last O_t ready
    static constexpr int B_STATS = B_OFULL + 2;            // [2] softmax -> correction: alpha ready
    static constexpr int B_FINAL = B_STATS + 2;            // [parity][2] softmax -> correction: 1/l, lse ready
    static constexpr int B_FIN = B_FINAL + 4;
    // unit ring: the TMA lane publishes the work-unit indices it took, the MMA,
    // softmax and correction roles read them
    static constexpr int NUNIT = 2;
    static constexpr int B_UFULL = B_FIN + 1;              // [NUNIT] TMA lane -> other roles
    static constexpr int B_UEMPTY = B_UFULL + NUNIT;       // [NUNIT] other roles -> TMA lane
    static constexpr int NBAR = B_UEMPTY + NUNIT;
    // misc: tmem base (u32), abort flag (u32), pad, unit ring (int[NUNIT])
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    static constexpr int UNIT_OFF = MISC_OFF + 16;
    static constexpr int BYTES = UNIT_OFF + NUNIT * 4;
    static constexpr int ALLOC = BYTES + 1024;             // slack for 1 KiB alignment
};

struct KParams {
    CUtensorMap tmap_q;
    CUtensorMap tmap_k;
    CUtensorMap tmap_v;
    uint8_t* o;
    float* lse;    // [B, H, Sq] contiguous
    long long o_sb, o_sh, o_ss;  // byte strides of O over b, h and the query row
    int BH;
    int H;
    int Sq;        // query rows per head
    int Sk;        // keys per head
    int n_mblk;    // 256-row query blocks per head
    int n_units;
    int nkv;       // key tiles per head
    int causal;
    int causal_off;  // Sk - Sq: query i sees keys j <= i + causal_off under the mask
    const uint8_t* mask;         // explicit boolean mask (nonzero = attend), or null
    long long m_sb, m_sh, m_ss;  // its element strides over b, h and the query row (keys contiguous)
    float scale_log2;
    unsigned int* sched;  // zeroed unit counter (claim order), or null for the static order
    // sched[1] counts the CTAs that have finished; the last one zeroes both
    // words for the next launch on the same stream (no memset between launches)
    int sched_reset;
    // dropout (DROP kernels): threshold in every byte, generator key, counter word 3, 1 / (1 - p)
    uint32_t drop_p8x4, seed_lo, seed_hi, drop_offset;
    float keep_scale;
};

// Threads that read each published unit index: MMA lane, two softmax
// warpgroups and the correction warpgroup.
constexpr uint32_t UNIT_READERS = 1 + 2 * BLOCK_M + BLOCK_M;

// ------------------------------------------------------------------ PTX helpers

#include "sm100_helpers.cuh"

// 32 lanes x 64 consecutive 32-bit columns (a 64-key score row per thread).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float* v) {
    uint32_t r[64];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

// Instruction descriptor for kind::f16 with fp32 accumulate, M = 128.
__host__ __device__ constexpr uint32_t make_idesc(bool bf16, int N, bool b_mn_major) {
    return (1u << 4)                                   // D format: f32
           | ((bf16 ? 1u : 0u) << 7)                   // A format
           | ((bf16 ? 1u : 0u) << 10)                  // B format
           | (0u << 15)                                // A K-major
           | ((b_mn_major ? 1u : 0u) << 16)            // B major
           | ((uint32_t)(N >> 3) << 17)                // N / 8
           | ((uint32_t)(BLOCK_M >> 4) << 24);         // M / 16
}

// The 128 mask bytes of keys [kbase, kbase + 128) of one query row as a 128-bit
// mask (bit c of word c / 32 = key kbase + c may be attended).  Keys at or past
// Sk read as 0.  Whole 16-byte loads when the tile is complete (the row and the
// tile start are 16-byte aligned), byte loads on the ragged last tile.
__device__ __forceinline__ void load_mask_bits(const uint8_t* mrow, int kbase, int Sk, uint32_t (&bits)[4]) {
    if (kbase + BLOCK_N <= Sk) {
        const uint4* src = reinterpret_cast<const uint4*>(mrow + kbase);
        uint4 w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = __ldg(src + i);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t acc = 0;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint4 x = w[2 * q + h];
                const uint32_t ws[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    // one bit per nonzero byte, gathered into a nibble (byte i -> bit i)
                    const uint32_t t = __vcmpne4(ws[e], 0u) & 0x01010101u;
                    acc |= ((t * 0x01020408u) >> 24 & 0xFu) << (16 * h + 4 * e);
                }
            }
            bits[q] = acc;
        }
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) bits[q] = 0u;
        for (int c = 0; c < Sk - kbase; ++c)
            if (mrow[kbase + c]) bits[c >> 5] |= 1u << (c & 31);
    }
}

struct Unit {
    int bh;
    int q0[2];   // first query row of each tile
    int n[2];    // key tiles visited by each tile (0 = tile beyond S)
    int N;       // key tiles streamed for the unit
};

// Causal units are ordered longest first within groups of CAUSAL_HEAD_GROUP
// heads (0: one group of all heads): the K/V of the heads that CTAs work on at
// the same time then fit in L2 (8 heads x 2 x S x D x 2 bytes = 64 MiB at
// S = 16384, D = 128) while claimed scheduling keeps the makespan balanced.
constexpr int CAUSAL_HEAD_GROUP = 8;

// Work-unit order: with the causal mask, longest units first (query block
// descending) within head groups, heads innermost; without it, heads
// outermost so that CTAs running together share one head's K/V in L2.
template <int BN, int QT>
__device__ __forceinline__ Unit decode_unit(const KParams& p, int u) {
    constexpr int ROWS = QT * BLOCK_M;  // query rows per unit
    Unit U;
    int mb;
    if (p.causal) {
        if (CAUSAL_HEAD_GROUP > 0 && p.BH > CAUSAL_HEAD_GROUP) {
            const int per_group = CAUSAL_HEAD_GROUP * p.n_mblk;
            const int g = u / per_group;
            const int within = u - g * per_group;
            const int gh = min(CAUSAL_HEAD_GROUP, p.BH - g * CAUSAL_HEAD_GROUP);  // heads in this group
            mb = p.n_mblk - 1 - within / gh;
            U.bh = g * CAUSAL_HEAD_GROUP + within % gh;
        } else {
            mb = p.n_mblk - 1 - u / p.BH;
            U.bh = u % p.BH;
        }
    } else {
        U.bh = u / p.n_mblk;
        mb = u % p.n_mblk;
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int q0 = mb * ROWS + t * BLOCK_M;
        U.q0[t] = q0;
        int n = 0;
        if (t < QT && q0 < p.Sq) {
            // diagonal bound: key tile j is visited iff its first key j*BN is
            // not after the last key that the tile's last query row sees,
            // q0 + BLOCK_M - 1 + causal_off
            n = p.causal ? min((q0 + BLOCK_M - 1 + p.causal_off) / BN + 1, p.nkv) : p.nkv;
        }
        U.n[t] = n;
    }
    U.N = max(U.n[0], U.n[1]);
    return U;
}

// ------------------------------------------------------------------ roles

// Reads the work-unit indices published by the TMA lane, in order.
// next() returns the unit, -1 when the CTA has no more work, -2 on abort.
template <int D, int BN, int QT, int NQB>
struct UnitReader {
    int slot = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ int next(uint8_t* smem, volatile uint32_t* abort_flag, int site) {
        using L = Smem<D, BN, QT, NQB>;
        const uint32_t bar0 = smem_u32(smem) + L::BAR_OFF;
        if (!mbar_wait(bar0 + 8u * (uint32_t)(L::B_UFULL + slot), phase, abort_flag, site)) return -2;
        const int u = reinterpret_cast<volatile int*>(smem + L::UNIT_OFF)[slot];
        mbar_arrive(bar0 + 8u * (uint32_t)(L::B_UEMPTY + slot));
        if (++slot == L::NUNIT) { slot = 0; phase ^= 1u; }
        return u;
    }
};

template <int D, int BN, int QT, int NQB>
__device__ void producer_role(const KParams& p, uint8_t* smem, volatile uint32_t* abort_flag) {
    using L = Smem<D, BN, QT, NQB>;
    const uint32_t base = smem_u32(smem);
    const uint32_t bar0 = base + L::BAR_OFF;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    int stage = 0;
    uint32_t phase = 0;
    int qk = 0;                  // Q fills issued
    uint32_t q_fill_mask = 0;    // Q buffers with a fill issued
    uint32_t q_fill_parity = 0;  // parity of each Q buffer's last fill
    uint32_t fill_mask = 0;    // stages with a fill issued
    uint32_t fill_parity = 0;  // parity of each stage's last fill
    bool ok = true;
    volatile int* ring = reinterpret_cast<volatile int*>(smem + L::UNIT_OFF);
    int uslot = 0;
    uint32_t uphase = 0;

    // Work units: with a counter (the causal mask, where units differ in
    // length) the next unit is claimed when this CTA is about to start it, so
    // CTAs that finish early take more units and the longest-first order of
    // decode_unit holds across the grid; without one the CTA takes units
    // blockIdx.x, blockIdx.x + gridDim.x, ...  Each index is published to the
    // other roles through the unit ring.
    for (int k = 0;; ++k) {
        int u = p.sched ? (int)atomicAdd(p.sched, 1u) : (int)blockIdx.x + k * (int)gridDim.x;
        if (u >= p.n_units) u = -1;
        if (!mbar_wait(bar(L::B_UEMPTY + uslot), uphase ^ 1u, abort_flag, 30)) { ok = false; break; }
        ring[uslot] = u;
        mbar_arrive(bar(L::B_UFULL + uslot));
        if (++uslot == L::NUNIT) { uslot = 0; uphase ^= 1u; }
        if (u < 0) break;
        const Unit U = decode_unit<BN, QT>(p, u);
        const int ub = U.bh / p.H, uh = U.bh - ub * p.H;  // tensor-map coordinates of the head
        // Q buffer of this unit: fill number qk of the CTA goes to buffer qk mod NQB
        const int qb = qk % L::NQB;
        const uint32_t qph = (uint32_t)(qk / L::NQB) & 1u;
        ++qk;
        if (!mbar_wait(bar(L::B_QEMPTY + qb), qph ^ 1u, abort_flag, 1)) { ok = false; break; }
        const uint32_t qbytes = (U.n[0] > 0 ? L::Q_TILE_BYTES : 0) + (U.n[1] > 0 ? L::Q_TILE_BYTES : 0);
        mbar_expect_tx(bar(L::B_QFULL + qb), qbytes);
        q_fill_mask |= 1u << qb;
        q_fill_parity = (q_fill_parity & ~(1u << qb)) | (qph << qb);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            if (U.n[t] == 0) continue;
            const uint32_t dst = base + L::Q_OFF + qb * L::QBUF_BYTES + t * L::Q_TILE_BYTES;
#pragma unroll
            for (int c = 0; c < L::CHUNKS; ++c)
                tma_load_4d(dst + c * L::Q_CHUNK_BYTES, &p.tmap_q, bar(L::B_QFULL + qb), c * 64, U.q0[t], uh, ub);
        }
        // stages 0..N: stage s = (V_{s-1} if s >= 1, K_s if s < N)
        for (int st = 0; st <= U.N; ++st) {
            if (!mbar_wait(bar(L::B_STEMPTY + stage), phase ^ 1u, abort_flag, 2)) { ok = false; break; }
            const uint32_t bytes = (st >= 1 ? L::KV_TILE_BYTES : 0) + (st < U.N ? L::KV_TILE_BYTES : 0);
            mbar_expect_tx(bar(L::B_STFULL + stage), bytes);
            fill_mask |= 1u << stage;
            fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
            const uint32_t dst = base + L::KV_OFF + stage * L::STAGE_BYTES;
            if (st < U.N) {
#pragma unroll
                for (int c = 0; c < L::CHUNKS; ++c)
                    tma_load_4d(dst + L::STAGE_K + c * L::KV_CHUNK_BYTES, &p.tmap_k, bar(L::B_STFULL + stage),
                                c * 64, st * BN, uh, ub);
            }
            if (st >= 1) {
#pragma unroll
                for (int c = 0; c < L::CHUNKS; ++c)
                    tma_load_4d(dst + L::STAGE_V + c * L::KV_CHUNK_BYTES, &p.tmap_v, bar(L::B_STFULL + stage),
                                c * 64, (st - 1) * BN, uh, ub);
            }
            if (++stage == L::NSTAGE) { stage = 0; phase ^= 1u; }
        }
    }
    if (!ok) {
        // drain the copies this thread issued before leaving
        for (int i = 0; i < L::NSTAGE; ++i)
            if (fill_mask & (1u << i)) mbar_drain(bar(L::B_STFULL + i), (fill_parity >> i) & 1u);
        for (int i = 0; i < L::NQB; ++i)
            if (q_fill_mask & (1u << i)) mbar_drain(bar(L::B_QFULL + i), (q_fill_parity >> i) & 1u);
    }
}

template <int D, bool BF16, int BN, int QT, int NQB>
__device__ void mma_role(const KParams& p, uint8_t* smem, uint32_t tmem, volatile uint32_t* abort_flag) {
    using L = Smem<D, BN, QT, NQB>;
    const uint32_t base = smem_u32(smem);
    const uint32_t bar0 = base + L::BAR_OFF;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    constexpr uint32_t IDESC_S = make_idesc(BF16, BN, false);
    constexpr uint32_t IDESC_PV = make_idesc(BF16, D, true);
    constexpr int KSTEPS_S = D / 16;        // QK^T: K = D
    constexpr int KSTEPS_PV = BN / 16;      // PV: K = BN keys

    // S_t = Q_t K^T : A = Q tile (K-major), B = K tile (K-major), 128-byte swizzle,
    // 8-row groups 1024 bytes apart; K steps of 16 elements advance 32 bytes
    // inside a swizzle atom and 16 KiB across the 64-column chunks.
    // O_t += P_t V : A = P in TMEM (16-bit pairs packed per column, 8 columns per
    // 16 keys), B = V tile read MN-major (D contiguous): 64-element chunks 16 KiB
    // apart (leading byte offset; with D = 64 there is a single chunk and the
    // field is unused), 8-key groups 1024 bytes apart (stride byte offset);
    // K steps of 16 keys advance 2 KiB.
    // Descriptors are built once; a start address (< 256 KiB, 14 bits after >> 4)
    // plus any offset used here stays inside the low half's field.
    constexpr uint32_t V_LBO = (D == 128) ? (uint32_t)L::KV_CHUNK_BYTES : 1024u;
    const uint64_t dq = sw128_desc(base + L::Q_OFF, 16, 1024);
    const uint64_t dk = sw128_desc(base + L::KV_OFF, 16, 1024);
    const uint64_t dv = sw128_desc(base + L::KV_OFF, V_LBO, 1024);
    const uint32_t dq_lo = (uint32_t)dq, dq_hi = (uint32_t)(dq >> 32);
    const uint32_t dk_lo = (uint32_t)dk, dk_hi = (uint32_t)(dk >> 32);
    const uint32_t dv_lo = (uint32_t)dv, dv_hi = (uint32_t)(dv >> 32);
    constexpr uint32_t TILE16 = (uint32_t)L::Q_TILE_BYTES >> 4;

    constexpr uint32_t STAGE16 = (uint32_t)L::STAGE_BYTES >> 4;
    uint32_t qbuf16 = 0;  // this unit's Q buffer offset (16-byte units)
    auto issue_s = [&](int t, int st) {
        const uint32_t a_lo = dq_lo + qbuf16 + (uint32_t)t * TILE16;
        const uint32_t b_lo = dk_lo + (uint32_t)st * STAGE16 + ((uint32_t)L::STAGE_K >> 4);
        const uint32_t d_tmem = tmem + (t == 0 ? COL_S0 : COL_S1);
#pragma unroll
        for (int ks = 0; ks < KSTEPS_S; ++ks) {
            const uint32_t a_off = (uint32_t)(((ks & 3) * 32 + (ks >> 2) * L::Q_CHUNK_BYTES) >> 4);
            const uint32_t b_off = (uint32_t)(((ks & 3) * 32 + (ks >> 2) * L::KV_CHUNK_BYTES) >> 4);
            tc_mma_ss2(d_tmem, a_lo + a_off, dq_hi, b_lo + b_off, dk_hi, IDESC_S, ks > 0 ? 1u : 0u);
        }
    };
    auto issue_pv = [&](int t, int st, bool accumulate) {
        const uint32_t b_lo = dv_lo + (uint32_t)st * STAGE16 + ((uint32_t)L::STAGE_V >> 4);
        const uint32_t a_tmem = tmem + (t == 0 ? COL_S0 : COL_S1);
        const uint32_t d_tmem = tmem + (t == 0 ? COL_O0 : COL_O1);
#pragma unroll
        for (int ks = 0; ks < KSTEPS_PV; ++ks) {
            tc_mma_ts2(d_tmem, a_tmem + (uint32_t)(ks * 8), b_lo + (uint32_t)(ks * (2048 >> 4)), dv_hi, IDESC_PV,
                       (accumulate || ks > 0) ? 1u : 0u);
        }
    };

    int stage = 0;
    uint32_t phase = 0;
    int qk = 0;  // units whose Q was used
    uint32_t p_phase[2] = {0u, 0u};
    bool ok = true;

    // Wait for what PV_t needs besides V: P_t and O_t (one barrier, armed by the
    // softmax and the correction warpgroups).  Waits of this thread queue behind
    // its MMAs that the tensor pipe has not taken yet, so each wait point costs
    // pipe time: the loop below has three per key tile (K, P1, V + P0).
    auto wait_pv_inputs = [&](int t, int site) -> bool {
        if (!mbar_wait(bar(L::B_PFULL + t), p_phase[t], abort_flag, site)) return false;
        p_phase[t] ^= 1u;
        tc_fence_after();  // P_t and O_t were written by tcgen05.st of other threads
        return true;
    };

    // Issue order per key tile j (tile 1 lags tile 0 by one step), stage j
    // holding V_{j-1} and K_j:
    //   [P1] O1 += P1 V_{j-1};  S1 = Q1 K_j^T;  release stage j;
    //   [stage j+1, P0] O0 += P0 V_j;  S0 = Q0 K_{j+1}^T
    // Each P.V is followed directly by the next S of the same tile (the S/P
    // columns are free once that P.V is issued; MMAs of one thread run in
    // order).  Waits and commits of this thread queue behind its MMAs not yet
    // taken by the tensor pipe, so there are as few of them as possible:
    // per key tile three waits (P1, stage, P0) and three commits.
    auto wait_stage = [&](int site) -> int {
        const int st = stage;
        if (!mbar_wait(bar(L::B_STFULL + st), phase, abort_flag, site)) return -1;
        if (++stage == L::NSTAGE) { stage = 0; phase ^= 1u; }
        return st;
    };
    // A unit's prologue: its Q, stage 0 (K_0), S0 = Q0 K_0^T.
    auto start_unit = [&](const Unit& Un, int& cur_out, int& qb_out) -> bool {
        const int qbn = qk % L::NQB;
        if (!mbar_wait(bar(L::B_QFULL + qbn), (uint32_t)(qk / L::NQB) & 1u, abort_flag, 3)) return false;
        ++qk;
        qbuf16 = (uint32_t)(qbn * L::QBUF_BYTES) >> 4;
        const int c0 = wait_stage(4);
        if (c0 < 0) return false;
        issue_s(0, c0);
        tc_commit(bar(L::B_SFULL + 0));
        if (Un.N == 1 && Un.n[1] != Un.N) tc_commit(bar(L::B_QEMPTY + qbn));
        cur_out = c0;
        qb_out = qbn;
        return true;
    };
    UnitReader<D, BN, QT, NQB> units;
    int u = units.next(smem, abort_flag, 32);
    Unit U{};
    int cur = -1, qb = 0;
    if (u >= 0) {
        U = decode_unit<BN, QT>(p, u);
        if (!start_unit(U, cur, qb)) ok = false;
    }
    while (ok && u >= 0) {
        const bool tile1_last = U.n[1] == U.N;  // which tile issues the unit's last S
        for (int j = 0; j < U.N; ++j) {
            // ---- tile 1 on stage j: O1 += P1 V_{j-1}, S1 = Q1 K_j^T
            if (j >= 1 && j - 1 < U.n[1]) {
                if (!wait_pv_inputs(1, 5)) { ok = false; break; }
                issue_pv(1, cur, j - 1 > 0);
            }
            if (j < U.n[1]) {
                issue_s(1, cur);
                tc_commit(bar(L::B_SFULL + 1));
            }
            tc_commit(bar(L::B_STEMPTY + cur));  // V_{j-1} and K_j: last readers issued
            if (j == U.N - 1 && tile1_last) tc_commit(bar(L::B_QEMPTY + qb));
            // ---- tile 0 on stage j+1: O0 += P0 V_j, S0 = Q0 K_{j+1}^T
            const int nxt = wait_stage(6);
            if (nxt < 0) { ok = false; break; }
            if (j < U.n[0]) {
                if (!wait_pv_inputs(0, 9)) { ok = false; break; }
                issue_pv(0, nxt, j > 0);
                if (j == U.n[0] - 1) tc_commit(bar(L::B_OFULL + 0));
            }
            if (j + 1 < U.n[0]) {
                issue_s(0, nxt);
                tc_commit(bar(L::B_SFULL + 0));
                if (j + 1 == U.N - 1 && !tile1_last) tc_commit(bar(L::B_QEMPTY + qb));
            }
            cur = nxt;
        }
        if (!ok) break;
        // stage N holds V_{N-1}: O1 += P1 V_{N-1}, then release it.  With two Q
        // buffers the next unit's first S goes first, so that its tile 0 starts
        // while this unit's tile 1 finishes (as between key tiles of a unit).
        auto finish_unit = [&]() -> bool {
            if (U.n[1] > 0) {
                if (!wait_pv_inputs(1, 12)) return false;
                issue_pv(1, cur, U.N - 1 > 0);
                tc_commit(bar(L::B_OFULL + 1));
            }
            tc_commit(bar(L::B_STEMPTY + cur));
            return true;
        };
        if constexpr (L::NQB == 1) {
            if (!finish_unit()) { ok = false; break; }
        }
        const int u2 = units.next(smem, abort_flag, 32);
        Unit U2{};
        int cur2 = -1, qb2 = 0;
        if (u2 >= 0) {
            U2 = decode_unit<BN, QT>(p, u2);
            if (!start_unit(U2, cur2, qb2)) { ok = false; break; }
        }
        if constexpr (L::NQB == 2) {
            if (!finish_unit()) { ok = false; break; }
        }
        u = u2;
        U = U2;
        cur = cur2;
        qb = qb2;
    }
    // all MMAs issued by this thread have completed once B_FIN fires
    tc_commit(bar(L::B_FIN));
    mbar_drain(bar(L::B_FIN), 0u);
}

template <int D, bool BF16, bool MASK, bool DROP, int BN, int QT, int NQB>
__device__ void softmax_role(const KParams& p, uint8_t* smem, uint32_t tmem, int t, int warp_in_group,
                             volatile uint32_t* abort_flag) {
    using L = Smem<D, BN, QT, NQB>;
    static_assert(BN == BLOCK_N || (!MASK && !DROP), "the mask and dropout paths take 128-key tiles");
    const uint32_t base = smem_u32(smem);
    const uint32_t bar0 = base + L::BAR_OFF;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    const int lane = threadIdx.x & 31;
    const int row_in_tile = warp_in_group * 32 + lane;
    const uint32_t lane_sel = (uint32_t)(warp_in_group * 32) << 16;
    const uint32_t ts = tmem + lane_sel + (t == 0 ? COL_S0 : COL_S1);
    float* alpha_buf = reinterpret_cast<float*>(smem + L::ALPHA_OFF) + t * BLOCK_M + row_in_tile;
    float2* fin_buf = reinterpret_cast<float2*>(smem + L::FIN_OFF) + t * BLOCK_M + row_in_tile;
    int fin_par = 0;  // parity of this tile's active units
    const float sl2 = p.scale_log2;
    const float2 sl2x2 = make_float2(sl2, sl2);

    uint32_t s_phase = 0;
    UnitReader<D, BN, QT, NQB> units;
    for (;;) {
        const int u = units.next(smem, abort_flag, 33);
        if (!__all_sync(0xffffffffu, u != -2)) return;
        if (u < 0) break;
        const Unit U = decode_unit<BN, QT>(p, u);
        const int n = U.n[t];
        if (n == 0) continue;
        const int row = U.q0[t] + row_in_tile;
        const int key_limit = p.causal ? min(row + p.causal_off, p.Sk - 1) : p.Sk - 1;  // last visible key
        float m_use = -INFINITY;  // reference max in log2 units
        float l = 0.f;            // running sum of the weights relative to m_use (fp32)
        float lr = 0.f;           // the same sum over the weights as rounded for P.V
        // explicit mask: this row's bits for the next key tile, loaded while the
        // previous tile's MMAs run (rows past Sq read the last row)
        const uint8_t* mrow = nullptr;
        uint32_t mbits[4] = {0u, 0u, 0u, 0u};
        if constexpr (MASK) {
            const int ub = U.bh / p.H, uh = U.bh - ub * p.H;
            mrow = p.mask + (long long)ub * p.m_sb + (long long)uh * p.m_sh + (long long)min(row, p.Sq - 1) * p.m_ss;
            load_mask_bits(mrow, 0, p.Sk, mbits);
        }
        for (int j = 0; j < n; ++j) {
            // the result is made warp-uniform: the TMEM accesses below need the whole warp
            if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_SFULL + t), s_phase, abort_flag, 16 + t))) return;
            s_phase ^= 1u;
            tc_fence_after();
            float s[BN];
            if constexpr (BN == 128) tmem_ld128(ts, s); else tmem_ld64(ts, s);
            const int kbase = j * BN;
            const bool need_mask =
                (kbase + BN > p.Sk) || (p.causal && kbase + BN - 1 > U.q0[t] + p.causal_off);
            if (need_mask) {
                const int lim = key_limit - kbase;
#pragma unroll
                for (int c = 0; c < BN; ++c)
                    if (c > lim) s[c] = -INFINITY;
            }
            if constexpr (MASK) {
#pragma unroll
                for (int c = 0; c < BLOCK_N; ++c)
                    if (!((mbits[c >> 5] >> (c & 31)) & 1u)) s[c] = -INFINITY;
            }
            float mx0 = max3(s[0], s[1], s[2]), mx1 = max3(s[3], s[4], s[5]);
            float mx2 = max3(s[6], s[7], s[8]), mx3 = max3(s[9], s[10], s[11]);
#pragma unroll
            for (int c = 12; c < BN - 4; c += 8) {
                mx0 = max3(mx0, s[c], s[c + 1]);
                mx1 = max3(mx1, s[c + 2], s[c + 3]);
                mx2 = max3(mx2, s[c + 4], s[c + 5]);
                mx3 = max3(mx3, s[c + 6], s[c + 7]);
            }
            mx0 = max3(mx0, s[BN - 4], s[BN - 3]);
            mx1 = max3(mx1, s[BN - 2], s[BN - 1]);
            const float m_blk = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
            bool grow = m_blk > m_use + Policy<BF16>::TAU;
            if constexpr (BF16) grow = grow || (m_blk > m_use && ex2(m_blk - m_use) > RESCALE_KAPPA * lr);
            float alpha = 1.f;
            if (grow) {
                alpha = (m_use == -INFINITY) ? 0.f : ex2(m_use - m_blk);
                m_use = m_blk;
                l *= alpha;
                lr *= alpha;
            }
            if (j > 0) {
                // the correction warpgroup rescales this O row by alpha before P.V
                *alpha_buf = alpha;
                mbar_arrive(bar(L::B_STATS + t));
            }
            const float neg_m = (m_use == -INFINITY) ? 0.f : -m_use;
            const float2 negm2 = make_float2(neg_m, neg_m);
            float2 lsum0 = make_float2(0.f, 0.f), lsum1 = make_float2(0.f, 0.f);
            float2 rsum0 = make_float2(0.f, 0.f), rsum1 = make_float2(0.f, 0.f);
            // Weights of a quarter row (16 pairs) into packed 16-bit P, stored to
            // TMEM right away (fewer live registers).
            auto quarter_row = [&](int qr) {
                uint32_t pk[16];
                // dropout: keep masks of the quarter's 32 keys (two 16-key generator blocks)
                uint32_t km[8];
                if constexpr (DROP) {
                    const uint32_t g0 = (uint32_t)(kbase + 32 * qr) >> 4;
                    const uint4 a = dropout_keep_bytes(g0, (uint32_t)row, (uint32_t)U.bh, p.drop_offset, p.seed_lo,
                                                       p.seed_hi, p.drop_p8x4);
                    const uint4 b = dropout_keep_bytes(g0 + 1u, (uint32_t)row, (uint32_t)U.bh, p.drop_offset,
                                                       p.seed_lo, p.seed_hi, p.drop_p8x4);
                    km[0] = a.x; km[1] = a.y; km[2] = a.z; km[3] = a.w;
                    km[4] = b.x; km[5] = b.y; km[6] = b.z; km[7] = b.w;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 x = __ffma2_rn(make_float2(s[32 * qr + 2 * i], s[32 * qr + 2 * i + 1]), sl2x2, negm2);
                    const float2 e = make_float2(ex2(x.x), ex2(x.y));
                    pk[i] = pack2<BF16>(e.x, e.y);
                    if (i & 1) lsum1 = __fadd2_rn(lsum1, e); else lsum0 = __fadd2_rn(lsum0, e);
                    if constexpr (Policy<BF16>::NORM_BY_ROUNDED_P) {
                        // the rounded weights as the MMA sees them (bf16 -> fp32 is exact)
                        if (i & 1) rsum1 = add_bf16x2(rsum1, pk[i]); else rsum0 = add_bf16x2(rsum0, pk[i]);
                    }
                    // the sums keep every weight; P.V sees only the kept ones (keys 2i and
                    // 2i + 1 are bytes 2i and 2i + 1 of the quarter's mask: each byte fills a half)
                    if constexpr (DROP) pk[i] &= __byte_perm(km[i >> 1], 0u, (i & 1) ? 0x3322u : 0x1100u);
                }
                // P (16-bit, two per column) overwrites the first 64 columns of S
                tmem_st16(ts + 16 * qr, pk);
            };
#pragma unroll
            for (int qr = 0; qr < BN / 32; ++qr) quarter_row(qr);
            const float2 ls = __fadd2_rn(lsum0, lsum1);
            l += ls.x + ls.y;
            if constexpr (Policy<BF16>::NORM_BY_ROUNDED_P) {
                const float2 rs = __fadd2_rn(rsum0, rsum1);
                lr += rs.x + rs.y;
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(L::B_PFULL + t));
            if constexpr (MASK) {
                if (j + 1 < n) load_mask_bits(mrow, kbase + BLOCK_N, p.Sk, mbits);
            }
        }
        // final statistics for the epilogue: 1/l for O, LSE = (m + log2 l) ln 2;
        // a row with no visible key (possible only with an explicit mask) gets
        // O = 0 and LSE = -inf
        const float norm = Policy<BF16>::NORM_BY_ROUNDED_P ? lr : l;
        fin_buf[fin_par * 2 * BLOCK_M] = (l > 0.f)
            ? make_float2((DROP ? p.keep_scale : 1.f) / norm, (m_use + __log2f(l)) * 0.69314718055994530942f)
            : make_float2(0.f, -INFINITY);
        mbar_arrive(bar(L::B_FINAL + 2 * fin_par + t));
        fin_par ^= 1;
    }
}

template <int D, bool BF16, int BN, int QT, int NQB>
__device__ void correction_role(const KParams& p, uint8_t* smem, uint32_t tmem, int warp_in_group,
                                volatile uint32_t* abort_flag) {
    using L = Smem<D, BN, QT, NQB>;
    const uint32_t base = smem_u32(smem);
    const uint32_t bar0 = base + L::BAR_OFF;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    const int lane = threadIdx.x & 31;
    const int row_in_tile = warp_in_group * 32 + lane;
    const uint32_t lane_sel = (uint32_t)(warp_in_group * 32) << 16;
    const float* alpha_buf = reinterpret_cast<const float*>(smem + L::ALPHA_OFF);
    const float2* fin_buf = reinterpret_cast<const float2*>(smem + L::FIN_OFF);
    uint32_t st_phase[2] = {0u, 0u}, of_phase[2] = {0u, 0u};
    // O_t of the first unit needs no read-out: arm both tiles' first P barrier phase
    mbar_arrive(bar(L::B_PFULL + 0));
    mbar_arrive(bar(L::B_PFULL + 1));
    uint32_t fi_phase[2][2] = {{0u, 0u}, {0u, 0u}};  // [unit parity][tile]
    int fin_par[2] = {0, 0};

    // O_t row *= alpha for iteration j of tile t (warp-uniform skip when all alpha == 1)
    auto correct = [&](int t) -> bool {
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_STATS + t), st_phase[t], abort_flag, 24 + t)))
            return false;
        st_phase[t] ^= 1u;
        const float alpha = alpha_buf[t * BLOCK_M + row_in_tile];
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
            tc_fence_after();
            const uint32_t to = tmem + lane_sel + (t == 0 ? COL_O0 : COL_O1);
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32u(to + 32 * c, r);
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const float2 v = __fmul2_rn(make_float2(__uint_as_float(r[i]), __uint_as_float(r[i + 1])),
                                                make_float2(alpha, alpha));
                    r[i] = __float_as_uint(v.x);
                    r[i + 1] = __float_as_uint(v.y);
                }
                tmem_st32(to + 32 * c, r);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(bar(L::B_PFULL + t));
        return true;
    };

    // O_t / l -> 16 bits -> global, LSE -> global; then O_t is free for the next unit
    auto epilogue = [&](const Unit& U, int t) -> bool {
        const int fp = fin_par[t];
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_FINAL + 2 * fp + t), fi_phase[fp][t], abort_flag, 26 + t)))
            return false;
        fi_phase[fp][t] ^= 1u;
        fin_par[t] ^= 1;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_OFULL + t), of_phase[t], abort_flag, 28 + t)))
            return false;
        of_phase[t] ^= 1u;
        tc_fence_after();
        const float2 fin = fin_buf[(fp * 2 + t) * BLOCK_M + row_in_tile];
        const int row = U.q0[t] + row_in_tile;
        const bool valid = row < p.Sq;
        const int ub = U.bh / p.H, uh = U.bh - ub * p.H;
        uint8_t* orow = p.o + (long long)ub * p.o_sb + (long long)uh * p.o_sh + (long long)(valid ? row : 0) * p.o_ss;
        const uint32_t to = tmem + lane_sel + (t == 0 ? COL_O0 : COL_O1);
        const float2 inv2 = make_float2(fin.x, fin.x);
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32u(to + 32 * c, r);
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float2 v = __fmul2_rn(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), inv2);
                w[i] = pack2<BF16>(v.x, v.y);
            }
            if (valid) {
                uint4* dst = reinterpret_cast<uint4*>(orow + c * 64);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
            }
        }
        if (valid) p.lse[(size_t)U.bh * (size_t)p.Sq + row] = fin.y;
        // O_t is free for the next unit's first P.V: arm that P barrier phase
        tc_fence_before();
        mbar_arrive(bar(L::B_PFULL + t));
        return true;
    };

    UnitReader<D, BN, QT, NQB> units;
    for (;;) {
        const int u = units.next(smem, abort_flag, 34);
        if (!__all_sync(0xffffffffu, u != -2)) return;
        if (u < 0) break;
        const Unit U = decode_unit<BN, QT>(p, u);
        for (int j = 1; j < U.N; ++j) {
            if (j < U.n[0] && !correct(0)) return;
            if (j < U.n[1] && !correct(1)) return;
        }
        if (U.n[0] > 0 && !epilogue(U, 0)) return;
        if (U.n[1] > 0 && !epilogue(U, 1)) return;
    }
}

template <int D, bool BF16, bool MASK, bool DROP, int BN = BLOCK_N, int QT = Q_TILES_PER_CTA, int NQB = 1>
__global__ void __launch_bounds__(NUM_THREADS, 1) fa_fwd_kernel(const __grid_constant__ KParams p) {
    using L = Smem<D, BN, QT, NQB>;
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
            uint32_t count = 1;  // TMA transaction or tcgen05.commit arrivals
            if ((i >= L::B_STATS && i < L::B_STATS + 2) || (i >= L::B_FINAL && i < L::B_FINAL + 4))
                count = BLOCK_M;      // one arrival per thread of a 128-thread warpgroup
            if (i >= L::B_PFULL && i < L::B_PFULL + 2)
                count = 2 * BLOCK_M;  // softmax and correction warpgroups
            if (i >= L::B_UEMPTY && i < L::B_UEMPTY + L::NUNIT) count = UNIT_READERS;
            mbar_init(base + L::BAR_OFF + 8 * i, count);
        }
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == WARP_TMA && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmap_q)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmap_k)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmap_v)) : "memory");
    }
    if (warp == WARP_MMA) {
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
        softmax_role<D, BF16, MASK, DROP, BN, QT, NQB>(p, smem, tmem, wg, warp & 3, abort_flag);
    } else if (wg == 2) {
        setmaxnreg_dec<REG_CORR>();
        correction_role<D, BF16, BN, QT, NQB>(p, smem, tmem, warp & 3, abort_flag);
    } else {
        setmaxnreg_dec<REG_CTRL>();
        if (warp == WARP_TMA) {
            if (lane == 0) producer_role<D, BN, QT, NQB>(p, smem, abort_flag);
        } else if (warp == WARP_MMA) {
            if (lane == 0) mma_role<D, BF16, BN, QT, NQB>(p, smem, tmem, abort_flag);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS)
                     : "memory");
    }
    if (p.sched_reset && threadIdx.x == 0) {
        // this CTA's claims are done (its producer has left); the last CTA to
        // get here clears the counter and the count for the stream's next launch
        __threadfence();
        if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1u) {
            __threadfence();
            atomicExch(p.sched, 0u);
            atomicExch(p.sched + 1, 0u);
        }
    }
}

// Diagnostic kernel for the failure path: thread 0 waits on an mbarrier that
// nothing arrives on, with a short deadline; it then raises the abort flag and
// the status word.  Thread 32 waits on another barrier and leaves on the abort
// flag; TMEM held by the CTA is released before the kernel ends.
__global__ void __launch_bounds__(64, 1) selftest_timeout_kernel(long long deadline_cycles) {
    grid_dependency_sync();
    __shared__ __align__(8) uint64_t bars[2];
    __shared__ uint32_t tm;
    __shared__ uint32_t abort_s;
    const int warp = threadIdx.x >> 5;
    const uint32_t b0 = smem_u32(&bars[0]), b1 = smem_u32(&bars[1]);
    if (threadIdx.x == 0) {
        mbar_init(b0, 1);
        mbar_init(b1, 1);
        abort_s = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tm)), "r"(32u)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    volatile uint32_t* abort_flag = &abort_s;
    if (threadIdx.x == 0) mbar_wait(b0, 0u, abort_flag, SELFTEST_SITE, deadline_cycles);
    if (threadIdx.x == 32) mbar_wait(b1, 0u, abort_flag, SELFTEST_SITE + 1, 8 * deadline_cycles);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm), "r"(32u) : "memory");
    }
}

template <int D, bool BF16, bool MASK, bool DROP = false, int BN = BLOCK_N, int QT = Q_TILES_PER_CTA, int NQB = 1>
cudaError_t launch_impl(const LaunchArgs& a, cudaStream_t stream) {
    using L = Smem<D, BN, QT, NQB>;
    static_assert(L::ALLOC <= 232448, "shared memory budget exceeded");
    auto kern = fa_fwd_kernel<D, BF16, MASK, DROP, BN, QT, NQB>;
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), L::ALLOC);
    if (e != cudaSuccess) return e;
    KParams p;
    p.tmap_q = a.tmap_q;
    p.tmap_k = a.tmap_k;
    p.tmap_v = a.tmap_v;
    p.o = reinterpret_cast<uint8_t*>(a.o);
    p.lse = a.lse;
    p.o_sb = a.o_stride[0] * 2;
    p.o_sh = a.o_stride[1] * 2;
    p.o_ss = a.o_stride[2] * 2;
    p.BH = a.B * a.H;
    p.H = a.H;
    p.Sq = a.Sq;
    p.Sk = a.Sk;
    p.n_mblk = (a.Sq + QT * BLOCK_M - 1) / (QT * BLOCK_M);
    p.n_units = p.BH * p.n_mblk;
    p.nkv = (a.Sk + BN - 1) / BN;
    p.causal = a.causal;
    p.causal_off = a.Sk - a.Sq;
    p.mask = a.mask;
    p.m_sb = a.mask_stride[0];
    p.m_sh = a.mask_stride[1];
    p.m_ss = a.mask_stride[2];
    p.scale_log2 = a.scale_log2;
    p.sched = a.sched;
    p.sched_reset = a.sched_reset;
    p.drop_p8x4 = a.drop.p8 * 0x01010101u;
    p.seed_lo = a.drop.seed_lo;
    p.seed_hi = a.drop.seed_hi;
    p.drop_offset = a.drop.offset;
    p.keep_scale = a.drop.enabled ? a.drop.keep_scale : 1.f;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.grid, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = L::ALLOC;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    set_programmatic_launch(cfg, attr);
    return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

// Manual tilings (attention without an explicit mask or dropout): key tiles of
// 64 or 128 rows, one or two 128-row query tiles per work unit.
template <int D, bool BF16>
cudaError_t launch_tiled(const LaunchArgs& a, cudaStream_t stream) {
    if (a.block_n == 64)
        return a.q_tiles == 1 ? launch_impl<D, BF16, false, false, 64, 1>(a, stream)
                              : launch_impl<D, BF16, false, false, 64, 2>(a, stream);
    return a.q_tiles == 1 ? launch_impl<D, BF16, false, false, 128, 1>(a, stream)
                          : launch_impl<D, BF16, false, false, 128, 2>(a, stream);
}

cudaError_t launch_fwd_sm100(const LaunchArgs& a, cudaStream_t stream) {
    if (a.block_n != BLOCK_N || a.q_tiles != Q_TILES_PER_CTA) {
        if (a.mask || a.drop.enabled) return cudaErrorInvalidValue;  // rejected by the host layer first
        if (a.D == 128) return a.dtype == 1 ? launch_tiled<128, true>(a, stream) : launch_tiled<128, false>(a, stream);
        return a.dtype == 1 ? launch_tiled<64, true>(a, stream) : launch_tiled<64, false>(a, stream);
    }
    if (a.drop.enabled) {
        if (a.mask) {
            if (a.D == 128)
                return a.dtype == 1 ? launch_impl<128, true, true, true>(a, stream)
                                    : launch_impl<128, false, true, true>(a, stream);
            return a.dtype == 1 ? launch_impl<64, true, true, true>(a, stream) : launch_impl<64, false, true, true>(a, stream);
        }
        if (a.D == 128)
            return a.dtype == 1 ? launch_impl<128, true, false, true>(a, stream)
                                : launch_impl<128, false, false, true>(a, stream);
        return a.dtype == 1 ? launch_impl<64, true, false, true>(a, stream) : launch_impl<64, false, false, true>(a, stream);
    }
    if (a.D == 128) {
        if (a.mask) return a.dtype == 1 ? launch_impl<128, true, true>(a, stream) : launch_impl<128, false, true>(a, stream);
        return a.dtype == 1 ? launch_impl<128, true, false>(a, stream) : launch_impl<128, false, false>(a, stream);
    }
    if (a.mask) return a.dtype == 1 ? launch_impl<64, true, true>(a, stream) : launch_impl<64, false, true>(a, stream);
    // two Q buffers when a CTA runs two or more units (more shared memory per
    // CTA; for one unit per CTA they cannot help)
    const int n_units = a.B * a.H * ((a.Sq + Q_TILES_PER_CTA * BLOCK_M - 1) / (Q_TILES_PER_CTA * BLOCK_M));
    if (n_units >= 2 * a.grid)
        return a.dtype == 1 ? launch_impl<64, true, false, false, BLOCK_N, Q_TILES_PER_CTA, 2>(a, stream)
                            : launch_impl<64, false, false, false, BLOCK_N, Q_TILES_PER_CTA, 2>(a, stream);
    return a.dtype == 1 ? launch_impl<64, true, false>(a, stream) : launch_impl<64, false, false>(a, stream);
}

cudaError_t launch_selftest_timeout(cudaStream_t stream) {
    // about 50 ms at the maximum SM clock
    return launch_kernel(selftest_timeout_kernel, dim3(1), dim3(64), 0, stream, 100000000ll);
}

namespace {

// Device address of a static array in the current context, looked up once per
// context.  In host code the array's name is only a stand-in, not a device
// address; cudaGetSymbolAddress gives the address with that context current.
template <typename T, size_t N>
cudaError_t symbol_address_per_context(const T (&symbol)[N], std::mutex& mu,
                                       std::map<unsigned long long, unsigned int*>& cache, unsigned int** out) {
    unsigned long long ctx = 0;
    cudaError_t e = current_context_id(&ctx);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(ctx);
    if (it == cache.end()) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, symbol);
        if (e != cudaSuccess) return e;
        it = cache.emplace(ctx, static_cast<unsigned int*>(ptr)).first;
    }
    *out = it->second;
    return cudaSuccess;
}

}  // namespace

cudaError_t noalloc_scratch_address(unsigned int** out) {
    static std::mutex mu;
    static std::map<unsigned long long, unsigned int*> cache;
    return symbol_address_per_context(g_noalloc_scratch, mu, cache, out);
}

cudaError_t sched_pool_address(unsigned int** out) {
    static std::mutex mu;
    static std::map<unsigned long long, unsigned int*> cache;
    return symbol_address_per_context(g_sched_pool, mu, cache, out);
}

cudaError_t read_and_clear_status(cudaStream_t stream, int* status, int* site) {
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
