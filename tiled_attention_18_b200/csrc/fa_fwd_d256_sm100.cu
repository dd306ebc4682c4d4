// fa_fwd_d256_sm100.cu -- attention forward pass for head dimension 256 on B200
// (sm_100a).  Same operation, numerics policy and C ABI as the D = 64/128
// kernel (fa_fwd_sm100.cu); a different tiling, because two 128-row query tiles
// with D = 256 would need 2 x (128 + 256) TMEM columns (512 exist) and 256 KiB
// of shared memory for Q and one K/V stage (227 KiB exist).  The pages name
// 256 among the common head dimensions their 128 x 128 tiles serve
// ("FlashAttention-2 在昇腾 NPU 上如何做到 3 倍加速？", section 3.2).
//
// Work unit = (b, h, 128-row query tile).  Keys and values stream in 64-row
// tiles through separate two-slot rings (K_j is released once S_j is
// computed, V_j once P_j V_j is), so a K tile loads while the previous V tile is
// still in use.  Tensor memory: S of two consecutive key tiles (64 columns
// each, double-buffered: the MMA lane computes S_{j+1} while the softmax
// warpgroup works on S_j) and O (256 columns).
//
// Roles (12 warps): warpgroup 0 = softmax (one query row per thread), warpgroup
// 1 = correction (O rescale when a row's reference max moves, and the
// epilogue), warp 8 lane 0 = every tcgen05.mma, warp 9 lane 0 = every TMA load
// and the unit claims, warps 10-11 idle.  Every wait is bounded as in the
// other kernels.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa_internal.h"

namespace fa {
namespace {

// Status words of this translation unit (see read_and_clear_status_d256).
__device__ int g_status = 0;
__device__ int g_status_site = 0;

#include "sm100_helpers.cuh"

constexpr int DH = 256;             // head dimension
constexpr int BM = 128;             // query rows per unit
constexpr int BN = 64;              // keys per tile
constexpr int THREADS = 384;
constexpr int W_MMA = 8;
constexpr int W_TMA = 9;
constexpr uint32_t TMEM_COLS_D256 = 512;
constexpr uint32_t COL_S = 0;       // S buffers at 0 and 64
constexpr uint32_t COL_O = 128;     // O: 256 columns
constexpr int HEAD_GROUP = 8;       // causal claim order: longest first within groups of heads
constexpr uint32_t READERS = 1 + 2 * BM;  // MMA lane + softmax + correction warpgroups

template <bool BF16>
struct Pol {
    static constexpr float TAU = 8.0f;
    static constexpr bool NORM_BY_ROUNDED_P = BF16;
};
constexpr float KAPPA = 0.125f;

struct L {
    static constexpr int Q_CHUNK = BM * 128;        // [128 rows][64 cols]
    static constexpr int KV_CHUNK = BN * 128;       // [64 rows][64 cols]
    static constexpr int Q_BYTES = BM * DH * 2;     // 64 KiB
    static constexpr int KV_BYTES = BN * DH * 2;    // 32 KiB
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_BYTES;                  // 2 slots
    static constexpr int V_OFF = K_OFF + 2 * KV_BYTES;     // 2 slots
    static constexpr int ALPHA_OFF = V_OFF + 2 * KV_BYTES;  // float[2][128]
    static constexpr int FIN_OFF = ALPHA_OFF + 2 * BM * 4;  // float2[2][128]
    static constexpr int BAR_OFF = FIN_OFF + 2 * BM * 8;
    enum {
        B_QFULL = 0,
        B_QEMPTY,
        B_OREADY,               // P_j V_j has completed (O may be rescaled)
        B_OFULL,                // the unit's last P.V has completed
        B_FIN,
        B_KFULL,                // [2]
        B_KEMPTY = B_KFULL + 2,
        B_VFULL = B_KEMPTY + 2,
        B_VEMPTY = B_VFULL + 2,
        B_SFULL = B_VEMPTY + 2,  // [2] per S buffer
        B_PFULL = B_SFULL + 2,   // [2] softmax + correction
        B_STATS = B_PFULL + 2,   // [2] rescale factors ready
        B_FINAL = B_STATS + 2,   // [2] by unit parity
        B_UFULL = B_FINAL + 2,
        B_UEMPTY = B_UFULL + 2,
        NBAR = B_UEMPTY + 2
    };
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    static constexpr int UNIT_OFF = MISC_OFF + 16;
    static constexpr int BYTES = UNIT_OFF + 8;
    static constexpr int ALLOC = BYTES + 1024;
};
static_assert(L::ALLOC <= 232448, "shared memory budget exceeded");

struct Params {
    CUtensorMap tmap_q;   // box {64, 128, 1, 1}
    CUtensorMap tmap_k;   // box {64, 64, 1, 1}
    CUtensorMap tmap_v;
    uint8_t* o;
    float* lse;
    long long o_sb, o_sh, o_ss;  // byte strides of O
    int BH, H, Sq, Sk, n_mtiles, n_units, nkv, causal, causal_off;
    float scale_log2;
    unsigned int* sched;
    int sched_reset;  // the last CTA to finish zeroes sched[0] and sched[1] for the next launch
    const uint8_t* mask;         // explicit boolean mask (MASK kernels): nonzero = attend
    long long m_sb, m_sh, m_ss;  // its element strides over b, h and the query row
    uint32_t drop_p8x4, seed_lo, seed_hi, drop_offset;  // dropout (DROP kernels)
    float keep_scale;            // 1 / (1 - p), or 1
};

// The mask bytes of keys [kbase, kbase + 64) of one query row as 64 bits (bit c
// of word c / 32 = key kbase + c may be attended); keys at or past Sk read as
// 0.  Four 16-byte loads for a whole tile (row and tile start 16-byte
// aligned), byte loads on the ragged last one.
__device__ __forceinline__ void mask_bits64(const uint8_t* mrow, int kbase, int Sk, uint32_t (&bits)[2]) {
    if (kbase + BN <= Sk) {
        const uint4* src = reinterpret_cast<const uint4*>(mrow + kbase);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            uint32_t acc = 0;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const uint4 x = __ldg(src + 2 * q + hh);
                const uint32_t ws[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    // one bit per nonzero byte, gathered into a nibble (byte i -> bit i)
                    const uint32_t t = __vcmpne4(ws[e], 0u) & 0x01010101u;
                    acc |= ((t * 0x01020408u) >> 24 & 0xFu) << (16 * hh + 4 * e);
                }
            }
            bits[q] = acc;
        }
    } else {
        bits[0] = bits[1] = 0u;
        for (int c = 0; c < Sk - kbase; ++c)
            if (mrow[kbase + c]) bits[c >> 5] |= 1u << (c & 31);
    }
}

struct U256 {
    int bh, q0, n;  // head, first query row, key tiles visited
};

__device__ __forceinline__ U256 decode(const Params& p, int u) {
    U256 U;
    int m;
    if (p.causal) {
        const int per_group = HEAD_GROUP * p.n_mtiles;
        const int g = u / per_group;
        const int within = u - g * per_group;
        const int gh = min(HEAD_GROUP, p.BH - g * HEAD_GROUP);
        m = p.n_mtiles - 1 - within / gh;
        U.bh = g * HEAD_GROUP + within % gh;
    } else {
        U.bh = u / p.n_mtiles;
        m = u - U.bh * p.n_mtiles;
    }
    U.q0 = m * BM;
    U.n = p.causal ? min((U.q0 + BM - 1 + p.causal_off) / BN + 1, p.nkv) : p.nkv;
    return U;
}

__host__ __device__ constexpr uint32_t idesc(bool bf16, int N, bool b_mn) {
    return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

template <bool BF16>
__device__ __forceinline__ uint32_t pk2(float lo, float hi) {
    uint32_t r;
    if constexpr (BF16) asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    else asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float2 add_bf16_pair(float2 acc, uint32_t pk) {
    float2 r;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "mov.b32 {lo, hi}, %2;\n\t"
        "add.rn.f32.bf16 %0, lo, %3;\n\t"
        "add.rn.f32.bf16 %1, hi, %4;\n\t}"
        : "=r"(*reinterpret_cast<uint32_t*>(&r.x)), "=r"(*reinterpret_cast<uint32_t*>(&r.y))
        : "r"(pk), "f"(acc.x), "f"(acc.y));
    return r;
}

struct Reader {
    int slot = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ int next(uint8_t* smem, volatile uint32_t* abort_flag, int site) {
        const uint32_t bar0 = smem_u32(smem) + L::BAR_OFF;
        if (!mbar_wait(bar0 + 8u * (uint32_t)(L::B_UFULL + slot), phase, abort_flag, site)) return -2;
        const int u = reinterpret_cast<volatile int*>(smem + L::UNIT_OFF)[slot];
        mbar_arrive(bar0 + 8u * (uint32_t)(L::B_UEMPTY + slot));
        if (++slot == 2) { slot = 0; phase ^= 1u; }
        return u;
    }
};

__device__ void producer(const Params& p, uint8_t* smem, volatile uint32_t* abort_flag) {
    const uint32_t base = smem_u32(smem);
    const uint32_t bar0 = base + L::BAR_OFF;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    volatile int* ring = reinterpret_cast<volatile int*>(smem + L::UNIT_OFF);
    int uslot = 0;
    uint32_t uphase = 0, qe_phase = 0;
    uint32_t kq = 0, vq = 0;  // global K and V tile counts (ring slot = count & 1)
    bool ok = true;
    int last_q = -1;
    uint32_t kmask = 0, kpar = 0, vmask = 0, vpar = 0;
    auto load_k = [&](const U256& U, int b, int h, int j) -> bool {
        const int s = (int)(kq & 1u);
        const uint32_t ph = (kq >> 1) & 1u;
        if (!mbar_wait(bar(L::B_KEMPTY + s), ph ^ 1u, abort_flag, 81)) return false;
        mbar_expect_tx(bar(L::B_KFULL + s), L::KV_BYTES);
        kmask |= 1u << s;
        kpar = (kpar & ~(1u << s)) | (ph << s);
#pragma unroll
        for (int c = 0; c < 4; ++c)
            tma_load_4d(base + L::K_OFF + s * L::KV_BYTES + c * L::KV_CHUNK, &p.tmap_k, bar(L::B_KFULL + s), c * 64,
                        j * BN, h, b);
        ++kq;
        return true;
    };
    auto load_v = [&](const U256& U, int b, int h, int j) -> bool {
        const int s = (int)(vq & 1u);
        const uint32_t ph = (vq >> 1) & 1u;
        if (!mbar_wait(bar(L::B_VEMPTY + s), ph ^ 1u, abort_flag, 82)) return false;
        mbar_expect_tx(bar(L::B_VFULL + s), L::KV_BYTES);
        vmask |= 1u << s;
        vpar = (vpar & ~(1u << s)) | (ph << s);
#pragma unroll
        for (int c = 0; c < 4; ++c)
            tma_load_4d(base + L::V_OFF + s * L::KV_BYTES + c * L::KV_CHUNK, &p.tmap_v, bar(L::B_VFULL + s), c * 64,
                        j * BN, h, b);
        ++vq;
        return true;
    };
    for (int k = 0;; ++k) {
        int u = p.sched ? (int)atomicAdd(p.sched, 1u) : (int)blockIdx.x + k * (int)gridDim.x;
        if (u >= p.n_units) u = -1;
        if (!mbar_wait(bar(L::B_UEMPTY + uslot), uphase ^ 1u, abort_flag, 80)) { ok = false; break; }
        ring[uslot] = u;
        mbar_arrive(bar(L::B_UFULL + uslot));
        if (++uslot == 2) { uslot = 0; uphase ^= 1u; }
        if (u < 0) break;
        const U256 U = decode(p, u);
        const int b = U.bh / p.H, h = U.bh - b * p.H;
        if (!mbar_wait(bar(L::B_QEMPTY), qe_phase ^ 1u, abort_flag, 83)) { ok = false; break; }
        mbar_expect_tx(bar(L::B_QFULL), L::Q_BYTES);
        last_q = (int)qe_phase;
        qe_phase ^= 1u;
#pragma unroll
        for (int c = 0; c < 4; ++c)
            tma_load_4d(base + L::Q_OFF + c * L::Q_CHUNK, &p.tmap_q, bar(L::B_QFULL), c * 64, U.q0, h, b);
        // K runs two tiles ahead of V: K_0, K_1, then V_j, K_{j+2}
        if (!load_k(U, b, h, 0)) { ok = false; break; }
        if (U.n > 1 && !load_k(U, b, h, 1)) { ok = false; break; }
        for (int j = 0; j < U.n; ++j) {
            if (!load_v(U, b, h, j)) { ok = false; break; }
            if (j + 2 < U.n && !load_k(U, b, h, j + 2)) { ok = false; break; }
        }
        if (!ok) break;
    }
    if (!ok) {
        for (int i = 0; i < 2; ++i) {
            if (kmask & (1u << i)) mbar_drain(bar(L::B_KFULL + i), (kpar >> i) & 1u);
            if (vmask & (1u << i)) mbar_drain(bar(L::B_VFULL + i), (vpar >> i) & 1u);
        }
        if (last_q >= 0) mbar_drain(bar(L::B_QFULL), (uint32_t)last_q);
    }
}

template <bool BF16>
__device__ void mma(const Params& p, uint8_t* smem, uint32_t tmem, volatile uint32_t* abort_flag) {
    const uint32_t base = smem_u32(smem);
    const uint32_t bar0 = base + L::BAR_OFF;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    constexpr uint32_t ID_S = idesc(BF16, BN, false);   // S = Q K^T: N = 64 keys
    constexpr uint32_t ID_PV = idesc(BF16, DH, true);   // O += P V: N = 256, V read MN-major
    // Q (K-major, [128 rows][256], 64-column chunks 16 KiB apart), K (K-major,
    // [64 rows][256], chunks 8 KiB apart): a K step of 16 elements is +32 bytes
    // in a chunk.  V (MN-major, [64 keys][256]): 64-column chunks 8 KiB apart
    // (leading byte offset), 8-row groups 1 KiB apart, 16 keys +2 KiB.
    const uint64_t dq = sw128_desc(base + L::Q_OFF, 16, 1024);
    const uint64_t dk = sw128_desc(base + L::K_OFF, 16, 1024);
    const uint64_t dv = sw128_desc(base + L::V_OFF, (uint32_t)L::KV_CHUNK, 1024);
    const uint32_t dq_lo = (uint32_t)dq, dq_hi = (uint32_t)(dq >> 32);
    const uint32_t dk_lo = (uint32_t)dk, dk_hi = (uint32_t)(dk >> 32);
    const uint32_t dv_lo = (uint32_t)dv, dv_hi = (uint32_t)(dv >> 32);
    constexpr uint32_t KV16 = (uint32_t)L::KV_BYTES >> 4;

    uint32_t kq = 0, vq = 0, qf_phase = 0, uo = 0;
    uint32_t p_phase[2] = {0u, 0u};
    bool ok = true;
    // S_j = Q K_j^T into S buffer sb; releases K_j
    auto issue_s = [&](int sb) -> bool {
        const int s = (int)(kq & 1u);
        if (!mbar_wait(bar(L::B_KFULL + s), (kq >> 1) & 1u, abort_flag, 84)) return false;
        ++kq;
#pragma unroll
        for (int ks = 0; ks < DH / 16; ++ks) {
            const uint32_t qo = (uint32_t)(((ks & 3) * 32 + (ks >> 2) * L::Q_CHUNK) >> 4);
            const uint32_t ko = (uint32_t)(((ks & 3) * 32 + (ks >> 2) * L::KV_CHUNK) >> 4);
            tc_mma_ss2(tmem + COL_S + 64u * (uint32_t)sb, dq_lo + qo, dq_hi, dk_lo + (uint32_t)s * KV16 + ko, dk_hi, ID_S,
                       ks > 0 ? 1u : 0u);
        }
        tc_commit(bar(L::B_SFULL + sb));
        tc_commit(bar(L::B_KEMPTY + s));
        return true;
    };
    Reader units;
    for (;;) {
        const int u = units.next(smem, abort_flag, 85);
        if (u < 0) break;
        const U256 U = decode(p, u);
        if (!mbar_wait(bar(L::B_QFULL), qf_phase, abort_flag, 86)) { ok = false; break; }
        qf_phase ^= 1u;
        if (!issue_s(0)) { ok = false; break; }
        if (U.n > 1 && !issue_s(1)) { ok = false; break; }
        if (U.n <= 2) tc_commit(bar(L::B_QEMPTY));  // the unit's last S has been issued
        for (int j = 0; j < U.n; ++j) {
            const int sb = j & 1;
            // P_j written and O corrected for tile j
            if (!mbar_wait(bar(L::B_PFULL + sb), p_phase[sb], abort_flag, 87)) { ok = false; break; }
            p_phase[sb] ^= 1u;
            tc_fence_after();
            const int vs = (int)(vq & 1u);
            if (!mbar_wait(bar(L::B_VFULL + vs), (vq >> 1) & 1u, abort_flag, 88)) { ok = false; break; }
            ++vq;
#pragma unroll
            for (int ks = 0; ks < BN / 16; ++ks)
                tc_mma_ts2(tmem + COL_O, tmem + COL_S + 64u * (uint32_t)sb + (uint32_t)(ks * 8),
                           dv_lo + (uint32_t)vs * KV16 + (uint32_t)(ks * (2048 >> 4)), dv_hi, ID_PV,
                           (j > 0 || ks > 0) ? 1u : 0u);
            tc_commit(bar(L::B_VEMPTY + vs));
            tc_commit(bar(L::B_OREADY));
            if (j == U.n - 1) tc_commit(bar(L::B_OFULL));
            if (j + 2 < U.n) {
                // S_{j+2} reuses buffer sb: P_j has been read by the P.V above (in order)
                if (!issue_s(sb)) { ok = false; break; }
                if (j + 2 == U.n - 1) tc_commit(bar(L::B_QEMPTY));
            }
        }
        if (!ok) break;
        ++uo;
    }
    (void)uo;
    tc_commit(bar(L::B_FIN));
    mbar_drain(bar(L::B_FIN), 0u);
}

template <bool BF16, bool MASK, bool DROP>
__device__ void softmax(const Params& p, uint8_t* smem, uint32_t tmem, int warp_in_group,
                        volatile uint32_t* abort_flag) {
    const uint32_t base = smem_u32(smem);
    const uint32_t bar0 = base + L::BAR_OFF;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    const int lane = threadIdx.x & 31;
    const int r_in = warp_in_group * 32 + lane;
    const uint32_t lane_sel = (uint32_t)(warp_in_group * 32) << 16;
    float* alpha_buf = reinterpret_cast<float*>(smem + L::ALPHA_OFF);
    float2* fin_buf = reinterpret_cast<float2*>(smem + L::FIN_OFF);
    const float sl2 = p.scale_log2;
    uint32_t s_phase[2] = {0u, 0u};
    int fin_par = 0;
    Reader units;
    for (;;) {
        const int u = units.next(smem, abort_flag, 89);
        if (!__all_sync(0xffffffffu, u != -2)) return;
        if (u < 0) break;
        const U256 U = decode(p, u);
        const int row = U.q0 + r_in;
        const int key_limit = p.causal ? min(row + p.causal_off, p.Sk - 1) : p.Sk - 1;
        float m_use = -INFINITY, l = 0.f, lr = 0.f;
        // explicit mask: this row's bits for the next key tile, loaded while the
        // previous tile's MMAs run (rows past Sq read the last row)
        const uint8_t* mrow = nullptr;
        uint32_t mbits[2] = {0u, 0u};
        if constexpr (MASK) {
            const int ub = U.bh / p.H, uh = U.bh - ub * p.H;
            mrow = p.mask + (long long)ub * p.m_sb + (long long)uh * p.m_sh + (long long)min(row, p.Sq - 1) * p.m_ss;
            mask_bits64(mrow, 0, p.Sk, mbits);
        }
        for (int j = 0; j < U.n; ++j) {
            const int sb = j & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_SFULL + sb), s_phase[sb], abort_flag, 90))) return;
            s_phase[sb] ^= 1u;
            tc_fence_after();
            const uint32_t ts = tmem + lane_sel + COL_S + 64u * (uint32_t)sb;
            uint32_t sr0[32], sr1[32];
            tmem_ld32u(ts, sr0);
            tmem_ld32u(ts + 32, sr1);
            float s[BN];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                s[c] = __uint_as_float(sr0[c]);
                s[32 + c] = __uint_as_float(sr1[c]);
            }
            const int kbase = j * BN;
            const bool need_mask = (kbase + BN > p.Sk) || (p.causal && kbase + BN - 1 > U.q0 + p.causal_off);
            if (need_mask) {
                const int lim = key_limit - kbase;
#pragma unroll
                for (int c = 0; c < BN; ++c)
                    if (c > lim) s[c] = -INFINITY;
            }
            if constexpr (MASK) {
#pragma unroll
                for (int c = 0; c < BN; ++c)
                    if (!((mbits[c >> 5] >> (c & 31)) & 1u)) s[c] = -INFINITY;
            }
            float mx = s[0];
#pragma unroll
            for (int c = 1; c < BN; ++c) mx = fmaxf(mx, s[c]);
            const float m_blk = mx * sl2;
            bool grow = m_blk > m_use + Pol<BF16>::TAU;
            if constexpr (BF16) grow = grow || (m_blk > m_use && ex2(m_blk - m_use) > KAPPA * lr);
            float alpha = 1.f;
            if (grow) {
                alpha = (m_use == -INFINITY) ? 0.f : ex2(m_use - m_blk);
                m_use = m_blk;
                l *= alpha;
                lr *= alpha;
            }
            if (j > 0) {
                alpha_buf[sb * BM + r_in] = alpha;
                mbar_arrive(bar(L::B_STATS + sb));
            }
            const float neg_m = (m_use == -INFINITY) ? 0.f : -m_use;
            float ls = 0.f;
            float2 rs = make_float2(0.f, 0.f);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t pk[16];
                // dropout: keep masks of the half's 32 keys (two 16-key generator blocks)
                uint32_t km[8];
                if constexpr (DROP) {
                    const uint32_t g0 = (uint32_t)(kbase + 32 * h) >> 4;
                    const uint4 a = dropout_keep_bytes(g0, (uint32_t)row, (uint32_t)U.bh, p.drop_offset, p.seed_lo,
                                                       p.seed_hi, p.drop_p8x4);
                    const uint4 b = dropout_keep_bytes(g0 + 1u, (uint32_t)row, (uint32_t)U.bh, p.drop_offset,
                                                       p.seed_lo, p.seed_hi, p.drop_p8x4);
                    km[0] = a.x; km[1] = a.y; km[2] = a.z; km[3] = a.w;
                    km[4] = b.x; km[5] = b.y; km[6] = b.z; km[7] = b.w;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float e0 = ex2(fmaf(s[32 * h + 2 * i], sl2, neg_m));
                    const float e1 = ex2(fmaf(s[32 * h + 2 * i + 1], sl2, neg_m));
                    pk[i] = pk2<BF16>(e0, e1);
                    ls += e0 + e1;
                    if constexpr (Pol<BF16>::NORM_BY_ROUNDED_P) rs = add_bf16_pair(rs, pk[i]);
                    // the sums keep every weight; P.V sees only the kept ones (keys 2i and
                    // 2i + 1 are bytes 2i and 2i + 1 of the half's mask: each byte fills a half)
                    if constexpr (DROP) pk[i] &= __byte_perm(km[i >> 1], 0u, (i & 1) ? 0x3322u : 0x1100u);
                }
                // P (16-bit pairs) over the first 32 columns of this S buffer
                tmem_st16(ts + 16 * h, pk);
            }
            l += ls;
            if constexpr (Pol<BF16>::NORM_BY_ROUNDED_P) lr += rs.x + rs.y;
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(L::B_PFULL + sb));
            if constexpr (MASK) {
                if (j + 1 < U.n) mask_bits64(mrow, kbase + BN, p.Sk, mbits);
            }
        }
        const float norm = Pol<BF16>::NORM_BY_ROUNDED_P ? lr : l;
        fin_buf[fin_par * BM + r_in] = (l > 0.f)
            ? make_float2(p.keep_scale / norm, (m_use + __log2f(l)) * 0.69314718055994530942f)
            : make_float2(0.f, -INFINITY);
        mbar_arrive(bar(L::B_FINAL + fin_par));
        fin_par ^= 1;
    }
}

template <bool BF16>
__device__ void correction(const Params& p, uint8_t* smem, uint32_t tmem, int warp_in_group,
                           volatile uint32_t* abort_flag) {
    const uint32_t base = smem_u32(smem);
    const uint32_t bar0 = base + L::BAR_OFF;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    const int lane = threadIdx.x & 31;
    const int r_in = warp_in_group * 32 + lane;
    const uint32_t lane_sel = (uint32_t)(warp_in_group * 32) << 16;
    const uint32_t to = tmem + lane_sel + COL_O;
    const float* alpha_buf = reinterpret_cast<const float*>(smem + L::ALPHA_OFF);
    const float2* fin_buf = reinterpret_cast<const float2*>(smem + L::FIN_OFF);
    uint32_t st_phase[2] = {0u, 0u}, fi_phase[2] = {0u, 0u}, of_phase = 0;
    uint32_t npv = 0;  // P.V completions so far (B_OREADY)
    int fin_par = 0;
    Reader units;
    for (;;) {
        const int u = units.next(smem, abort_flag, 91);
        if (!__all_sync(0xffffffffu, u != -2)) return;
        if (u < 0) break;
        const U256 U = decode(p, u);
        for (int j = 0; j < U.n; ++j) {
            const int sb = j & 1;
            if (j > 0) {
                // this tile's factors, and P_{j-1} V_{j-1} complete, before touching O
                if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_STATS + sb), st_phase[sb], abort_flag, 92))) return;
                st_phase[sb] ^= 1u;
                if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_OREADY), (npv - 1u) & 1u, abort_flag, 93))) return;
                const float alpha = alpha_buf[sb * BM + r_in];
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < DH / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld32u(to + 32 * c, r);
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                        tmem_st32(to + 32 * c, r);
                    }
                    tmem_wait_st();
                }
            }
            tc_fence_before();
            mbar_arrive(bar(L::B_PFULL + sb));
            ++npv;
        }
        // epilogue: O / l -> 16 bits -> global; LSE
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_FINAL + fin_par), fi_phase[fin_par], abort_flag, 94)))
            return;
        fi_phase[fin_par] ^= 1u;
        const float2 fin = fin_buf[fin_par * BM + r_in];
        fin_par ^= 1;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_OFULL), of_phase, abort_flag, 95))) return;
        of_phase ^= 1u;
        tc_fence_after();
        const int row = U.q0 + r_in;
        const bool valid = row < p.Sq;
        const int ub = U.bh / p.H, uh = U.bh - ub * p.H;
        uint8_t* orow = p.o + (long long)ub * p.o_sb + (long long)uh * p.o_sh + (long long)(valid ? row : 0) * p.o_ss;
#pragma unroll 1
        for (int c = 0; c < DH / 32; ++c) {
            uint32_t r[32];
            tmem_ld32u(to + 32 * c, r);
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                w[i] = pk2<BF16>(__uint_as_float(r[2 * i]) * fin.x, __uint_as_float(r[2 * i + 1]) * fin.x);
            if (valid) {
                uint4* dst = reinterpret_cast<uint4*>(orow + c * 64);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
            }
        }
        if (valid) p.lse[(size_t)U.bh * (size_t)p.Sq + row] = fin.y;
        // O is read: the next unit's first P.V may overwrite it (its tile-0 arrival
        // on B_PFULL comes after this point in this warpgroup's program order)
        tc_fence_before();
    }
}

template <bool BF16, bool MASK, bool DROP>
__global__ void __launch_bounds__(THREADS, 1) fa_fwd_kernel_d256(const __grid_constant__ Params p) {
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
            if ((i >= L::B_STATS && i < L::B_STATS + 2) || (i >= L::B_FINAL && i < L::B_FINAL + 2)) count = BM;
            if (i >= L::B_PFULL && i < L::B_PFULL + 2) count = 2 * BM;
            if (i >= L::B_UEMPTY && i < L::B_UEMPTY + 2) count = READERS;
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
    }
    if (warp == W_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(misc)),
                     "r"(TMEM_COLS_D256)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    grid_dependency_sync();  // the previous kernel in the stream has completed
    if (wg == 0) {
        softmax<BF16, MASK, DROP>(p, smem, tmem, warp & 3, abort_flag);
    } else if (wg == 1) {
        correction<BF16>(p, smem, tmem, warp & 3, abort_flag);
    } else {
        if (warp == W_TMA && lane == 0) producer(p, smem, abort_flag);
        if (warp == W_MMA && lane == 0) mma<BF16>(p, smem, tmem, abort_flag);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == W_MMA) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS_D256)
                     : "memory");
    }
    if (p.sched_reset && threadIdx.x == 0) {
        // as in the D = 64/128 kernel: the last CTA clears the counter and the count
        __threadfence();
        if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1u) {
            __threadfence();
            atomicExch(p.sched, 0u);
            atomicExch(p.sched + 1, 0u);
        }
    }
}

template <bool BF16, bool MASK, bool DROP>
cudaError_t launch_impl(const LaunchArgs& a, cudaStream_t stream) {
    auto kern = fa_fwd_kernel_d256<BF16, MASK, DROP>;
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), L::ALLOC);
    if (e != cudaSuccess) return e;
    Params p;
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
    p.n_mtiles = (a.Sq + BM - 1) / BM;
    p.n_units = p.BH * p.n_mtiles;
    p.nkv = (a.Sk + BN - 1) / BN;
    p.causal = a.causal;
    p.causal_off = a.Sk - a.Sq;
    p.scale_log2 = a.scale_log2;
    p.sched = a.sched;
    p.sched_reset = a.sched_reset;
    p.mask = a.mask;
    p.m_sb = a.mask_stride[0];
    p.m_sh = a.mask_stride[1];
    p.m_ss = a.mask_stride[2];
    p.drop_p8x4 = a.drop.p8 * 0x01010101u;
    p.seed_lo = a.drop.seed_lo;
    p.seed_hi = a.drop.seed_hi;
    p.drop_offset = a.drop.offset;
    p.keep_scale = a.drop.enabled ? a.drop.keep_scale : 1.f;
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

int64_t num_units_d256(int64_t BH, int64_t Sq) { return BH * ((Sq + BM - 1) / BM); }

template <bool BF16>
cudaError_t launch_dtype(const LaunchArgs& a, cudaStream_t stream) {
    if (a.drop.enabled)
        return a.mask ? launch_impl<BF16, true, true>(a, stream) : launch_impl<BF16, false, true>(a, stream);
    return a.mask ? launch_impl<BF16, true, false>(a, stream) : launch_impl<BF16, false, false>(a, stream);
}

cudaError_t launch_fwd_d256_sm100(const LaunchArgs& a, cudaStream_t stream) {
    return a.dtype == 1 ? launch_dtype<true>(a, stream) : launch_dtype<false>(a, stream);
}

cudaError_t read_and_clear_status_d256(cudaStream_t stream, int* status, int* site) {
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
