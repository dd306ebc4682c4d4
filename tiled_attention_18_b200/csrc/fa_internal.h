// fa_internal.h -- declarations shared by the host layer (fa_api.cpp) and the
// sm_100a kernel translation unit (fa_fwd_sm100.cu).  Not part of the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace fa {

// Tile shape of the forward kernel: a CTA owns two query tiles of BLOCK_M
// rows each and streams keys/values in tiles of BLOCK_N rows.
constexpr int BLOCK_M = 128;
constexpr int BLOCK_N = 128;
constexpr int Q_TILES_PER_CTA = 2;
constexpr int ROWS_PER_UNIT = BLOCK_M * Q_TILES_PER_CTA;
// Short key sets (at most one key tile per head) take the short-key kernel
// when the tiling is automatic and there is no explicit mask or dropout.
constexpr int SHORT_SK_MAX = 128;
// The backward's fp32 dK/dV partial sums, used when a key set of at most this
// many keys gives fewer work units than SMs (the query range is then split
// across units): [B*H][KV_ACC_ROWS][D] each, in the workspace.
constexpr int KV_ACC_ROWS = 128;

// Device-side status codes written to the status word by the kernel.
constexpr int DEV_OK = 0;
constexpr int DEV_TIMEOUT = 1;
// Wait-site code of the diagnostic timeout kernel (low byte of the site word).
constexpr int SELFTEST_SITE = 100;

// Attention dropout after the softmax: the weight of query q and key j of
// head bh is kept iff byte j mod 16 of Philox4x32-10(counter (j / 16, q, bh,
// offset), key (seed_lo, seed_hi)) is >= p8; kept weights are scaled by
// keep_scale = 256 / (256 - p8).
struct DropoutArgs {
    int enabled;
    uint32_t p8;            // drop threshold in 1/256 units, 0 .. 255
    uint32_t seed_lo, seed_hi;
    uint32_t offset;
    float keep_scale;
};

struct LaunchArgs {
    CUtensorMap tmap_q;     // 4-D maps over [B][H][S][D] (innermost first: D, S, H, B) with
    CUtensorMap tmap_k;     // the tensors' own strides, box {64, 128, 1, 1}, 128-byte swizzle
    CUtensorMap tmap_v;
    CUtensorMap tmap_o;     // short-key kernel only: the output, box {64, 128, 1, 1}
    void* o;                // [B,H,Sq,D] 16-bit at o_stride
    float* lse;             // [B,H,Sq] fp32, contiguous
    long long o_stride[3];  // element strides of O over b, h, s (d is contiguous)
    const uint8_t* mask;    // explicit boolean mask (nonzero = attend) or null
    long long mask_stride[3];  // its element strides over b, h, query row (keys contiguous)
    DropoutArgs drop;       // dropout (drop.enabled = 0: none)
    int B;
    int H;
    int Sq;                 // query rows per head
    int Sk;                 // key/value rows per head (Sk >= Sq under the causal mask)
    int D;
    int dtype;              // 0 fp16, 1 bf16
    int causal;
    float scale_log2;       // scale * log2(e)
    int grid;               // persistent CTAs
    unsigned int* sched;    // zeroed device counter for claimed-unit scheduling, or null
    int sched_reset;        // the launch zeroes sched[0] and sched[1] again as its last CTA ends
    int block_n;            // keys per key tile: 128 (default) or 64 (D = 64/128 kernel)
    int q_tiles;            // 128-row query tiles per work unit: 2 (default) or 1
};

// Backward pass (fa_bwd): tensor maps as for the forward pass (Q, dO over
// [B][H][Sq][D]; K, V over [B][H][Sk][D]), the forward outputs O and LSE, the
// gradients, and the caller's workspace carved as bwd_workspace_layout says.
struct BwdLaunchArgs {
    CUtensorMap tmap_q;
    CUtensorMap tmap_k;
    CUtensorMap tmap_v;
    CUtensorMap tmap_do;
    CUtensorMap tmap_dq;    // fp32 dQ accumulator [BH][Sq][D], box {128, 64, 1}, for bulk reduce-add
    const void* o;          // [B,H,Sq,D] 16-bit at o_stride
    const void* dout;       // [B,H,Sq,D] 16-bit at do_stride
    // element strides over b, h and the row (d contiguous) of O, dO and the gradients
    long long o_stride[3], do_stride[3], dq_stride[3], dk_stride[3], dv_stride[3];
    const float* lse;       // [B,H,Sq] fp32 (natural log)
    void* dq;               // [B,H,Sq,D] 16-bit
    void* dk;               // [B,H,Sk,D] 16-bit
    void* dv;               // [B,H,Sk,D] 16-bit
    float* dq_acc;          // workspace: [B*H][Sq][D] fp32
    float* dk_acc;          // workspace: [B*H][KV_ACC_ROWS][D] fp32 dK partial sums (split query range)
    float* dv_acc;          // workspace: the same for dV
    float* lse2;            // workspace: [B*H][Sq_pad] fp32
    float* delta;           // workspace: [B*H][Sq_pad] fp32
    unsigned int* sched;    // workspace: unit counter
    int* dq_flags;          // workspace: deterministic-mode turn counters, or null (atomic mode)
    const uint8_t* mask;    // explicit boolean mask or null
    long long mask_stride[3];
    DropoutArgs drop;       // dropout (drop.enabled = 0: none)
    int B;
    int H;
    int Sq;
    int Sk;
    int D;
    int dtype;
    int causal;
    float scale;
    int grid;
    int sms;                // SMs of the device (the split decision sizes units against it)
};

// Byte offsets of the backward workspace parts (each 256-byte aligned) and
// its total size.  Sq_pad = Sq rounded up to a multiple of 128.
struct BwdWorkspace {
    int64_t dq_acc, lse2, delta, flags, flags_bytes, sched, kv_acc, total;
};
inline BwdWorkspace bwd_workspace_layout(int64_t BH, int64_t Sq, int64_t D) {
    auto up = [](int64_t x) { return (x + 255) / 256 * 256; };
    const int64_t Sq_pad = (Sq + 127) / 128 * 128;
    BwdWorkspace w;
    w.dq_acc = 0;
    w.lse2 = up(BH * Sq * D * 4);
    w.delta = w.lse2 + up(BH * Sq_pad * 4);
    w.flags = w.delta + up(BH * Sq_pad * 4);
    w.flags_bytes = BH * ((Sq + 63) / 64) * (D == 256 ? 2 : 1) * 4 * 4;  // [BH][64-row steps][D/128 halves][4 warps] int
    w.sched = w.flags + up(w.flags_bytes);
    w.kv_acc = w.sched + 256;
    w.total = w.kv_acc + up(2 * BH * KV_ACC_ROWS * D * 4);
    return w;
}

// LSE-weighted merge of a partial attention result into a running fp32 one,
// and the conversion of the running O to 16 bits (fa_merge_sm100.cu).
// Raises `kernel`'s dynamic shared-memory limit to `bytes` in the current
// context, once per (kernel, context) for the life of the process: later
// launches make no attribute call, so host threads launching at the same time
// never set an attribute of a kernel that another thread is launching.  A
// context re-created after cudaDeviceReset has a new id and is set again.
cudaError_t ensure_smem_limit(const void* kernel, int bytes);

// Programmatic dependent launch.  Every kernel of this library is launched
// with programmatic stream serialization: it may start while the kernel before
// it in the stream is still running (its CTAs take SMs as that kernel's CTAs
// leave them), does its set-up (barriers, tensor memory, descriptor
// prefetches), and then waits in grid_dependency_sync() until that kernel has
// completed and its memory writes are visible, before touching global memory.
// Each kernel also lets its own successor start early.  A kernel launched
// without the attribute, or after work that is not a kernel, passes the wait
// at once.
inline void set_programmatic_launch(cudaLaunchConfig_t& cfg, cudaLaunchAttribute (&attr)[1]) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
}

#ifdef __CUDACC__
// Called by every thread of a CTA before its first global-memory access.
__device__ __forceinline__ void grid_dependency_sync() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
#endif

// Launches `kernel` on `stream` (as a programmatic dependent launch: the
// kernel must call grid_dependency_sync() first) and returns the status of
// this launch alone (cudaGetLastError after a <<<>>> launch would also return
// an error that other code left pending in the calling thread).
template <typename... Expected, typename... Actual>
cudaError_t launch_kernel(void (*kernel)(Expected...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                          Actual&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    set_programmatic_launch(cfg, attr);
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Actual>(args)...);
}

cudaError_t launch_merge_partial(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                                 long long rows, int D, int dtype, cudaStream_t stream);
cudaError_t launch_accumulate(float* acc, const void* x, long long n, int dtype, cudaStream_t stream);
cudaError_t launch_merge_finalize(const float* o_acc, void* o, long long n, int dtype, cudaStream_t stream);

// Launch the three backward kernels (prep, main, post) on `stream`.
cudaError_t launch_bwd_sm100(const BwdLaunchArgs& a, cudaStream_t stream);

// Status words of the backward kernels (same protocol as read_and_clear_status).
cudaError_t read_and_clear_status_bwd(cudaStream_t stream, int* status, int* site);

// Number of work units (b, h, query block of q_tiles x 128 rows).
inline int64_t num_units(int64_t BH, int64_t S, int q_tiles = Q_TILES_PER_CTA) {
    const int64_t rows = (int64_t)q_tiles * BLOCK_M;
    return BH * ((S + rows - 1) / rows);
}

// Launch the persistent forward kernel on `stream`.  Returns a cudaError_t.
cudaError_t launch_fwd_sm100(const LaunchArgs& a, cudaStream_t stream);

// Head dimension 256: its own kernel (one 128-row query tile per work unit,
// 64-key tiles; K/V tensor maps with 64-row boxes), its units and status words.
cudaError_t launch_fwd_d256_sm100(const LaunchArgs& a, cudaStream_t stream);
int64_t num_units_d256(int64_t BH, int64_t Sq);
cudaError_t read_and_clear_status_d256(cudaStream_t stream, int* status, int* site);

// Launch the short-key forward kernel (Sk <= SHORT_SK_MAX, D = 64/128, no mask
// or dropout; K/V maps with a box of Sk rounded up to 16 rows, tmap_o set).
cudaError_t launch_fwd_short_sm100(const LaunchArgs& a, cudaStream_t stream);
// Status word of the short-key kernel's translation unit.
cudaError_t read_and_clear_status_short(cudaStream_t stream, int* status, int* site);

// fa_fwd_noalloc: size of its static scratch array (256 bytes; word 0 is the
// causal unit counter) and the largest number of unit claims the counter
// serves (work units + CTAs, read back as a non-negative int).
constexpr int NOALLOC_SCRATCH_WORDS = 64;
constexpr long long NOALLOC_MAX_CLAIMS = 0x7FFFFFFFll;

// Device address of the static scratch array in the current context (looked
// up once per context, so a context re-created after cudaDeviceReset gets a
// fresh lookup).
cudaError_t noalloc_scratch_address(unsigned int** out);

// Causal work-unit counters of the other forward entries: a static pool of
// SCHED_POOL_SLOTS counters in the library's own device memory, one slot per
// (context, stream) that has launched a causal forward, 32 bytes apart.  The
// pool is part of the loaded module: handing out a slot allocates nothing.
constexpr int SCHED_POOL_SLOTS = 2048;
constexpr int SCHED_SLOT_WORDS = 8;
cudaError_t sched_pool_address(unsigned int** out);

// Unique id of the CUDA context current in the calling thread (the device's
// primary context unless the caller made another current); binds the
// current device's primary context to the thread first if none is current.
cudaError_t current_context_id(unsigned long long* id);

// Launch the diagnostic kernel whose first wait is never satisfied.
cudaError_t launch_selftest_timeout(cudaStream_t stream);

// Read (after synchronising `stream`) and clear the device status word of
// the current device.  *status receives DEV_OK or an error code; *site the
// diagnostic word of the first failing wait.
cudaError_t read_and_clear_status(cudaStream_t stream, int* status, int* site);

}  // namespace fa
