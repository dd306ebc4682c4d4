// fa_api.cpp -- host side of libfa.so: argument validation, TMA tensor-map
// encoding, persistent-grid sizing and the launch (declared in include/fa.h).
//
// The host layer plays the part of the pages' host tiling step (block sizes,
// block counts: "FlashAttention-2 在昇腾 NPU 上如何做到 3 倍加速？" section 3.2)
// and of the host operator entry that returns a status code (the lanjinlin.com.cn
// page "解析CANN ops-transformer的FlashAttention算子", host Compute function),
// except that it never synchronises the stream.
#include "fa.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "fa_internal.h"

namespace {

constexpr int FA_VERSION = 100;  // 0.1.0

// Per-device facts read once: compute capability and SM count.
struct DeviceInfo {
    bool known = false;
    int major = 0;
    int minor = 0;
    int sms = 0;
};

constexpr int MAX_DEVICES = 64;
DeviceInfo g_dev[MAX_DEVICES];
std::mutex g_dev_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

thread_local int t_last_site = 0;

// The CUDA failure behind this thread's most recent FA_ERR_LAUNCH: the
// cudaError_t (or CUresult) code and the name of the call that returned it.
thread_local int t_err_code = 0;
thread_local const char* t_err_site = "";

// Records a failed CUDA call, clears the calling thread's pending error that the
// failure may have left, and returns FA_ERR_LAUNCH.
int cuda_fail(int code, const char* site) {
    t_err_code = code;
    t_err_site = site;
    cudaGetLastError();
    return FA_ERR_LAUNCH;
}

// Causal work-unit counters: (context id, stream) -> its slot in the library's
// static counter pool.  Launches on one stream are ordered, so they can share
// a counter; launches on different streams never do.  Context ids are unique
// for the life of the process, so a context re-created after cudaDeviceReset
// starts with fresh slots (the pool's address is looked up again there).
std::mutex g_ws_mu;
std::map<std::pair<unsigned long long, cudaStream_t>, unsigned int*> g_ws;
std::map<unsigned long long, int> g_ws_used;  // slots handed out per context
// Held from a causal call's counter reset to its launch: two host threads
// launching on one stream must not interleave reset A, reset B, kernel A,
// kernel B (kernel B would find the counter spent and skip its units).
std::mutex g_launch_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_current = nullptr;
CtxGetIdFn g_ctx_id = nullptr;
std::once_flag g_ctx_once;

}  // namespace

namespace fa {

cudaError_t current_context_id(unsigned long long* id) {
    std::call_once(g_ctx_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(fn);
        fn = nullptr;
        q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_id = reinterpret_cast<CtxGetIdFn>(fn);
    });
    if (!g_ctx_current || !g_ctx_id) return cudaErrorNotSupported;
    CUcontext ctx = nullptr;
    if (g_ctx_current(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
    if (!ctx) {
        // no context bound to this thread yet: bind the current device's primary one
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaSetDevice(dev);
        if (e != cudaSuccess) return e;
        if (g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorDeviceUninitialized;
    }
    return g_ctx_id(ctx, id) == CUDA_SUCCESS ? cudaSuccess : cudaErrorDeviceUninitialized;
}

cudaError_t ensure_smem_limit(const void* kernel, int bytes) {
    static std::mutex mu;
    static std::map<std::pair<const void*, unsigned long long>, int> done;  // (kernel, context) -> bytes set
    unsigned long long ctx = 0;
    cudaError_t e = current_context_id(&ctx);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_pair(kernel, ctx);
    auto it = done.find(key);
    if (it != done.end() && it->second >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done[key] = bytes;
    return e;
}

}  // namespace fa

namespace {

// The counter of `stream` in the current context: its slot of the static pool,
// handed out on the stream's first causal launch.  FA_ERR_LIMIT once every slot
// of the context is taken.
int sched_counter(cudaStream_t stream, unsigned int** out) {
    unsigned long long ctx = 0;
    cudaError_t e = fa::current_context_id(&ctx);
    if (e != cudaSuccess) return cuda_fail(e, "cuCtxGetId");
    std::lock_guard<std::mutex> lock(g_ws_mu);
    const auto key = std::make_pair(ctx, stream);
    auto it = g_ws.find(key);
    if (it != g_ws.end()) {
        *out = it->second;
        return FA_OK;
    }
    int& used = g_ws_used[ctx];
    if (used >= fa::SCHED_POOL_SLOTS) return FA_ERR_LIMIT;
    unsigned int* pool = nullptr;
    e = fa::sched_pool_address(&pool);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scheduler pool)");
    unsigned int* ctr = pool + (size_t)used * fa::SCHED_SLOT_WORDS;
    ++used;
    g_ws[key] = ctr;
    *out = ctr;
    return FA_OK;
}

int device_info(DeviceInfo* out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= MAX_DEVICES) return cuda_fail(cudaErrorInvalidDevice, "device index");
    std::lock_guard<std::mutex> lock(g_dev_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.known) {
        e = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        d.known = true;
    }
    *out = d;
    return FA_OK;
}

// cuTensorMapEncodeTiled is a driver call and needs a context current in the
// calling thread; the runtime calls made before it (attribute and pointer
// queries) do not bind one in a thread that has made no other CUDA call.
// Binds the current device's primary context when none is current.
int bind_context() {
    unsigned long long ctx = 0;
    const cudaError_t e = fa::current_context_id(&ctx);
    return e == cudaSuccess ? FA_OK : cuda_fail(e, "cuCtxGetCurrent / cudaSetDevice (binding a context)");
}

EncodeTiledFn encoder() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    });
    return g_encode;
}

// 4-D map over a [B][H][S][D] tensor with the given element strides
// (innermost first: D, S, H, B), box {64, 128, 1, 1}: one 128-byte-wide column
// chunk of 128 rows of one head, 128-byte swizzle (the swizzle atom the
// tcgen05 operand descriptors expect).  Rows past S read as zeros and never
// bleed into the next head, whatever the layout.
// Returns true on success; on failure records the CUresult for fa_last_cuda_error.
bool encode_tensor(CUtensorMap* map, const void* ptr, int B, int H, int S, int D, const long long st[3],
                   int dtype, int box_rows = fa::BLOCK_M) {
    EncodeTiledFn enc = encoder();
    if (!enc) {
        cuda_fail(cudaErrorNotSupported, "cuTensorMapEncodeTiled entry point");
        return false;
    }
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)S, (cuuint64_t)H, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)st[2] * 2, (cuuint64_t)st[1] * 2, (cuuint64_t)st[0] * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
    const cuuint32_t elem[4] = {1, 1, 1, 1};
    const CUtensorMapDataType dt =
        dtype == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUresult r = enc(map, dt, 4, const_cast<void*>(ptr), dims, strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        cuda_fail((int)r, "cuTensorMapEncodeTiled");
        return false;
    }
    return true;
}

// Element strides (b, h, s) of one tensor: the caller's, or contiguous BHSD
// when `given` is null.  A stride over an extent of 1 never moves the address
// and is replaced by the contiguous one.  Returns FA_OK or FA_ERR_STRIDE.
constexpr long long MAX_STRIDE = 1ll << 36;  // elements: 2^37 bytes, well inside TMA's 2^40
int resolve_strides(const long long* given, int B, int H, int S, int D, long long out[3]) {
    const long long contig[3] = {(long long)H * S * D, (long long)S * D, (long long)D};
    const int ext[3] = {B, H, S};
    for (int i = 0; i < 3; ++i) {
        if (!given || ext[i] == 1) {
            out[i] = contig[i];
            continue;
        }
        const long long x = given[i];
        if (x <= 0 || x % 8 != 0 || x >= MAX_STRIDE) return FA_ERR_STRIDE;
        out[i] = x;
    }
    return FA_OK;
}

int check_device_pointer(const void* p, int dev) {
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();  // clear the sticky-free error of a failed query
        return FA_ERR_PTR;
    }
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged) return FA_ERR_PTR;
    if (attr.type == cudaMemoryTypeDevice && attr.device != dev) return FA_ERR_PTR;
    return FA_OK;
}

}  // namespace

extern "C" {

long long fa_num_units(int B, int H, int S) {
    if (B < 0 || H < 0 || S < 0) return FA_ERR_SHAPE;
    if (B == 0 || H == 0 || S == 0) return 0;
    return (long long)fa::num_units((int64_t)B * H, S);
}

}  // extern "C"

namespace {

// Dropout probability -> threshold in 1/256 units (nearest, halves up) and the
// scale of the kept weights; false when p is not finite, negative or rounds to
// 256 (every weight dropped).
bool make_dropout(float p, unsigned long long seed, unsigned int offset, fa::DropoutArgs* d) {
    if (!std::isfinite(p) || p < 0.f) return false;
    const double t = std::floor((double)p * 256.0 + 0.5);
    if (t > 255.0) return false;
    d->enabled = 1;
    d->p8 = (uint32_t)t;
    d->seed_lo = (uint32_t)(seed & 0xffffffffull);
    d->seed_hi = (uint32_t)(seed >> 32);
    d->offset = offset;
    d->keep_scale = (float)(256.0 / (256.0 - t));
    return true;
}

// Where the causal scheduler's counter lives.
enum class Scratch { Allocated, Static };

// The one implementation behind fa_fwd, fa_fwd_ex and fa_fwd_noalloc: checks
// in the documented order, tensor maps, grid size, scheduler counter, launch.
int forward(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Sq, int Sk, int D,
            const long long* q_stride, const long long* k_stride, const long long* v_stride,
            const long long* o_stride, float scale, int causal, int dtype, cudaStream_t stream, Scratch scratch,
            const uint8_t* mask = nullptr, const long long* mask_stride = nullptr,
            const fa::DropoutArgs* drop = nullptr, int block_n = 0, int q_tiles = 0) {
    if (B < 0 || H < 0 || Sq < 0 || Sk < 0) return FA_ERR_SHAPE;
    if (D != 64 && D != 128 && D != 256) return FA_ERR_HEADDIM;
    if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_DTYPE;
    if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_SCALE;
    if (causal != 0 && causal != 1) return FA_ERR_ARG;
    // tiling: 0 = automatic (128-key tiles, two 128-row query tiles per unit);
    // manual tilings for D = 64/128 without an explicit mask or dropout
    if ((block_n != 0 && block_n != 64 && block_n != 128) || (q_tiles < 0 || q_tiles > 2)) return FA_ERR_ARG;
    const bool auto_tiling = block_n == 0 && q_tiles == 0;
    if (block_n == 0) block_n = fa::BLOCK_N;
    if (q_tiles == 0) q_tiles = fa::Q_TILES_PER_CTA;
    const bool manual = block_n != fa::BLOCK_N || q_tiles != fa::Q_TILES_PER_CTA;
    if (manual && (D == 256 || mask || (drop && drop->enabled))) return FA_ERR_ARG;
    if (B == 0 || H == 0 || Sq == 0) return FA_OK;  // empty problem
    // every query row must see at least one key
    if (Sk == 0 || (causal && Sq > Sk)) return FA_ERR_SHAPE;
    const int64_t BH = (int64_t)B * H;
    if (BH > INT_MAX || BH * (int64_t)Sq > INT_MAX || Sq > INT_MAX - 512 || Sk > INT_MAX - 512) return FA_ERR_SHAPE;
    if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
    long long qs[3], ks[3], vs[3], os[3];
    int rc = resolve_strides(q_stride, B, H, Sq, D, qs);
    if (rc == FA_OK) rc = resolve_strides(k_stride, B, H, Sk, D, ks);
    if (rc == FA_OK) rc = resolve_strides(v_stride, B, H, Sk, D, vs);
    if (rc == FA_OK) rc = resolve_strides(o_stride, B, H, Sq, D, os);
    if (rc != FA_OK) return rc;
    long long ms[3] = {0, 0, 0};
    if (mask) {
        // element strides over b, h, query row: 0 broadcasts over b or h; rows
        // at least Sk apart and 16-byte aligned (whole 16-byte loads)
        for (int i = 0; i < 3; ++i) ms[i] = mask_stride[i];
        if (ms[0] < 0 || ms[1] < 0 || ms[0] >= MAX_STRIDE || ms[1] >= MAX_STRIDE || ms[2] >= MAX_STRIDE)
            return FA_ERR_STRIDE;
        if ((ms[2] < Sk && Sq > 1) || ms[2] % 16 != 0 || ms[0] % 16 != 0 || ms[1] % 16 != 0) return FA_ERR_STRIDE;
    }
    const uintptr_t a16 = (uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)o | (uintptr_t)mask;
    if ((a16 & 15u) != 0 || ((uintptr_t)lse & 3u) != 0) return FA_ERR_ALIGN;

    DeviceInfo dev;
    rc = device_info(&dev);
    if (rc != FA_OK) return rc;
    if (dev.major != 10 || dev.minor != 0) return FA_ERR_ARCH;
    rc = bind_context();
    if (rc != FA_OK) return rc;
    int cur = 0;
    const cudaError_t de = cudaGetDevice(&cur);
    if (de != cudaSuccess) return cuda_fail(de, "cudaGetDevice");
    const void* ptrs[6] = {q, k, v, o, lse, mask ? (const void*)mask : (const void*)q};
    for (const void* p : ptrs) {
        rc = check_device_pointer(p, cur);
        if (rc != FA_OK) return rc;
    }
    // every key of a head in one tile: the short-key kernel (query tiles of 128
    // rows, keys and values loaded once per head), with automatic tiling
    const bool short_keys = auto_tiling && D != 256 && !mask && !(drop && drop->enabled) && Sk <= fa::SHORT_SK_MAX;
    const int64_t units = short_keys ? BH * ((Sq + fa::BLOCK_M - 1) / fa::BLOCK_M)
                          : (D == 256) ? fa::num_units_d256(BH, Sq) : fa::num_units(BH, Sq, q_tiles);
    const int grid = (int)(units < dev.sms ? units : dev.sms);
    // fa_fwd_noalloc's counter is read back as an int: the claims of all CTAs must fit
    if (scratch == Scratch::Static && !short_keys && units + grid > fa::NOALLOC_MAX_CLAIMS) return FA_ERR_SHAPE;

    fa::LaunchArgs a;
    std::memset(&a, 0, sizeof(a));
    // the D = 256 kernel streams keys and values in 64-row tiles; the short-key
    // kernel loads all Sk keys of a head at once (rounded up to 16 rows)
    const int kv_box = short_keys ? (Sk + 15) / 16 * 16 : (D == 256) ? 64 : block_n;
    if (!encode_tensor(&a.tmap_q, q, B, H, Sq, D, qs, dtype) ||
        !encode_tensor(&a.tmap_k, k, B, H, Sk, D, ks, dtype, kv_box) ||
        !encode_tensor(&a.tmap_v, v, B, H, Sk, D, vs, dtype, kv_box) ||
        (short_keys && !encode_tensor(&a.tmap_o, o, B, H, Sq, D, os, dtype)))
        return FA_ERR_LAUNCH;
    a.o = o;
    a.lse = lse;
    for (int i = 0; i < 3; ++i) a.o_stride[i] = os[i];
    a.mask = mask;
    for (int i = 0; i < 3; ++i) a.mask_stride[i] = ms[i];
    if (drop) a.drop = *drop;
    a.B = B;
    a.H = H;
    a.Sq = Sq;
    a.Sk = Sk;
    a.D = D;
    a.dtype = dtype;
    a.causal = causal;
    a.scale_log2 = (float)((double)scale * 1.4426950408889634074);  // scale * log2(e)
    a.grid = grid;
    a.sched = nullptr;
    a.block_n = block_n;
    a.q_tiles = q_tiles;
    std::unique_lock<std::mutex> launch_lock(g_launch_mu, std::defer_lock);
    if (causal && !short_keys) {
        // units differ in length under the mask: CTAs claim them from a counter
        launch_lock.lock();
        unsigned int* ctr = nullptr;
        if (scratch == Scratch::Static) {
            const cudaError_t e = fa::noalloc_scratch_address(&ctr);
            if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(fa_fwd_noalloc scratch)");
        } else {
            rc = sched_counter(stream, &ctr);
            if (rc != FA_OK) return rc;
        }
        if (scratch == Scratch::Static) {
            // the shared no-allocation counter keeps the previous call's value:
            // clear it on this stream
            const cudaError_t e = cudaMemsetAsync(ctr, 0, sizeof(unsigned int), stream);
            if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(scheduler counter)");
        } else {
            // a stream's own slot starts zeroed (static memory) and every launch
            // leaves it zeroed: no memset, so the launch can overlap the tail of
            // the kernel before it in the stream
            a.sched_reset = 1;
        }
        a.sched = ctr;
    }
    if (short_keys) {
        const cudaError_t le = fa::launch_fwd_short_sm100(a, stream);
        if (le != cudaSuccess) return cuda_fail(le, "launch(fa_fwd_kernel_short)");
        return FA_OK;
    }
    const cudaError_t le = (D == 256) ? fa::launch_fwd_d256_sm100(a, stream) : fa::launch_fwd_sm100(a, stream);
    if (le != cudaSuccess) return cuda_fail(le, D == 256 ? "launch(fa_fwd_kernel_d256)" : "launch(fa_fwd_kernel)");
    return FA_OK;
}

}  // namespace

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int S, int D,
           float scale, int causal, int dtype, cudaStream_t stream) {
    return forward(q, k, v, o, lse, B, H, S, S, D, nullptr, nullptr, nullptr, nullptr, scale, causal, dtype, stream,
                   Scratch::Allocated);
}

int fa_fwd_mask(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Sq, int Sk,
                int D, const void* mask, const long long* mask_stride, float scale, int causal, int dtype,
                cudaStream_t stream) {
    if (B < 0 || H < 0 || Sq < 0 || Sk < 0) return FA_ERR_SHAPE;
    if (B > 0 && H > 0 && Sq > 0 && (!mask || !mask_stride)) return FA_ERR_NULL;
    return forward(q, k, v, o, lse, B, H, Sq, Sk, D, nullptr, nullptr, nullptr, nullptr, scale, causal, dtype, stream,
                   Scratch::Allocated, static_cast<const uint8_t*>(mask), mask_stride);
}

int fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Sq, int Sk,
                   int D, float scale, int causal, float dropout_p, unsigned long long seed, unsigned int offset,
                   int dtype, cudaStream_t stream) {
    fa::DropoutArgs d;
    std::memset(&d, 0, sizeof(d));
    if (!make_dropout(dropout_p, seed, offset, &d)) return FA_ERR_ARG;
    return forward(q, k, v, o, lse, B, H, Sq, Sk, D, nullptr, nullptr, nullptr, nullptr, scale, causal, dtype, stream,
                   Scratch::Allocated, nullptr, nullptr, &d);
}

int fa_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Sq, int Sk, int D,
              const long long* q_stride, const long long* k_stride, const long long* v_stride,
              const long long* o_stride, float scale, int causal, int dtype, cudaStream_t stream) {
    return forward(q, k, v, o, lse, B, H, Sq, Sk, D, q_stride, k_stride, v_stride, o_stride, scale, causal, dtype,
                   stream, Scratch::Allocated);
}

// For callers that cannot allocate device memory (for example code running
// where cudaMalloc is unavailable or forbidden: inside an allocator, a
// pre-allocated-memory runtime, or a process that must not grow its device
// footprint).  Same computation and arguments as fa_fwd; the causal scheduler's
// counter lives in the library's static scratch array instead of memory the
// library allocates.  Nothing here allocates.
int fa_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int S, int D,
                   float scale, int causal, int dtype, cudaStream_t stream) {
    return forward(q, k, v, o, lse, B, H, S, S, D, nullptr, nullptr, nullptr, nullptr, scale, causal, dtype, stream,
                   Scratch::Static);
}

long long fa_bwd_workspace_size(int B, int H, int Sq, int D) {
    if (B < 0 || H < 0 || Sq < 0) return FA_ERR_SHAPE;
    if (D != 64 && D != 128 && D != 256) return FA_ERR_HEADDIM;
    if (B == 0 || H == 0 || Sq == 0) return 0;
    return (long long)fa::bwd_workspace_layout((int64_t)B * H, Sq, D).total;
}

}  // extern "C"

namespace {

int backward(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse, void* dq,
             void* dk, void* dv, void* workspace, long long workspace_bytes, int B, int H, int Sq, int Sk, int D,
             float scale, int causal, int deterministic, int dtype, cudaStream_t stream, const uint8_t* mask,
             const long long* mask_stride, const fa::DropoutArgs* drop = nullptr,
             const long long* const* strides = nullptr) {
    if (B < 0 || H < 0 || Sq < 0 || Sk < 0) return FA_ERR_SHAPE;
    if (D != 64 && D != 128 && D != 256) return FA_ERR_HEADDIM;
    if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_DTYPE;
    if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_SCALE;
    if (causal != 0 && causal != 1) return FA_ERR_ARG;
    if (deterministic != 0 && deterministic != 1) return FA_ERR_ARG;
    if (B == 0 || H == 0 || (Sq == 0 && Sk == 0)) return FA_OK;  // empty problem
    if (Sk == 0 || (causal && Sq > Sk)) return FA_ERR_SHAPE;     // a query would see no key
    const int64_t BH = (int64_t)B * H;
    if (BH > INT_MAX || BH * (int64_t)Sq > INT_MAX || BH * (int64_t)Sk > INT_MAX || Sq > INT_MAX - 512 ||
        Sk > INT_MAX - 512)
        return FA_ERR_SHAPE;
    // strides (elements over b, h, row) of q, k, v, o, dout, dq, dk, dv; NULL = contiguous
    long long st[8][3];
    {
        const int rows[8] = {Sq, Sk, Sk, Sq, Sq, Sq, Sk, Sk};
        for (int t = 0; t < 8; ++t) {
            const int rc = resolve_strides(strides ? strides[t] : nullptr, B, H, rows[t], D, st[t]);
            if (rc != FA_OK) return rc;
        }
    }
    if (Sq == 0) {
        // no query: the key and value gradients are zero
        if (!dk || !dv) return FA_ERR_NULL;
        if (strides && (strides[6] || strides[7])) return FA_ERR_STRIDE;  // zeroed as whole contiguous blocks
        const size_t bytes = (size_t)BH * (size_t)Sk * (size_t)D * 2;
        cudaError_t e = cudaMemsetAsync(dk, 0, bytes, stream);
        if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, bytes, stream);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(dk, dv)");
        return FA_OK;
    }
    if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_NULL;
    long long ms[3] = {0, 0, 0};
    if (mask) {
        for (int i = 0; i < 3; ++i) ms[i] = mask_stride[i];
        if (ms[0] < 0 || ms[1] < 0 || ms[0] >= MAX_STRIDE || ms[1] >= MAX_STRIDE || ms[2] >= MAX_STRIDE)
            return FA_ERR_STRIDE;
        if ((ms[2] < Sk && Sq > 1) || ms[2] % 16 != 0 || ms[0] % 16 != 0 || ms[1] % 16 != 0) return FA_ERR_STRIDE;
        if (((uintptr_t)mask & 15u) != 0) return FA_ERR_ALIGN;
    }
    const fa::BwdWorkspace ws = fa::bwd_workspace_layout(BH, Sq, D);
    if (!workspace || ((uintptr_t)workspace & 255u) != 0 || workspace_bytes < ws.total) return FA_ERR_WORKSPACE;
    const uintptr_t a16 = (uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)o | (uintptr_t)dout |
                          (uintptr_t)dq | (uintptr_t)dk | (uintptr_t)dv;
    if ((a16 & 15u) != 0 || ((uintptr_t)lse & 3u) != 0) return FA_ERR_ALIGN;

    DeviceInfo dev;
    int rc = device_info(&dev);
    if (rc != FA_OK) return rc;
    if (dev.major != 10 || dev.minor != 0) return FA_ERR_ARCH;
    rc = bind_context();
    if (rc != FA_OK) return rc;
    int cur = 0;
    const cudaError_t de = cudaGetDevice(&cur);
    if (de != cudaSuccess) return cuda_fail(de, "cudaGetDevice");
    const void* ptrs[11] = {q, k, v, o, dout, lse, dq, dk, dv, workspace, mask ? (const void*)mask : q};
    for (const void* p : ptrs) {
        rc = check_device_pointer(p, cur);
        if (rc != FA_OK) return rc;
    }
    fa::BwdLaunchArgs a;
    std::memset(&a, 0, sizeof(a));
    // the backward kernel steps through 64 query rows at a time
    const int q_box = 64;
    if (!encode_tensor(&a.tmap_q, q, B, H, Sq, D, st[0], dtype, q_box) ||
        !encode_tensor(&a.tmap_do, dout, B, H, Sq, D, st[4], dtype, q_box) ||
        !encode_tensor(&a.tmap_k, k, B, H, Sk, D, st[1], dtype) ||
        !encode_tensor(&a.tmap_v, v, B, H, Sk, D, st[2], dtype))
        return FA_ERR_LAUNCH;
    for (int i = 0; i < 3; ++i) {
        a.o_stride[i] = st[3][i];
        a.do_stride[i] = st[4][i];
        a.dq_stride[i] = st[5][i];
        a.dk_stride[i] = st[6][i];
        a.dv_stride[i] = st[7][i];
    }
    uint8_t* w = static_cast<uint8_t*>(workspace);
    // the fp32 dQ accumulator as a 3-D tensor [B*H][Sq][D] for the TMA engine's
    // bulk reduce-add (D = 64, 128): boxes of 64 rows x D values, rows past Sq clipped
    if (D == 64 || D == 128) {
        EncodeTiledFn enc = encoder();
        if (!enc) return cuda_fail(cudaErrorNotSupported, "cuTensorMapEncodeTiled entry point");
        const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Sq, (cuuint64_t)BH};
        const cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)Sq * D * 4};
        const cuuint32_t box[3] = {(cuuint32_t)D, 64, 1};
        const cuuint32_t elem[3] = {1, 1, 1};
        const CUresult r = enc(&a.tmap_dq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, w + ws.dq_acc, dims, strides, box, elem,
                               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cuda_fail((int)r, "cuTensorMapEncodeTiled (dQ accumulator)");
    }
    a.o = o;
    a.dout = dout;
    a.lse = lse;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.dq_acc = reinterpret_cast<float*>(w + ws.dq_acc);
    a.dk_acc = reinterpret_cast<float*>(w + ws.kv_acc);
    a.dv_acc = a.dk_acc + BH * fa::KV_ACC_ROWS * D;
    a.lse2 = reinterpret_cast<float*>(w + ws.lse2);
    a.delta = reinterpret_cast<float*>(w + ws.delta);
    a.sched = reinterpret_cast<unsigned int*>(w + ws.sched);
    a.mask = mask;
    for (int i = 0; i < 3; ++i) a.mask_stride[i] = ms[i];
    if (drop) a.drop = *drop;
    a.dq_flags = nullptr;
    if (deterministic) {
        a.dq_flags = reinterpret_cast<int*>(w + ws.flags);  // cleared by the backward's first kernel
    }
    a.B = B;
    a.H = H;
    a.Sq = Sq;
    a.Sk = Sk;
    a.D = D;
    a.dtype = dtype;
    a.causal = causal;
    a.scale = scale;
    // D = 256: a unit is (head, key tile, half of the head dimension)
    const int64_t units = BH * ((Sk + 127) / 128) * (D == 256 ? 2 : 1);
    a.grid = (int)(units < dev.sms ? units : dev.sms);
    a.sms = dev.sms;  // a split query range (short key sets) resizes the grid
    const cudaError_t le = fa::launch_bwd_sm100(a, stream);
    if (le != cudaSuccess) return cuda_fail(le, "launch(backward kernels)");
    return FA_OK;
}

}  // namespace

extern "C" {

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse, void* dq,
           void* dk, void* dv, void* workspace, long long workspace_bytes, int B, int H, int Sq, int Sk, int D,
           float scale, int causal, int deterministic, int dtype, cudaStream_t stream) {
    return backward(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H, Sq, Sk, D, scale, causal,
                    deterministic, dtype, stream, nullptr, nullptr);
}

int fa_bwd_ex(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse, void* dq,
              void* dk, void* dv, void* workspace, long long workspace_bytes, int B, int H, int Sq, int Sk, int D,
              const long long* q_stride, const long long* k_stride, const long long* v_stride,
              const long long* o_stride, const long long* do_stride, const long long* dq_stride,
              const long long* dk_stride, const long long* dv_stride, float scale, int causal, int deterministic,
              int dtype, cudaStream_t stream) {
    const long long* const strides[8] = {q_stride, k_stride, v_stride, o_stride, do_stride, dq_stride, dk_stride,
                                         dv_stride};
    return backward(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H, Sq, Sk, D, scale, causal,
                    deterministic, dtype, stream, nullptr, nullptr, nullptr, strides);
}

int fa_bwd_mask(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                void* dq, void* dk, void* dv, void* workspace, long long workspace_bytes, int B, int H, int Sq, int Sk,
                int D, const void* mask, const long long* mask_stride, float scale, int causal, int deterministic,
                int dtype, cudaStream_t stream) {
    if (B < 0 || H < 0 || Sq < 0 || Sk < 0) return FA_ERR_SHAPE;
    if (B > 0 && H > 0 && Sq > 0 && (!mask || !mask_stride)) return FA_ERR_NULL;
    return backward(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H, Sq, Sk, D, scale, causal,
                    deterministic, dtype, stream, static_cast<const uint8_t*>(mask), mask_stride);
}

int fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                   void* dq, void* dk, void* dv, void* workspace, long long workspace_bytes, int B, int H, int Sq,
                   int Sk, int D, float scale, int causal, float dropout_p, unsigned long long seed,
                   unsigned int offset, int deterministic, int dtype, cudaStream_t stream) {
    fa::DropoutArgs d;
    std::memset(&d, 0, sizeof(d));
    if (!make_dropout(dropout_p, seed, offset, &d)) return FA_ERR_ARG;
    return backward(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H, Sq, Sk, D, scale, causal,
                    deterministic, dtype, stream, nullptr, nullptr, &d);
}

int fa_forward(const fa_fwd_params* p, cudaStream_t stream) {
    if (!p) return FA_ERR_NULL;
    if (p->B < 0 || p->H < 0 || p->Sq < 0 || p->Sk < 0) return FA_ERR_SHAPE;
    fa::DropoutArgs d;
    std::memset(&d, 0, sizeof(d));
    if (p->dropout_p != 0.f && !make_dropout(p->dropout_p, p->seed, p->offset, &d)) return FA_ERR_ARG;
    if (p->B > 0 && p->H > 0 && p->Sq > 0 && p->mask && !p->mask_stride) return FA_ERR_NULL;
    return forward(p->q, p->k, p->v, p->o, p->lse, p->B, p->H, p->Sq, p->Sk, p->D, p->q_stride, p->k_stride,
                   p->v_stride, p->o_stride, p->scale, p->causal, p->dtype, stream, Scratch::Allocated,
                   static_cast<const uint8_t*>(p->mask), p->mask_stride, d.enabled ? &d : nullptr, p->block_n,
                   p->q_tiles);
}

int fa_backward(const fa_bwd_params* p, cudaStream_t stream) {
    if (!p) return FA_ERR_NULL;
    if (p->B < 0 || p->H < 0 || p->Sq < 0 || p->Sk < 0) return FA_ERR_SHAPE;
    fa::DropoutArgs d;
    std::memset(&d, 0, sizeof(d));
    if (p->dropout_p != 0.f && !make_dropout(p->dropout_p, p->seed, p->offset, &d)) return FA_ERR_ARG;
    if (p->B > 0 && p->H > 0 && p->Sq > 0 && p->mask && !p->mask_stride) return FA_ERR_NULL;
    const long long* const strides[8] = {p->q_stride,  p->k_stride,  p->v_stride,  p->o_stride,
                                         p->do_stride, p->dq_stride, p->dk_stride, p->dv_stride};
    return backward(p->q, p->k, p->v, p->o, p->dout, p->lse, p->dq, p->dk, p->dv, p->workspace, p->workspace_bytes,
                    p->B, p->H, p->Sq, p->Sk, p->D, p->scale, p->causal, p->deterministic, p->dtype, stream,
                    static_cast<const uint8_t*>(p->mask), p->mask_stride, d.enabled ? &d : nullptr, strides);
}

int fa_merge_partial(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, long long rows, int D,
                     int dtype, cudaStream_t stream) {
    if (rows < 0 || rows > (1LL << 33)) return FA_ERR_SHAPE;  // 8 rows per block, grid < 2^31
    if (D < 1 || D > 1024) return FA_ERR_HEADDIM;
    if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_DTYPE;
    if (rows == 0) return FA_OK;
    if (!o_acc || !lse_acc || !o_part || !lse_part) return FA_ERR_NULL;
    if ((((uintptr_t)o_acc | (uintptr_t)lse_acc | (uintptr_t)lse_part) & 3u) != 0 || ((uintptr_t)o_part & 1u) != 0)
        return FA_ERR_ALIGN;
    int cur = 0;
    const cudaError_t de = cudaGetDevice(&cur);
    if (de != cudaSuccess) return cuda_fail(de, "cudaGetDevice");
    const void* ptrs[4] = {o_acc, lse_acc, o_part, lse_part};
    for (const void* p : ptrs) {
        const int rc = check_device_pointer(p, cur);
        if (rc != FA_OK) return rc;
    }
    const cudaError_t le = fa::launch_merge_partial(o_acc, lse_acc, o_part, lse_part, rows, D, dtype, stream);
    if (le != cudaSuccess) return cuda_fail(le, "launch(fa_merge_partial)");
    return FA_OK;
}

int fa_merge_finalize(const float* o_acc, void* o, long long n, int dtype, cudaStream_t stream) {
    if (n < 0) return FA_ERR_SHAPE;
    if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_DTYPE;
    if (n == 0) return FA_OK;
    if (!o_acc || !o) return FA_ERR_NULL;
    if (((uintptr_t)o_acc & 3u) != 0 || ((uintptr_t)o & 1u) != 0) return FA_ERR_ALIGN;
    int cur = 0;
    const cudaError_t de = cudaGetDevice(&cur);
    if (de != cudaSuccess) return cuda_fail(de, "cudaGetDevice");
    int rc = check_device_pointer(o_acc, cur);
    if (rc == FA_OK) rc = check_device_pointer(o, cur);
    if (rc != FA_OK) return rc;
    const cudaError_t le = fa::launch_merge_finalize(o_acc, o, n, dtype, stream);
    if (le != cudaSuccess) return cuda_fail(le, "launch(fa_merge_finalize)");
    return FA_OK;
}

int fa_accumulate(float* acc, const void* x, long long n, int dtype, cudaStream_t stream) {
    if (n < 0) return FA_ERR_SHAPE;
    if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_DTYPE;
    if (n == 0) return FA_OK;
    if (!acc || !x) return FA_ERR_NULL;
    if (((uintptr_t)acc & 3u) != 0 || ((uintptr_t)x & 1u) != 0) return FA_ERR_ALIGN;
    int cur = 0;
    const cudaError_t de = cudaGetDevice(&cur);
    if (de != cudaSuccess) return cuda_fail(de, "cudaGetDevice");
    int rc = check_device_pointer(acc, cur);
    if (rc == FA_OK) rc = check_device_pointer(x, cur);
    if (rc != FA_OK) return rc;
    const cudaError_t le = fa::launch_accumulate(acc, x, n, dtype, stream);
    if (le != cudaSuccess) return cuda_fail(le, "launch(fa_accumulate)");
    return FA_OK;
}

int fa_check_status(cudaStream_t stream) {
    // one status word per kernel translation unit; all are read and cleared
    int st[4] = {0, 0, 0, 0}, site[4] = {0, 0, 0, 0};
    cudaError_t e = fa::read_and_clear_status(stream, &st[0], &site[0]);
    if (e == cudaSuccess) e = fa::read_and_clear_status_bwd(stream, &st[1], &site[1]);
    if (e == cudaSuccess) e = fa::read_and_clear_status_d256(stream, &st[2], &site[2]);
    if (e == cudaSuccess) e = fa::read_and_clear_status_short(stream, &st[3], &site[3]);
    if (e != cudaSuccess) return cuda_fail(e, "fa_check_status (stream synchronize / status word copy)");
    for (int i = 0; i < 4; ++i) {
        if (st[i] != fa::DEV_OK) {
            t_last_site = site[i];
            return FA_ERR_TIMEOUT;
        }
    }
    return FA_OK;
}

int fa_last_timeout_site(void) { return t_last_site; }

int fa_last_cuda_error(const char** site) {
    if (site) *site = t_err_site;
    return t_err_code;
}

int fa_selftest_timeout(cudaStream_t stream) {
    DeviceInfo dev;
    int rc = device_info(&dev);
    if (rc != FA_OK) return rc;
    if (dev.major != 10 || dev.minor != 0) return FA_ERR_ARCH;
    const cudaError_t le = fa::launch_selftest_timeout(stream);
    if (le != cudaSuccess) return cuda_fail(le, "launch(selftest_timeout_kernel)");
    return FA_OK;
}

const char* fa_status_string(int status) {
    switch (status) {
        case FA_OK: return "ok";
        case FA_ERR_NULL: return "a required pointer is NULL";
        case FA_ERR_SHAPE: return "invalid B, H, Sq or Sk (or causal with Sq > Sk)";
        case FA_ERR_HEADDIM: return "head dimension must be 64, 128 or 256";
        case FA_ERR_DTYPE: return "dtype must be FA_FP16 or FA_BF16";
        case FA_ERR_ALIGN: return "q, k, v, o must be 16-byte aligned and lse 4-byte aligned";
        case FA_ERR_ARCH: return "the current device is not sm_100 (B200)";
        case FA_ERR_LAUNCH: return "CUDA runtime error (fa_last_cuda_error names the call)";
        case FA_ERR_TIMEOUT: return "a device-side wait exceeded its bound";
        case FA_ERR_SCALE: return "scale must be finite and > 0";
        case FA_ERR_ARG: return "causal or deterministic not 0/1, dropout_p out of range, or an unsupported tiling";
        case FA_ERR_PTR: return "pointer is not device memory of the current device";
        case FA_ERR_STRIDE: return "a stride is not positive, a multiple of 8 elements and below 2^36";
        case FA_ERR_WORKSPACE: return "workspace is NULL, not 256-byte aligned or smaller than fa_bwd_workspace_size";
        case FA_ERR_LIMIT: return "every scheduler-counter slot of this context is taken (too many streams)";
        default: return "unknown status";
    }
}

int fa_version(void) { return FA_VERSION; }

}  // extern "C"
