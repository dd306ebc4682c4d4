// fa_merge_sm100.cu -- merging partial attention results by their log-sum-exp
// and accumulating partial gradients (declared in include/fa.h:
// fa_merge_partial, fa_merge_finalize, fa_accumulate).
//
// Attention over a key set split into blocks is the LSE-weighted combination
// of the attention over each block: with (O_a, L_a) and (O_b, L_b) for two
// disjoint key sets, L = log(e^L_a + e^L_b) and O = (e^(L_a - L) O_a +
// e^(L_b - L) O_b).  This is what lets the sequence be split across devices
// ("FlashAttention-2 在昇腾 NPU 上如何做到 3 倍加速？", section 6.4: each device
// computes the attention of its part of the sequence while K/V move between
// devices) and is the same rescaling the online softmax applies tile by tile
// inside one kernel (section 2.2).
//
// One warp per row, its lanes striding over the row's D values.  The running
// result is fp32 (o_acc, lse_acc); a partial is 16-bit O with fp32 LSE, as
// fa_fwd_ex produces them.  An empty side (LSE = -inf) contributes nothing.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa_internal.h"

namespace fa {
namespace {

template <bool BF16>
__device__ __forceinline__ float to_f32(uint16_t x) {
    if constexpr (BF16) return __bfloat162float(__ushort_as_bfloat16(x));
    else return __half2float(__ushort_as_half(x));
}

template <bool BF16>
__device__ __forceinline__ uint16_t from_f32(float x) {
    if constexpr (BF16) return __bfloat16_as_ushort(__float2bfloat16_rn(x));
    else return __half_as_ushort(__float2half_rn(x));
}

template <bool BF16>
__device__ __forceinline__ float4 load4_f32(const uint16_t* p) {
    const uint2 raw = *reinterpret_cast<const uint2*>(p);
    return make_float4(to_f32<BF16>((uint16_t)(raw.x & 0xffffu)), to_f32<BF16>((uint16_t)(raw.x >> 16)),
                       to_f32<BF16>((uint16_t)(raw.y & 0xffffu)), to_f32<BF16>((uint16_t)(raw.y >> 16)));
}

// VEC: D % 4 == 0 with 16-byte aligned o_acc and 8-byte aligned o_part, so a
// lane moves four consecutive values per access (one float4, one 8-byte load).
template <bool BF16, bool VEC>
__global__ void __launch_bounds__(256) merge_kernel(float* __restrict__ o_acc, float* __restrict__ lse_acc,
                                                    const uint16_t* __restrict__ o_part,
                                                    const float* __restrict__ lse_part, long long rows, int D) {
    grid_dependency_sync();
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float la = lse_acc[row], lb = lse_part[row];
    const float m = fmaxf(la, lb);
    if (m == -INFINITY) return;  // neither side saw a key
    const float wa = (la == -INFINITY) ? 0.f : expf(la - m);
    const float wb = (lb == -INFINITY) ? 0.f : expf(lb - m);
    const float inv = 1.f / (wa + wb);
    const float ca = wa * inv, cb = wb * inv;
    float* oa = o_acc + row * D;
    const uint16_t* ob = o_part + row * D;
    // an accumulator that has seen no key yet (ca = 0) is overwritten, not read
    if constexpr (VEC) {
        for (int d = 4 * lane; d < D; d += 128) {
            const float4 b = load4_f32<BF16>(ob + d);
            float4 r;
            if (ca != 0.f) {
                const float4 a = *reinterpret_cast<const float4*>(oa + d);
                r = make_float4(ca * a.x + cb * b.x, ca * a.y + cb * b.y, ca * a.z + cb * b.z, ca * a.w + cb * b.w);
            } else {
                r = make_float4(cb * b.x, cb * b.y, cb * b.z, cb * b.w);
            }
            *reinterpret_cast<float4*>(oa + d) = r;
        }
    } else {
        for (int d = lane; d < D; d += 32)
            oa[d] = (ca != 0.f ? ca * oa[d] : 0.f) + cb * to_f32<BF16>(ob[d]);
    }
    __syncwarp();
    if (lane == 0) lse_acc[row] = m + logf(wa + wb);
}

template <bool BF16>
__global__ void __launch_bounds__(256) finalize_kernel(const float* __restrict__ o_acc, uint16_t* __restrict__ o,
                                                       long long n) {
    grid_dependency_sync();
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        o[i] = from_f32<BF16>(o_acc[i]);
}

// acc += x for n values: fp32 accumulators of partial gradients (16-bit x),
// four per thread when n, acc and x allow it.
template <bool BF16>
__global__ void __launch_bounds__(256) accumulate_kernel(float* __restrict__ acc, const uint16_t* __restrict__ x,
                                                         long long n) {
    grid_dependency_sync();
    const long long step = (long long)gridDim.x * blockDim.x;
    long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if ((n & 3) == 0 && ((uintptr_t)acc & 15) == 0 && ((uintptr_t)x & 7) == 0) {
        for (; i < n / 4; i += step) {
            const uint2 r = reinterpret_cast<const uint2*>(x)[i];
            float4 a = reinterpret_cast<float4*>(acc)[i];
            a.x += to_f32<BF16>((uint16_t)(r.x & 0xffffu));
            a.y += to_f32<BF16>((uint16_t)(r.x >> 16));
            a.z += to_f32<BF16>((uint16_t)(r.y & 0xffffu));
            a.w += to_f32<BF16>((uint16_t)(r.y >> 16));
            reinterpret_cast<float4*>(acc)[i] = a;
        }
    } else {
        for (; i < n; i += step) acc[i] += to_f32<BF16>(x[i]);
    }
}

}  // namespace

cudaError_t launch_accumulate(float* acc, const void* x, long long n, int dtype, cudaStream_t stream) {
    const long long want = (n / 4 + 255) / 256 + 1;
    const unsigned blocks = (unsigned)(want < 148 * 32 ? want : 148 * 32);
    const uint16_t* xs = static_cast<const uint16_t*>(x);
    return dtype == 1 ? launch_kernel(accumulate_kernel<true>, dim3(blocks), dim3(256), 0, stream, acc, xs, n)
                      : launch_kernel(accumulate_kernel<false>, dim3(blocks), dim3(256), 0, stream, acc, xs, n);
}

cudaError_t launch_merge_partial(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                                 long long rows, int D, int dtype, cudaStream_t stream) {
    const unsigned blocks = (unsigned)((rows + 7) / 8);
    const uint16_t* ob = static_cast<const uint16_t*>(o_part);
    const bool vec = (D % 4 == 0) && ((uintptr_t)o_acc % 16 == 0) && ((uintptr_t)o_part % 8 == 0);
    auto kern = dtype == 1 ? (vec ? merge_kernel<true, true> : merge_kernel<true, false>)
                           : (vec ? merge_kernel<false, true> : merge_kernel<false, false>);
    return launch_kernel(kern, dim3(blocks), dim3(256), 0, stream, o_acc, lse_acc, ob, lse_part, rows, D);
}

cudaError_t launch_merge_finalize(const float* o_acc, void* o, long long n, int dtype, cudaStream_t stream) {
    const long long want = (n + 255) / 256;
    const unsigned blocks = (unsigned)(want < 148 * 32 ? want : 148 * 32);
    uint16_t* out = static_cast<uint16_t*>(o);
    return dtype == 1 ? launch_kernel(finalize_kernel<true>, dim3(blocks), dim3(256), 0, stream, o_acc, out, n)
                      : launch_kernel(finalize_kernel<false>, dim3(blocks), dim3(256), 0, stream, o_acc, out, n);
}

}  // namespace fa
