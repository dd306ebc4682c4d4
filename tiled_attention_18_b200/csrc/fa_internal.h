// fa_internal.h -- declarations shared by the host layer (fa_api.cpp) and the
// sm_100a kernel translation unit (fa_fwd_sm100.cu).  Not part of the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

// Tile shape of the forward kernel: a CTA owns two query tiles of BLOCK_M
// rows each and streams keys/values in tiles of BLOCK_N rows.
constexpr int BLOCK_M = 128;
constexpr int BLOCK_N = 128;
constexpr int Q_TILES_PER_CTA = 2;
constexpr int ROWS_PER_UNIT = BLOCK_M * Q_TILES_PER_CTA;

// Device-side status codes written to the status word by the kernel.
constexpr int DEV_OK = 0;
constexpr int DEV_TIMEOUT = 1;
// Wait-site code of the diagnostic timeout kernel (low byte of the site word).
constexpr int SELFTEST_SITE = 100;

struct LaunchArgs {
    CUtensorMap tmap_q;     // 4-D maps over [B][H][S][D] (innermost first: D, S, H, B) with
    CUtensorMap tmap_k;     // the tensors' own strides, box {64, 128, 1, 1}, 128-byte swizzle
    CUtensorMap tmap_v;
    void* o;                // [B,H,Sq,D] 16-bit at o_stride
    float* lse;             // [B,H,Sq] fp32, contiguous
    long long o_stride[3];  // element strides of O over b, h, s (d is contiguous)
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
};

// Number of work units (b, h, 256-row query block).
inline int64_t num_units(int64_t BH, int64_t S) {
    return BH * ((S + ROWS_PER_UNIT - 1) / ROWS_PER_UNIT);
}

// Launch the persistent forward kernel on `stream`.  Returns a cudaError_t.
cudaError_t launch_fwd_sm100(const LaunchArgs& a, cudaStream_t stream);

// fa_fwd_noalloc: size of its static scratch array (256 bytes; word 0 is the
// causal unit counter) and the largest number of unit claims the counter
// serves (work units + CTAs, read back as a non-negative int).
constexpr int NOALLOC_SCRATCH_WORDS = 64;
constexpr long long NOALLOC_MAX_CLAIMS = 0x7FFFFFFFll;

// Device address of the static scratch array on the current device (looked
// up once per device).
cudaError_t noalloc_scratch_address(unsigned int** out);

// Launch the diagnostic kernel whose first wait is never satisfied.
cudaError_t launch_selftest_timeout(cudaStream_t stream);

// Read (after synchronising `stream`) and clear the device status word of
// the current device.  *status receives DEV_OK or an error code; *site the
// diagnostic word of the first failing wait.
cudaError_t read_and_clear_status(cudaStream_t stream, int* status, int* site);

}  // namespace fa
