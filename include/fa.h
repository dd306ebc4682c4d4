/*
 * fa.h -- C ABI of libfa.so: fused attention (FlashAttention-2 style) for
 * NVIDIA B200 (sm_100a): the forward pass (fa_fwd, fa_fwd_ex, fa_fwd_noalloc,
 * head dimension 64/128/256), its explicit-mask and dropout variants
 * (fa_fwd_mask, fa_fwd_dropout), the backward pass (fa_bwd, fa_bwd_ex,
 * fa_bwd_mask, fa_bwd_dropout) and the log-sum-exp merge of partial results
 * for a sequence split across devices (fa_merge_partial, fa_merge_finalize).
 *
 * The operation, per batch b, head h and query row i of BHSD tensors
 * (contiguous for fa_fwd; any b, h, s strides and Sq != Sk for fa_fwd_ex):
 *
 *   O[b,h,i,:]  = sum_j softmax_j( scale * Q[b,h,i,:] . K[b,h,j,:] ) * V[b,h,j,:]
 *   LSE[b,h,i]  = log( sum_j exp( scale * Q[b,h,i,:] . K[b,h,j,:] ) )   (natural log)
 *
 * with j over [0, S), or over [0, i] when causal (each position sees only
 * itself and earlier tokens; top-left aligned, Sq = Sk = S).
 *
 * Sources (page title, section):
 *  - the attention equation softmax(QK^T / sqrt(d_k)) V and the tiled,
 *    online-softmax evaluation that never stores the S x S score matrix:
 *    "FlashAttention-2 在昇腾 NPU 上如何做到 3 倍加速？深度拆解 ops-transformer 的实现",
 *    sections 1, 2.1 and 2.2;
 *  - the operator call flash_attention(Q, K, V, causal=True) on [B, H, S, D]
 *    tensors: "ops-transformer FlashAttention 算子实战：让昇腾NPU算力彻底释放",
 *    section 4.1;
 *  - the [batch, heads, seq_len, head_dim] row-major layout, FP16/BF16 inputs
 *    and in-kernel causal tile skipping: the gsyq.cn catlass FlashAttention
 *    page, sections on precision choice, data layout and "Causal Mask的实现差异";
 *  - the explicit softmax scale (the caller passes it; there is no default):
 *    the omica.com.cn cann-learning-hub FlashAttention tutorial, the step that
 *    compares against SDPA.
 * The per-row LSE is not defined on the pages; it is the natural log of the
 * softmax denominator of the scaled scores.
 *
 * All calls return an fa_status code; none aborts.  FA_ERR_LAUNCH reports
 * the failure of this call's own CUDA calls and launches, never an error that
 * other code left pending in the calling thread; fa_last_cuda_error names the
 * failed call and its error code.  Calls from several host threads at once
 * are safe: a causal call takes its stream's work counter and launches under
 * one lock (the counter is cleared by the last CTA of each launch, so no
 * memset precedes a causal launch except in fa_fwd_noalloc, whose counter all
 * streams share), and each kernel's shared-memory limit is set once per
 * context.
 *
 * Every kernel is launched with programmatic stream serialization: it may
 * begin (barrier set-up, tensor memory, descriptor prefetch) while the kernel
 * before it in the stream is still running, and it waits for that kernel to
 * complete, with its writes visible, before it reads or writes any tensor.
 * Work of other code in the stream (kernels, copies, memsets, event waits)
 * orders with these calls exactly as with ordinary launches.
 */
#ifndef FA_H_
#define FA_H_

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { FA_FP16 = 0, FA_BF16 = 1 } fa_dtype;

typedef enum {
    FA_OK = 0,
    FA_ERR_NULL = -1,     /* a required pointer is NULL */
    FA_ERR_SHAPE = -2,    /* B, H or S negative, or too large for 32-bit indexing */
    FA_ERR_HEADDIM = -3,  /* D is not 64, 128 or 256 */
    FA_ERR_DTYPE = -4,    /* dtype is not FA_FP16 or FA_BF16 */
    FA_ERR_ALIGN = -5,    /* q, k, v, o not 16-byte aligned, or lse not 4-byte aligned */
    FA_ERR_ARCH = -6,     /* the current device is not compute capability 10.0 (sm_100) */
    FA_ERR_LAUNCH = -7,   /* a CUDA runtime error (launch, tensor-map encoding, sync) */
    FA_ERR_TIMEOUT = -8,  /* a device-side wait exceeded its bound (reported by fa_check_status) */
    FA_ERR_SCALE = -9,    /* scale is not finite and > 0 */
    FA_ERR_ARG = -10,     /* causal (or fa_bwd's deterministic) is not 0 or 1, or dropout_p is out of range */
    FA_ERR_PTR = -11,     /* a pointer is not device memory of the current device */
    FA_ERR_STRIDE = -12,  /* fa_fwd_ex, fa_bwd_ex: a stride is negative, zero over an extent > 1,
                             not a multiple of 8 elements (16 bytes), or not below 2^36 elements;
                             the mask entries: a mask stride breaks their rules */
    FA_ERR_WORKSPACE = -13, /* the fa_bwd entries: workspace NULL, not 256-byte aligned or too small */
    FA_ERR_LIMIT = -14      /* causal forward: more streams of one context have launched causal
                               forwards than the library's 2048 scheduler-counter slots */
} fa_status;

/*
 * fa_fwd -- attention forward pass with per-row log-sum-exp.
 *
 * q, k, v : device pointers, [B, H, S, D] contiguous (BHSD, row-major), dtype
 *           elements; 16-byte aligned.  Read only.
 * o       : device pointer, [B, H, S, D] contiguous, dtype; 16-byte aligned.
 *           Written.  Must not overlap q, k, v or lse.
 * lse     : device pointer, [B, H, S] contiguous fp32, 4-byte aligned.
 *           Written (natural log).  Required.
 * B, H, S : batch, heads, sequence length (queries = keys = S).  Any of them
 *           0 is an empty problem: FA_OK, nothing is launched and the pointers
 *           are not inspected.  B*H*S must fit in 31 bits.
 * D       : head dimension, 64, 128 or 256.  D = 256 runs a kernel of its own
 *           (one 128-row query tile per work unit, 64-key tiles); the pages
 *           name 64, 128 and 256 as the common head dimensions
 *           ("FlashAttention-2 在昇腾 NPU 上如何做到 3 倍加速？", section 3.2).
 * scale   : softmax scale (commonly 1/sqrt(D)); finite and > 0.
 * causal  : 0 = attend to all keys; 1 = key j attends to query i iff j <= i.
 * dtype   : FA_FP16 or FA_BF16 (inputs and output).  Scores, the softmax
 *           statistics and the accumulation are fp32; the softmax weights
 *           are rounded to dtype before the P.V product; O is rounded to
 *           nearest even.
 * stream  : the CUDA stream to launch on (0 = legacy default stream).
 *
 * Ownership: the caller owns every buffer and the stream; fa_fwd allocates
 * nothing.  With causal = 1 the library's work scheduler uses a counter
 * (claimed units and finished CTAs): one slot per (context, stream) of a
 * fixed pool of 2048 slots in libfa.so's own static device memory (64 KiB,
 * part of the loaded module), handed out by the stream's first causal call;
 * the slot starts zeroed and the last CTA of every causal launch zeroes it
 * again, so no memset precedes the launch.  More than 2048 distinct streams
 * of one context launching causal forwards gives FA_ERR_LIMIT.  The first
 * call in a context looks up the pool's device address (a host-side query,
 * no device work).  Synchronicity: asynchronous on `stream`; fa_fwd never
 * synchronises.  Errors: argument checks run before any launch and return a
 * negative fa_status with nothing launched; a launch failure returns
 * FA_ERR_LAUNCH.  A device-side wait that exceeds its bound (about two
 * seconds) makes the kernel stop early and is reported by fa_check_status.
 */
FA_API int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int S,
           int D, float scale, int causal, int dtype, cudaStream_t stream);

/*
 * fa_fwd_noalloc -- fa_fwd for callers that cannot allocate device memory
 * (code that runs where cudaMalloc is unavailable or not allowed, such as
 * inside a memory allocator, a runtime that works only in pre-allocated
 * memory, or a process whose device footprint must not grow).  The pages have
 * no counterpart; it is a deployment variant.  Same arguments, checks, result
 * and error codes as fa_fwd, but it allocates nothing: the causal work
 * scheduler's counter lives in a fixed 256-byte array inside libfa.so's own
 * device memory, held on every GPU that loads the library until the process
 * exits.  The first call on a device looks up that array's device address
 * (once per device, with that device current), so make that first call
 * before any stream capture.  Limit: the work units plus the CTAs of one call
 * must stay below 2^31 (always true for shapes fa_fwd accepts); otherwise it
 * returns FA_ERR_SHAPE.  Every call shares the one array, and each causal call
 * zeroes its counter on `stream` before the launch: calls that overlap on the
 * GPU (for example on two streams at once) race on it and may compute wrong
 * results; issue them one after another.
 */
FA_API int fa_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                          int S, int D, float scale, int causal, int dtype, cudaStream_t stream);

/*
 * fa_fwd_ex -- fa_fwd for general shapes: Sq queries and Sk keys per head
 * (cross-attention, e.g. image tokens attending to 77 text tokens:
 * "解析CANN ops-transformer的FlashAttention算子：注意力机制的内存优化",
 * section "Stable Diffusion中的优化") and tensors at arbitrary b, h, s strides,
 * so that [batch, seq_len, heads, head_dim] (BSHD) data is read in place
 * instead of being transposed and copied first (the layout pitfall of the
 * gsyq.cn catlass FlashAttention page, section on data layout).
 *
 *   O[b,h,i,:] = sum_j softmax_j( scale * Q[b,h,i,:] . K[b,h,j,:] ) * V[b,h,j,:]
 *
 * with j over [0, Sk); with causal = 1, j over [0, i + Sk - Sq]: the queries
 * are the last Sq of the Sk positions (bottom-right alignment; with Sq = Sk
 * this is fa_fwd's mask).  The pages do not say how the mask aligns when
 * Sq != Sk; this is the reading taken.
 *
 * q       : [B, H, Sq, D] elements at q_stride; k, v : [B, H, Sk, D] at
 *           k_stride, v_stride; o : [B, H, Sq, D] at o_stride.  Each *_stride
 *           is a host array of 3 element strides for the b, h and s
 *           dimensions (d is contiguous), or NULL for the contiguous BHSD
 *           layout of that shape.  A stride over an extent of 1 is ignored.
 *           Every other stride must be > 0, a multiple of 8 elements (16
 *           bytes) and below 2^36 elements (else FA_ERR_STRIDE).  o must not
 *           overlap itself, q, k, v or lse.
 * lse     : [B, H, Sq] contiguous fp32 (natural log).  Required.
 * B, H, Sq: B, H or Sq 0 is an empty problem (FA_OK, nothing launched,
 *           pointers not inspected).  Sk must be >= 1, and >= Sq when
 *           causal = 1 (else FA_ERR_SHAPE: some query would see no key).
 *           B*H*Sq must fit in 31 bits and Sq, Sk must stay below 2^31 - 512.
 * D, scale, causal, dtype, stream, ownership, scheduler scratch, errors:
 *           as fa_fwd.  fa_fwd(q, k, v, o, lse, B, H, S, D, ...) computes the
 *           same as fa_fwd_ex with Sq = Sk = S and NULL strides.
 */
FA_API int fa_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Sq,
                     int Sk, int D, const long long* q_stride, const long long* k_stride,
                     const long long* v_stride, const long long* o_stride, float scale, int causal, int dtype,
                     cudaStream_t stream);

/*
 * fa_fwd_mask -- fa_fwd_ex (contiguous BHSD, Sq queries, Sk keys) with an
 * explicit boolean mask fused into the kernel: query i of head (b, h) attends
 * to key j only where mask[b][h][i][j] != 0 (and, with causal = 1, j <= i + Sk
 * - Sq).  A masked score becomes -infinity before the softmax
 * ("FlashAttention-2 在昇腾 NPU 上如何做到 3 倍加速？", section 3.4, the fused
 * mask; the explicit mask matrix of the gsyq.cn catlass page, "Causal Mask的
 * 实现差异", mode 1).  A row that sees no key gets O = 0 and LSE = -infinity
 * (the pages do not say; this is the reading taken).
 *
 * mask        : device, uint8 (0 = masked, nonzero = attend), keys contiguous.
 * mask_stride : host array of 3 element strides over b, h and the query row;
 *               0 over b or h broadcasts one mask to every batch or head.  All
 *               three must be multiples of 16 and the row stride >= Sk (else
 *               FA_ERR_STRIDE); mask must be 16-byte aligned (FA_ERR_ALIGN).
 * Other arguments, ownership and errors: as fa_fwd_ex.  The mask costs a
 * 16-byte load per 16 keys of every query row and tile; key tiles above the
 * causal diagonal are still skipped.
 */
FA_API int fa_fwd_mask(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Sq,
                       int Sk, int D, const void* mask, const long long* mask_stride, float scale, int causal,
                       int dtype, cudaStream_t stream);

/*
 * fa_bwd_workspace_size -- bytes of device workspace fa_bwd needs for B*H
 * heads of Sq query rows of dimension D: an fp32 dQ accumulator
 * [B*H][Sq][D], two fp32 row-statistic arrays [B*H][Sq rounded up to 128],
 * the deterministic mode's turn counters [B*H][Sq/64 rounded up][1, or 2 at
 * D = 256][4] int, a
 * 256-byte scheduler counter and two fp32 arrays [B*H][128][D] for the
 * partial sums of dK and dV (used when Sk <= 128 and the (head, key tile)
 * units are fewer than the SMs: the query range is then split across units),
 * each part 256-byte aligned.  0 for an empty problem, a negative fa_status
 * on invalid sizes.  Host only.
 */
FA_API long long fa_bwd_workspace_size(int B, int H, int Sq, int D);

/*
 * fa_bwd -- backward pass of fa_fwd / fa_fwd_ex (contiguous BHSD tensors):
 * the gradients dQ, dK, dV of the attention output for the upstream gradient
 * dO, recomputing the scores and weights tile by tile from Q, K and the
 * forward pass's LSE instead of storing them ("FlashAttention-2 在昇腾 NPU 上
 * 如何做到 3 倍加速？", the recomputation row of the core-optimisation table
 * and section 6.2; the backward configuration on the gsyq.cn catlass page,
 * "反向传播的特殊处理").  With P_ij = exp(scale q_i.k_j - LSE_i) over the keys
 * query i sees (the mask of fa_fwd_ex: all keys, or j <= i + Sk - Sq) and
 * Delta_i = sum_d dO_id O_id:
 *
 *   dV_j = sum_i P_ij dO_i,    dS_ij = P_ij (dO_i.v_j - Delta_i),
 *   dQ_i = scale sum_j dS_ij k_j,    dK_j = scale sum_i dS_ij q_i.
 *
 * q, o, dout : device, [B, H, Sq, D] contiguous, dtype.  o and lse must be the
 *              forward outputs for these q, k, v, scale and mask.
 * k, v       : device, [B, H, Sk, D] contiguous, dtype.
 * lse        : device, [B, H, Sq] contiguous fp32 (natural log).
 * dq         : device, [B, H, Sq, D] contiguous, dtype.  Written.
 * dk, dv     : device, [B, H, Sk, D] contiguous, dtype.  Written.
 * workspace  : device, at least fa_bwd_workspace_size(B, H, Sq, D) bytes,
 *              256-byte aligned (else FA_ERR_WORKSPACE); contents on entry do
 *              not matter; used only during the call's kernels on `stream`, so
 *              calls that may overlap on the GPU need separate workspaces.
 * B, H, Sq, Sk, D, scale, causal, dtype: as fa_fwd_ex (D = 64, 128 or 256).
 *              B or H 0 is an empty problem (FA_OK, nothing launched); Sq = 0
 *              zeroes dK and dV.  D = 256 forms each 128-key tile's gradients
 *              in two passes, one per half of the head dimension, each
 *              recomputing the full-width scores (the pages name 64, 128 and 256
 *              as the common head dimensions: "FlashAttention-2 在昇腾 NPU 上
 *              如何做到 3 倍加速？", section 3.2).
 * deterministic: 0 = dQ is accumulated in fp32 across key tiles with atomic
 *              adds (fastest; its last bits may differ between runs); 1 = the
 *              key tiles of a head add their dQ parts in key-tile order (the
 *              catlass page's deterministic mode), so every output is bitwise
 *              repeatable.  Mode 1 makes CTAs wait (bounded) for one another, so
 *              all of the call's CTAs must be able to run at once: do not run
 *              other kernels beside it that hold SMs it needs, or the waits may
 *              time out (reported by fa_check_status as FA_ERR_TIMEOUT).  dK and
 *              dV are bitwise repeatable in both modes.
 * Numerics: S, P, dP, dS, Delta and all accumulation in fp32; P and dS are
 * rounded to dtype before their products; the outputs are rounded to nearest
 * even.
 * Kernels alone run on `stream`, with no memset or copy between them: row
 * statistics (which also clears the workspace parts the call needs zeroed:
 * the dQ accumulator, the turn counters, the dK/dV partial sums), the fused
 * backward, then the dQ conversion, or with a split query range the dK/dV
 * conversion (plus the dQ conversion at D = 256); Sq = 0 runs two memsets of
 * dK and dV instead.  Nothing is allocated; asynchronous.  Errors as fa_fwd.
 */
FA_API int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                  void* dq, void* dk, void* dv, void* workspace, long long workspace_bytes, int B, int H, int Sq,
                  int Sk, int D, float scale, int causal, int deterministic, int dtype, cudaStream_t stream);

/*
 * fa_bwd_ex -- fa_bwd with each tensor at its own (b, h, s) element strides,
 * d contiguous, as fa_fwd_ex takes them (NULL = contiguous BHSD): BSHD data,
 * packed QKV and padded gradient buffers are read and written in place.
 * q_stride, o_stride, do_stride, dq_stride: host arrays of 3 strides for the
 * [B][H][Sq][D] tensors; k_stride, v_stride, dk_stride, dv_stride for the
 * [B][H][Sk][D] ones.  Each stride > 0, a multiple of 8 elements and below
 * 2^36 (a stride over an extent of 1 is ignored), else FA_ERR_STRIDE; with
 * Sq = 0 the dK/dV strides must be NULL.  The gradients must not overlap
 * each other or the inputs.  Other arguments, workspace, modes and errors as
 * fa_bwd (the workspace size does not depend on the strides).
 */
FA_API int fa_bwd_ex(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                     void* dq, void* dk, void* dv, void* workspace, long long workspace_bytes, int B, int H, int Sq,
                     int Sk, int D, const long long* q_stride, const long long* k_stride,
                     const long long* v_stride, const long long* o_stride, const long long* do_stride,
                     const long long* dq_stride, const long long* dk_stride, const long long* dv_stride,
                     float scale, int causal, int deterministic, int dtype, cudaStream_t stream);

/*
 * fa_bwd_mask -- fa_bwd for the explicitly masked attention of fa_fwd_mask:
 * the same mask (device uint8, nonzero = attend; mask_stride = element strides
 * over b, h and the query row, 0 broadcasting over b or h; all multiples of 16,
 * row stride >= Sk; 16-byte aligned).  Masked (query, key) pairs contribute no
 * gradient; rows that saw no key (LSE = -inf) get dQ = 0.  o and lse must come
 * from fa_fwd_mask with the same mask.  D = 64, 128 or 256; other arguments, modes
 * and errors as fa_bwd.
 */
FA_API int fa_bwd_mask(const void* q, const void* k, const void* v, const void* o, const void* dout,
                       const float* lse, void* dq, void* dk, void* dv, void* workspace, long long workspace_bytes,
                       int B, int H, int Sq, int Sk, int D, const void* mask, const long long* mask_stride,
                       float scale, int causal, int deterministic, int dtype, cudaStream_t stream);

/*
 * fa_fwd_dropout -- fa_fwd_ex (contiguous BHSD, Sq queries, Sk keys, bottom-right
 * causal mask) with attention dropout fused into the kernel: after the softmax
 * each weight P_ij is kept or zeroed, and the kept weights are scaled by
 * 1 / (1 - p), so O_i = sum_j P_ij z_ij v_j with z_ij in {0, 1 / (1 - p)}
 * ("FlashAttention-2 在昇腾 NPU 上如何做到 3 倍加速？", sections 3.4 and 6.3: dropout
 * fused into the kernel with random numbers drawn on the device).  The LSE is
 * that of the undropped softmax (what fa_bwd_dropout needs).
 *
 * The keep decisions are reproducible from (seed, offset): for head
 * bh = b * H + h, query row i and key j, Philox4x32-10 (Salmon, Moraes, Dror,
 * Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011) of the
 * counter (j / 16, i, bh, offset) under the key (seed mod 2^32, seed / 2^32)
 * gives four 32-bit words; key j takes byte j mod 16 of them (word
 * (j mod 16) / 4, little-endian byte j mod 4) and is kept iff that byte is
 * >= p8 = floor(256 dropout_p + 1/2).  The drop probability is therefore
 * p8 / 256 and the kept weights are scaled by 256 / (256 - p8).
 *
 * dropout_p : 0 <= dropout_p and p8 <= 255 (else FA_ERR_ARG); 0 keeps every
 *             weight (the result equals fa_fwd_ex's).
 * seed, offset : the generator's key and the counter's last word; use a new
 *             offset (or seed) for every call that needs fresh decisions.
 * D = 64, 128 or 256 (else FA_ERR_HEADDIM).  Other arguments, ownership and
 * errors as fa_fwd_ex with NULL strides.
 */
FA_API int fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Sq,
                          int Sk, int D, float scale, int causal, float dropout_p, unsigned long long seed,
                          unsigned int offset, int dtype, cudaStream_t stream);

/*
 * fa_bwd_dropout -- fa_bwd for the attention with dropout of fa_fwd_dropout:
 * with the same dropout_p, seed and offset the kernel regenerates the same
 * keep decisions, and dV_j = sum_i P_ij z_ij dO_i, dP_ij = z_ij dO_i . v_j,
 * dS_ij = P_ij (dP_ij - dO_i . O_i).  o and lse must come from fa_fwd_dropout
 * with the same arguments.  D = 64, 128 or 256; other arguments, modes and errors
 * as fa_bwd; dropout_p as fa_fwd_dropout.
 */
FA_API int fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o, const void* dout,
                          const float* lse, void* dq, void* dk, void* dv, void* workspace, long long workspace_bytes,
                          int B, int H, int Sq, int Sk, int D, float scale, int causal, float dropout_p,
                          unsigned long long seed, unsigned int offset, int deterministic, int dtype,
                          cudaStream_t stream);

/*
 * fa_forward / fa_backward -- every option of the forward and backward
 * passes in one call, in any combination: Sq != Sk with the bottom-right
 * causal mask, per-tensor (b, h, s) strides, an explicit mask, dropout.
 * The fields mean what the arguments of the same names mean for fa_fwd_ex,
 * fa_fwd_mask and fa_fwd_dropout (fa_bwd_ex, fa_bwd_mask, fa_bwd_dropout):
 * a NULL stride array is contiguous, a NULL mask is no mask, dropout_p = 0 is
 * no dropout.  fa_forward and fa_backward take D = 64, 128 or 256
 * (with or without a mask and dropout).  The caller owns the
 * struct (read during the call only) and everything it points to.  Errors:
 * FA_ERR_NULL for a NULL params pointer, else those of the separate entries.
 * o and lse given to fa_backward must come from fa_forward with the same
 * mask and dropout arguments.
 */
typedef struct fa_fwd_params {
    const void* q;
    const void* k;
    const void* v;
    void* o;
    float* lse;
    int B, H, Sq, Sk, D;
    const long long* q_stride; /* each: 3 element strides over b, h, s, or NULL */
    const long long* k_stride;
    const long long* v_stride;
    const long long* o_stride;
    const void* mask;          /* uint8 [B|1][H|1][Sq][Sk], nonzero = attend, or NULL */
    const long long* mask_stride;
    float dropout_p;           /* 0: no dropout */
    unsigned long long seed;
    unsigned int offset;
    float scale;
    int causal;
    int dtype;
    /* Tiling (0 = automatic: 128-key tiles, two 128-row query tiles per work
     * unit).  block_n: keys per key tile, 64 or 128; q_tiles: 128-row query
     * tiles per work unit, 1 or 2.  A manual tiling takes D = 64 or 128 and no
     * mask or dropout; otherwise FA_ERR_ARG.  The FlashAttention-2 page lets
     * the caller set the block sizes by hand for particular shapes ("FlashAttention-2
     * 在昇腾 NPU 上如何做到 3 倍加速？", section 6.1); the catlass page tabulates
     * block_m x block_n against throughput (section "分块策略不是越大越好"). */
    int block_n;
    int q_tiles;
} fa_fwd_params;

typedef struct fa_bwd_params {
    const void* q;
    const void* k;
    const void* v;
    const void* o;
    const void* dout;
    const float* lse;
    void* dq;
    void* dk;
    void* dv;
    void* workspace;           /* fa_bwd_workspace_size(B, H, Sq, D) bytes, 256-byte aligned */
    long long workspace_bytes;
    int B, H, Sq, Sk, D;
    const long long* q_stride; /* each: 3 element strides over b, h, s, or NULL */
    const long long* k_stride;
    const long long* v_stride;
    const long long* o_stride;
    const long long* do_stride;
    const long long* dq_stride;
    const long long* dk_stride;
    const long long* dv_stride;
    const void* mask;
    const long long* mask_stride;
    float dropout_p;
    unsigned long long seed;
    unsigned int offset;
    float scale;
    int causal;
    int deterministic;
    int dtype;
} fa_bwd_params;

FA_API int fa_forward(const fa_fwd_params* p, cudaStream_t stream);
FA_API int fa_backward(const fa_bwd_params* p, cudaStream_t stream);

/*
 * fa_merge_partial -- fold a partial attention result into a running one by
 * log-sum-exp weights.  For two disjoint key sets with results (O_a, L_a) and
 * (O_b, L_b): L = log(e^L_a + e^L_b), O = e^(L_a - L) O_a + e^(L_b - L) O_b, the
 * attention over their union.  This combines the blocks of a sequence split
 * across devices ("FlashAttention-2 在昇腾 NPU 上如何做到 3 倍加速？", section
 * 6.4) and is the rescaling the online softmax applies tile by tile (section
 * 2.2).
 *
 * o_acc   : device, [rows][D] fp32, the running O; updated in place.
 * lse_acc : device, [rows] fp32 (natural log), the running LSE; updated.  Start
 *           with -inf (no key yet); a row whose sides are both -inf is left
 *           unchanged.
 * o_part  : device, [rows][D] 16-bit (dtype), a partial O, e.g. from fa_fwd_ex.
 * lse_part: device, [rows] fp32, its LSE (-inf: the partial saw no key).
 * rows, D : contiguous rows of D values (0 <= rows <= 2^33, 1 <= D <= 1024).
 * Asynchronous on stream; errors as fa_fwd (argument checks first).
 */
FA_API int fa_merge_partial(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, long long rows,
                            int D, int dtype, cudaStream_t stream);

/*
 * fa_merge_finalize -- round n fp32 values (a running O) to the 16-bit dtype
 * (nearest even) into o.  Device pointers; asynchronous on stream.
 */
FA_API int fa_merge_finalize(const float* o_acc, void* o, long long n, int dtype, cudaStream_t stream);

/*
 * fa_accumulate -- acc[i] += x[i] for n values: fp32 accumulators (device,
 * 4-byte aligned) of 16-bit partial results x (device, dtype), e.g. the
 * gradients of one K/V block in the sequence-parallel backward pass, which
 * sums the contributions of every block.  Asynchronous on stream; errors as
 * fa_merge_partial.
 */
FA_API int fa_accumulate(float* acc, const void* x, long long n, int dtype, cudaStream_t stream);

/*
 * fa_check_status -- synchronise `stream`, then report and clear the device
 * status word of the current device: FA_OK, FA_ERR_TIMEOUT if a kernel
 * stopped on a bounded wait since the last call, or FA_ERR_LAUNCH on a CUDA
 * error.  Meant for tests and diagnostics; it blocks the host.
 */
FA_API int fa_check_status(cudaStream_t stream);

/*
 * fa_last_timeout_site -- diagnostic word of the first failed wait recorded
 * by the last fa_check_status that returned FA_ERR_TIMEOUT:
 * (wait site) | (CTA index << 8).  0 if none.
 */
FA_API int fa_last_timeout_site(void);

/*
 * fa_last_cuda_error -- the CUDA failure behind the calling thread's most
 * recent FA_ERR_LAUNCH from any entry of this library: returns the cudaError_t
 * (or, for the tensor-map encoder, the CUresult) code, 0 if no call of this
 * thread has failed, and sets *site (if site is not NULL) to a static string
 * naming the call that failed.  Per host thread; a later success does not
 * clear it.  Diagnostic; the pages have no counterpart.
 */
FA_API int fa_last_cuda_error(const char** site);

/*
 * fa_selftest_timeout -- diagnostic for the failure path (no counterpart on
 * the pages): launches on `stream` a one-CTA kernel whose first mbarrier wait
 * is never satisfied.  After about 50 ms the wait gives up, the kernel
 * records a timeout in the device status word (wait site 100), releases its
 * tensor memory and ends; the context stays usable.  A following
 * fa_check_status returns FA_ERR_TIMEOUT.  Returns FA_OK when launched.
 */
FA_API int fa_selftest_timeout(cudaStream_t stream);

/* fa_status_string -- static, NUL-terminated description of a status code. */
FA_API const char* fa_status_string(int status);

/* fa_version -- library version as major*10000 + minor*100 + patch. */
FA_API int fa_version(void);

/*
 * fa_num_units -- number of work units (b, h, 256-row query block) that
 * fa_fwd distributes over persistent CTAs for the given shape; 0 for an empty
 * problem, negative fa_status on invalid sizes.  Host only, no CUDA call.
 */
FA_API long long fa_num_units(int B, int H, int S);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
