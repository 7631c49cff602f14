/*
 * rfb_attn.h -- C ABI of the B200 (sm_100a) library for attention with an
 * additive rank-factorised bias:
 *
 *     S   = s * Q K^T + U W^T                    (per batch b, head h)
 *     O   = softmax_rows(S) V
 *     LSE = log(sum_j exp(S_ij))                 (natural log, per row i)
 *
 * Where the operation comes from:
 *   - "FlashBias: Fast Computation of Attention with Bias", Abstract: attention
 *     with bias adds a bias matrix to the query-key scores; a low-rank bias
 *     lets the fused (FlashAttention-style) pipeline stay intact.
 *   - "Rank-Factorized Implicit Neural Bias: Scaling Super-Resolution
 *     Transformer with FlashAttention", Abstract: the positional bias is a
 *     low-rank product whose factors are concatenated with the content tokens
 *     along channels, so the element-wise bias addition becomes part of one
 *     dot product.  Here U, W are those factors; the library evaluates
 *     [Q | U/s] . [K | W]^T inside one fused kernel and never forms the N x N
 *     bias.
 *   - The scale s multiplies Q K^T only (the bias is added after scaling).
 *
 * Entry points: the per-window forward / backward (rfb_attn_fwd,
 * rfb_attn_bwd, rfb_attn_bwd_noalloc); variants with one factor pair per head
 * shared by all windows (rfb_attn_*_shared_bias); shifted-window attention on
 * feature maps (rfb_attn_fwd_image_windows, rfb_attn_bwd_image_windows); a dense-bias
 * comparator (rfb_attn_fwd_dense_bias); the factoriser's products
 * (rfb_bias_project); diagnostics and test hooks.  Each declaration below
 * states what differs from these conventions.
 *
 * Conventions for every entry point
 *   - Layout: all tensors are contiguous row-major.  Q, K, V, O, dO and their
 *     gradients are [B, H, N, d] bf16; U, W, dU, dW are [B, H, N, r] bf16;
 *     LSE is [B, H, N] fp32.  The bias factors are per (batch, head).
 *   - Pointers are DEVICE pointers (CUDA global memory of the current device)
 *     and must be 16-byte aligned.  The caller owns every buffer; the library
 *     allocates no device memory.
 *   - `stream` is a cudaStream_t passed as void*; NULL means the legacy
 *     default stream.  Calls are asynchronous on that stream: a return value
 *     of RFB_OK means the work was enqueued, not that it finished.  Stream
 *     order holds as usual; the short kernels are launched with programmatic
 *     stream serialisation, so they may begin while the kernel before them
 *     on the stream finishes, and wait for it before touching memory.  The
 *     calls may be captured into CUDA graphs.
 *   - Supported shapes: d in {32, 64}; r in {0, 8, 16, ..., 64} (a multiple of
 *     8); B, H, N >= 0.  B*H*N == 0 is a no-op that returns RFB_OK without
 *     touching any pointer.  When r == 0, u / w / du / dw may be NULL.
 *   - Outputs must not alias inputs.
 *   - Errors are reported only through the return code; nothing is thrown
 *     across the ABI.  Argument checks happen on the host before anything is
 *     enqueued.
 */
#ifndef RFB_ATTN_H_
#define RFB_ATTN_H_

#include <stddef.h>

#if defined(__GNUC__)
#define RFB_API __attribute__((visibility("default")))
#else
#define RFB_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RFB_OK = 0,
  RFB_ERR_INVALID_ARG = 1,    /* NULL pointer, negative size, scale not finite and > 0 */
  RFB_ERR_UNSUPPORTED = 2,    /* d or r outside the supported set, sizes beyond int32 */
  RFB_ERR_ALIGNMENT = 3,      /* a pointer is not 16-byte aligned */
  RFB_ERR_WORKSPACE = 4,      /* workspace missing or smaller than required */
  RFB_ERR_CUDA = 5,           /* a CUDA runtime / driver call failed */
  RFB_ERR_DEVICE_TIMEOUT = 6  /* a kernel's bounded wait expired (see rfb_last_device_error) */
} rfb_status;

/*
 * Forward.  Computes O and LSE as defined above.
 *   q, k, v : [B, H, N, d] bf16 inputs.
 *   u, w    : [B, H, N, r] bf16 bias factors (NULL allowed iff r == 0).
 *   o       : [B, H, N, d] bf16 output.
 *   lse     : [B, H, N] fp32 output (natural-log log-sum-exp of each score row,
 *             consumed by rfb_attn_bwd).
 *   scale   : s, finite and > 0 (usually 1/sqrt(d)); anything else is
 *             RFB_ERR_INVALID_ARG.
 */
RFB_API int rfb_attn_fwd(const void* q, const void* k, const void* v, const void* u, const void* w,
                 void* o, float* lse, int B, int H, int N, int d, int r, float scale,
                 void* stream);

/*
 * Bytes of device workspace rfb_attn_bwd needs for these sizes (fp32 row
 * statistics and the fp32 dQ | dU accumulator).  Returns 0 for unsupported or
 * empty shapes.
 */
RFB_API size_t rfb_attn_bwd_workspace_size(int B, int H, int N, int d, int r);

/*
 * Backward.  Given the forward inputs, the forward outputs o and lse, and the
 * upstream gradient dout = dL/dO, writes
 *     dq = s dS K,  dk = s dS^T Q,  dv = P^T dO,  du = dS W,  dw = dS^T U,
 * with P = softmax(S), dS = P o (dO V^T - rowsum(dO o O)).
 *   dq, dk, dv : [B, H, N, d] bf16 outputs.
 *   du, dw     : [B, H, N, r] bf16 outputs (NULL allowed iff r == 0).
 *   workspace  : device buffer of at least rfb_attn_bwd_workspace_size() bytes,
 *                16-byte aligned, owned by the caller, contents irrelevant on
 *                entry and scratch afterwards.  It must not be used by another
 *                call that runs concurrently.
 */
RFB_API int rfb_attn_bwd(const void* q, const void* k, const void* v, const void* u, const void* w,
                 const void* o, const float* lse, const void* dout, void* dq, void* dk, void* dv,
                 void* du, void* dw, void* workspace, size_t workspace_bytes, int B, int H,
                 int N, int d, int r, float scale, void* stream);

/*
 * Backward that allocates nothing (the pages have no counterpart; this is an
 * integration aid).  Same inputs, outputs and results as rfb_attn_bwd, but
 * without the workspace argument: the scratch the backward needs (per-row
 * statistics and the fp32 dQ|dU accumulator) lives in one fixed array of
 * RFB_NOALLOC_SCRATCH_BYTES bytes compiled into the library.
 *
 * Who it is for: callers that may not allocate device memory while they run
 * and have no workspace to lend -- for example a serving runtime that carves
 * up all device memory when it starts and forbids cudaMalloc afterwards, or a
 * plugin host that owns the allocator and hands its plugins nothing but their
 * input and output buffers.
 *
 * Limit: the call accepts exactly the problems for which
 * rfb_attn_bwd_workspace_size(B, H, N, d, r) <= RFB_NOALLOC_SCRATCH_BYTES,
 * i.e. about 32 + 4 (d + r) + 2 r bytes per row of B*H*N (the row
 * statistics -LSE / s and -D as six bf16 parts in a 32-byte row, with N
 * rounded up to a multiple of 128; the fp32 dQ | dU accumulator; bf16 U / s):
 * up to about 69,900 rows for d = 64, r = 32 and 161,000 rows for d = 32,
 * r = 8.  Larger problems are rejected with
 * RFB_ERR_WORKSPACE before anything is enqueued.  The call makes no
 * cudaMalloc, cudaFree or other allocating call.
 *
 * Cost and set-up: the array is device memory that CUDA reserves on a GPU
 * when this library's kernels are loaded there -- with CUDA's lazy module
 * loading, at the first library call on that device that launches a kernel
 * or looks up the array, not when the library is opened -- and keeps until
 * the process exits.  A caller that reserves the rest of the device's memory
 * up front must therefore make one library call on the device before it
 * does.  An empty call of this function (B, H or N == 0, with a supported d
 * and r and a valid scale) is enough: it loads the kernels, which reserves
 * the array, and caches the array's device address (cudaGetSymbolAddress,
 * with that device current), launching nothing.  The first call on a device,
 * empty or not, does that set-up, so make it before any stream capture on
 * the device.  An empty call returns RFB_ERR_CUDA if the set-up fails.
 *
 * Sharing: all calls on one device use the same array, which keeps whatever
 * the previous call left; each call clears the parts that must start at zero.
 * Calls whose kernels overlap on the GPU (e.g. on two unordered streams) race
 * on the array and produce wrong gradients -- order them, e.g. on one stream.
 */
#define RFB_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
RFB_API int rfb_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* u,
                                 const void* w, const void* o, const float* lse, const void* dout,
                                 void* dq, void* dk, void* dv, void* du, void* dw, int B, int H,
                                 int N, int d, int r, float scale, void* stream);

/*
 * Shared bias factors: one pair U, W per head, used by every window.
 * "Rank-Factorized Implicit Neural Bias" (Abstract) produces the bias of a
 * head from an implicit neural representation of relative positions, the same
 * for all windows of an image; these entry points take that form.  Window-head
 * (b, h) uses U[h], W[h]:
 *     O[b, h] = softmax(s Q[b, h] K[b, h]^T + U[h] W[h]^T) V[b, h].
 * Arguments, layouts, ownership and errors as in rfb_attn_fwd / rfb_attn_bwd,
 * except:
 *   u, w   : [H, N, r] bf16 (NULL allowed iff r == 0).
 *   du, dw : [H, N, r] bf16 outputs, the sums over the B windows of the
 *            per-window gradients (dU[h] = sum_b dS[b, h] W[h],
 *            dW[h] = sum_b dS[b, h]^T U[h]), accumulated in fp32.
 *   workspace : at least rfb_attn_bwd_shared_bias_workspace_size() bytes
 *            (adds fp32 [B, H, N, r] for the per-window dW).
 * With data-parallel windows on several GPUs, each rank passes its own windows
 * and sums du, dw over the ranks afterwards (an all-reduce); the library
 * itself makes no collective call.
 */
RFB_API int rfb_attn_fwd_shared_bias(const void* q, const void* k, const void* v, const void* u,
                                     const void* w, void* o, float* lse, int B, int H, int N,
                                     int d, int r, float scale, void* stream);
RFB_API size_t rfb_attn_bwd_shared_bias_workspace_size(int B, int H, int N, int d, int r);
RFB_API int rfb_attn_bwd_shared_bias(const void* q, const void* k, const void* v,
                                     const void* u, const void* w, const void* o,
                                     const float* lse, const void* dout, void* dq, void* dk,
                                     void* dv, void* du, void* dw, void* workspace,
                                     size_t workspace_bytes, int B, int H, int N, int d, int r,
                                     float scale, void* stream);

/*
 * Materialised-bias comparator (not the method): the same attention with the
 * bias given as a dense bf16 matrix per head,
 *     O[b, h] = softmax(s Q[b, h] K[b, h]^T + bias[z]) V[b, h],
 *     z = h (bias_heads == H, one matrix per head shared by all windows) or
 *     z = b H + h (bias_heads == B H),
 * i.e. the conventional form whose N x N read the rank-factorised bias avoids
 * ("FlashBias: Fast Computation of Attention with Bias", Abstract: low-rank
 * bias keeps attention fast where a materialised bias slows it down).  Forward
 * only; used to measure that difference on this hardware.
 *   bias : [bias_heads, N, N] bf16, row i holding the bias of query i.
 *   q, k, v, o, lse, scale, stream : as rfb_attn_fwd (r = 0).
 * Errors as rfb_attn_fwd; RFB_ERR_INVALID_ARG if bias_heads is neither H nor
 * B*H; RFB_ERR_UNSUPPORTED if N is not a multiple of 8 (bias rows must be
 * whole 16-byte units for the copy engine).
 */
RFB_API int rfb_attn_fwd_dense_bias(const void* q, const void* k, const void* v, const void* bias,
                                    void* o, float* lse, int B, int H, int N, int d,
                                    int bias_heads, float scale, void* stream);

/*
 * Shifted-window attention straight from feature maps (forward): the window
 * partition and the cyclic shift of SR window transformers happen in the copy
 * engine's addressing, with the bias in the rank-factorised form of
 * "Rank-Factorized Implicit Neural Bias" (Abstract).  For each image b, the
 * map rolled by (-shift, -shift) is cut into win x win windows (raster order);
 * per window and head h,
 *     O = softmax(s Q K^T + U[h] W[h]^T + M) V,
 * where M is 0 between tokens of the same region of the rolled map and -inf
 * between tokens of different regions (regions: rows [0, H-win), [H-win,
 * H-shift), [H-shift, H) times the same split of columns; all one region when
 * shift == 0); every token's O and LSE are written at its place in the
 * unrolled map.  Nothing is copied or rolled in memory.
 *   q, k, v, o : [B, img_h, img_w, heads, d] bf16 (channels-last maps).
 *   u, w       : [heads, win*win, r] bf16, row = raster position in the
 *                window (one pair per head for all windows); NULL iff r == 0.
 *   lse        : [B, img_h, img_w, heads] fp32 (natural log).
 *   win        : 8 (64 tokens per window); shift : 0 or 4.
 *   img_h, img_w : multiples of 8.
 * Errors as rfb_attn_fwd; RFB_ERR_UNSUPPORTED for other win / shift / map
 * sizes, or when the factors of all heads do not fit in shared memory at once
 * ((heads + 1) * 64 * r_pad * 4 bytes beside the input ring; up to 15 heads
 * at r <= 16, 7 at r = 32, 3 at r = 64 for d = 32; 11, 5, 2 for d = 64).
 */
RFB_API int rfb_attn_fwd_image_windows(const void* q, const void* k, const void* v,
                                       const void* u, const void* w, void* o, float* lse, int B,
                                       int img_h, int img_w, int heads, int d, int r, int win,
                                       int shift, float scale, void* stream);

/*
 * Backward of rfb_attn_fwd_image_windows: dQ, dK, dV at the tokens' map
 * positions and dU, dW of the shared factors, summed over all windows (the
 * chain rule through the roll, the window cut and the masked window
 * attention; the mask gives P = 0 between regions).  The maps are gathered
 * into window tensors (the rolled window cut, raster order inside each
 * window) in the workspace, the shared-factor backward runs on them with the
 * shifted-window mask, and dQ, dK, dV are scattered back.
 *   q, k, v, o, dout   : [B, img_h, img_w, heads, d] bf16; o and lse as
 *                        written by rfb_attn_fwd_image_windows for the same
 *                        inputs, win and shift.
 *   u, w               : [heads, win*win, r] bf16 (raster position in the
 *                        window); NULL iff r == 0.
 *   lse                : [B, img_h, img_w, heads] fp32.
 *   dq, dk, dv         : [B, img_h, img_w, heads, d] bf16 outputs.
 *   du, dw             : [heads, win*win, r] bf16 outputs (fp32 sums over the
 *                        windows, rounded once); NULL iff r == 0.
 *   workspace          : device, 16-byte aligned, at least
 *                        rfb_attn_bwd_image_windows_workspace_size() bytes
 *                        (eight bf16 window tensors, the gathered LSE and the
 *                        shared-factor backward's workspace); the caller owns
 *                        it and may reuse it once the call has completed on
 *                        the stream.
 *   win = 8, shift = 0 or 4, img_h and img_w multiples of 8.
 * Errors as rfb_attn_bwd_shared_bias; RFB_ERR_UNSUPPORTED for other win /
 * shift / map sizes.
 */
RFB_API size_t rfb_attn_bwd_image_windows_workspace_size(int B, int img_h, int img_w, int heads,
                                                         int d, int r);
RFB_API int rfb_attn_bwd_image_windows(const void* q, const void* k, const void* v,
                                       const void* u, const void* w, const void* o,
                                       const float* lse, const void* dout, void* dq, void* dk,
                                       void* dv, void* du, void* dw, void* workspace,
                                       size_t workspace_bytes, int B, int img_h, int img_w,
                                       int heads, int d, int r, int win, int shift, float scale,
                                       void* stream);

/*
 * The N x N products of the low-rank factoriser of a materialised bias (the
 * step before the attention path that turns a dense per-head bias into the
 * factors U, W; "FlashBias: Fast Computation of Attention with Bias",
 * Abstract: low-rank bias approximation):
 *     transpose == 0:  out[h] = bias[h] . x[h]
 *     transpose != 0:  out[h] = bias[h]^T . x[h]
 *   bias : [H, N, N] fp32 device pointer (row i, column j = bias[h][i][j]).
 *   x    : [H, N, k] fp32 device pointer, 1 <= k <= 80.
 *   out  : [H, N, k] fp32 device pointer, written (must not alias bias or x).
 * Accumulation in fp32; pointers 16-byte aligned.  Asynchronous on stream.
 * Errors: RFB_ERR_INVALID_ARG (negative sizes, k < 1, NULL pointers),
 * RFB_ERR_UNSUPPORTED (k > 80), RFB_ERR_ALIGNMENT.  H or N == 0 is a no-op.
 */
RFB_API int rfb_bias_project(const float* bias, const float* x, float* out, int H, int N, int k,
                             int transpose, void* stream);

/* Human-readable text for a status code (static storage). */
RFB_API const char* rfb_strerror(int status);

/*
 * Reads and clears the current device's error word, which kernels set when a
 * bounded wait expires (RFB_ERR_DEVICE_TIMEOUT in the low byte, the wait site
 * in the next byte).  Synchronises the device first.  Returns 0 if no error
 * was recorded, -RFB_ERR_CUDA if the word could not be read.
 */
RFB_API int rfb_last_device_error(void);

/*
 * Diagnostics for RFB_ERR_CUDA: the error code of the last CUDA runtime /
 * driver call that failed inside the library (a cudaError_t, or a CUresult
 * for tensor-map encoding), and in *site (if not NULL) which call it was:
 * 1 device query, 2 attribute query, 3 symbol address, 4 driver entry point,
 * 5 tensor-map encoding, 6 kernel attribute, 7 kernel launch, 8 synchronise.
 * Returns 0 if nothing has failed.
 */
RFB_API int rfb_last_cuda_error(int* site);

/*
 * Failure-detection self test: launches one CTA whose bounded wait is on an
 * mbarrier that nothing ever arrives at, with a limit of `timeout_us`
 * microseconds.  The wait expires, the kernel records RFB_ERR_DEVICE_TIMEOUT in
 * the error word and returns normally, leaving the context usable.  Returns
 * the launch status; read the outcome with rfb_last_device_error().
 */
RFB_API int rfb_selftest_wait_timeout(unsigned int timeout_us, void* stream);

/*
 * Failure-detection test hook for the attention kernels' own waits (not for
 * production use).  Every kernel launched after this call gets:
 *   limit_us  : the limit of each main-loop wait on a copy, an MMA or another
 *               role of the same CTA, in microseconds (0 restores the default
 *               of 2 s).  The exit-path waits for copies and MMAs already in
 *               flight keep 2 s.
 *   fail_site : a wait site number (the value stored in bits 8..15 of the
 *               error word) whose wait gives up at once, as if its limit had
 *               expired, or -1 for none.
 * A wait that gives up raises its CTA's abort flag and records
 * RFB_ERR_DEVICE_TIMEOUT | site << 8 in the error word; the CTA's other roles
 * leave their loops, let in-flight copies and MMAs land, free TMEM and return.
 * The call's outputs are then incomplete; the context stays usable.  The
 * setting is process-wide: restore it with rfb_debug_set_wait_limit(0, -1).
 * Returns RFB_ERR_INVALID_ARG if fail_site is outside [-1, 255].
 */
RFB_API int rfb_debug_set_wait_limit(unsigned int limit_us, int fail_site);

/*
 * Optional per-kernel timing.  While enabled, every kernel launch made by
 * rfb_attn_fwd / rfb_attn_bwd is bracketed by two CUDA events recorded on the
 * call's stream.  rfb_profile_read synchronises on those events and returns,
 * per kernel id (0 forward, 1 backward row statistics, 2 backward main,
 * 3 backward gradient cast; RFB_PROFILE_KERNELS ids in all), the summed
 * milliseconds and the number of launches since the last read, then clears
 * them.  Arrays must hold RFB_PROFILE_KERNELS entries.  The events are created
 * by the library (no device memory is allocated).
 */
#define RFB_PROFILE_KERNELS 4
RFB_API int rfb_profile_enable(int on);
RFB_API int rfb_profile_read(float* ms, int* launches);
RFB_API const char* rfb_profile_kernel_name(int id);

/*
 * Self test of the software exp2 that the kernels use for part of the softmax
 * exponentials: y[i] = 2^x[i] for i < n, computed on the device by that code
 * path (x, y device pointers, fp32).  Inputs below -125 return about 2^-125.
 */
RFB_API int rfb_selftest_soft_exp2(const float* x, float* y, int n, void* stream);

/* Library version string. */
RFB_API const char* rfb_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RFB_ATTN_H_ */
