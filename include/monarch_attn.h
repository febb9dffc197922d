/*
 * monarch_attn.h -- C ABI of the MonarchAttention forward pass on B200 (sm_100a).
 *
 * What it computes (one head; the library loops over B*H independent heads):
 *
 *   MonarchAttention replaces softmax(Q K^T / sqrt(d)) V by M V, where M is a
 *   Monarch matrix M = P L P^T R with block-diagonal L and R (MonarchRT
 *   summary, "Method" (1)) found by T steps of alternating maximisation of
 *   the softmax variational objective  f(M) = <M, Q K^T / sqrt(d)> + H(M)
 *   over block rank-one factors (MonarchAttention AI summary, "Approach";
 *   OpenReview discussion of MonarchAttention, eq. (6) and "Alternating
 *   Maximization with Constraints").  M V is applied without forming the
 *   N x N matrix; compute is Theta(N sqrt(N) d) and I/O Theta(N d)
 *   (MonarchAttention abstract).  The tiled variant cuts every Monarch block
 *   into c1 x c2 independently rank-one sub-tiles (MonarchRT summary,
 *   "Key claims", Theorem 4.1; "Method" (2)).
 *
 *   Token n = l*b2 + i (l in [b1] the chunk, i in [b2] the position in the
 *   chunk).  For a (f,h,w) video latent flattened row-major, (b1,b2) = (f*h, w)
 *   is the aligned (fh,w) layout (MonarchRT summary, "Key claims").
 *   Row groups p of l and column groups q of j are contiguous, sizes
 *   differing by at most one, larger groups first.
 *   One step = R-update then L-update; the initial L and R are uniform;
 *   T = 0 returns the uniform Monarch matrix applied to V.
 *
 * Layout: q, k, v, out are contiguous row-major (B, H, N, d) with
 *   N = b1*b2, i.e. element (b, h, n, x) at ((b*H + h)*N + n)*d + x.
 *
 * Ownership: the caller owns q, k, v, out.  `out` must not overlap any input.
 *   Device pointers must be 16-byte aligned.  The library owns one cached
 *   device workspace per device (allocated on first use, grown on demand,
 *   freed by monarch_attn_release_workspace); calls on one device that may
 *   overlap on the GPU must be ordered on one stream, because they share it.
 *
 * Semantics: asynchronous on `stream` (host-buffer variant excepted).
 *   Deterministic: no atomics in any reduction.
 *
 * Errors: every entry point returns 0 on success or a negative status:
 *   MONARCH_ERR_INVALID_ARG  null/misaligned pointer, B,H,b1,b2 < 1, T < 0,
 *                            c1 not in [1,b1], c2 not in [1,b2], size overflow.
 *   MONARCH_ERR_UNSUPPORTED  d not in [1, 256] (d a multiple of 8 on the
 *                            tensor-core path, which otherwise falls back).
 *   MONARCH_ERR_CUDA         a CUDA launch, copy or allocation failed (the
 *                            CUDA error string is kept, see strerror).
 *   MONARCH_ERR_DEVICE_TIMEOUT a bounded device wait expired; the kernel
 *                            stopped and the context stays usable.  Reported
 *                            by monarch_attn_check() (and by the host-buffer
 *                            entry point, which checks before returning).
 *   MONARCH_ERR_NO_MEMORY    the workspace could not be allocated.
 *   MONARCH_ERR_SCRATCH_LIMIT the shape needs more scratch than the static
 *                            array of monarch_attn_fwd_noalloc holds.
 */
#ifndef MONARCH_ATTN_H
#define MONARCH_ATTN_H

#include <stddef.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MONARCH_API __attribute__((visibility("default")))
#else
#define MONARCH_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MONARCH_OK                  0
#define MONARCH_ERR_INVALID_ARG    -1
#define MONARCH_ERR_UNSUPPORTED    -2
#define MONARCH_ERR_CUDA           -3
#define MONARCH_ERR_DEVICE_TIMEOUT -4
#define MONARCH_ERR_NO_MEMORY      -5  /* also forced by MONARCH_ATTN_FAIL_ALLOC=1 (see below) */
#define MONARCH_ERR_SCRATCH_LIMIT  -6

#define MONARCH_DTYPE_BF16 0
#define MONARCH_DTYPE_F32  1

/* Forward pass, bf16 in/out, fp32 accumulation.
 * q, k, v, out: device pointers to __nv_bfloat16, (B, H, N, d), N = b1*b2.
 * (Pages: MonarchAttention abstract and AI summary "Approach"; MonarchRT
 * summary "Method" (2)-(3) for c1, c2 > 1.) */
MONARCH_API int monarch_attn_fwd(const void* q, const void* k, const void* v, void* out,
                     int B, int H, int b1, int b2, int d, int T, int c1, int c2,
                     cudaStream_t stream);

/* Same computation with float32 in/out and float32 arithmetic throughout
 * (no TF32). */
MONARCH_API int monarch_attn_fwd_f32(const float* q, const float* k, const float* v, float* out,
                         int B, int H, int b1, int b2, int d, int T, int c1, int c2,
                         cudaStream_t stream);

/* Same computation on HOST buffers (dtype MONARCH_DTYPE_BF16 or _F32).
 * Copies q, k, v to cached device staging buffers, runs the forward pass and
 * copies the result into out_host, in groups of heads (up to 12, each with
 * at least 32 MiB of q, k and v; smaller calls take one group): a group's
 * copy-in (on a copy stream of the library's own), its forward pass (on
 * `stream`) and its copy-out (on a second copy stream) overlap the
 * neighbouring groups', ordered by events after the work already on
 * `stream`.  The output is bit-identical to monarch_attn_fwd's (every group
 * runs the kernels of the whole call).  Synchronises `stream` and both copy
 * streams before returning, on success and on error.  Pinned host memory
 * gives full PCIe/C2C bandwidth and the overlap; pageable memory works but
 * is slower. */
MONARCH_API int monarch_attn_fwd_host(int dtype, const void* q_host, const void* k_host,
                          const void* v_host, void* out_host,
                          int B, int H, int b1, int b2, int d, int T, int c1, int c2,
                          cudaStream_t stream);

/* Forward pass, bf16, that allocates nothing.  The pages have no
 * counterpart of this entry point: it is for callers that cannot allocate
 * device memory when they call, such as a real-time frame loop (cudaMalloc
 * and cudaFree can synchronise the device and stall a frame past its
 * deadline) or a host framework that reserves all device memory for its own
 * pool and leaves a plugin no room for a cache of its own.
 *
 * Arguments, layout and result are those of monarch_attn_fwd, and it runs
 * the same kernels, so the output is bit-identical to monarch_attn_fwd's on
 * the same inputs.  Only the shapes those kernels take run here (d = 64 or
 * 128 and T >= 1; small untiled heads with T >= 2 need no scratch at all);
 * any other shape returns MONARCH_ERR_UNSUPPORTED.  The caller still passes
 * q, k, v and out.
 *
 * Scratch: one static device array of 64 MiB (67108864 bytes) on every
 * device that loads this library, held until the process exits.  A shape
 * whose scratch (monarch_attn_workspace_bytes(..., MONARCH_DTYPE_BF16))
 * exceeds it returns MONARCH_ERR_SCRATCH_LIMIT (the 720p config does).
 * CUDA loads device code lazily by default: the first call on a device
 * looks up the array's device address, which loads it there and commits the
 * 64 MiB, so make that first call at initialisation, while device memory is
 * still free and before any stream capture.  Later calls of a shape that
 * already ran on the device neither allocate nor change the device's free
 * memory (the first call of another shape may make CUDA load the code of
 * kernels not run before).  Every call on a device shares the
 * array and leaves the last call's contents in it; the kernels write every
 * scratch entry before they read it.  Calls that overlap on the GPU (other
 * streams, or unordered host threads) race on the array: order them on one
 * stream.  No cudaMalloc, cudaFree or other allocating routine is called.
 *
 * A bounded device wait that expires (the kernel stops early and out is
 * invalid) sets the library's device status word, which is a static device
 * variable too: monarch_attn_check() reports it as
 * MONARCH_ERR_DEVICE_TIMEOUT and clears it. */
MONARCH_API int monarch_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                         int B, int H, int b1, int b2, int d, int T, int c1,
                                         int c2, cudaStream_t stream);

/* Aligned block layouts of a video latent with f frames of h x w tokens,
 * stored in raster order (token n = (t*h + y)*w + x for frame t, row y,
 * column x).  A layout names the axes that form the Monarch row index l
 * (first) and the position index i (second); b1 is the product of the first
 * group's sizes, b2 of the second's (MonarchRT summary, "Key claims" and
 * "Method": block sizes aligned with the latent's (f, h, w) axes).  Inside a
 * group the axes keep the order written. */
#define MONARCH_LAYOUT_FH_W 0  /* l = (f, h), i = w:      b1 = f*h, b2 = w   */
#define MONARCH_LAYOUT_W_FH 1  /* l = w,      i = (f, h): b1 = w,   b2 = f*h */
#define MONARCH_LAYOUT_F_HW 2  /* l = f,      i = (h, w): b1 = f,   b2 = h*w */
#define MONARCH_LAYOUT_HW_F 3  /* l = (h, w), i = f:      b1 = h*w, b2 = f   */
#define MONARCH_LAYOUT_FW_H 4  /* l = (f, w), i = h:      b1 = f*w, b2 = h   */
#define MONARCH_LAYOUT_H_FW 5  /* l = h,      i = (f, w): b1 = h,   b2 = f*w */

/* Forward pass on a video latent in one of the aligned layouts above.
 * q, k, v, out: device pointers (B, H, N, d) in raster token order,
 * N = f*h*w, dtype MONARCH_DTYPE_BF16 (__nv_bfloat16) or MONARCH_DTYPE_F32.
 * The result is monarch_attn_fwd / _f32 applied to the tokens reordered
 * into the layout's Monarch order (token l*b2 + i), with the output put back
 * into raster order.  (fh, w) and (f, hw) are already in Monarch order and
 * run directly.  (w, fh) and (hw, f) are its transpose (raster token
 * i*b1 + l), which the bf16 tensor-core kernels read and write in place when
 * they run every step of the shape.  Otherwise, and for (fw, h) and (h, fw),
 * the layout gathers q, k, v into a cached device
 * buffer of 4*B*H*N*d elements (allocated on first use, grown on demand,
 * freed by monarch_attn_release_workspace) and scatters the output back: one
 * extra read and write of each tensor.  The gather uses a table of N raster
 * indices per (f, h, w, layout) and device, built and uploaded with a
 * synchronous copy on its first use and kept until
 * monarch_attn_release_workspace.  Otherwise asynchronous on `stream`; errors
 * as for monarch_attn_fwd, plus MONARCH_ERR_INVALID_ARG for an unknown
 * layout. */
MONARCH_API int monarch_attn_fwd_video(int dtype, const void* q, const void* k, const void* v,
                                       void* out, int B, int H, int f, int h, int w, int layout,
                                       int d, int T, int c1, int c2, cudaStream_t stream);

/* Forward pass on n_real <= b1*b2 tokens per head, padded to the b1*b2
 * grid (MonarchAttention OpenReview discussion, author response on choosing
 * block sizes: the chunk count is the ceiling of N over the block size, and
 * ViT's 197 tokens are pre-padded).  The n_pad = b1*b2 - n_real pad tokens
 * sit before the real ones (pad_front = 1, pre-padding) or after them
 * (pad_front = 0).  The objective is taken over the real tokens only: pad
 * keys get zero R weight, a column group without a real key zero L weight,
 * and pad query rows are left out of the aggregations.
 *
 * dtype: MONARCH_DTYPE_BF16 (__nv_bfloat16) or MONARCH_DTYPE_F32.
 * q, k, v, out: device pointers, (B, H, n_real, d) contiguous, real tokens
 * only.  Small untiled bf16 heads (b1, b2 <= 16, d = 64, T >= 2) run in
 * place; other shapes copy q, k, v into a cached device buffer of
 * 4*B*H*b1*b2*d elements in grid order (allocated on first use, grown on
 * demand, freed by monarch_attn_release_workspace), run the masked forward
 * pass there and copy the real output rows back.  n_real = b1*b2 is
 * monarch_attn_fwd / _f32.  Asynchronous on `stream`.  Errors as for
 * monarch_attn_fwd, plus MONARCH_ERR_INVALID_ARG for n_real outside
 * [1, b1*b2], pad_front not 0 or 1, or an unknown dtype. */
MONARCH_API int monarch_attn_fwd_padded(int dtype, const void* q, const void* k, const void* v,
                                        void* out, int B, int H, int n_real, int b1, int b2,
                                        int pad_front, int d, int T, int c1, int c2,
                                        cudaStream_t stream);

/* Backward pass of the T = 1 forward (one refinement step, the setting the
 * pages finetune with: MonarchRT summary, "Method" (3), forward and
 * backward kernels): dq, dk, dv = gradients of sum(O * dout) with respect
 * to q, k, v, where O = monarch_attn_fwd / _f32(q, k, v, ..., T = 1).
 *
 * dtype: MONARCH_DTYPE_BF16 or MONARCH_DTYPE_F32; all seven pointers are
 * device buffers of that type, (B, H, N, d) contiguous, N = b1*b2,
 * 16-byte aligned; dq, dk, dv must not overlap each other or any input.
 * The forward intermediates are recomputed.  bf16 calls with d in {64, 128},
 * b1 c2 <= 128 and row groups of <= 128 rows run the L side on the tensor
 * cores (bf16 operands, fp32 accumulation), and with c1 = c2 = 1 and
 * b2 <= 128 the R side too; every other case, and the final sum of dq,
 * runs in fp32 on SIMT kernels.  The library keeps a cached workspace per
 * device of about G (1.5 c1 b2 d + 7 N c1 c2 d + 2 N c1 c2 + N d + 2 N +
 * 2 b1 c1 b2^2) floats (G = B*H; allocated on first use, grown on demand,
 * freed by monarch_attn_release_workspace).  Deterministic (fixed-order
 * reductions, no atomics).  Asynchronous on `stream`.  Errors as for
 * monarch_attn_fwd, plus MONARCH_ERR_DEVICE_TIMEOUT from monarch_attn_check
 * if a tensor-core kernel's bounded wait expired; T other than 1 returns
 * MONARCH_ERR_UNSUPPORTED. */
MONARCH_API int monarch_attn_bwd(int dtype, const void* q, const void* k, const void* v,
                                 const void* dout, void* dq, void* dk, void* dv, int B, int H,
                                 int b1, int b2, int d, int T, int c1, int c2,
                                 cudaStream_t stream);

/* Bytes of device workspace a call with these arguments uses (0 on invalid
 * arguments).  dtype is MONARCH_DTYPE_BF16 or MONARCH_DTYPE_F32. */
MONARCH_API size_t monarch_attn_workspace_bytes(int B, int H, int b1, int b2, int d, int T,
                                    int c1, int c2, int dtype);

/* Fault injection for tests: while the environment variable
 * MONARCH_ATTN_FAIL_ALLOC is "1", every device allocation the library would
 * make for its workspace or staging buffers fails with
 * MONARCH_ERR_NO_MEMORY before any device call (calls whose cached buffers
 * are already large enough are unaffected). */

/* Free the cached workspace and staging buffers of every device.  Must not
 * be called while a forward pass is still running on the GPU. */
MONARCH_API void monarch_attn_release_workspace(void);

/* Synchronise `stream` and report a device-side failure (a bounded wait that
 * expired, in any entry point) recorded on the current device since the
 * last check; clears the flag.  The flag is a static device variable: this
 * call reads it with a 4-byte copy and allocates nothing. */
MONARCH_API int monarch_attn_check(cudaStream_t stream);

/* Human-readable text for a status code (includes the last CUDA error text
 * for MONARCH_ERR_CUDA). */
MONARCH_API const char* monarch_attn_strerror(int status);

/* Number of kernels the most recent forward call on this host thread
 * launched (for launch accounting in benchmarks). */
MONARCH_API int monarch_attn_last_launches(void);

/* Per-kernel timing (a profiling aid; off by default).  While enabled, every
 * kernel a forward call launches is bracketed by two CUDA events recorded on
 * the call's stream.  Returns the previous setting. */
MONARCH_API int monarch_attn_timing_enable(int enable);

/* Synchronise on the recorded events and report, per kernel name, the summed
 * device milliseconds and launch count since the previous read (which this
 * read clears).  Up to max_kernels entries are written: names as
 * NUL-terminated strings of at most name_len bytes at names + i*name_len,
 * ms_total[i], launches[i].  Returns the number of distinct kernels, or a
 * negative status. */
MONARCH_API int monarch_attn_timing_read(int max_kernels, char* names, int name_len,
                                         double* ms_total, long* launches);

/* Self-test of the device-timeout path (not part of the method): launches
 * one CTA on `stream` that waits on a barrier nothing arrives on; after
 * limit_ns nanoseconds (at most 10 s) the wait gives up, records the timeout
 * in the device status word and the kernel returns normally, leaving the
 * context usable.  A following monarch_attn_check() returns
 * MONARCH_ERR_DEVICE_TIMEOUT.  Returns MONARCH_OK once launched. */
MONARCH_API int monarch_attn_selftest_timeout(unsigned long long limit_ns, cudaStream_t stream);

/* Library version, (major << 16) | minor. */
MONARCH_API int monarch_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MONARCH_ATTN_H */
