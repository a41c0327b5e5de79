/*
 * causalconv.h -- C ABI of the B200 (sm_100a) causal sequence convolution.
 *
 * Operation (Caracal: Causal Architecture via Spectral Mixing, "Key design 1:
 * Multi-Head Fourier module" and "Key design 2: frequency-domain causal
 * mask"): for every batch b and channel d of channel-last tensors,
 *
 *     r[b, t, d] = sum_{j=0..t} v[b, j, d] * g[b, t-j, d],     0 <= t < L,
 *
 * computed the way the pages describe: each (b, d) row is zero-padded to
 * N >= 2L, Fourier-transformed, multiplied pointwise, inverse-transformed and
 * truncated to its first L entries.  x_v (value stream) and x_g (gate stream)
 * of the Multi-Head Fourier module are v and g here.
 *
 * Layout: v, g and r are contiguous row-major [B, L, D] arrays ("channel
 * last"): element (b, t, d) is at index (b*L + t)*D + d.
 *
 * Ownership and execution: every pointer named *_dev or taken by the three
 * conv entry points is a DEVICE pointer on the calling thread's current CUDA
 * device, owned by the caller.  Work is enqueued on `stream` (a cudaStream_t;
 * NULL = the legacy default stream) and the call returns without
 * synchronising.  The library never allocates device memory on these calls;
 * its small twiddle/constant tables are static device arrays filled once per
 * device on the first call (that first call synchronises `stream` once).
 *
 * Errors: every argument check runs on the host before any launch; a failed
 * check returns a non-zero cc_status and enqueues nothing.  CC_ERR_CUDA means
 * a CUDA API call or the launch itself failed (cudaGetLastError after launch).
 * Errors raised later by the asynchronous kernel surface at the caller's next
 * synchronisation, as with any CUDA kernel.
 */
#ifndef CAUSALCONV_H
#define CAUSALCONV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CC_API __attribute__((visibility("default")))
#else
#define CC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CC_OK = 0,
    CC_ERR_INVALID_ARG = 1, /* null pointer, B/L/D < 1, size overflow, bad dtype */
    CC_ERR_UNSUPPORTED = 2, /* L beyond the supported range for this dtype      */
    CC_ERR_ALIAS = 3,       /* r overlaps v or g                                */
    CC_ERR_WORKSPACE = 4,   /* workspace smaller than causal_conv_workspace_bytes */
    CC_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed      */
    CC_ERR_NOT_DEVICE = 6,  /* a pointer is not device memory of the current device */
    CC_ERR_SCRATCH_LIMIT = 7 /* beyond the fixed scratch of causal_conv_decode_f32_noalloc */
} cc_status;

typedef enum {
    CC_DTYPE_F32 = 0,  /* float32 in, float32 out, float32 arithmetic        */
    CC_DTYPE_BF16 = 1, /* bfloat16 in/out (uint16 bit patterns), float32 arithmetic */
    CC_DTYPE_I32 = 2   /* int32 in/out, exact arithmetic mod p = 2013265921   */
} cc_dtype;

/*
 * causal_fftconv_f32 -- float32 causal convolution via a fused
 * pad -> FFT -> multiply -> inverse FFT -> truncate kernel.
 *
 *   v, g  [B, L, D] float32 inputs (device).   r  [B, L, D] float32 output
 *   (device), must not overlap v or g.  B, L, D >= 1.
 *   workspace / workspace_bytes: device scratch of at least
 *   causal_conv_workspace_bytes(CC_DTYPE_F32, B, L, D) bytes (0 for every
 *   supported L: NULL, 0 is valid).  A workspace of at least
 *   causal_conv_fast_workspace_bytes(...) bytes (nonzero for 4096 < L),
 *   16-byte aligned, makes long rows take the four-step path through it; it
 *   must then not overlap v, g or r (CC_ERR_ALIAS).  Caller-owned; its
 *   contents are scratch, undefined after the call.
 *
 * Accuracy: |r - r_exact| <= 1e-5 * sum_j |v_j g_{t-j}| per element on the
 * tested workloads; outputs with t < 32 are summed directly (no transform),
 * because the rounding error of a float transform is spread evenly over a row
 * and exceeds that per-element bound where the exact sum is tiny
 * ("Catastrophic Token Leakage in Convolutional Sequence Modeling", TL;DR).
 * Supported: 1 <= L <= 65536.
 */
CC_API int causal_fftconv_f32(const float *v, const float *g, float *r,
                       int64_t B, int64_t L, int64_t D,
                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * causal_fftconv_bf16 -- as causal_fftconv_f32 with bfloat16 inputs and
 * output (raw 16-bit patterns), float32 transform arithmetic and
 * round-to-nearest-even on the output.  Supported: 1 <= L <= 65536.
 */
CC_API int causal_fftconv_bf16(const uint16_t *v, const uint16_t *g, uint16_t *r,
                        int64_t B, int64_t L, int64_t D,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * causal_ntt_conv_i32 -- exact integer causal convolution through a
 * number-theoretic transform mod p = 2013265921 = 15 * 2^27 + 1 (primitive
 * root 31), the leakage-free primitive proposed in "Catastrophic Token Leakage
 * in Convolutional Sequence Modeling and How to Mitigate It" (abstract).
 *
 *   v, g  [B, L, D] int32 (device); negative values are taken mod p.
 *   r     [B, L, D] int32 (device): the centered residue of the true sum,
 *         i.e. the unique value in [-(p-1)/2, (p-1)/2] congruent to it mod p.
 *         It equals the true sum whenever |sum| <= (p-1)/2, e.g. whenever
 *         L * max|v| * max|g| <= 1006632960 (documented precondition; not
 *         checked, since checking would read the inputs).
 * The result is bit-exact and deterministic.  Supported: 1 <= L <= 8192.
 */
CC_API int causal_ntt_conv_i32(const int32_t *v, const int32_t *g, int32_t *r,
                        int64_t B, int64_t L, int64_t D,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * causal_fftconv_bwd_f32 -- gradients of the causal convolution for training
 * (the models on "Caracal: Causal Architecture via Spectral Mixing" train with
 * next-token cross-entropy, "Loss / training strategy").  Given
 * dr = dLoss/dr, per (b, d) row:
 *
 *     dv[b, j, d] = sum_{t=j..L-1} dr[b, t, d] * g[b, t-j, d]
 *     dg[b, k, d] = sum_{t=k..L-1} dr[b, t, d] * v[b, t-k, d]
 *
 * Both are anti-causal correlations; with rev(x)_t = x_{L-1-t} they equal
 * rev(conv(rev(dr), g)) and rev(conv(rev(dr), v)), which is how they are
 * computed: two launches of the forward kernels with time-reversed input and
 * output indexing (no extra copies).  For L <= 1024 the dg launch runs on a
 * library-owned stream of the device, forked from `stream` by an event and
 * joined back to it, so it fills the SMs the dv launch's last wave leaves
 * idle; `stream` still orders everything after the call (capturable in a
 * CUDA graph like any fork and join).
 *   dr, v, g  [B, L, D] float32 (device); dv, dg [B, L, D] float32 outputs
 *   (device), overlapping none of the inputs or each other.
 * Accuracy, ranges, workspace and errors as causal_fftconv_f32, with the
 * bound taken against sum_t |dr_t g_{t-j}| (resp. |dr_t v_{t-k}|).
 */
CC_API int causal_fftconv_bwd_f32(const float *dr, const float *v, const float *g, float *dv, float *dg,
                                  int64_t B, int64_t L, int64_t D,
                                  void *workspace, size_t workspace_bytes, void *stream);

/* causal_fftconv_bwd_bf16 -- as causal_fftconv_bwd_f32 with bfloat16 I/O. */
CC_API int causal_fftconv_bwd_bf16(const uint16_t *dr, const uint16_t *v, const uint16_t *g, uint16_t *dv,
                                   uint16_t *dg, int64_t B, int64_t L, int64_t D,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * causal_conv_decode_f32 -- one autoregressive step: the output of the newest
 * position t from cached value and gate streams (next-token prediction in
 * "Caracal: Causal Architecture via Spectral Mixing", framework figure):
 *
 *     r[b, d] = sum_{j=0..t} v[b, j, d] * g[b, t-j, d]
 *
 *   v, g   [B, Lcap, D] float32 caches (device), positions 0..t filled
 *   r      [B, D] float32 output (device), overlapping neither cache
 *   t      0 <= t < Lcap, the same position for every batch row
 *   workspace  device scratch of at least causal_conv_decode_workspace_bytes()
 *              bytes (fp64 partial sums of the split reduction; required)
 * Direct O(t) summation (no transform), split over j across the GPU, fp64
 * accumulation, fixed-order reduction: deterministic and within one float
 * rounding of the exact sum.  B <= 65535.  Errors as causal_fftconv_f32;
 * int32 is CC_ERR_UNSUPPORTED.
 */
CC_API int causal_conv_decode_f32(const float *v, const float *g, float *r, int64_t B, int64_t Lcap, int64_t D,
                                  int64_t t, void *workspace, size_t workspace_bytes, void *stream);

/* causal_conv_decode_bf16 -- as causal_conv_decode_f32 with bfloat16 caches and output. */
CC_API int causal_conv_decode_bf16(const uint16_t *v, const uint16_t *g, uint16_t *r, int64_t B, int64_t Lcap,
                                   int64_t D, int64_t t, void *workspace, size_t workspace_bytes, void *stream);

/*
 * causal_conv_decode_f32_noalloc -- causal_conv_decode_f32 for callers that
 * cannot allocate device memory: code that runs inside an engine which owns
 * all device memory through its own pool and forbids allocations behind its
 * back, or code on a path that must not pay the device-wide synchronisation
 * cudaFree implies.  The pages have no counterpart; this is a library entry
 * point, not part of the method.
 *
 * Arguments and result are those of causal_conv_decode_f32 without the
 * workspace: the caller still passes the caches v, g and the output r.  The
 * fp64 partial sums go to one static device buffer of 8 MiB inside the
 * library, which every GPU that loads the library holds until the process
 * exits.  The first call on a device looks the buffer's address up (once,
 * with that device current; again after a cudaDeviceReset replaced the
 * device's context); make that first call before any stream capture.
 * The function calls no cudaMalloc, cudaFree or other allocating routine.
 * Under CUDA's lazy module loading (the default since CUDA 12) the first call
 * into this library on a device -- any entry point -- loads the library's
 * device code there, and that load reserves all its static device memory at
 * once: this 8 MiB buffer plus under 1 MiB of transform tables.  A caller
 * whose memory pool must see no reservation later should make one warm-up
 * call (of this or any entry point) before it hands memory control to the
 * pool; after that, calls reserve nothing.
 *
 * Limit: a problem whose partial sums need more than 8 MiB, i.e. for which
 * causal_conv_decode_workspace_bytes(CC_DTYPE_F32, B, D, t) > 8388608 (the
 * small_f32 shape B = 8, D = 768, t = 1023 needs 768 KiB), returns
 * CC_ERR_SCRATCH_LIMIT before anything is enqueued.  Every call on a device
 * shares the one buffer and leaves its partial sums there; nothing in it has
 * to start at zero (each call writes every slot it reads), but calls whose
 * work overlaps on the GPU (other streams, other host threads) race on the
 * buffer: order them.
 */
CC_API int causal_conv_decode_f32_noalloc(const float *v, const float *g, float *r, int64_t B, int64_t Lcap,
                                          int64_t D, int64_t t, void *stream);

/* Workspace bytes causal_conv_decode_* needs for (B, D, t); (size_t)-1 if invalid. */
CC_API size_t causal_conv_decode_workspace_bytes(int dtype, int64_t B, int64_t D, int64_t t);

/*
 * causal_conv_from_host -- the same convolution for HOST buffers: the copy of
 * v_host and g_host into the caller's device buffers v_dev and g_dev, the
 * convolution into r_dev, and the copy of r_dev back into r_host, ordered
 * after the work already on `stream`; `stream` waits for the last copy back
 * (asynchronous: synchronise `stream` before reading r_host; pass pinned host
 * memory, or the copies are synchronous).  With B >= 2 the batches go in up
 * to 4 pieces on two library-owned streams of the device, so the upload and
 * transform of one piece overlap the download of the previous one (copies in
 * both directions at once); concurrent calls on one device are serialised
 * while they enqueue.
 *   dtype: a cc_dtype.  All six buffers hold B*L*D elements of that type.
 * Errors as for the device entry points; nothing is enqueued on an argument
 * error (a CUDA error part-way may leave earlier pieces enqueued).
 */
CC_API int causal_conv_from_host(int dtype, const void *v_host, const void *g_host, void *r_host,
                          void *v_dev, void *g_dev, void *r_dev,
                          int64_t B, int64_t L, int64_t D,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * causal_conv_fast_workspace_bytes -- optional workspace for rows longer than
 * one CTA holds (4096 < L <= 65536, float paths; transform length N = 131072).
 * Without it such a row is transformed by a cluster of 8 CTAs reading the
 * channel-last tensors straight (time steps D elements apart; 8-CTA clusters
 * fit 120 of B200's 148 SMs).  When causal_fftconv_f32/bf16 and the backward
 * entry points receive a 16-byte-aligned workspace of at least this many
 * bytes they take the four-step path instead (Caracal, limitations: 100k+
 * contexts): per row the sums of squares of v and g, the 256-point DFTs over
 * n2 of t = n1 + 512 n2, the 512-point DFTs over n1 with the spectral product
 * and the first half of the real-output inverse, then the last inverse step
 * with the stores -- each pass on every SM, exchanging the partial transforms
 * through the workspace (N x B x D float2, rows innermost, then 64 float2 of
 * norm partials and one float2 of scales per row).  Same convolution, same
 * accuracy bound, a different summation order from the single-pass path.
 * The workspace must not overlap any tensor of the call (CC_ERR_ALIAS); its
 * contents are scratch.  A smaller or misaligned workspace (or none) selects
 * the single-pass path.  Returns 0 when no such path applies (L <= 4096, the
 * NTT path, B x D beyond INT32_MAX) and for invalid arguments.
 */
CC_API size_t causal_conv_fast_workspace_bytes(int dtype, int64_t B, int64_t L, int64_t D);

/* Device workspace bytes the conv entry points need for this problem (0 when
 * no scratch is needed).  Returns (size_t)-1 for an invalid dtype/shape. */
CC_API size_t causal_conv_workspace_bytes(int dtype, int64_t B, int64_t L, int64_t D);

/* Largest supported L for a dtype (0 for an unknown dtype). */
CC_API int64_t causal_conv_max_len(int dtype);

/* Static text for a cc_status value. */
CC_API const char *causal_conv_strerror(int status);

/*
 * causal_ntt_params -- host-only query of the transform constants the NTT
 * path uses for transform length N (a power of two, 2 <= N <= 2^27):
 *   out[0] = p, out[1] = omega_N = 31^((p-1)/N) mod p (an element of order
 *   exactly N), out[2] = omega_N^-1 mod p, out[3] = N^-1 mod p,
 *   out[4] = p^-1 mod 2^32 (Montgomery reduction with R = 2^32),
 *   out[5] = 2^64 mod p (R^2 mod p).
 * Returns CC_OK, or CC_ERR_INVALID_ARG for a bad N or NULL out.  Launches
 * nothing and touches no device.
 */
CC_API int causal_ntt_params(int64_t N, uint32_t out[6]);

/*
 * causal_mhf_gate_f32 / _bf16 -- the gate stream of the Multi-Head Fourier
 * block (Caracal: Causal Architecture via Spectral Mixing, "Key design 1":
 * x_g = Conv1d_G2(sigma(Linear_G1(x_norm))), a 1-D convolution grouped by
 * head), starting from a = Linear_G1(x_norm):
 *
 *   g[b,t,hC+n] = bias[hC+n]
 *               + sum_{k<K} sum_{c<C} w[hC+n][c][k] * sigmoid(a[b, t-(K-1)+k, hC+c])
 *
 * with C = D / H channels a head and terms with t-(K-1)+k < 0 left out (a
 * causal convolution: K-1 zeros on the left).  sigma is the logistic
 * function.  Readings where the page is silent: causal padding (a centred
 * kernel would let g_t see future tokens), kernel size K a parameter, bias
 * as in a default Conv1d.
 *   a     [B, L, D] device array, channel-last (bf16: uint16 bit patterns);
 *   w     [D, C, K] float32 device array (the grouped Conv1d weight layout:
 *         output channel, input channel within the head, tap);
 *   bias  [D] float32 device array, or NULL for no bias;
 *   g     [B, L, D] device output, same dtype as a (bf16: rounded to nearest
 *         even); must not overlap a, w or bias (CC_ERR_ALIAS);
 *   H     number of heads, D % H == 0 (else CC_ERR_INVALID_ARG); the head
 *         width C = D / H must be 16, 32 or 64 and 1 <= K <= 4, else
 *         CC_ERR_UNSUPPORTED; L is limited as for causal_fftconv_f32.
 * The contraction runs on the tensor cores (tf32 with each operand split
 * into two tf32 parts, fp32 accumulation), so g carries fp32-level error:
 * |g - g_exact| stays far below 1e-6 * (|bias| + sum |w| sigmoid(a)).
 * Stream-ordered and asynchronous on `stream`; allocates nothing.  Returns
 * CC_OK or an error status before launching anything.
 */
CC_API int causal_mhf_gate_f32(const float *a, const float *w, const float *bias, float *g, int64_t B, int64_t L,
                               int64_t D, int64_t H, int64_t K, void *stream);
CC_API int causal_mhf_gate_bf16(const uint16_t *a, const float *w, const float *bias, uint16_t *g, int64_t B,
                                int64_t L, int64_t D, int64_t H, int64_t K, void *stream);

/*
 * causal_mhf_gated_conv_f32 / _bf16 -- the gate stream followed by the
 * causal convolution: r = causal_fftconv(v, causal_mhf_gate(a, w, bias)).
 * v, a, r are [B, L, D] device arrays of the entry's dtype; w, bias as for
 * causal_mhf_gate_f32.  The gate is written once into the caller's
 * workspace (at least causal_mhf_gated_conv_workspace_bytes() bytes of
 * device memory, overlapping none of the arrays: CC_ERR_WORKSPACE /
 * CC_ERR_ALIAS), then the convolution reads it.  r must overlap no input.
 * Two launches on `stream`; allocates nothing.
 */
CC_API int causal_mhf_gated_conv_f32(const float *v, const float *a, const float *w, const float *bias, float *r,
                                     int64_t B, int64_t L, int64_t D, int64_t H, int64_t K, void *workspace,
                                     size_t workspace_bytes, void *stream);
CC_API int causal_mhf_gated_conv_bf16(const uint16_t *v, const uint16_t *a, const float *w, const float *bias,
                                      uint16_t *r, int64_t B, int64_t L, int64_t D, int64_t H, int64_t K,
                                      void *workspace, size_t workspace_bytes, void *stream);

/* Workspace of the gated convolution: B*L*D elements of the dtype (the gate
 * stream), or (size_t)-1 for invalid sizes or dtype (only F32 and BF16). */
CC_API size_t causal_mhf_gated_conv_workspace_bytes(int dtype, int64_t B, int64_t L, int64_t D);

/*
 * causal_dwconv_f32 / _bf16 -- the causal depthwise convolution that opens the
 * Multi-Head Fourier block (Caracal: Causal Architecture via Spectral Mixing,
 * "Key design 1": a causal depthwise 1-D convolution, kernel size 3):
 *
 *   y[b,t,d] = bias[d] + sum_{k<K} w[d][k] * x[b, t-(K-1)+k, d]
 *
 * terms with t-(K-1)+k < 0 left out (K-1 zeros on the left, none on the
 * right).  The output is the convolution alone (any residual connection is
 * the caller's).
 *   x     [B, L, D] device array, channel-last (bf16: uint16 bit patterns);
 *   w     [D, K] float32 device array (a depthwise Conv1d weight [D, 1, K]);
 *   bias  [D] float32 device array, or NULL;
 *   y     [B, L, D] device output of x's dtype (bf16: rounded to nearest
 *         even), overlapping neither x, w nor bias (CC_ERR_ALIAS);
 *   K     1..8 taps (the page's value is 3), else CC_ERR_UNSUPPORTED
 *         (K < 1: CC_ERR_INVALID_ARG).  L is not limited by a transform length.
 * fp32 arithmetic (fused multiply-adds in tap order).  Stream-ordered and
 * asynchronous; allocates nothing; errors are returned before any launch.
 */
CC_API int causal_dwconv_f32(const float *x, const float *w, const float *bias, float *y, int64_t B, int64_t L,
                             int64_t D, int64_t K, void *stream);
CC_API int causal_dwconv_bf16(const uint16_t *x, const float *w, const float *bias, uint16_t *y, int64_t B, int64_t L,
                              int64_t D, int64_t K, void *stream);

/*
 * causal_conv_fault_flags -- the library's per-device fault word.  The pages
 * have no counterpart: it reports waits inside the kernels that ran out of
 * time.  Every wait in the kernels (on an asynchronous copy, an mbarrier) is
 * bounded to about two seconds; a wait that runs out sets a bit here and its
 * kernel returns early, leaving its outputs incomplete, instead of hanging the
 * device.  Bit 0: a TMA staging copy did not complete.  Bit 1: the
 * tensor-core MMAs of the gate stream did not signal completion.
 *   device  CUDA device ordinal;
 *   flags   host pointer, receives the word;
 *   clear   non-zero: reset the word to 0 after reading it.
 * Synchronises the device (the word is read after all queued work ends).
 * Returns CC_OK, CC_ERR_INVALID_ARG (NULL flags, bad device) or CC_ERR_CUDA.
 */
CC_API int causal_conv_fault_flags(int device, unsigned int *flags, int clear);

#ifdef __cplusplus
}
#endif

#endif /* CAUSALCONV_H */
