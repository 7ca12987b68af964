/*
 * rank_fp8_residual.h -- C ABI of the B200 (sm_100a) LiteLinear forward.
 *
 * The layer stores a weight as a low-rank pair plus an FP8 residual and
 * evaluates (LiteLinear README, introduction, the display formula):
 *
 *     W ~= A*B + Q_fp8,
 *     y  = (x B^T) A^T + scale * (x Q_fp8^T) + bias
 *
 * Storage formats (README "Features"): A and B bf16, Q_fp8 e4m3fn (the
 * NVIDIA variant), bf16 activations in and out (README "Usage").  Factor
 * shapes as in SVDLinearLayer (tt_compressor page, class SVDLinearLayer:
 * A is (out, r), B is (r, in)); Q is shaped like nn.Linear.weight.
 *
 *   x     [M, K]  bf16, row-major (K contiguous)
 *   B     [r, K]  bf16, row-major
 *   A     [N, r]  bf16, row-major
 *   Q     [N, K]  e4m3fn codes, one byte each, row-major
 *   scale [N] fp32 (LL_SCALE_PER_ROW, one per output feature) or [1] fp32
 *         (LL_SCALE_PER_TENSOR).  It multiplies the x*Q^T term only (the
 *         README's "scale"; its state-dict key is Q_scale_inv, and it is
 *         applied as a multiplier).
 *   bias  [N] bf16, or NULL for no bias
 *   y     [M, N]  bf16, row-major
 *
 * All pointers passed to the compute calls are device pointers on the
 * device that was current when the layer was created.  Every call is
 * thread-compatible: one handle must not be used from two host threads at
 * the same time, and a handle's forward calls must be ordered on one
 * stream (they share the handle's workspace).  Distinct handles are
 * independent.
 *
 * Error behaviour: every int-returning call returns LL_OK (0) or one of
 * the LL_ERR_* codes below; ll_create returns NULL on error and records
 * the code for ll_last_error().  Argument errors are reported
 * synchronously and leave the handle unchanged.  Asynchronous device
 * faults surface at the next synchronising CUDA call; a device-side wait
 * that exceeded its time limit is reported by ll_status() after the
 * stream has been synchronised.
 */
#ifndef RANK_FP8_RESIDUAL_H
#define RANK_FP8_RESIDUAL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ll_layer *ll_handle;

enum { LL_SCALE_PER_TENSOR = 0, LL_SCALE_PER_ROW = 1 };

enum {
  LL_OK = 0,
  LL_ERR_INVALID_ARG = 1,    /* null / misaligned pointer, bad size or mode */
  LL_ERR_UNSUPPORTED = 2,    /* valid request this build does not handle */
  LL_ERR_NOT_READY = 3,      /* forward before ll_set_weights succeeded */
  LL_ERR_NAN_CODE = 4,       /* Q holds an e4m3fn NaN code (0x7F or 0xFF) */
  LL_ERR_OOM = 5,            /* device allocation failed */
  LL_ERR_CUDA = 6,           /* a CUDA runtime/driver call failed */
  LL_ERR_DEVICE_TIMEOUT = 7, /* a device-side wait ran past its limit */
  LL_ERR_SCRATCH_LIMIT = 8   /* request too large for ll_forward_noalloc's scratch */
};

/* Kernel variants for ll_set_variant (no counterpart on the pages).  AUTO:
 * GEMV for M == 1 (when x fits), STREAM for M <= 64, TC_PAIR for
 * 64 < M <= 256, above TC or FP8_SPLIT
 * (FP8_SPLIT on wide layers: N >= 2K, or N >= K at M >= 4096; the
 * measured crossovers).  TC: one-CTA fused
 * kernel, 128 features x up to 256 tokens per tile, low-rank factor folded
 * as A / scale (bf16 pair).  TC_PAIR: the same on CTA pairs (256 features
 * per MMA, tiles as narrow as 32 tokens).  SMALL: one-CTA
 * kernel, 128 x 128 tiles, separate residual and low-rank accumulators.
 * STREAM (M <= 64 only; larger M runs SMALL): one CTA per 128 features
 * streaming Q in 32 KB boxes, all tokens in one MMA, exact A.  FP8_SPLIT:
 * e4m3 tensor cores (kind::f8f6f4) with Q as stored and x carried per
 * token as the two-term e4m3fn expansion of ll_quantize_x: CTA pairs on
 * 256 x 256 tiles above 64 tokens; up to 64 tokens (except with the GEGLU
 * epilogue) a streaming kernel that deals Q's bytes out evenly to the SMs.
 * These variants meet the same accuracy bound.  FP8_ACT: the same kernel
 * on one e4m3fn term per token, the FP8-activation variant: its result is
 * the layer's formula evaluated on x quantised per token as by
 * ll_quantize_x with terms == 1 (that rounding of x is part of the
 * variant's definition).  GEMV (M <= 4 with x in shared memory beside the
 * 128 KB load ring, 2*M*K + 128 KB + 128 bytes <= 227 KB; otherwise SMALL):
 * CUDA cores only, every weight element used by M fused multiply-adds and
 * warp reductions, t in fp32; it meets the same accuracy bound. */
enum {
  LL_VARIANT_AUTO = 0,
  LL_VARIANT_TC = 1,
  LL_VARIANT_SMALL = 2,
  LL_VARIANT_TC_PAIR = 3,
  LL_VARIANT_STREAM = 4,
  LL_VARIANT_FP8_SPLIT = 5,
  LL_VARIANT_FP8_ACT = 6,
  LL_VARIANT_GEMV = 7
};

/* LiteLinear README, "Usage": the layer constructor
 * LiteLinear(in_features, out_features, bias, rank) -- here K = in_features,
 * N = out_features, r = rank, and whether a bias exists is decided by
 * ll_set_weights.  The scale granularity (one per output feature or one
 * per tensor) is not stated on the page; scale_mode selects it.
 *
 * Create a layer with N output features, K input features and rank r on
 * the current CUDA device.  Requires N >= 1 and N % 8 == 0, K >= 16 and
 * K % 16 == 0, 0 <= r <= 512, scale_mode one of LL_SCALE_*.  The handle is
 * host-allocated; device memory for the factors is allocated here.
 * Returns NULL on error (see ll_last_error()): LL_ERR_INVALID_ARG for bad
 * sizes or mode, LL_ERR_UNSUPPORTED for r > 512 or a GPU other than
 * sm_100, LL_ERR_OOM / LL_ERR_CUDA when the device allocation fails. */
ll_handle ll_create(int N, int K, int r, int scale_mode);

/* LiteLinear README, "Features": the factors a converted layer holds, its
 * state-dict keys A, B, Q_fp8, Q_scale_inv and bias (A, B bf16; Q_fp8
 * e4m3fn; Q_scale_inv is the "scale" of the introduction's formula and is
 * applied as a multiplier).
 *
 * Copy the factors into handle-owned device memory (device-to-device;
 * the caller may free its buffers once the call returns -- the call
 * synchronises the device).  A: bf16 [N, r]; B: bf16 [r, K] (both may be
 * NULL when r == 0); Q: e4m3fn codes [N, K]; scale: fp32 [N] or [1] by
 * the layer's scale_mode; bias: bf16 [N] or NULL.  A, B and Q must be
 * 16-byte aligned device pointers, scale 4-byte and bias 2-byte aligned
 * (LL_ERR_INVALID_ARG otherwise).  The rank is zero-padded internally to a multiple of
 * 32 (exact).  The call also prepares A / scale as a bf16 pair for the
 * fused large-M kernel.  Returns LL_ERR_NAN_CODE if any Q code is 0x7F or
 * 0xFF; LL_ERR_INVALID_ARG for null/misaligned/non-device pointers or a
 * non-finite scale; LL_ERR_UNSUPPORTED if some nonzero |A[n,j] / scale[n]|
 * lies outside [2^-100, 2^100] (rows with scale 0 count as scale 1). */
int ll_set_weights(ll_handle h, const void *A, const void *B, const void *Q, const float *scale,
                   const void *bias);

/* LiteLinear README, "Usage": y = layer(x), evaluating the introduction's
 * display formula y = (x B^T) A^T + scale * (x Q_fp8^T) + bias.
 *
 * y = forward(x) for M rows on `stream` (a cudaStream_t; NULL is the
 * legacy default stream).  x: bf16 [M, K], y: bf16 [M, N], both 16-byte
 * aligned device pointers that must not overlap.  M == 0 is a no-op.  The
 * call is asynchronous; x and y are borrowed until the stream reaches the
 * end of the call.  The first call with a larger M than any before grows
 * the handle's workspace with stream-ordered allocation (call ll_reserve
 * beforehand to avoid that, e.g. before graph capture). */
int ll_forward(ll_handle h, const void *x, void *y, int M, void *stream);

/* No counterpart on the pages: the forward from host memory.
 *
 * ll_forward on HOST buffers: copies x (host, bf16 [M, K]) to the device,
 * runs the forward and copies y back to the host (bf16 [M, N]).  The rows
 * go in up to four chunks of whole 256-token tiles, so that the copy of
 * one chunk into the device, the forward of the one before and the copy
 * out of the one before that overlap (two handle-owned copy streams; the
 * forwards run on `stream`, which waits for the last copy out).  Pinned
 * host buffers make the copies asynchronous; the caller synchronises
 * `stream` once before reading y.  Device staging buffers are
 * handle-owned and grown on demand.  Errors as ll_forward. */
int ll_forward_host(ll_handle h, const void *x_host, void *y_host, int M, void *stream);

/* No counterpart on the pages.  Pre-size the workspace for forwards of up
 * to max_M rows (synchronous). */
int ll_reserve(ll_handle h, int max_M);

/* Activation fused into the epilogue (ll_set_epilogue).  The LTX-Video
 * transformers the LiteLinear README converts wrap the first linear of each
 * feed-forward in a GEGLU ("Usage": replace_activation_proj_ routes the
 * GEGLU's projection through LiteLinear): proj(x) is split into a value
 * half h and a gate half g, and the block computes h * gelu(g), with GELU
 * in its tanh form gelu(v) = v / 2 * (1 + tanh(sqrt(2/pi) (v + 0.044715
 * v^3))).  LL_EPILOGUE_GELU_TANH applies gelu to every output;
 * LL_EPILOGUE_GEGLU_TANH returns y[m, j] = h[m, j] * gelu(g[m, j]) with
 * h = outputs 0 .. N/2 - 1 and g = outputs N/2 .. N - 1 of the formula, so
 * y is [M, N/2]. */
enum { LL_EPILOGUE_NONE = 0, LL_EPILOGUE_GELU_TANH = 1, LL_EPILOGUE_GEGLU_TANH = 2 };

/* Select the epilogue activation (no counterpart on the pages beyond the
 * GEGLU above).  The activation is applied to the fp32 result before its
 * one rounding to bf16.  GEGLU needs N % 256 == 0 (LL_ERR_UNSUPPORTED
 * otherwise), runs on the FP8-operand kernel (AUTO and the two FP8
 * variants; the others return LL_ERR_UNSUPPORTED from ll_forward), and
 * stores the weights in its own row order: switching GEGLU on or off
 * requires ll_set_weights again (a forward before that returns
 * LL_ERR_NOT_READY).  LL_ERR_INVALID_ARG for an unknown epilogue. */
int ll_set_epilogue(ll_handle h, int epilogue);

/* No counterpart on the pages.  Select a kernel variant (LL_VARIANT_AUTO
 * picks by M).  LL_ERR_INVALID_ARG for an unknown variant. */
int ll_set_variant(ll_handle h, int variant);

/* The plan a forward of M tokens would follow on a layer of shape
 * (N, K, r) with the given variant, on a GPU with num_sms SMs; host
 * arithmetic only (no CUDA call, no handle), so it also runs without a GPU.
 * The pages have no counterpart: this reports this library's dispatch
 * (the kernel variants above) and its tile planning.
 *   kernel:      the variant that runs (LL_VARIANT_TC, _TC_PAIR, _SMALL or
 *                _STREAM; never AUTO).
 *   tile_tokens: tokens per tile of that kernel (TC: the joint plan's
 *                width; TC_PAIR: tokens per 256-feature pair tile; SMALL:
 *                128; STREAM: M rounded up to 16).
 *   lr_splits:   K splits of the down-projection t = x B^T (1 when r == 0).
 * The CTA-pair plan assumes every pair of SMs can hold one cluster (a
 * forward asks the occupancy calculator).  Any of the three out-pointers
 * may be NULL.  Errors: LL_ERR_INVALID_ARG for shapes ll_create would
 * reject, M < 1, num_sms < 2 or an unknown variant; LL_ERR_UNSUPPORTED for
 * r > 512. */
int ll_plan(int N, int K, int r, int M, int num_sms, int variant, int *kernel, int *tile_tokens, int *lr_splits);

/* No counterpart on the pages.  Device status word of the handle: LL_OK, or LL_ERR_DEVICE_TIMEOUT if a
 * kernel of this handle gave up on a wait.  Synchronises the device;
 * call after the stream of the forward has been synchronised.  Reading
 * the status clears it. */
int ll_status(ll_handle h);

/* No counterpart on the pages.  Debug controls: timeout_ns bounds every device-side wait (default 2 s);
 * withhold_producer != 0 makes the main kernel's loader issue nothing, so
 * its consumers run into the timeout (used to test the timeout path). */
int ll_set_debug(ll_handle h, int withhold_producer, uint64_t timeout_ns);

/* LiteLinear README, "Usage": LiteLinear.from_dense, the SVD-based
 * decomposition of a dense weight (and "Features": the factors A, B, Q_fp8,
 * Q_scale_inv).  After the SVD, which the caller runs (A = U_r S_r and
 * B = V_r^T rounded to bf16, as the MoDeGPT compressor keeps them), this
 * call quantises the residual:
 *
 *   R[n, k] = W[n, k] - sum_j A[n, j] B[j, k]   (binary64, j in order)
 *   scale   = max |R| / 448 rounded to binary32, per row ([N]) or over the
 *             whole tensor ([1]) by scale_mode; 0 for an all-zero residual
 *   Q[n, k] = e4m3fn code nearest to binary32(R[n, k] / scale) (ties to
 *             even, saturating at 448); 0 where the scale is 0
 *
 * The pages do not state how the scale is chosen; this maps each row's (or
 * the tensor's) largest residual to the largest e4m3fn value.  Device
 * pointers: W bf16 [N, K], A bf16 [N, r] and B bf16 [r, K] (NULL when
 * r == 0), Q uint8 [N, K], scale fp32 [N] or [1]; 2-byte alignment for
 * the bf16 arrays, 4 for scale.  Asynchronous on `stream` (a per-tensor
 * scale uses a stream-ordered allocation of N doubles).  Errors:
 * LL_ERR_INVALID_ARG for bad sizes, mode or pointers, LL_ERR_UNSUPPORTED
 * for K + r beyond 29,000 (the residual row is kept in shared memory),
 * LL_ERR_OOM, LL_ERR_CUDA. */
int ll_quantize_residual(const void *W, const void *A, const void *B, int N, int K, int r, int scale_mode, void *Q,
                         float *scale, void *stream);

/* The per-token e4m3fn quantisation of activations that the FP8-operand
 * variants apply before the residual product (the FP8-activation reading
 * of the README's "Features" list and its fused benchmark kernel): for
 * each token row m of x (bf16 [M, K], device, 16-byte aligned) it writes
 * e_out[m] (int32 [M]), the smallest e in [-126, 126] with
 * max_k |x[m, k]| <= 448 * 2^e (0 for an all-zero row), and the e4m3fn
 * codes hi[m, k] = rne(x[m, k] / 2^e) (uint8 [M, K], 16-byte aligned);
 * with terms == 2 also lo[m, k] = rne(x[m, k] / 2^e - hi[m, k]), so that
 * 2^e * (hi + lo) equals x wherever |x| >= 2^e / 4 and lies within
 * 2^(e - 10) of it elsewhere.  rne rounds to the nearest e4m3fn value,
 * ties to the even code.  K % 16 == 0.  Asynchronous on `stream`;
 * LL_ERR_INVALID_ARG for bad sizes, terms, or null / misaligned /
 * non-device pointers. */
int ll_quantize_x(const void *x, int M, int K, int terms, int *e_out, void *hi, void *lo, void *stream);

/* No counterpart on the pages.  Release the handle and all device memory
 * it owns (synchronises). */
void ll_destroy(ll_handle h);

/* No counterpart on the pages.  Code of the last failed call on this host
 * thread (LL_OK if none). */
int ll_last_error(void);

/* No counterpart on the pages.  Static description of a status code. */
const char *ll_status_string(int code);

/* No counterpart on the pages.  Number of kernels the last ll_forward on
 * this handle launched. */
int ll_last_launch_count(ll_handle h);

/* No counterpart on the pages.  Profiling mode (enable != 0): every later ll_forward records CUDA events
 * on its stream around each kernel it launches, and launches them without
 * programmatic overlap so each duration is that kernel's alone.  All work
 * is still done.  Off by default. */
int ll_set_profiling(ll_handle h, int enable);

/* No counterpart on the pages.  Device durations in milliseconds of the kernels the last profiled
 * ll_forward launched, in launch order, written to ms[0 .. n).  Waits for
 * the events.  Returns the number of kernels (may exceed n), or -1 if the
 * last forward was not profiled. */
int ll_kernel_times(ll_handle h, float *ms, int n);

/* No counterpart on the pages.  Name of the i-th kernel of the last
 * ll_forward (static string), or NULL. */
const char *ll_kernel_name(ll_handle h, int i);

/* ---------------------------------------------------------------------
 * ll_forward_noalloc: the forward without any device allocation.
 *
 * The paper has no counterpart to this call; it serves callers that may
 * not allocate device memory at all.  Examples: a host framework whose
 * caching allocator already holds the GPU's memory (an outside cudaMalloc
 * fails, or fragments that pool behind its back), a plug-in whose host
 * only lets it use buffers the host hands over, and a latency-critical
 * loop where cudaMalloc / cudaFree would stall on device-wide
 * synchronisation.  Such a caller cannot use ll_create (it copies the
 * factors into library-owned memory) or ll_forward (it grows a workspace
 * on demand).  This call takes no handle: the caller passes every input
 * and the output, and the intermediate t = x B^T (bf16 hi + lo), a device
 * status word and, for a per-tensor scale, the scale broadcast to N rows
 * live in one static device array of LL_NOALLOC_SCRATCH_BYTES.  Every GPU
 * on which the library's device code is loaded holds that array until the
 * process exits.
 *
 * y is the forward of ll_forward with the SMALL variant (residual and
 * low-rank terms in separate accumulators, A used as given) and meets the
 * same accuracy bound.  Arguments are laid out as described at the top of
 * this header: x bf16 [M, K], A bf16 [N, r] and B bf16 [r, K] (both NULL
 * when r == 0), Q e4m3fn codes [N, K], scale fp32 [N] (LL_SCALE_PER_ROW) or
 * [1] (LL_SCALE_PER_TENSOR), bias bf16 [N] or NULL, y bf16 [M, N]; all
 * device pointers of the current device; x, y, A, B and Q 16-byte
 * aligned, scale 4-byte, bias 2-byte; y must not overlap any input.  Shapes follow
 * ll_create (N % 8 == 0, K % 16 == 0, K >= 16, 0 <= r <= 512) and, since
 * A is read in place, r % 8 == 0.  M == 0 is a no-op.
 *
 * Limit: with r32 = r rounded up to a multiple of 32, the call needs
 *     256 + 4 * M * r32 bytes  (+ 4 * N rounded up to 256 for a per-tensor
 *     scale), at most LL_NOALLOC_SCRATCH_BYTES.
 * A larger request returns LL_ERR_SCRATCH_LIMIT and launches nothing
 * (e.g. r = 512 allows M up to 8191, r = 64 up to 65535).
 *
 * Not checked here: the weights are read as given on every call, with no
 * scan for NaN codes or non-finite scales (ll_set_weights does those
 * checks); a Q code 0x7F or 0xFF gives meaningless values.
 *
 * Shared scratch: every call on a device uses the same array, and the
 * array keeps the last call's contents.  Each call clears the status word
 * and fully rewrites t before reading it.  Calls whose kernels overlap on
 * the GPU (issued on two streams without ordering, or from two host
 * threads) race on the array and give wrong results: order them on one
 * stream or with events.
 *
 * Set-up: the first successful call on each device (made with that
 * device current) looks up the array's device address and sets kernel
 * attributes; make that first call before any stream capture.  A set-up
 * that fails is not kept: the next call tries again.  cudaDeviceReset
 * invalidates the set-up; do not call this entry point on a device after
 * resetting it in the same process.
 *
 * Errors: LL_ERR_INVALID_ARG for bad shapes, modes, null / misaligned
 * pointers, pointers that are not device memory of the current device, or
 * y overlapping any input; LL_ERR_UNSUPPORTED for r % 8 != 0;
 * LL_ERR_SCRATCH_LIMIT as above; LL_ERR_CUDA when a launch fails.  A
 * device-side wait that runs past its limit (2 s) ends the kernels early
 * and leaves y incomplete; this call has no way to report that
 * afterwards. */
#define LL_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
int ll_forward_noalloc(const void *x, const void *A, const void *B, const void *Q, const float *scale,
                       int scale_mode, const void *bias, void *y, int M, int N, int K, int r, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* RANK_FP8_RESIDUAL_H */
