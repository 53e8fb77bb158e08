/*
 * sq.h -- C ABI of libsq.so, the sm_100a (B200) implementation of the
 * SmoothQuant W8A8 smoothed linear layer.
 *
 * Method ("SmoothQuant (activation smoothing quantization)", jisaku.com
 * glossary page):
 *   - "The mathematics of the smoothing transformation":
 *       Y = X W = (X diag(s)^-1)(diag(s) W) = X~ W~
 *   - "Hyper-parameter alpha (migration strength)":
 *       s_j = max|X_j|^alpha / max|W_j|^(1-alpha), alpha = 0.5 by default
 *   - "Why activation quantization is hard": INT8 codes, a row is scaled so
 *     that its largest magnitude maps to 127
 *   - comparison table: the product runs directly on INT8 tensor cores
 *   - usage example: get_act_scales (calibration) -> smooth_lm(alpha)
 *     -> quantize_model.
 * The four compute calls below follow that order.
 *
 * Conventions shared by every call
 *   - Every data pointer is DEVICE memory on the current device, allocated
 *     and owned by the caller.  The library allocates nothing, never
 *     synchronises, and enqueues all work on `stream` (asynchronous with
 *     respect to the host).  Buffers must stay alive until the work ends.
 *   - Matrices are row-major with a leading dimension `ld*` counted in
 *     ELEMENTS of the matrix's own type.
 *   - Alignment: every pointer 16-byte aligned; every leading dimension a
 *     multiple of 16 bytes; K and N multiples of 16.
 *   - Arithmetic is IEEE fp32 with round-to-nearest-even; no operation is
 *     contracted into an FMA.  INT8 codes, scales, s and int32 sums are
 *     therefore reproducible bit for bit on any input.
 *   - Quantization of a row v with absmax m: scale = m / 127 and
 *     q = clamp(rne(v / scale), -127, 127) with an IEEE division (the
 *     kernels reach the same codes with a reciprocal multiply and an exact
 *     check, dividing only next to a rounding boundary); an all-zero row
 *     gives scale 0 and codes 0.  -128 is never produced.
 *   - Inputs must be finite; NaN/Inf give unspecified results.
 *   - Errors: argument checks run on the host before anything is enqueued
 *     and return SQ_ERR_INVALID_ARG / SQ_ERR_UNSUPPORTED with no side
 *     effect.  A failed launch returns SQ_ERR_CUDA.  Work that is empty
 *     (T == 0 or M == 0) returns SQ_OK and enqueues nothing.  Every wait
 *     inside a kernel is bounded in time; a wait that runs out makes the
 *     kernel stop and records SQ_ERR_TIMEOUT, which sq_check_device_error
 *     reports.  No C++ exception crosses this interface.
 */
#ifndef SQ_H_
#define SQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream; NULL is the legacy default stream. */
typedef struct CUstream_st *sq_stream_t;

typedef enum {
  SQ_OK = 0,
  SQ_ERR_INVALID_ARG = 1, /* null pointer, bad size, alignment or alpha   */
  SQ_ERR_UNSUPPORTED = 2, /* valid request this build does not implement  */
  SQ_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed            */
  SQ_ERR_TIMEOUT = 4      /* a bounded in-kernel wait ran out             */
} sq_status;

typedef enum { SQ_F32 = 0, SQ_F16 = 1, SQ_BF16 = 2 } sq_dtype;

/* Layout of the weight matrix W (input channel j, output channel n). */
typedef enum {
  SQ_W_KN = 0, /* W[K][N]: Y = X W as the page writes it            */
  SQ_W_NK = 1  /* W[N][K]: output-major, as torch.nn.Linear stores it */
} sq_wlayout;

/*
 * Calibration: running per-input-channel activation maximum
 * (get_act_scales in the page's usage example; the max|X_j| of the alpha
 * formula).
 *   x     [T][ldx] of type xt (f32/f16/bf16), T tokens of K channels.
 *   amax  [K] fp32, in-out: amax_j <- max(amax_j, max_t |x_tj|).  The caller
 *         zero-fills it once and then calls this once per calibration chunk;
 *         max is exact and order-free, so any chunking gives the same bits.
 * T == 0 is a no-op.  K % 16 == 0, ldx >= K.
 */
sq_status sq_calib_absmax(const void *x, sq_dtype xt, int64_t T, int64_t K,
                          int64_t ldx, float *amax, sq_stream_t stream);

/*
 * Smoothing and weight quantization (smooth_lm(alpha) then quantize_model).
 *   w         weights of type wt; layout SQ_W_KN: [K][ldw], SQ_W_NK: [N][ldw].
 *   amax      [K] fp32 calibration maxima from sq_calib_absmax.
 *   alpha     migration strength in [0, 1].
 *   wq        [N][K] int8 OUT, K contiguous (row n = output channel n):
 *             Wq = clamp(rne(W~ / w_scale_n)), W~ = diag(s) W.
 *   w_scale   [N] fp32 OUT, per-output-channel scale max_j|W~_jn| / 127.
 *   smooth    [K] fp32 OUT, s_j (also used as scratch during the call).
 *   inv_smooth[K] fp32 OUT, 1/s_j (what sq_quant_act multiplies by).
 * s_j uses a_j and w_j = max_n |W_jn| floored at 1e-5.  For alpha in
 * {0, 0.25, 0.5, 0.75, 1} the power is formed from IEEE square roots
 * (bit-reproducible); other alphas use double-precision pow, rounded once.
 * K % 16 == 0, N % 16 == 0, ldw >= K (NK) or >= N (KN).
 */
sq_status sq_smooth_quant_weight(const void *w, sq_dtype wt, sq_wlayout layout,
                                 int64_t K, int64_t N, int64_t ldw,
                                 const float *amax, float alpha, int8_t *wq,
                                 float *w_scale, float *smooth,
                                 float *inv_smooth, sq_stream_t stream);

/*
 * Runtime activation smoothing and per-token dynamic quantization
 * (X~ = X diag(s)^-1, then INT8 with the largest magnitude mapped to 127).
 *   x          [M][ldx] of type xt.
 *   inv_smooth [K] fp32 (from sq_smooth_quant_weight).
 *   xq         [M][K] int8 OUT (row stride K).
 *   x_scale    [M] fp32 OUT, max_j |x_tj * inv_s_j| / 127.
 * M == 0 is a no-op.  K % 16 == 0, ldx >= K.
 */
sq_status sq_quant_act(const void *x, sq_dtype xt, int64_t M, int64_t K,
                       int64_t ldx, const float *inv_smooth, int8_t *xq,
                       float *x_scale, sq_stream_t stream);

/*
 * Fold diag(s)^-1 into the weight of the norm that produces X, once per
 * layer, the way sq_smooth_quant_weight folds diag(s) into W: smooth_lm(alpha)
 * in the page's usage example moves the smoothing out of the run-time path.
 *   gs_j = gamma_j * inv_smooth_j   (fp32, IEEE round to nearest even)
 *   gamma, inv_smooth [K] fp32 IN; gs [K] fp32 OUT (may alias gamma).
 * K > 0; 16-byte aligned device pointers.
 */
sq_status sq_fold_smooth_into_norm(const float *gamma, const float *inv_smooth,
                                   int64_t K, float *gs, sq_stream_t stream);

/*
 * Upstream producer: RMS normalisation of each token with the folded weight
 * gs (sq_fold_smooth_into_norm), then per-token INT8, in one pass; in
 * transformer blocks this replaces norm + sq_quant_act:
 *   r_t  = 1 / sqrt(sum_j x_tj^2 / K + eps)   (squares summed in double
 *          precision in an unspecified order, root and reciprocal in double,
 *          rounded once to fp32)
 *   v_tj = (x_tj * r_t) * gs_j   (fp32, in that order)
 *   then per-token quantization of v exactly as sq_quant_act.
 *   gs [K] fp32, eps >= 0 and finite.  Other arguments as sq_quant_act.
 * Because the order of the double-precision sum is unspecified, r_t may
 * differ from another implementation's by one fp32 ulp, which moves a code
 * by one only where v / scale lies within ~2^-20 of a rounding
 * boundary.  K <= 16384 for 16-bit x, <= 8192 for fp32 x, else
 * SQ_ERR_UNSUPPORTED.
 */
sq_status sq_rmsnorm_quant_act(const void *x, sq_dtype xt, int64_t M, int64_t K,
                               int64_t ldx, const float *gs, float eps,
                               int8_t *xq, float *x_scale, sq_stream_t stream);

/*
 * Upstream producer for models whose linears are fed by a LayerNorm with a
 * bias (the OPT models of the page's speed-up and perplexity tables): fold
 * diag(s)^-1 into both, gs = gamma * inv_smooth and bs = beta * inv_smooth
 * (sq_fold_smooth_into_norm computes either product), then per token
 *   mu_t  = sum_j x_tj / K
 *   var_t = sum_j (x_tj - mu_t)^2 / K
 *          (both in double precision: this library takes one pass over
 *          the deviations from the token's first value, in an unspecified
 *          order, which keeps var_t within 2^-31 (relative) and mu_t within
 *          2^-40 standard deviations of their exact values for K <= 16384;
 *          mu_t and r_t = 1 / sqrt(var_t + eps) each rounded once to fp32)
 *   n_tj  = (x_tj - mu_t) * r_t              (fp32, in that order)
 *   v_tj  = fma(n_tj, gs_j, bs_j)            (one rounding)
 *   then per-token quantization of v exactly as sq_quant_act.
 *   gs [K] fp32; bs [K] fp32 or NULL (no bias); eps > 0 and finite (a
 *   constant token has var_t = 0).  Other arguments as sq_quant_act.
 * As for sq_rmsnorm_quant_act, mu_t and r_t may differ from another
 * implementation's by one fp32 ulp, which moves a code by one only next to
 * a rounding boundary.  K <= 16384 for 16-bit x, <= 8192 for fp32 x, else
 * SQ_ERR_UNSUPPORTED.
 */
sq_status sq_layernorm_quant_act(const void *x, sq_dtype xt, int64_t M, int64_t K,
                                 int64_t ldx, const float *gs, const float *bs,
                                 float eps, int8_t *xq, float *x_scale,
                                 sq_stream_t stream);

/*
 * Static per-tensor activation scale, the alternative to per-token scales
 * (the page notes activations change per prompt, which is why the main path
 * measures each token at run time).  After smoothing, channel j's
 * calibrated maximum is amax_j * inv_smooth_j, so
 *   *delta = max_j(amax_j * inv_smooth_j) / 127   (one fp32 on the device).
 */
sq_status sq_static_act_scale(const float *amax, const float *inv_smooth, int64_t K,
                              float *delta, sq_stream_t stream);

/*
 * Static quantization with that scale: xq = clamp(rne((x * inv_smooth) /
 * *delta), -127, 127) -- values beyond the calibrated range
 * saturate -- and x_scale_t = *delta for every token, so sq_w8a8_linear
 * consumes the result unchanged.  delta is a device pointer (*delta > 0).
 * Other arguments as sq_quant_act.
 */
sq_status sq_quant_act_static(const void *x, sq_dtype xt, int64_t M, int64_t K,
                              int64_t ldx, const float *inv_smooth,
                              const float *delta, int8_t *xq, float *x_scale,
                              sq_stream_t stream);

/*
 * W8A8 linear on the tensor cores (tcgen05, kind::i8): exact int32
 * accumulation acc_tn = sum_j xq_tj * wq_nj, then the dequant epilogue
 * y_tn = round_yt(((float)acc_tn * x_scale_t) * w_scale_n).
 *   xq [M][K] int8, wq [N][K] int8, x_scale [M], w_scale [N] fp32.
 *   y  [M][ldy] of type yt (f32/f16/bf16) OUT.
 *   workspace / workspace_bytes: device scratch of at least
 *         sq_w8a8_linear_workspace_size(M, N, K) bytes, which must be ZERO
 *         on the first call; the library leaves it zero again when each
 *         call ends.  May be NULL when that size is 0.  Calls that share a
 *         workspace must be stream-ordered.
 * M == 0 is a no-op.  K % 16 == 0, N % 16 == 0, ldy >= N.
 * Decode-shaped calls (1 <= M <= 64) stream Wq over the SMs.  With at most
 * 32 tokens and more 128-row tiles of Wq than SMs, a stream-K kernel shares
 * the (tile, k-block) items evenly over all SMs and adds the partial sums
 * of split tiles in the workspace.  Every other decode shape runs on
 * clusters of CTAs that split tiles' K ranges and add their partials
 * through distributed shared memory, with no workspace.
 */
sq_status sq_w8a8_linear(const int8_t *xq, const float *x_scale,
                         const int8_t *wq, const float *w_scale, int64_t M,
                         int64_t N, int64_t K, void *y, sq_dtype yt,
                         int64_t ldy, void *workspace, size_t workspace_bytes,
                         sq_stream_t stream);

/* Bytes of workspace sq_w8a8_linear needs for this shape on the current
 * device: the stream-K decode kernel's partial sums and tile counters where
 * that kernel runs (see sq_w8a8_linear), 0 for every other shape.  Where no
 * device can be queried, the stream-K kernel's need for any 1 <= M <= 64. */
size_t sq_w8a8_linear_workspace_size(int64_t M, int64_t N, int64_t K);

/*
 * The integer product alone: acc[M][ldacc] int32 OUT = xq . wq^T, computed
 * by the same tensor-core kernels as sq_w8a8_linear (same tiling and
 * dispatch on M), for verifying the exact accumulators.  Same workspace
 * contract as sq_w8a8_linear.
 */
sq_status sq_w8a8_accumulate(const int8_t *xq, const int8_t *wq, int64_t M,
                             int64_t N, int64_t K, int32_t *acc, int64_t ldacc,
                             void *workspace, size_t workspace_bytes,
                             sq_stream_t stream);

/*
 * Column-parallel linear: the output-channel shard of one rank, stored into
 * several destinations in the same pass.  With G ranks each holding the rows
 * [n0, n0 + N) of Wq and w_scale (a shard of the output channels) and the
 * same xq / x_scale, every rank's call produces Y[:, n0:n0+N] and writes each
 * tile into all n_dst destination matrices -- its own Y and the other ranks'
 * copies, which may be peer-mapped device pointers (plain stores over
 * NVLink) -- so that after every rank's call (and a barrier that orders it)
 * each rank holds the full Y without a separate all-gather.  The page's
 * OPT-175B runs use 8 GPUs; this is how the linear shards over them.
 *   y_dst      HOST array of n_dst (1..8) device pointers; y_dst[d] points at
 *              the destination's element (row 0, column n0), row stride ldy
 *              elements of type yt, 16-byte aligned.
 * Other arguments, workspace and errors as sq_w8a8_linear (N is the shard's
 * width).  Writes from different ranks go to disjoint columns.
 */
sq_status sq_w8a8_linear_scatter(const int8_t *xq, const float *x_scale,
                                 const int8_t *wq, const float *w_scale, int64_t M,
                                 int64_t N, int64_t K, void *const *y_dst, int n_dst,
                                 sq_dtype yt, int64_t ldy, void *workspace,
                                 size_t workspace_bytes, sq_stream_t stream);

/*
 * Outlier handling beyond smoothing: a butterfly rotation before the INT8
 * quantization ("ButterflyQuant", lifetechia.com: an orthogonal transform
 * built from Givens rotations in an FFT butterfly, O(n log n), with the
 * Hadamard transform as the special case of every angle pi/4).  Rows are
 * rotated block by block, blocks of n = 2^L channels (K % n == 0):
 *   stage i = 0 .. L-1 pairs positions p and p + 2^i (bit i of p clear);
 *   the pair's index is j = ((p >> (i + 1)) << i) | (p mod 2^i);
 *   (a, b) -> (c a - s b, s a + c b), (c, s) = rot_cs[i][j][0..1],
 *   each product and sum an IEEE fp32 operation.
 * As the rotation R is orthogonal, (R x~) . (R w~_n) = x~ . w~_n: rotating
 * both the smoothed activations and the smoothed weights' K-vectors keeps
 * the product while spreading outliers over a block.
 *   rot_cs   [L][n / 2][2] fp32 (cos, sin) pairs, device memory.
 *   n        a power of two, 2 <= n, dividing K (n = K rotates the whole
 *            row); K <= 16384 (16-bit rows) or 8192 (fp32 rows), else
 *            SQ_ERR_UNSUPPORTED; other n give SQ_ERR_INVALID_ARG.  Blocks
 *            of up to 256 channels (128 for fp32) rotate in registers;
 *            wider blocks through a row staged in shared memory (slower).
 * sq_quant_act_rotated: xq, x_scale of R(x * inv_smooth), as sq_quant_act.
 * sq_smooth_quant_weight_rotated: s and 1/s as sq_smooth_quant_weight
 *   (layout SQ_W_NK only), then wq, w_scale of R(s * w_n) per output
 *   channel n.
 */
sq_status sq_quant_act_rotated(const void *x, sq_dtype xt, int64_t M, int64_t K,
                               int64_t ldx, const float *inv_smooth, int64_t n,
                               const float *rot_cs, int8_t *xq, float *x_scale,
                               sq_stream_t stream);
sq_status sq_smooth_quant_weight_rotated(const void *w, sq_dtype wt, int64_t K,
                                         int64_t N, int64_t ldw, const float *amax,
                                         float alpha, int64_t n, const float *rot_cs,
                                         int8_t *wq, float *w_scale, float *smooth,
                                         float *inv_smooth, sq_stream_t stream);

/*
 * FP8 (E4M3) variant.  The glossary page "Quantization Calibration
 * GPTQ/AWQ/SmoothQuant 2026" (jisaku.com glossary) lists FP8 SmoothQuant:
 * the same smoothing, with FP8 operands.  Both operands are E4M3 codes (1
 * sign, 4 exponent bits of bias 7, 3 mantissa bits, no infinities,
 * S.1111.111 = NaN, largest finite 448) with the INT8 path's granularity:
 *   scale = m / 448 for a row with absmax m, and
 *   code  = e4m3(v / scale) (IEEE division), nearest value, ties to even,
 *           saturating at +-448;  an all-zero row gives scale 0, codes +0.
 * Smoothing (s, 1/s) is computed exactly as for INT8.  The product runs on
 * the tensor cores' FP8 path with an fp32 accumulator: every product of
 * two E4M3 values is exact, the additions are fp32 in the hardware's own
 * order, so the sum is within K * 2^-22 * sum_j |x_j w_j| of the exact one
 * (and deterministic: the same inputs and launch give the same bits).
 *
 * sq_smooth_quant_weight_e4m3: as sq_smooth_quant_weight, with wq [N][K]
 *   E4M3 codes (uint8) and w_scale = max_j|W~_jn| / 448.
 * sq_quant_act_e4m3: as sq_quant_act, with xq [M][K] E4M3 codes and
 *   x_scale = max_j|X~_tj| / 448.
 * sq_w8a8_linear_e4m3: y = round_yt((acc_tn * x_scale_t) * w_scale_n) with
 *   the fp32 accumulator acc; arguments, workspace
 *   (sq_w8a8_linear_workspace_size) and errors as sq_w8a8_linear.
 * sq_w8a8_accumulate_e4m3: the fp32 accumulator alone, acc [M][ldacc].
 */
sq_status sq_smooth_quant_weight_e4m3(const void *w, sq_dtype wt, sq_wlayout layout,
                                      int64_t K, int64_t N, int64_t ldw,
                                      const float *amax, float alpha, uint8_t *wq,
                                      float *w_scale, float *smooth,
                                      float *inv_smooth, sq_stream_t stream);
sq_status sq_quant_act_e4m3(const void *x, sq_dtype xt, int64_t M, int64_t K,
                            int64_t ldx, const float *inv_smooth, uint8_t *xq,
                            float *x_scale, sq_stream_t stream);
sq_status sq_w8a8_linear_e4m3(const uint8_t *xq, const float *x_scale,
                              const uint8_t *wq, const float *w_scale, int64_t M,
                              int64_t N, int64_t K, void *y, sq_dtype yt,
                              int64_t ldy, void *workspace, size_t workspace_bytes,
                              sq_stream_t stream);
sq_status sq_w8a8_accumulate_e4m3(const uint8_t *xq, const uint8_t *wq, int64_t M,
                                  int64_t N, int64_t K, float *acc, int64_t ldacc,
                                  void *workspace, size_t workspace_bytes,
                                  sq_stream_t stream);

/*
 * Allocation-free variant of sq_w8a8_linear for decode-shaped calls.
 * (This has no counterpart in the SmoothQuant page; it is a deployment
 * convenience of this library.)
 *
 * Some callers cannot allocate device memory at the point of the call:
 * plugins whose host framework owns all device memory through its own pool
 * and forbids side allocations, latency-critical loops that cannot accept
 * cudaMalloc's implicit device-wide synchronisation, and code running inside
 * an allocator's own callbacks.  sq_w8a8_linear needs a caller-provided
 * workspace for the decode shapes that take its stream-K kernel (at most 32
 * tokens, more 128-row tiles of Wq than SMs); this entry point instead uses
 * a scratch array
 * of SQ_DECODE_STATIC_SCRATCH_BYTES compiled into the library (a static
 * device array that every GPU which loads the library holds until the
 * process exits).  It allocates nothing and calls no allocating routine.
 *
 * Arguments, layouts and results are those of sq_w8a8_linear (minus the
 * workspace); the results are identical.
 *   - 1 <= M <= 64 and sq_w8a8_linear_workspace_size(M, N, K) <=
 *     SQ_DECODE_STATIC_SCRATCH_BYTES, else SQ_ERR_UNSUPPORTED (nothing is
 *     enqueued).  M == 0 is a no-op.  A shape whose size query is 0 runs
 *     without touching the scratch.
 *   - The first call on a device that needs the scratch looks up the
 *     array's device address (once per device, with that device current);
 *     make that first call outside any stream capture.
 *   - Every call on a device shares the one scratch array.  A shape whose
 *     product takes the stream-K kernel (see sq_w8a8_linear) clears the part
 *     it uses on `stream` before using it; any other shape uses no scratch
 *     and clears nothing.  Calls whose work overlaps on the GPU (different
 *     streams without ordering, or several host threads) race on the
 *     scratch and give wrong results: serialise them.
 */
#define SQ_DECODE_STATIC_SCRATCH_BYTES ((size_t)8 << 20) /* 8 MiB */
/* The size of that scratch array as built into this library, for bindings
 * that cannot read the macro. */
size_t sq_decode_static_scratch_bytes(void);
sq_status sq_w8a8_linear_decode_noalloc(const int8_t *xq, const float *x_scale,
                                        const int8_t *wq, const float *w_scale,
                                        int64_t M, int64_t N, int64_t K,
                                        void *y, sq_dtype yt, int64_t ldy,
                                        sq_stream_t stream);

/*
 * Self-test of the failure path.  Launches one block whose thread waits on a
 * shared-memory barrier that nothing ever arrives at; the wait gives up
 * after `limit_ms` milliseconds (1..5000), records SQ_ERR_TIMEOUT in the
 * device error word, and the kernel returns normally, so the device stays
 * usable.  The next sq_check_device_error(stream) then reports
 * SQ_ERR_TIMEOUT.  Every wait in the other kernels uses the same mechanism
 * (with a 2 s limit).  Returns SQ_ERR_INVALID_ARG for a limit out of range.
 */
sq_status sq_selftest_wait_timeout(int limit_ms, sq_stream_t stream);

/*
 * Synchronises `stream`, then reports (and clears) a timeout that any
 * kernel of this library recorded on the current device since the last
 * check: SQ_ERR_TIMEOUT, else SQ_OK (or SQ_ERR_CUDA if the sync failed).
 */
sq_status sq_check_device_error(sq_stream_t stream);

/* Static, human-readable name of a status code. */
const char *sq_status_string(sq_status status);

#ifdef __cplusplus
}
#endif

#endif /* SQ_H_ */
