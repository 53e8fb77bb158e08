// sq_internal.h -- launchers shared between the ABI shim and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stddef.h>
#include <stdint.h>

#include "sq.h"

namespace sq {

// An NVTX range named after the ABI call, open for the call's host-side
// duration (validation and launches), so a profiler's timeline shows which
// call enqueued which kernels.  Without a profiler attached NVTX calls
// return at once and allocate nothing.
struct TraceRange {
  explicit TraceRange(const char *name) { nvtxRangePushA(name); }
  ~TraceRange() { nvtxRangePop(); }
  TraceRange(const TraceRange &) = delete;
  TraceRange &operator=(const TraceRange &) = delete;
};
#define SQ_TRACE_CALL() const sq::TraceRange sq_trace_range_(__func__)

// Number of SMs of the current device (cached per device).
int num_sms();
// Address of the current device's error word (cached per device).
unsigned *device_error_word();


// amax[c] = max(amax[c], max_r |x[r][c]| (* row_scale[r] when given)).
// keep_in_l2: x is read again by the next kernel (weights), so its lines
// are loaded with evict-last priority; otherwise evict-first.
cudaError_t launch_absmax_cols(const void *x, sq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                               const float *row_scale, float *amax, bool keep_in_l2, cudaStream_t st);
// out[r] = max_c |x[r][c]|.
cudaError_t launch_absmax_rows(const void *x, sq_dtype xt, int64_t rows, int64_t cols, int64_t ld, float *out,
                               cudaStream_t st);
// One block waits on a barrier nobody arrives at, up to limit_ns.
cudaError_t launch_wait_timeout_selftest(unsigned long long limit_ns, cudaStream_t st);
// p[0..n) = 0 (a kernel, so that it chains with its neighbours).
cudaError_t launch_zero_fill(float *p, int64_t n, cudaStream_t st);
// s[j] (holding w_j on entry) <- s_j, inv_s[j] <- 1/s_j from amax[j], w_j.
cudaError_t launch_smooth_factor(const float *amax, float *s_inout, float *inv_s, int64_t K, float alpha,
                                 cudaStream_t st);
// Code format of a quantizer: symmetric INT8 (absmax -> 127) or FP8 E4M3
// (absmax -> 448).
enum class QFmt { I8, E4M3 };
// Row-wise: v = x[r][c] * col_scale[c]; per row absmax -> scale, codes.
cudaError_t launch_quant_rows(const void *x, sq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                              const float *col_scale, int8_t *q, float *row_scale_out, QFmt fmt, cudaStream_t st);
// W[K][N] -> Wq[N][K] with v = s[j] * W[j][n] quantized per column n with
// the column maxima colmax[n]; then colmax[n] <- colmax[n] / Q.
cudaError_t launch_quant_cols_transpose(const void *w, sq_dtype wt, int64_t K, int64_t N, int64_t ld,
                                        const float *s, float *colmax_to_scale, int8_t *wq, QFmt fmt,
                                        cudaStream_t st);

// gs[j] = gamma[j] * inv_s[j].
cudaError_t launch_fold_norm_weight(const float *gamma, const float *inv_s, int64_t K, float *gs, cudaStream_t st);
// RMSNorm with the folded weight gs (eps) + per-token INT8 (K <= 16384 at
// 16 bits, 8192 at 32; cudaErrorNotSupported beyond).
cudaError_t launch_rmsnorm_quant(const void *x, sq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                                 const float *gs, float eps, int8_t *q, float *row_scale_out, cudaStream_t st);
cudaError_t launch_layernorm_quant(const void *x, sq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                                   const float *gs, const float *bs, float eps, int8_t *q, float *row_scale_out,
                                   cudaStream_t st);
// *delta = max_j(amax_j * inv_s_j) / 127.
cudaError_t launch_static_scale(const float *amax, const float *inv_s, int64_t K, float *delta, cudaStream_t st);
// Static per-tensor quantization with the device scalar *delta.
cudaError_t launch_quant_static(const void *x, sq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                                const float *inv_s, const float *delta, int8_t *q, float *row_scale_out,
                                cudaStream_t st);

// Rows of x * col_scale rotated per block of n = 2^logn channels by the
// butterfly with (cos, sin) pairs cs [logn][n / 2][2], then per-row INT8
// (K <= 16384 at 16 bits, 8192 at 32; cudaErrorNotSupported beyond).  Blocks
// of up to one warp's channels (256 at 16 bits, 128 at 32) rotate in
// registers; wider blocks through a row staged in shared memory.
cudaError_t launch_rot_quant_rows(const void *x, sq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                                  const float *col_scale, int logn, const float *cs, int8_t *q, float *row_scale_out,
                                  cudaStream_t st);

// Output kinds of the tensor-core GEMM epilogue (I32: the raw 32-bit
// accumulator -- an int32 sum for INT8 operands, an f32 sum for E4M3).
enum class OutKind { F32, F16, BF16, I32 };
// Where the epilogue stores Y: n destination matrices (this rank's Y and,
// for a column-parallel linear, peers' copies -- possibly peer-mapped
// pointers), each [M][ldy] and already offset to this shard's first column.
// Every tile is written to all n with plain stores.
constexpr int kMaxDest = 8;
struct YDest {
  void *p[kMaxDest];
  int n;
};
// Operands are INT8 codes (fmt I8) or E4M3 codes (fmt E4M3), both [rows][K].
cudaError_t launch_w8a8_gemm_dest(const int8_t *xq, const float *x_scale, const int8_t *wq, const float *w_scale,
                                  int64_t M, int64_t N, int64_t K, const YDest &dst, OutKind kind, int64_t ldy,
                                  void *workspace, cudaStream_t st, QFmt fmt);
cudaError_t launch_w8a8_gemm(const int8_t *xq, const float *x_scale, const int8_t *wq, const float *w_scale,
                             int64_t M, int64_t N, int64_t K, void *y, OutKind kind, int64_t ldy, void *workspace,
                             size_t workspace_bytes, cudaStream_t st, QFmt fmt);
// Workspace bytes the product of this shape needs on the current device:
// the stream-K decode kernel's partial sums and tile counters, or 0 (the
// cluster split and the prefill kernels use none).  Without a device to plan
// for, the stream-K kernel's need for any decode-shaped M.
size_t w8a8_workspace_bytes(int64_t M, int64_t N, int64_t K);
// Whether the decode-shaped product (1 <= M <= 64) of this shape takes the
// stream-K kernel on the current device.
bool w8a8_decode_uses_workspace(int64_t M, int64_t N, int64_t K);

}  // namespace sq
