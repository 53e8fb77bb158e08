// sq_abi.cu -- the extern "C" boundary of libsq.so: argument validation,
// dispatch to the kernels, status mapping.  See include/sq.h for the
// contract of each call.
#include <cuda_runtime.h>

#include <mutex>

#include "sq_internal.h"

namespace sq {

// One word per device; kernels OR kDevErrTimeout into it.
__device__ unsigned g_device_error;

namespace {
constexpr int kMaxDevices = 64;

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return 0;
  return d;
}
}  // namespace

int num_sms() {
  static int cache[kMaxDevices] = {};
  const int d = current_device();
  if (d >= kMaxDevices) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d);
    return n > 0 ? n : 1;
  }
  if (cache[d] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d);
    cache[d] = n > 0 ? n : 1;
  }
  return cache[d];
}

unsigned *device_error_word() {
  static unsigned *cache[kMaxDevices] = {};
  static std::mutex mu;
  const int d = current_device();
  std::lock_guard<std::mutex> lock(mu);
  if (d < kMaxDevices && cache[d] != nullptr) return cache[d];
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
  if (d < kMaxDevices) cache[d] = static_cast<unsigned *>(p);
  return static_cast<unsigned *>(p);
}

}  // namespace sq

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool valid_dtype(int t) { return t == SQ_F32 || t == SQ_F16 || t == SQ_BF16; }
int64_t dsize(sq_dtype t) { return t == SQ_F32 ? 4 : 2; }
constexpr int64_t kMaxDim = (int64_t)1 << 31;

sq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SQ_OK : SQ_ERR_CUDA; }

// A [rows][ld] matrix of dtype t whose rows hold `cols` elements.
bool valid_matrix(const void *p, sq_dtype t, int64_t rows, int64_t cols, int64_t ld) {
  if (p == nullptr || !aligned16(p)) return false;
  if (rows < 0 || rows >= kMaxDim || cols <= 0 || cols >= kMaxDim) return false;
  if (ld < cols || (ld * dsize(t)) % 16 != 0) return false;
  return true;
}

bool valid_vec(const void *p) { return p != nullptr && aligned16(p); }

}  // namespace

extern "C" {

const char *sq_status_string(sq_status s) {
  switch (s) {
    case SQ_OK: return "SQ_OK";
    case SQ_ERR_INVALID_ARG: return "SQ_ERR_INVALID_ARG: invalid argument";
    case SQ_ERR_UNSUPPORTED: return "SQ_ERR_UNSUPPORTED: unsupported request";
    case SQ_ERR_CUDA: return "SQ_ERR_CUDA: a CUDA call failed";
    case SQ_ERR_TIMEOUT: return "SQ_ERR_TIMEOUT: an in-kernel wait ran out";
  }
  return "unknown sq_status";
}

sq_status sq_calib_absmax(const void *x, sq_dtype xt, int64_t T, int64_t K, int64_t ldx, float *amax,
                          sq_stream_t stream) {
  SQ_TRACE_CALL();
  if (!valid_dtype(xt) || K <= 0 || K % 16 != 0 || K >= kMaxDim || T < 0 || T >= kMaxDim) return SQ_ERR_INVALID_ARG;
  if (!valid_vec(amax)) return SQ_ERR_INVALID_ARG;
  if (ldx < K || (ldx * dsize(xt)) % 16 != 0) return SQ_ERR_INVALID_ARG;
  if (T == 0) return SQ_OK;
  if (!valid_matrix(x, xt, T, K, ldx)) return SQ_ERR_INVALID_ARG;
  return from_cuda(sq::launch_absmax_cols(x, xt, T, K, ldx, nullptr, amax, false, (cudaStream_t)stream));
}

static sq_status smooth_quant_weight_impl(const void *w, sq_dtype wt, sq_wlayout layout, int64_t K, int64_t N,
                                          int64_t ldw, const float *amax, float alpha, int8_t *wq, float *w_scale,
                                          float *smooth, float *inv_smooth, sq::QFmt fmt, sq_stream_t stream) {
  if (!valid_dtype(wt) || (layout != SQ_W_KN && layout != SQ_W_NK)) return SQ_ERR_INVALID_ARG;
  if (K <= 0 || N <= 0 || K % 16 != 0 || N % 16 != 0) return SQ_ERR_INVALID_ARG;
  if (!(alpha >= 0.0f && alpha <= 1.0f)) return SQ_ERR_INVALID_ARG;
  const bool kn = layout == SQ_W_KN;
  if (!valid_matrix(w, wt, kn ? K : N, kn ? N : K, ldw)) return SQ_ERR_INVALID_ARG;
  if (!valid_vec(amax) || !valid_vec(wq) || !valid_vec(w_scale) || !valid_vec(smooth) || !valid_vec(inv_smooth))
    return SQ_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  // w_j = max_n |W_jn| into `smooth`
  if (kn) {
    e = sq::launch_absmax_rows(w, wt, K, N, ldw, smooth, st);
  } else {
    e = sq::launch_zero_fill(smooth, K, st);
    if (e == cudaSuccess) e = sq::launch_absmax_cols(w, wt, N, K, ldw, nullptr, smooth, true, st);
  }
  if (e != cudaSuccess) return SQ_ERR_CUDA;
  // s_j, 1/s_j
  e = sq::launch_smooth_factor(amax, smooth, inv_smooth, K, alpha, st);
  if (e != cudaSuccess) return SQ_ERR_CUDA;
  // W~ = diag(s) W, per-output-channel INT8
  if (kn) {
    e = sq::launch_zero_fill(w_scale, N, st);
    if (e == cudaSuccess) e = sq::launch_absmax_cols(w, wt, K, N, ldw, smooth, w_scale, true, st);
    if (e == cudaSuccess) e = sq::launch_quant_cols_transpose(w, wt, K, N, ldw, smooth, w_scale, wq, fmt, st);
  } else {
    e = sq::launch_quant_rows(w, wt, N, K, ldw, smooth, wq, w_scale, fmt, st);
  }
  return from_cuda(e);
}

sq_status sq_smooth_quant_weight(const void *w, sq_dtype wt, sq_wlayout layout, int64_t K, int64_t N, int64_t ldw,
                                 const float *amax, float alpha, int8_t *wq, float *w_scale, float *smooth,
                                 float *inv_smooth, sq_stream_t stream) {
  SQ_TRACE_CALL();
  return smooth_quant_weight_impl(w, wt, layout, K, N, ldw, amax, alpha, wq, w_scale, smooth, inv_smooth,
                                  sq::QFmt::I8, stream);
}

sq_status sq_smooth_quant_weight_e4m3(const void *w, sq_dtype wt, sq_wlayout layout, int64_t K, int64_t N,
                                      int64_t ldw, const float *amax, float alpha, uint8_t *wq, float *w_scale,
                                      float *smooth, float *inv_smooth, sq_stream_t stream) {
  SQ_TRACE_CALL();
  return smooth_quant_weight_impl(w, wt, layout, K, N, ldw, amax, alpha, reinterpret_cast<int8_t *>(wq), w_scale,
                                  smooth, inv_smooth, sq::QFmt::E4M3, stream);
}

static sq_status quant_act_impl(const void *x, sq_dtype xt, int64_t M, int64_t K, int64_t ldx,
                                const float *inv_smooth, int8_t *xq, float *x_scale, sq::QFmt fmt,
                                sq_stream_t stream) {
  if (!valid_dtype(xt) || K <= 0 || K % 16 != 0 || K >= kMaxDim || M < 0 || M >= kMaxDim) return SQ_ERR_INVALID_ARG;
  if (ldx < K || (ldx * dsize(xt)) % 16 != 0) return SQ_ERR_INVALID_ARG;
  if (!valid_vec(inv_smooth)) return SQ_ERR_INVALID_ARG;
  if (M == 0) return SQ_OK;
  if (!valid_matrix(x, xt, M, K, ldx) || !valid_vec(xq) || !valid_vec(x_scale)) return SQ_ERR_INVALID_ARG;
  return from_cuda(sq::launch_quant_rows(x, xt, M, K, ldx, inv_smooth, xq, x_scale, fmt, (cudaStream_t)stream));
}

sq_status sq_quant_act(const void *x, sq_dtype xt, int64_t M, int64_t K, int64_t ldx, const float *inv_smooth,
                       int8_t *xq, float *x_scale, sq_stream_t stream) {
  SQ_TRACE_CALL();
  return quant_act_impl(x, xt, M, K, ldx, inv_smooth, xq, x_scale, sq::QFmt::I8, stream);
}

static int log2_exact(int64_t n) {
  int l = 0;
  while (l < 62 && ((int64_t)1 << l) < n) ++l;
  return ((int64_t)1 << l) == n ? l : -1;
}

static sq_status rot_checks(sq_dtype xt, int64_t K, int64_t n, const float *rot_cs, int *logn) {
  *logn = log2_exact(n);
  if (*logn < 1 || K % n != 0 || !valid_vec(rot_cs)) return SQ_ERR_INVALID_ARG;
  if (K > (xt == SQ_F32 ? 8192 : 16384)) return SQ_ERR_UNSUPPORTED;
  return SQ_OK;
}

sq_status sq_quant_act_rotated(const void *x, sq_dtype xt, int64_t M, int64_t K, int64_t ldx, const float *inv_smooth,
                               int64_t n, const float *rot_cs, int8_t *xq, float *x_scale, sq_stream_t stream) {
  SQ_TRACE_CALL();
  if (!valid_dtype(xt) || K <= 0 || K % 16 != 0 || K >= kMaxDim || M < 0 || M >= kMaxDim) return SQ_ERR_INVALID_ARG;
  if (ldx < K || (ldx * dsize(xt)) % 16 != 0 || !valid_vec(inv_smooth)) return SQ_ERR_INVALID_ARG;
  int logn = 0;
  const sq_status rs = rot_checks(xt, K, n, rot_cs, &logn);
  if (rs != SQ_OK) return rs;
  if (M == 0) return SQ_OK;
  if (!valid_matrix(x, xt, M, K, ldx) || !valid_vec(xq) || !valid_vec(x_scale)) return SQ_ERR_INVALID_ARG;
  return from_cuda(
      sq::launch_rot_quant_rows(x, xt, M, K, ldx, inv_smooth, logn, rot_cs, xq, x_scale, (cudaStream_t)stream));
}

sq_status sq_smooth_quant_weight_rotated(const void *w, sq_dtype wt, int64_t K, int64_t N, int64_t ldw,
                                         const float *amax, float alpha, int64_t n, const float *rot_cs, int8_t *wq,
                                         float *w_scale, float *smooth, float *inv_smooth, sq_stream_t stream) {
  SQ_TRACE_CALL();
  if (!valid_dtype(wt) || K <= 0 || N <= 0 || K % 16 != 0 || N % 16 != 0) return SQ_ERR_INVALID_ARG;
  if (!(alpha >= 0.0f && alpha <= 1.0f)) return SQ_ERR_INVALID_ARG;
  if (!valid_matrix(w, wt, N, K, ldw)) return SQ_ERR_INVALID_ARG;
  if (!valid_vec(amax) || !valid_vec(wq) || !valid_vec(w_scale) || !valid_vec(smooth) || !valid_vec(inv_smooth))
    return SQ_ERR_INVALID_ARG;
  int logn = 0;
  const sq_status rs = rot_checks(wt, K, n, rot_cs, &logn);
  if (rs != SQ_OK) return rs;
  cudaStream_t st = (cudaStream_t)stream;
  // w_j = max_n |W_jn| into `smooth`, then s_j and 1/s_j as without rotation
  cudaError_t e = sq::launch_zero_fill(smooth, K, st);
  if (e == cudaSuccess) e = sq::launch_absmax_cols(w, wt, N, K, ldw, nullptr, smooth, true, st);
  if (e == cudaSuccess) e = sq::launch_smooth_factor(amax, smooth, inv_smooth, K, alpha, st);
  // rows R(s * w_n), per-output-channel INT8
  if (e == cudaSuccess) e = sq::launch_rot_quant_rows(w, wt, N, K, ldw, smooth, logn, rot_cs, wq, w_scale, st);
  return from_cuda(e);
}

sq_status sq_quant_act_e4m3(const void *x, sq_dtype xt, int64_t M, int64_t K, int64_t ldx, const float *inv_smooth,
                            uint8_t *xq, float *x_scale, sq_stream_t stream) {
  SQ_TRACE_CALL();
  return quant_act_impl(x, xt, M, K, ldx, inv_smooth, reinterpret_cast<int8_t *>(xq), x_scale, sq::QFmt::E4M3,
                        stream);
}

sq_status sq_fold_smooth_into_norm(const float *gamma, const float *inv_smooth, int64_t K, float *gs,
                                   sq_stream_t stream) {
  SQ_TRACE_CALL();
  if (K <= 0 || K >= kMaxDim || !valid_vec(gamma) || !valid_vec(inv_smooth) || !valid_vec(gs))
    return SQ_ERR_INVALID_ARG;
  return from_cuda(sq::launch_fold_norm_weight(gamma, inv_smooth, K, gs, (cudaStream_t)stream));
}

sq_status sq_rmsnorm_quant_act(const void *x, sq_dtype xt, int64_t M, int64_t K, int64_t ldx, const float *gs,
                               float eps, int8_t *xq, float *x_scale, sq_stream_t stream) {
  SQ_TRACE_CALL();
  if (!valid_dtype(xt) || K <= 0 || K % 16 != 0 || K >= kMaxDim || M < 0 || M >= kMaxDim) return SQ_ERR_INVALID_ARG;
  if (ldx < K || (ldx * dsize(xt)) % 16 != 0) return SQ_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || eps > 3.0e38f) return SQ_ERR_INVALID_ARG;  // rejects NaN and infinity too
  if (!valid_vec(gs)) return SQ_ERR_INVALID_ARG;
  if (K > (xt == SQ_F32 ? 8192 : 16384)) return SQ_ERR_UNSUPPORTED;
  if (M == 0) return SQ_OK;
  if (!valid_matrix(x, xt, M, K, ldx) || !valid_vec(xq) || !valid_vec(x_scale)) return SQ_ERR_INVALID_ARG;
  return from_cuda(sq::launch_rmsnorm_quant(x, xt, M, K, ldx, gs, eps, xq, x_scale, (cudaStream_t)stream));
}

sq_status sq_layernorm_quant_act(const void *x, sq_dtype xt, int64_t M, int64_t K, int64_t ldx, const float *gs,
                                 const float *bs, float eps, int8_t *xq, float *x_scale, sq_stream_t stream) {
  SQ_TRACE_CALL();
  if (!valid_dtype(xt) || K <= 0 || K % 16 != 0 || K >= kMaxDim || M < 0 || M >= kMaxDim) return SQ_ERR_INVALID_ARG;
  if (ldx < K || (ldx * dsize(xt)) % 16 != 0) return SQ_ERR_INVALID_ARG;
  if (!(eps > 0.0f) || eps > 3.0e38f) return SQ_ERR_INVALID_ARG;  // rejects NaN and infinity too
  if (!valid_vec(gs) || (bs != nullptr && !valid_vec(bs))) return SQ_ERR_INVALID_ARG;
  if (K > (xt == SQ_F32 ? 8192 : 16384)) return SQ_ERR_UNSUPPORTED;
  if (M == 0) return SQ_OK;
  if (!valid_matrix(x, xt, M, K, ldx) || !valid_vec(xq) || !valid_vec(x_scale)) return SQ_ERR_INVALID_ARG;
  return from_cuda(sq::launch_layernorm_quant(x, xt, M, K, ldx, gs, bs, eps, xq, x_scale, (cudaStream_t)stream));
}

sq_status sq_static_act_scale(const float *amax, const float *inv_smooth, int64_t K, float *delta,
                              sq_stream_t stream) {
  SQ_TRACE_CALL();
  if (K <= 0 || K >= kMaxDim || !valid_vec(amax) || !valid_vec(inv_smooth)) return SQ_ERR_INVALID_ARG;
  if (delta == nullptr || (reinterpret_cast<uintptr_t>(delta) & 3u) != 0) return SQ_ERR_INVALID_ARG;
  return from_cuda(sq::launch_static_scale(amax, inv_smooth, K, delta, (cudaStream_t)stream));
}

sq_status sq_quant_act_static(const void *x, sq_dtype xt, int64_t M, int64_t K, int64_t ldx, const float *inv_smooth,
                              const float *delta, int8_t *xq, float *x_scale, sq_stream_t stream) {
  SQ_TRACE_CALL();
  if (!valid_dtype(xt) || K <= 0 || K % 16 != 0 || K >= kMaxDim || M < 0 || M >= kMaxDim) return SQ_ERR_INVALID_ARG;
  if (ldx < K || (ldx * dsize(xt)) % 16 != 0) return SQ_ERR_INVALID_ARG;
  if (!valid_vec(inv_smooth) || delta == nullptr || (reinterpret_cast<uintptr_t>(delta) & 3u) != 0)
    return SQ_ERR_INVALID_ARG;
  if (M == 0) return SQ_OK;
  if (!valid_matrix(x, xt, M, K, ldx) || !valid_vec(xq) || !valid_vec(x_scale)) return SQ_ERR_INVALID_ARG;
  return from_cuda(sq::launch_quant_static(x, xt, M, K, ldx, inv_smooth, delta, xq, x_scale, (cudaStream_t)stream));
}

static sq_status gemm_common(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K, const void *y,
                             int64_t ldy, int64_t ysize, void *workspace, size_t workspace_bytes) {
  if (M < 0 || M >= kMaxDim || N <= 0 || N >= kMaxDim || K <= 0 || K >= kMaxDim) return SQ_ERR_INVALID_ARG;
  if (K % 16 != 0 || N % 16 != 0) return SQ_ERR_INVALID_ARG;
  if (ldy < N || (ldy * ysize) % 16 != 0) return SQ_ERR_INVALID_ARG;
  if (!valid_vec(wq)) return SQ_ERR_INVALID_ARG;
  if (M == 0) return SQ_OK;
  if (!valid_vec(xq) || !valid_vec(y)) return SQ_ERR_INVALID_ARG;
  const size_t need = sq::w8a8_workspace_bytes(M, N, K);
  if (need > 0 && (workspace == nullptr || !aligned16(workspace) || workspace_bytes < need))
    return SQ_ERR_INVALID_ARG;
  return SQ_OK;
}

static sq_status linear_impl(const int8_t *xq, const float *x_scale, const int8_t *wq, const float *w_scale,
                             int64_t M, int64_t N, int64_t K, void *y, sq_dtype yt, int64_t ldy, void *workspace,
                             size_t workspace_bytes, sq::QFmt fmt, sq_stream_t stream) {
  if (!valid_dtype(yt)) return SQ_ERR_INVALID_ARG;
  if (!valid_vec(w_scale)) return SQ_ERR_INVALID_ARG;
  sq_status s = gemm_common(xq, wq, M, N, K, y, ldy, dsize(yt), workspace, workspace_bytes);
  if (s != SQ_OK || M == 0) return s;
  if (!valid_vec(x_scale)) return SQ_ERR_INVALID_ARG;
  const sq::OutKind kind = yt == SQ_F32 ? sq::OutKind::F32 : yt == SQ_F16 ? sq::OutKind::F16 : sq::OutKind::BF16;
  return from_cuda(sq::launch_w8a8_gemm(xq, x_scale, wq, w_scale, M, N, K, y, kind, ldy, workspace,
                                        workspace_bytes, (cudaStream_t)stream, fmt));
}

static sq_status accumulate_impl(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K, void *acc,
                                 int64_t ldacc, void *workspace, size_t workspace_bytes, sq::QFmt fmt,
                                 sq_stream_t stream) {
  sq_status s = gemm_common(xq, wq, M, N, K, acc, ldacc, 4, workspace, workspace_bytes);
  if (s != SQ_OK || M == 0) return s;
  return from_cuda(sq::launch_w8a8_gemm(xq, nullptr, wq, nullptr, M, N, K, acc, sq::OutKind::I32, ldacc, workspace,
                                        workspace_bytes, (cudaStream_t)stream, fmt));
}

sq_status sq_w8a8_linear(const int8_t *xq, const float *x_scale, const int8_t *wq, const float *w_scale, int64_t M,
                         int64_t N, int64_t K, void *y, sq_dtype yt, int64_t ldy, void *workspace,
                         size_t workspace_bytes, sq_stream_t stream) {
  SQ_TRACE_CALL();
  return linear_impl(xq, x_scale, wq, w_scale, M, N, K, y, yt, ldy, workspace, workspace_bytes, sq::QFmt::I8,
                     stream);
}

sq_status sq_w8a8_linear_e4m3(const uint8_t *xq, const float *x_scale, const uint8_t *wq, const float *w_scale,
                              int64_t M, int64_t N, int64_t K, void *y, sq_dtype yt, int64_t ldy, void *workspace,
                              size_t workspace_bytes, sq_stream_t stream) {
  SQ_TRACE_CALL();
  return linear_impl(reinterpret_cast<const int8_t *>(xq), x_scale, reinterpret_cast<const int8_t *>(wq), w_scale,
                     M, N, K, y, yt, ldy, workspace, workspace_bytes, sq::QFmt::E4M3, stream);
}

sq_status sq_w8a8_linear_scatter(const int8_t *xq, const float *x_scale, const int8_t *wq, const float *w_scale,
                                 int64_t M, int64_t N, int64_t K, void *const *y_dst, int n_dst, sq_dtype yt,
                                 int64_t ldy, void *workspace, size_t workspace_bytes, sq_stream_t stream) {
  SQ_TRACE_CALL();
  if (!valid_dtype(yt) || !valid_vec(w_scale)) return SQ_ERR_INVALID_ARG;
  if (y_dst == nullptr || n_dst < 1 || n_dst > sq::kMaxDest) return SQ_ERR_INVALID_ARG;
  sq::YDest dst{};
  for (int d = 0; d < n_dst; ++d) {
    if (!valid_vec(y_dst[d])) return SQ_ERR_INVALID_ARG;
    dst.p[d] = y_dst[d];
  }
  dst.n = n_dst;
  sq_status s = gemm_common(xq, wq, M, N, K, y_dst[0], ldy, dsize(yt), workspace, workspace_bytes);
  if (s != SQ_OK || M == 0) return s;
  if (!valid_vec(x_scale)) return SQ_ERR_INVALID_ARG;
  const sq::OutKind kind = yt == SQ_F32 ? sq::OutKind::F32 : yt == SQ_F16 ? sq::OutKind::F16 : sq::OutKind::BF16;
  return from_cuda(sq::launch_w8a8_gemm_dest(xq, x_scale, wq, w_scale, M, N, K, dst, kind, ldy, workspace,
                                             (cudaStream_t)stream, sq::QFmt::I8));
}

size_t sq_w8a8_linear_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  return sq::w8a8_workspace_bytes(M, N, K);
}

sq_status sq_w8a8_accumulate(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K, int32_t *acc,
                             int64_t ldacc, void *workspace, size_t workspace_bytes, sq_stream_t stream) {
  SQ_TRACE_CALL();
  return accumulate_impl(xq, wq, M, N, K, acc, ldacc, workspace, workspace_bytes, sq::QFmt::I8, stream);
}

sq_status sq_w8a8_accumulate_e4m3(const uint8_t *xq, const uint8_t *wq, int64_t M, int64_t N, int64_t K, float *acc,
                                  int64_t ldacc, void *workspace, size_t workspace_bytes, sq_stream_t stream) {
  SQ_TRACE_CALL();
  return accumulate_impl(reinterpret_cast<const int8_t *>(xq), reinterpret_cast<const int8_t *>(wq), M, N, K, acc,
                         ldacc, workspace, workspace_bytes, sq::QFmt::E4M3, stream);
}

sq_status sq_selftest_wait_timeout(int limit_ms, sq_stream_t stream) {
  SQ_TRACE_CALL();
  if (limit_ms < 1 || limit_ms > 5000) return SQ_ERR_INVALID_ARG;
  return from_cuda(sq::launch_wait_timeout_selftest((unsigned long long)limit_ms * 1000000ull, (cudaStream_t)stream));
}

sq_status sq_check_device_error(sq_stream_t stream) {
  SQ_TRACE_CALL();
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return SQ_ERR_CUDA;
  unsigned *word = sq::device_error_word();
  if (word == nullptr) return SQ_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpy(&v, word, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return SQ_ERR_CUDA;
  if (v != 0) {
    if (cudaMemset(word, 0, sizeof(v)) != cudaSuccess) return SQ_ERR_CUDA;
    return SQ_ERR_TIMEOUT;
  }
  return SQ_OK;
}

}  // extern "C"
