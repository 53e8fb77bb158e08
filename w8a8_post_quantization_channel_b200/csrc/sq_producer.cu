// sq_producer.cu -- the layer that produces X, with the smoothing folded in
// (sm_100a).  smooth_lm(alpha) in the usage example of "SmoothQuant
// (activation smoothing quantization)" (jisaku.com glossary) moves
// diag(s)^-1 out of the run-time path into the preceding layer; in
// transformer blocks that layer is an RMS normalisation, whose weight takes
// it.  Also the static per-tensor activation scale, the alternative to
// per-token scales that the same page contrasts with dynamic ones:
//   fold        gs_j = gamma_j * inv_s_j
//   producer    r_t = 1 / sqrt(sum_j x_tj^2 / K + eps), v = (x r) gs, INT8
//   static      delta = max_j(amax_j inv_s_j) / 127, q = sat(rne(x inv_s / delta))
#include <algorithm>

#include "sq_common.cuh"
#include "sq_internal.h"

namespace sq {

namespace {

constexpr int kRowMaxThreads = 512;  // largest CTA of the row producer
// Sum of the squares of one 16-byte row vector in double: each value is
// converted exactly, and fma(t, t, acc) adds its exact square with a single
// rounding, as a separate square and add would (one instruction fewer).
template <typename T>
__device__ __forceinline__ double sumsq_vec(uint4 raw) {
  constexpr int V = Vec<T>::N;
  float f[V];
  Vec<T>::to_f32(raw, f);
  double acc = 0.0;
#pragma unroll
  for (int e = 0; e < V; ++e) {
    const double t = (double)f[e];
    acc = __fma_rn(t, t, acc);
  }
  return acc;
}

// RMS normalisation whose weight already carries diag(s)^-1 (gs = gamma *
// inv_s, folded ahead of time), then per-token INT8.  Persistent like
// quant_rows_kernel: the folded weight stays in registers across rows and
// the next row is prefetched while the current one is reduced twice (sum of
// squares in double, then the absmax of v = (x * r) * gs, recomputed for
// the codes rather than held).
template <typename T, int kVPT>
__global__ void __launch_bounds__(kRowMaxThreads)
    rmsnorm_quant_rows_kernel(const T *__restrict__ x, int64_t rows, int64_t nvec, int64_t ld,
                              const float *__restrict__ gs, float eps, int8_t *__restrict__ q,
                              float *__restrict__ row_scale_out) {
  pdl_wait();  // the previous kernel's results are visible from here on
  pdl_trigger();
  constexpr int V = Vec<T>::N;
  __shared__ double red_ss[2][kRowMaxThreads / 32];
  __shared__ float red_m[2][kRowMaxThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  const int64_t K = nvec * V;
  const uint64_t policy = policy_evict_first();
  float g[kVPT][V];
#pragma unroll
  for (int i = 0; i < kVPT; ++i) {
    const int64_t v = tid + (int64_t)i * blockDim.x;
#pragma unroll
    for (int e4 = 0; e4 < V / 4; ++e4) {
      const float4 gv = v < nvec ? __ldg(reinterpret_cast<const float4 *>(gs + v * V) + e4) : make_float4(0, 0, 0, 0);
      g[i][4 * e4 + 0] = gv.x;
      g[i][4 * e4 + 1] = gv.y;
      g[i][4 * e4 + 2] = gv.z;
      g[i][4 * e4 + 3] = gv.w;
    }
  }
  uint4 cur[kVPT], nxt[kVPT];
  int64_t r = blockIdx.x;
#pragma unroll
  for (int i = 0; i < kVPT; ++i) {
    const int64_t v = tid + (int64_t)i * blockDim.x;
    cur[i] = (r < rows && v < nvec) ? ld_policy_v4(x + r * ld + v * V, policy) : make_uint4(0, 0, 0, 0);
  }
  int slot = 0;
  for (; r < rows; r += gridDim.x) {
    const int64_t rn = r + gridDim.x;
#pragma unroll
    for (int i = 0; i < kVPT; ++i) {
      const int64_t v = tid + (int64_t)i * blockDim.x;
      nxt[i] = (rn < rows && v < nvec) ? ld_policy_v4(x + rn * ld + v * V, policy) : make_uint4(0, 0, 0, 0);
    }
    // sum of squares in double (each square exact): one partial per
    // vector, then a tree -- the order of this sum is left open by the
    // definition
    double part[kVPT];
#pragma unroll
    for (int i = 0; i < kVPT; ++i) part[i] = sumsq_vec<T>(cur[i]);
#pragma unroll
    for (int w = kVPT / 2; w > 0; w >>= 1)
#pragma unroll
      for (int i = 0; i < w; ++i) part[i] = __dadd_rn(part[i], part[i + w]);
    double ss = part[0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
    if (lane == 0) red_ss[slot][warp] = ss;
    __syncthreads();
    ss = 0.0;
    for (int w = 0; w < nwarps; ++w) ss = __dadd_rn(ss, red_ss[slot][w]);
    // ss / K: an exact scaling when K is a power of two
    const double mean = (K & (K - 1)) == 0 ? __dmul_rn(ss, __drcp_rn((double)K)) : __ddiv_rn(ss, (double)K);
    const float rt = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(mean, (double)eps))));
    // absmax of v = (x * r) * gs (lanes past the row end hold x = gs = 0)
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < kVPT; ++i) {
      float f[V];
      Vec<T>::to_f32(cur[i], f);
#pragma unroll
      for (int e = 0; e < V; e += 2) {
        const float2 p = fmul2_rn(fmul2_rn(make_float2(f[e], f[e + 1]), make_float2(rt, rt)),
                                  make_float2(g[i][e], g[i][e + 1]));
        m = fmax3(m, fabsf(p.x), fabsf(p.y));
      }
    }
    m = warp_max(m);
    if (lane == 0) red_m[slot][warp] = m;
    __syncthreads();
    m = 0.0f;
    for (int w = 0; w < nwarps; ++w) m = fmaxf(m, red_m[slot][w]);
    slot ^= 1;
    const float delta = __fdiv_rn(m, 127.0f);
    const float rcp = m > 0.0f ? __frcp_rn(delta) : 0.0f;
    if (tid == 0) row_scale_out[r] = delta;
    int8_t *qrow = q + r * K;
#pragma unroll
    for (int i = 0; i < kVPT; ++i) {
      const int64_t v = tid + (int64_t)i * blockDim.x;
      if (v < nvec) {
        float f[V];
        Vec<T>::to_f32(cur[i], f);
        float val[V];
#pragma unroll
        for (int e = 0; e < V; e += 2) {
          const float2 p = fmul2_rn(fmul2_rn(make_float2(f[e], f[e + 1]), make_float2(rt, rt)),
                                    make_float2(g[i][e], g[i][e + 1]));
          val[e] = p.x;
          val[e + 1] = p.y;
        }
        if constexpr (V == 8) {
          *reinterpret_cast<uint2 *>(qrow + v * V) = codes8(val, delta, rcp);
        } else {
          *reinterpret_cast<uint32_t *>(qrow + v * V) = codes4(val, delta, rcp);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kVPT; ++i) cur[i] = nxt[i];
  }
}

// gs_j = gamma_j * inv_s_j: diag(s)^-1 folded into the norm's weight.
__global__ void fold_norm_weight_kernel(const float *__restrict__ gamma, const float *__restrict__ inv_s, int64_t K,
                                        float *__restrict__ gs) {
  pdl_wait();  // the previous kernel's results are visible from here on
  pdl_trigger();
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < K; j += (int64_t)gridDim.x * blockDim.x)
    gs[j] = __fmul_rn(gamma[j], inv_s[j]);
}

// Static per-tensor scale: *delta = max_j(amax_j * inv_s_j) / 127 (one block).
__global__ void __launch_bounds__(1024) static_scale_kernel(const float *__restrict__ amax,
                                                            const float *__restrict__ inv_s, int64_t K,
                                                            float *__restrict__ delta) {
  pdl_wait();  // the previous kernel's results are visible from here on
  pdl_trigger();
  __shared__ float red[32];
  float m = 0.0f;
  for (int64_t j = threadIdx.x; j < K; j += blockDim.x) m = fmaxf(m, __fmul_rn(amax[j], inv_s[j]));
  m = block_max(m, red);
  if (threadIdx.x == 0) *delta = __fdiv_rn(m, 127.0f);
}

// Static quantization: q = clamp(rne((x * inv_s) / delta)), every token's
// scale = delta.  Values beyond the calibrated range saturate.
// 2-D grid: x-blocks cover a row's 16-byte vectors, y-blocks stride rows.
constexpr int kStaticRows = 4;
template <typename T>
__global__ void __launch_bounds__(256) quant_static_kernel(const T *__restrict__ x, int64_t rows, int64_t nvec,
                                                           int64_t ld, const float *__restrict__ inv_s,
                                                           const float *__restrict__ delta, int8_t *__restrict__ q,
                                                           float *__restrict__ row_scale_out) {
  pdl_wait();  // the previous kernel's results are visible from here on
  pdl_trigger();
  constexpr int V = Vec<T>::N;
  const int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (v >= nvec) return;
  const float d = __ldg(delta);
  const float rcp = __frcp_rn(d);
  const float lim = __fmul_rn(127.0f, d);  // beyond +-lim every code saturates
  const int64_t K = nvec * V;
  float sc[V];
  const float4 *s4 = reinterpret_cast<const float4 *>(inv_s + v * V);
#pragma unroll
  for (int e4 = 0; e4 < V / 4; ++e4) {
    const float4 sv = __ldg(s4 + e4);
    sc[4 * e4 + 0] = sv.x;
    sc[4 * e4 + 1] = sv.y;
    sc[4 * e4 + 2] = sv.z;
    sc[4 * e4 + 3] = sv.w;
  }
  const uint64_t policy = policy_evict_first();
  // kStaticRows rows per pass, all loads issued before the first store
  const int64_t step = gridDim.y;
  for (int64_t t0 = blockIdx.y; t0 < rows; t0 += step * kStaticRows) {
    uint4 raw[kStaticRows];
#pragma unroll
    for (int u = 0; u < kStaticRows; ++u) {
      const int64_t t = t0 + u * step;
      raw[u] = t < rows ? ld_policy_v4(x + t * ld + v * V, policy) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kStaticRows; ++u) {
      const int64_t t = t0 + u * step;
      if (t >= rows) break;
      if (v == 0) row_scale_out[t] = d;
      float f[V];
      Vec<T>::to_f32(raw[u], f);
      float val[V];
#pragma unroll
      for (int e = 0; e < V; e += 2) {
        const float2 p = fmul2_rn(make_float2(f[e], f[e + 1]), make_float2(sc[e], sc[e + 1]));
        val[e] = clamp_to_range(p.x, lim);
        val[e + 1] = clamp_to_range(p.y, lim);
      }
      int8_t *qp = q + t * K + v * V;
      if constexpr (V == 8) {
        *reinterpret_cast<uint2 *>(qp) = codes8(val, d, rcp);
      } else {
        *reinterpret_cast<uint32_t *>(qp) = codes4(val, d, rcp);
      }
    }
  }
}

template <typename T>
cudaError_t rmsnorm_quant_t(const void *x, int64_t rows, int64_t cols, int64_t ld, const float *gs, float eps,
                            int8_t *q, float *row_scale_out, cudaStream_t st) {
  constexpr int V = Vec<T>::N;
  const int64_t nvec = cols / V;
  if (nvec > 4 * kRowMaxThreads) return cudaErrorNotSupported;
  // (two vectors per thread, for twice the resident warps, measured slower)
  const int vpt = nvec <= 4 * 32 ? 1 : 4;
  int64_t t = (nvec + vpt - 1) / vpt;
  const int threads = (int)std::max<int64_t>(32, ((t + 31) / 32) * 32);
  auto kern = vpt == 1 ? rmsnorm_quant_rows_kernel<T, 1> : rmsnorm_quant_rows_kernel<T, 4>;
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0);
  if (e != cudaSuccess) return e;
  const int64_t grid = std::min<int64_t>(rows, (int64_t)std::max(1, per_sm) * num_sms());
  return launch_pdl(kern, dim3((unsigned)grid), dim3(threads), 0, st, 1, (const T *)x, rows, nvec, ld, gs, eps, q,
                    row_scale_out);
}

template <typename T>
cudaError_t quant_static_t(const void *x, int64_t rows, int64_t cols, int64_t ld, const float *inv_s,
                           const float *delta, int8_t *q, float *row_scale_out, cudaStream_t st) {
  constexpr int V = Vec<T>::N;
  const int64_t nvec = cols / V;
  const int64_t bx = (nvec + 255) / 256;
  // about 16 resident 256-thread blocks per SM in total, each walking rows
  const int64_t groups = (rows + kStaticRows - 1) / kStaticRows;
  const int64_t by = std::max<int64_t>(1, std::min<int64_t>(groups, std::min<int64_t>(65535, num_sms() * 16 / bx + 1)));
  return launch_pdl(quant_static_kernel<T>, dim3((unsigned)bx, (unsigned)by), dim3(256), 0, st, 1, (const T *)x, rows,
                    nvec, ld, inv_s, delta, q, row_scale_out);
}

}  // namespace

cudaError_t launch_rmsnorm_quant(const void *x, sq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                                 const float *gs, float eps, int8_t *q, float *row_scale_out, cudaStream_t st) {
  switch (xt) {
    case SQ_F32: return rmsnorm_quant_t<float>(x, rows, cols, ld, gs, eps, q, row_scale_out, st);
    case SQ_F16: return rmsnorm_quant_t<__half>(x, rows, cols, ld, gs, eps, q, row_scale_out, st);
    default: return rmsnorm_quant_t<__nv_bfloat16>(x, rows, cols, ld, gs, eps, q, row_scale_out, st);
  }
}

cudaError_t launch_fold_norm_weight(const float *gamma, const float *inv_s, int64_t K, float *gs, cudaStream_t st) {
  const int64_t blocks = std::min<int64_t>((K + 255) / 256, 4 * (int64_t)num_sms());
  return launch_pdl(fold_norm_weight_kernel, dim3((unsigned)std::max<int64_t>(1, blocks)), dim3(256), 0, st, 1, gamma,
                    inv_s, K, gs);
}

cudaError_t launch_static_scale(const float *amax, const float *inv_s, int64_t K, float *delta, cudaStream_t st) {
  return launch_pdl(static_scale_kernel, dim3(1), dim3(1024), 0, st, 1, amax, inv_s, K, delta);
}

cudaError_t launch_quant_static(const void *x, sq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                                const float *inv_s, const float *delta, int8_t *q, float *row_scale_out,
                                cudaStream_t st) {
  switch (xt) {
    case SQ_F32: return quant_static_t<float>(x, rows, cols, ld, inv_s, delta, q, row_scale_out, st);
    case SQ_F16: return quant_static_t<__half>(x, rows, cols, ld, inv_s, delta, q, row_scale_out, st);
    default: return quant_static_t<__nv_bfloat16>(x, rows, cols, ld, inv_s, delta, q, row_scale_out, st);
  }
}

}  // namespace sq
