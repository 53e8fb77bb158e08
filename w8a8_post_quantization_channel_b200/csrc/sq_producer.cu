// sq_producer.cu -- the layer that produces X, with the smoothing folded in
// (sm_100a).  smooth_lm(alpha) in the usage example of "SmoothQuant
// (activation smoothing quantization)" (jisaku.com glossary) moves
// diag(s)^-1 out of the run-time path into the preceding layer; in
// transformer blocks that layer is a normalisation -- RMS (Llama) or a
// LayerNorm with a bias (the OPT models of the page's tables) -- whose
// weight and bias take it.  Also the static per-tensor activation scale, the alternative to
// per-token scales that the same page contrasts with dynamic ones:
//   fold        gs_j = gamma_j * inv_s_j
//   producer    r_t = 1 / sqrt(sum_j x_tj^2 / K + eps), v = (x r) gs, INT8
//   LayerNorm   mu_t = mean_j x_tj, r_t = 1 / sqrt(mean_j (x_tj - mu_t)^2 + eps),
//               v = fma((x - mu) r, gs, bs), INT8 (bs = beta * inv_s)
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

// Shifted sums of one 16-byte row vector in double: s += sum_e (x_e - c),
// q += sum_e (x_e - c)^2, each value converted exactly, in two chains per
// sum.  Lanes past the row end hold x = 0 and must add nothing: `live` is
// false there.
template <typename T>
__device__ __forceinline__ void shifted_sums_vec(uint4 raw, double c, bool live, double &s, double &q) {
  constexpr int V = Vec<T>::N;
  float f[V];
  Vec<T>::to_f32(raw, f);
  double s0 = 0.0, s1 = 0.0, q0 = 0.0, q1 = 0.0;
#pragma unroll
  for (int e = 0; e < V; e += 2) {
    const double d0 = __dsub_rn((double)f[e], c);
    const double d1 = __dsub_rn((double)f[e + 1], c);
    s0 = __dadd_rn(s0, d0);
    s1 = __dadd_rn(s1, d1);
    q0 = __fma_rn(d0, d0, q0);
    q1 = __fma_rn(d1, d1, q1);
  }
  if (live) {
    s = __dadd_rn(s, __dadd_rn(s0, s1));
    q = __dadd_rn(q, __dadd_rn(q0, q1));
  }
}

// Block-wide double sum of one per-thread partial through red[] (one slot
// per warp); every thread gets the total.
__device__ __forceinline__ double block_sum_d(double v, double *red, int lane, int warp, int nwarps) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) red[warp] = v;
  __syncthreads();
  v = 0.0;
  for (int w = 0; w < nwarps; ++w) v = __dadd_rn(v, red[w]);
  return v;
}

// Block-wide double sums of two per-thread partials through red[] (two
// slots per warp); every thread gets both totals.
__device__ __forceinline__ void block_sum_d2(double &a, double &b, double (*red)[2], int lane, int warp,
                                             int nwarps) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a = __dadd_rn(a, __shfl_xor_sync(0xffffffffu, a, o));
    b = __dadd_rn(b, __shfl_xor_sync(0xffffffffu, b, o));
  }
  if (lane == 0) {
    red[warp][0] = a;
    red[warp][1] = b;
  }
  __syncthreads();
  a = 0.0;
  b = 0.0;
  for (int w = 0; w < nwarps; ++w) {
    a = __dadd_rn(a, red[w][0]);
    b = __dadd_rn(b, red[w][1]);
  }
}

// x / K in double: an exact scaling when K is a power of two.
__device__ __forceinline__ double div_by_count(double x, int64_t K) {
  return (K & (K - 1)) == 0 ? __dmul_rn(x, __drcp_rn((double)K)) : __ddiv_rn(x, (double)K);
}

// Normalisation whose weight (and bias) already carry diag(s)^-1 (gs =
// gamma * inv_s, bs = beta * inv_s, folded ahead of time), then per-token
// INT8.  kLN false: RMS normalisation, v = (x * r) * gs with
// r = 1/sqrt(mean(x^2) + eps).  kLN true: layer normalisation,
// v = fma((x - mu) * r, gs, bs) with r = 1/sqrt(mean((x - mu)^2) + eps),
// the mean and variance from one shifted pass; bs may be null (no bias).  Persistent like quant_rows_kernel: the folded
// weight stays in registers across rows and the next row is prefetched
// while the current one is reduced (the statistics in double, then the
// absmax of v, recomputed for the codes rather than held).
template <typename T, int kVPT, bool kLN>
__global__ void __launch_bounds__(kRowMaxThreads)
    norm_quant_rows_kernel(const T *__restrict__ x, int64_t rows, int64_t nvec, int64_t ld,
                           const float *__restrict__ gs, const float *__restrict__ bs, float eps,
                           int8_t *__restrict__ q, float *__restrict__ row_scale_out) {
  pdl_wait();  // the previous kernel's results are visible from here on
  pdl_trigger();
  constexpr int V = Vec<T>::N;
  __shared__ double red_ss[2][kRowMaxThreads / 32];
  __shared__ double red_sq[kLN ? 2 : 1][kRowMaxThreads / 32][2];
  __shared__ float red_m[2][kRowMaxThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  const int64_t K = nvec * V;
  const uint64_t policy = policy_evict_first();
  float g[kVPT][V];
  float b[kLN ? kVPT : 1][V];
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
      if constexpr (kLN) {
        const float4 bv = (v < nvec && bs != nullptr) ? __ldg(reinterpret_cast<const float4 *>(bs + v * V) + e4)
                                                      : make_float4(0, 0, 0, 0);
        b[i][4 * e4 + 0] = bv.x;
        b[i][4 * e4 + 1] = bv.y;
        b[i][4 * e4 + 2] = bv.z;
        b[i][4 * e4 + 3] = bv.w;
      }
    }
  }
  uint4 cur[kVPT], nxt[kVPT];
  int64_t r = blockIdx.x;
#pragma unroll
  for (int i = 0; i < kVPT; ++i) {
    const int64_t v = tid + (int64_t)i * blockDim.x;
    cur[i] = (r < rows && v < nvec) ? ld_policy_v4(x + r * ld + v * V, policy) : make_uint4(0, 0, 0, 0);
  }
  // LayerNorm: the row's first value, the shift of its one-pass statistics
  double c_cur = 0.0, c_nxt = 0.0;
  if constexpr (kLN) c_cur = r < rows ? (double)Vec<T>::one(x + r * ld) : 0.0;
  int slot = 0;
  for (; r < rows; r += gridDim.x) {
    const int64_t rn = r + gridDim.x;
#pragma unroll
    for (int i = 0; i < kVPT; ++i) {
      const int64_t v = tid + (int64_t)i * blockDim.x;
      nxt[i] = (rn < rows && v < nvec) ? ld_policy_v4(x + rn * ld + v * V, policy) : make_uint4(0, 0, 0, 0);
    }
    if constexpr (kLN) c_nxt = rn < rows ? (double)Vec<T>::one(x + rn * ld) : 0.0;
    // the statistics in double -- the order of these sums is left open by
    // the definition
    double ms;  // the mean square under the root: mean(x^2), or var
    float muf = 0.0f;
    if constexpr (kLN) {
      // One pass over the deviations d = x - c from the row's first value
      // c: with S = sum d and Q = sum d^2, mu = c + S/K and
      // var = Q/K - (S/K)^2.  As c is one of the row's values,
      // (mu - c)^2 <= K var, so Q/K <= (K + 1) var: with about 44 rounding
      // steps per term in each double sum, var stays within ~132 (K + 1)
      // 2^-53 (relative; 2^-31 at K = 16384) of its exact value and mu
      // within 2^-40 standard deviations, far inside one fp32 ulp of r.
      double sh = 0.0, q = 0.0;
#pragma unroll
      for (int i = 0; i < kVPT; ++i)
        shifted_sums_vec<T>(cur[i], c_cur, tid + (int64_t)i * blockDim.x < nvec, sh, q);
      block_sum_d2(sh, q, red_sq[slot], lane, warp, nwarps);
      const double m1 = div_by_count(sh, K);
      ms = fmax(__fma_rn(-m1, m1, div_by_count(q, K)), 0.0);
      muf = __double2float_rn(__dadd_rn(c_cur, m1));
      c_cur = c_nxt;
    } else {
      double part[kVPT];
#pragma unroll
      for (int i = 0; i < kVPT; ++i) part[i] = sumsq_vec<T>(cur[i]);
#pragma unroll
      for (int w = kVPT / 2; w > 0; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) part[i] = __dadd_rn(part[i], part[i + w]);
      ms = div_by_count(block_sum_d(part[0], red_ss[slot], lane, warp, nwarps), K);
    }
    const float rt = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(ms, (double)eps))));
    // v for values e, e+1 of vector i: (x * r) * gs, or for LayerNorm
    // fma((x - mu) * r, gs, bs), the affine step rounded once
    auto value2 = [&](const float (&f)[V], int i, int e) -> float2 {
      if constexpr (kLN) {
        const float2 n = fmul2_rn(fsub2_rn(make_float2(f[e], f[e + 1]), make_float2(muf, muf)), make_float2(rt, rt));
        return ffma2_rn(n, make_float2(g[i][e], g[i][e + 1]), make_float2(b[i][e], b[i][e + 1]));
      } else {
        return fmul2_rn(fmul2_rn(make_float2(f[e], f[e + 1]), make_float2(rt, rt)), make_float2(g[i][e], g[i][e + 1]));
      }
    };
    // absmax of v (lanes past the row end hold x = gs = bs = 0 and give
    // v = 0, or -muf * r * 0 = +-0)
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < kVPT; ++i) {
      float f[V];
      Vec<T>::to_f32(cur[i], f);
#pragma unroll
      for (int e = 0; e < V; e += 2) {
        const float2 p = value2(f, i, e);
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
          const float2 p = value2(f, i, e);
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

template <typename T, bool kLN>
cudaError_t norm_quant_t(const void *x, int64_t rows, int64_t cols, int64_t ld, const float *gs, const float *bs,
                         float eps, int8_t *q, float *row_scale_out, cudaStream_t st) {
  constexpr int V = Vec<T>::N;
  const int64_t nvec = cols / V;
  if (nvec > 4 * kRowMaxThreads) return cudaErrorNotSupported;
  // (two vectors per thread, for twice the resident warps, measured slower)
  const int vpt = nvec <= 4 * 32 ? 1 : 4;
  int64_t t = (nvec + vpt - 1) / vpt;
  const int threads = (int)std::max<int64_t>(32, ((t + 31) / 32) * 32);
  auto kern = vpt == 1 ? norm_quant_rows_kernel<T, 1, kLN> : norm_quant_rows_kernel<T, 4, kLN>;
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0);
  if (e != cudaSuccess) return e;
  const int64_t grid = std::min<int64_t>(rows, (int64_t)std::max(1, per_sm) * num_sms());
  return launch_pdl(kern, dim3((unsigned)grid), dim3(threads), 0, st, 1, (const T *)x, rows, nvec, ld, gs, bs, eps,
                    q, row_scale_out);
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
    case SQ_F32: return norm_quant_t<float, false>(x, rows, cols, ld, gs, nullptr, eps, q, row_scale_out, st);
    case SQ_F16: return norm_quant_t<__half, false>(x, rows, cols, ld, gs, nullptr, eps, q, row_scale_out, st);
    default: return norm_quant_t<__nv_bfloat16, false>(x, rows, cols, ld, gs, nullptr, eps, q, row_scale_out, st);
  }
}

cudaError_t launch_layernorm_quant(const void *x, sq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                                   const float *gs, const float *bs, float eps, int8_t *q, float *row_scale_out,
                                   cudaStream_t st) {
  switch (xt) {
    case SQ_F32: return norm_quant_t<float, true>(x, rows, cols, ld, gs, bs, eps, q, row_scale_out, st);
    case SQ_F16: return norm_quant_t<__half, true>(x, rows, cols, ld, gs, bs, eps, q, row_scale_out, st);
    default: return norm_quant_t<__nv_bfloat16, true>(x, rows, cols, ld, gs, bs, eps, q, row_scale_out, st);
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

// ---------------------------------------------------------------------------
// Butterfly rotation before quantization ("ButterflyQuant", lifetechia.com:
// Givens rotations arranged as an FFT butterfly).  Each row v = x * col_scale
// is rotated block by block (blocks of n = 2^L channels); stage i pairs
// positions p and p + 2^i (bit i of p clear), pair j = ((p >> (i+1)) << i) |
// (p mod 2^i), and maps (a, b) to (c a - s b, s a + c b) with (c, s) =
// cs[i][j].  Then per-row INT8 as quant_rows_kernel.
// A warp holds 32 consecutive 16-byte vectors (32 V channels, aligned), so a
// block of n <= 32 V channels lives in one warp, and a lane's channel
// positions within its block are the same for every vector it holds and
// every row.  The CTA therefore lays the table out once per lane:
//   strides below V (both values in one thread), per pair k of the vector:
//     tin[i][k][lane] = (c, s, -s, c)  ->  (a', b') = (c a, s a) + (-s b, c b)
//   strides of whole lanes (partner lane ^ (h / V)), per value e:
//     tsh[i][e / 2][lane] = (c_e, c_e+1, s'_e, s'_e+1)  ->  x' = c x + s' y
//     with s' = -s in the pair's first position, +s in its second,
// so a warp reads 512 contiguous bytes per access (no bank conflicts) and
// the arithmetic runs on the packed fp32 pipe: the same products, negations
// (exact) and sums as the definition.
// ---------------------------------------------------------------------------
namespace sq {
namespace {

constexpr int kRotMaxStages = 8;  // n <= 256 in the warp-local kernel
constexpr int kRotSmemThreads = 512;

template <typename T, int kVPT>
__global__ void __launch_bounds__(kRowMaxThreads)
    rot_quant_rows_kernel(const T *__restrict__ x, int64_t rows, int64_t nvec, int64_t ld,
                          const float *__restrict__ col_scale, int logn, const float2 *__restrict__ cs,
                          int8_t *__restrict__ q, float *__restrict__ row_scale_out) {
  constexpr int V = Vec<T>::N;
  constexpr int kLogV = V == 8 ? 3 : 2;
  extern __shared__ float4 rtab[];  // [logn][V / 2][32]
  __shared__ float red[2][kRowMaxThreads / 32];
  const int n = 1 << logn;
  const int half = n >> 1;
  pdl_wait();  // the previous kernel's results are visible from here on
  pdl_trigger();
  // per-lane table: entry (st, k, l) for k < V / 2
  for (int idx = threadIdx.x; idx < logn * (V / 2) * 32; idx += blockDim.x) {
    const int l = idx & 31, k = (idx >> 5) % (V / 2), st = idx / (32 * (V / 2));
    const int h = 1 << st;
    const int base = (l * V) & (n - 1);  // this lane's first position in its block
    float4 t;
    if (h < V) {
      // k-th pair of the vector at this stride: lower element e
      const int e = ((k / h) * 2 * h) + (k % h);
      const int p = (base + e) & (n - 1);
      const float2 c = (st < logn) ? cs[st * half + (((p >> (st + 1)) << st) | (p & (h - 1)))] : make_float2(1, 0);
      t = make_float4(c.x, c.y, -c.y, c.x);
    } else {
      float cc[2], ss[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int p = base + 2 * k + u;
        const bool first = (p & h) == 0;
        const int pa = first ? p : p - h;
        const float2 c = cs[st * half + (((pa >> (st + 1)) << st) | (pa & (h - 1)))];
        cc[u] = c.x;
        ss[u] = first ? -c.y : c.y;
      }
      t = make_float4(cc[0], cc[1], ss[0], ss[1]);
    }
    rtab[idx] = t;
  }
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  const int64_t K = nvec * V;
  float sc[kVPT][V];
#pragma unroll
  for (int i = 0; i < kVPT; ++i) {
    const int64_t v = tid + (int64_t)i * blockDim.x;
#pragma unroll
    for (int e = 0; e < V; ++e) sc[i][e] = v < nvec ? __ldg(col_scale + v * V + e) : 0.0f;
  }
  __syncthreads();
  const uint64_t policy = policy_evict_first();
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
    float val[kVPT][V];
#pragma unroll
    for (int i = 0; i < kVPT; ++i) {
      float f[V];
      Vec<T>::to_f32(cur[i], f);
#pragma unroll
      for (int e = 0; e < V; e += 2) {
        const float2 p = fmul2_rn(make_float2(f[e], f[e + 1]), make_float2(sc[i][e], sc[i][e + 1]));
        val[i][e] = p.x;
        val[i][e + 1] = p.y;
      }
    }
    // strides below V: both values of a pair in this thread
#pragma unroll
    for (int st = 0; st < kLogV; ++st) {
      if (st < logn) {
        constexpr int kPairs = V / 2;
#pragma unroll
        for (int k = 0; k < kPairs; ++k) {
          const int h = 1 << st;
          const int e = ((k / h) * 2 * h) + (k % h);
          const float4 t = rtab[(st * kPairs + k) * 32 + lane];
#pragma unroll
          for (int i = 0; i < kVPT; ++i) {
            const float a = val[i][e], b = val[i][e + h];
            const float2 p1 = fmul2_rn(make_float2(a, a), make_float2(t.x, t.y));  // (c a, s a)
            const float2 p2 = fmul2_rn(make_float2(b, b), make_float2(t.z, t.w));  // (-s b, c b)
            val[i][e] = __fadd_rn(p1.x, p2.x);
            val[i][e + h] = __fadd_rn(p1.y, p2.y);
          }
        }
      }
    }
    // strides of whole lanes: every lane takes part in every shuffle
#pragma unroll
    for (int st = kLogV; st < kLogV + 5 && st < kRotMaxStages; ++st) {
      if (st < logn) {
        const int lm = (1 << st) / V;
#pragma unroll
        for (int e = 0; e < V; e += 2) {
          const float4 t = rtab[(st * (V / 2) + e / 2) * 32 + lane];
#pragma unroll
          for (int i = 0; i < kVPT; ++i) {
            const float y0 = __shfl_xor_sync(0xffffffffu, val[i][e], lm);
            const float y1 = __shfl_xor_sync(0xffffffffu, val[i][e + 1], lm);
            const float2 cx = fmul2_rn(make_float2(val[i][e], val[i][e + 1]), make_float2(t.x, t.y));
            const float2 sy = fmul2_rn(make_float2(y0, y1), make_float2(t.z, t.w));
            val[i][e] = __fadd_rn(cx.x, sy.x);
            val[i][e + 1] = __fadd_rn(cx.y, sy.y);
          }
        }
      }
    }
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < kVPT; ++i)
#pragma unroll
      for (int e = 0; e < V; e += 2) m = fmax3(m, fabsf(val[i][e]), fabsf(val[i][e + 1]));
    m = warp_max(m);
    if (lane == 0) red[slot][warp] = m;
    __syncthreads();
    m = 0.0f;
    for (int w = 0; w < nwarps; ++w) m = fmaxf(m, red[slot][w]);
    slot ^= 1;
    const float delta = __fdiv_rn(m, 127.0f);
    const float rcp = m > 0.0f ? __frcp_rn(delta) : 0.0f;
    if (tid == 0) row_scale_out[r] = delta;
    int8_t *qrow = q + r * K;
#pragma unroll
    for (int i = 0; i < kVPT; ++i) {
      const int64_t v = tid + (int64_t)i * blockDim.x;
      if (v < nvec) {
        if constexpr (V == 8) {
          *reinterpret_cast<uint2 *>(qrow + v * V) = codes8(val[i], delta, rcp);
        } else {
          *reinterpret_cast<uint32_t *>(qrow + v * V) = codes4(val[i], delta, rcp);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kVPT; ++i) cur[i] = nxt[i];
  }
}

// Blocks wider than a warp's 32 V channels: R rows (R <= 4) are staged in
// shared memory as fp32, and the stages run in radix-8 passes.  A pass
// takes stages i0, i0+1 and i0+2 at once on groups of 8 values at positions
// p0 + k 2^i0 (k < 8; p0 with bits i0..i0+2 clear): each thread loads a
// group, applies the three stages in registers -- stage i0+s pairs k and
// k + 2^s -- and stores it back, so a pass costs one barrier and one
// shared-memory round trip for three stages.  The first pass (stages 0-2,
// 8 contiguous values) runs as the rows are loaded.  The group's angles,
// cs[i][j] with j = ((p >> (i+1)) << i) | (p mod 2^i) for the pair's first
// position p, are read once for all R rows.  Shared-memory slots are padded
// by one word per 32 (slot p + p / 32), which spreads the stride-8 accesses
// of the first pass over all 32 banks; the 2^3-stride pass takes its groups
// in a permuted order for the same effect.  Persistent over groups of R rows;
// the codes follow as in the other row quantizers.
__device__ __forceinline__ int rot_slot(int p) { return p + (p >> 5); }

// Angles of r stages starting at i0 for the group whose first value sits at
// block position pb (bits i0..i0+r-1 clear): t[s][m] for pair m of stage
// i = i0 + s.  Pair m's first position is pb + k 2^i0 with k = m with a
// zero bit inserted at s; dropping bit i of it gives j = jb + m 2^i0, where
// jb drops bit i of pb.
template <int r>
__device__ __forceinline__ void group_angles(const float2 *__restrict__ cs, int half, int i0, int pb,
                                             float2 (&t)[r][1 << (r - 1)]) {
#pragma unroll
  for (int s = 0; s < r; ++s) {
    const int i = i0 + s;
    const float2 *row = cs + (int64_t)i * half + (((pb >> (i + 1)) << i) | (pb & ((1 << i) - 1)));
#pragma unroll
    for (int m = 0; m < (1 << (r - 1)); ++m) t[s][m] = __ldg(row + (m << i0));
  }
}

// r stages on the 2^r values of a group: (a, b) -> (c a - s b, s a + c b),
// every product and sum rounded as the definition states.  With t = (c, s)
// and ts = (s, c): (a, b) * t = (c a, s b) and (a, b) * ts = (s a, c b), so
// a butterfly is two packed products and two scalar sums.
template <int r>
__device__ __forceinline__ void group_stages(float (&v)[1 << r], const float2 (&t)[r][1 << (r - 1)],
                                             const float2 (&ts)[r][1 << (r - 1)]) {
#pragma unroll
  for (int s = 0; s < r; ++s) {
#pragma unroll
    for (int m = 0; m < (1 << (r - 1)); ++m) {
      const int k = ((m >> s) << (s + 1)) | (m & ((1 << s) - 1));
      const float2 ab = make_float2(v[k], v[k + (1 << s)]);
      const float2 p = fmul2_rn(ab, t[s][m]);   // (c a, s b)
      const float2 q = fmul2_rn(ab, ts[s][m]);  // (s a, c b)
      v[k] = __fsub_rn(p.x, p.y);
      v[k + (1 << s)] = __fadd_rn(q.x, q.y);
    }
  }
}

template <int r>
__device__ __forceinline__ void swap_angles(const float2 (&t)[r][1 << (r - 1)], float2 (&ts)[r][1 << (r - 1)]) {
#pragma unroll
  for (int s = 0; s < r; ++s)
#pragma unroll
    for (int m = 0; m < (1 << (r - 1)); ++m) ts[s][m] = make_float2(t[s][m].y, t[s][m].x);
}

// One pass of r stages from i0 over nr staged rows of K values.  For
// i0 >= 5 the group's slots are evenly spaced, slot(p0) + k (2^i0 +
// 2^(i0-5)); i0 = 3 takes the slot of each position.  The last pass also
// returns each row's largest magnitude over this thread's groups (mx).
template <int r, bool kLast>
__device__ __forceinline__ void rot_pass(float *rowbuf, int Kp, int nr, int K, int n, int i0,
                                         const float2 *__restrict__ cs, float (&mx)[4]) {
  const int half = n >> 1;
  const int step = i0 >= 5 ? (1 << i0) + (1 << (i0 - 5)) : 0;
  // The 2^3-stride pass with groups in order would put lanes 8 apart on the
  // same banks.  For loop index idx, taking the group gi = b + 8 a with
  // b = idx & 7, h = idx >> 5 and a = 16 (h >> 2) + 4 ((idx >> 3) & 3) +
  // (h & 3) gives a warp's lanes a values 4 apart: slot banks b + 2a + 8k
  // then differ across all 32 lanes.  A bijection of [0, K/8) when K/8 is a
  // multiple of 128.
  const bool permute = i0 == 3 && r == 3 && ((K >> 3) & 127) == 0;
  for (int idx = threadIdx.x; idx < (K >> r); idx += blockDim.x) {
    int gi = idx;
    if (permute) {
      const int h = idx >> 5;
      gi = (idx & 7) | ((((h >> 2) << 4) | (((idx >> 3) & 3) << 2) | (h & 3)) << 3);
    }
    const int p0 = ((gi >> i0) << (i0 + r)) | (gi & ((1 << i0) - 1));
    float2 t[r][1 << (r - 1)], ts[r][1 << (r - 1)];
    group_angles<r>(cs, half, i0, p0 & (n - 1), t);
    swap_angles<r>(t, ts);
    int slot[1 << r];
#pragma unroll
    for (int k = 0; k < (1 << r); ++k) slot[k] = step ? rot_slot(p0) + k * step : rot_slot(p0 + (k << i0));
#pragma unroll
    for (int u = 0; u < 4; ++u) {  // nr <= 4 rows; unrolled so that mx[u] stays in registers
      if (u >= nr) break;
      float *buf = rowbuf + u * Kp;
      float v[1 << r];
#pragma unroll
      for (int k = 0; k < (1 << r); ++k) v[k] = buf[slot[k]];
      group_stages<r>(v, t, ts);
#pragma unroll
      for (int k = 0; k < (1 << r); ++k) buf[slot[k]] = v[k];
      if constexpr (kLast) {
#pragma unroll
        for (int k = 0; k < (1 << r); k += 2) mx[u] = fmax3(mx[u], fabsf(v[k]), fabsf(v[k + 1]));
      }
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kRotSmemThreads, 2)
    rot_quant_rows_smem_kernel(const T *__restrict__ x, int64_t rows, int64_t nvec, int64_t ld,
                               const float *__restrict__ col_scale, int logn, const float2 *__restrict__ cs, int R,
                               int8_t *__restrict__ q, float *__restrict__ row_scale_out) {
  extern __shared__ float rowbuf[];  // [R][Kp]: value p of row u in slot u * Kp + rot_slot(p)
  __shared__ float red[32];
  constexpr int V = Vec<T>::N;
  constexpr int kVecs = 8 / V;  // 16-byte vectors per group of 8 values
  pdl_wait();  // the previous kernel's results are visible from here on
  pdl_trigger();
  const int K = (int)(nvec * V);  // <= 16384, a multiple of n >= 512
  const int Kp = rot_slot(K);
  const int n = 1 << logn;
  const int64_t groups = (rows + R - 1) / R;
  for (int64_t g = blockIdx.x; g < groups; g += gridDim.x) {
    const int64_t r0 = g * R;
    const int nr = (int)min((int64_t)R, rows - r0);
    // load, scale and stages 0-2 on groups of 8 contiguous values
    for (int gi = threadIdx.x; gi < (K >> 3); gi += blockDim.x) {
      const int p0 = gi << 3;
      float2 t[3][4], ts[3][4];
      group_angles<3>(cs, n >> 1, 0, p0 & (n - 1), t);
      swap_angles<3>(t, ts);
      float sc[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) sc[k] = __ldg(col_scale + p0 + k);
      for (int u = 0; u < nr; ++u) {
        const T *xr = x + (r0 + u) * ld + p0;
        float v[8];
#pragma unroll
        for (int w = 0; w < kVecs; ++w) {
          float f[V];
          Vec<T>::to_f32(ld_nc_v4(xr + w * V), f);
#pragma unroll
          for (int e = 0; e < V; ++e) v[w * V + e] = __fmul_rn(f[e], sc[w * V + e]);
        }
        group_stages<3>(v, t, ts);
        float *buf = rowbuf + u * Kp;
#pragma unroll
        for (int k = 0; k < 8; ++k) buf[rot_slot(p0 + k)] = v[k];
      }
    }
    __syncthreads();
    float mx[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // per staged row (R <= 4)
    for (int i0 = 3; i0 < logn; i0 += 3) {
      const int left = logn - i0;
      if (left > 3) {
        rot_pass<3, false>(rowbuf, Kp, nr, K, n, i0, cs, mx);
      } else if (left == 3) {
        rot_pass<3, true>(rowbuf, Kp, nr, K, n, i0, cs, mx);
      } else if (left == 2) {
        rot_pass<2, true>(rowbuf, Kp, nr, K, n, i0, cs, mx);
      } else {
        rot_pass<1, true>(rowbuf, Kp, nr, K, n, i0, cs, mx);
      }
      __syncthreads();
    }
    for (int u = 0; u < nr; ++u) {
      const float *buf = rowbuf + u * Kp;
      float m = 0.0f;
#pragma unroll
      for (int w = 0; w < 4; ++w) m = w == u ? mx[w] : m;  // mx[u] without a runtime index
      m = block_max(m, red);
      const float delta = __fdiv_rn(m, 127.0f);
      const float rcp = m > 0.0f ? __frcp_rn(delta) : 0.0f;
      if (threadIdx.x == 0) row_scale_out[r0 + u] = delta;
      int8_t *qrow = q + (r0 + u) * K;
      for (int v = threadIdx.x; v < (int)nvec; v += blockDim.x) {
        float val[V];
#pragma unroll
        for (int e = 0; e < V; ++e) val[e] = buf[rot_slot(v * V + e)];
        if constexpr (V == 8) {
          *reinterpret_cast<uint2 *>(qrow + v * V) = codes8(val, delta, rcp);
        } else {
          *reinterpret_cast<uint32_t *>(qrow + v * V) = codes4(val, delta, rcp);
        }
      }
    }
    __syncthreads();  // the buffers are reused by the next group
  }
}

template <typename T>
cudaError_t rot_quant_t(const void *x, int64_t rows, int64_t cols, int64_t ld, const float *col_scale, int logn,
                        const float *cs, int8_t *q, float *row_scale_out, cudaStream_t st) {
  constexpr int V = Vec<T>::N;
  const int64_t nvec = cols / V;
  if (nvec > 4 * kRowMaxThreads) return cudaErrorNotSupported;
  if ((1 << logn) > 32 * V) {  // blocks wider than a warp: the shared-memory kernel
    const size_t row_bytes = (size_t)(cols + cols / 32) * sizeof(float);  // padded slots
    const int R = (int)std::max<size_t>(1, std::min<size_t>(4, (200 * 1024) / row_bytes));
    const size_t smem = R * row_bytes;
    if (smem > 200 * 1024) return cudaErrorNotSupported;
    auto kern = rot_quant_rows_smem_kernel<T>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kRotSmemThreads, smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = std::min<int64_t>(rows, (int64_t)std::max(1, per_sm) * num_sms());
    const int64_t groups = (rows + R - 1) / R;
    return launch_pdl(kern, dim3((unsigned)std::min<int64_t>(grid, groups)), dim3(kRotSmemThreads), smem, st, 1,
                      (const T *)x, rows, nvec, ld, col_scale, logn, reinterpret_cast<const float2 *>(cs), R, q,
                      row_scale_out);
  }
  const int vpt = nvec <= 4 * 32 ? 1 : 4;
  const int64_t t = (nvec + vpt - 1) / vpt;
  const int threads = (int)std::max<int64_t>(32, ((t + 31) / 32) * 32);
  auto kern = vpt == 1 ? rot_quant_rows_kernel<T, 1> : rot_quant_rows_kernel<T, 4>;
  const size_t smem = (size_t)logn * (V / 2) * 32 * sizeof(float4);
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = std::min<int64_t>(rows, (int64_t)std::max(1, per_sm) * num_sms());
  return launch_pdl(kern, dim3((unsigned)grid), dim3(threads), smem, st, 1, (const T *)x, rows, nvec, ld, col_scale,
                    logn, reinterpret_cast<const float2 *>(cs), q, row_scale_out);
}

}  // namespace

cudaError_t launch_rot_quant_rows(const void *x, sq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                                  const float *col_scale, int logn, const float *cs, int8_t *q, float *row_scale_out,
                                  cudaStream_t st) {
  switch (xt) {
    case SQ_F32: return rot_quant_t<float>(x, rows, cols, ld, col_scale, logn, cs, q, row_scale_out, st);
    case SQ_F16: return rot_quant_t<__half>(x, rows, cols, ld, col_scale, logn, cs, q, row_scale_out, st);
    default: return rot_quant_t<__nv_bfloat16>(x, rows, cols, ld, col_scale, logn, cs, q, row_scale_out, st);
  }
}
}  // namespace sq
