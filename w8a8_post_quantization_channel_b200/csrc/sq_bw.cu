// sq_bw.cu -- the bandwidth-bound steps of the SmoothQuant path (sm_100a).
//
//   calibration maxima  max_t |X_tj|              ("Hyper-parameter alpha":
//   weight maxima       max_n |W_jn|               the max|X_j|, max|W_j|)
//   smoothing factor    s_j = a_j^alpha / w_j^(1-alpha), 1/s_j
//   row quantizer       per-token X~ = X / s and per-output-row W~ = s W
//   column quantizer    per-output-channel W~ for W stored [K][N]
// ("SmoothQuant (activation smoothing quantization)", jisaku.com glossary).
//
// Every kernel reads its input once with 16-byte vector loads, keeps
// per-thread partial maxima in registers and merges them with warp
// shuffles; results are independent of the launch shape (max is exact).
#include <algorithm>
#include <type_traits>

#include "sq_common.cuh"
#include "sq_internal.h"

namespace sq {

namespace {

constexpr int kColThreadsX = 32;  // 16-byte column vectors per CTA slab
constexpr int kColThreadsY = 8;   // row lanes per CTA
constexpr int kColUnroll = 8;     // independent row loads in flight per thread

// amax[c] = max(amax[c], max_r |v_rc|), v_rc = x[r][c] (* row_scale[r]).
// CTA (32 x 8): threadIdx.x picks a 16-byte column vector of a 32-vector
// slab, threadIdx.y a row lane; blockIdx.y splits the rows into chunks.
template <typename T, bool kScaled>
__global__ void __launch_bounds__(kColThreadsX *kColThreadsY)
    absmax_cols_kernel(const T *__restrict__ x, int64_t rows, int64_t nvec, int64_t ld,
                       const float *__restrict__ row_scale, float *__restrict__ amax, bool keep_in_l2) {
  pdl_wait();  // the previous kernel's results are visible from here on
  pdl_trigger();
  constexpr int V = Vec<T>::N;
  __shared__ float red[kColThreadsY][kColThreadsX * V];
  // data read again right after this kernel (the weights) is kept in L2,
  // read-once data (a calibration stream) is marked first to go
  const uint64_t policy = keep_in_l2 ? policy_evict_last() : policy_evict_first();
  const int64_t v = (int64_t)blockIdx.x * kColThreadsX + threadIdx.x;
  const int64_t chunk = (rows + gridDim.y - 1) / gridDim.y;
  const int64_t r0 = (int64_t)blockIdx.y * chunk;
  const int64_t r1 = min(rows, r0 + chunk);
  float m[V];
#pragma unroll
  for (int e = 0; e < V; ++e) m[e] = 0.0f;
  if (v < nvec) {
    const T *col = x + v * V;
    int64_t r = r0 + threadIdx.y;
    for (; r + (kColUnroll - 1) * kColThreadsY < r1; r += kColUnroll * kColThreadsY) {
      uint4 raw[kColUnroll];
#pragma unroll
      for (int u = 0; u < kColUnroll; ++u) raw[u] = ld_policy_v4(col + (r + u * kColThreadsY) * ld, policy);
#pragma unroll
      for (int u = 0; u < kColUnroll; u += 2) {
        float f0[V], f1[V];
        Vec<T>::to_f32(raw[u], f0);
        Vec<T>::to_f32(raw[u + 1], f1);
        const float s0 = kScaled ? __ldg(row_scale + r + u * kColThreadsY) : 1.0f;
        const float s1 = kScaled ? __ldg(row_scale + r + (u + 1) * kColThreadsY) : 1.0f;
#pragma unroll
        for (int e = 0; e < V; ++e)
          m[e] = fmax3(m[e], fabsf(kScaled ? __fmul_rn(s0, f0[e]) : f0[e]), fabsf(kScaled ? __fmul_rn(s1, f1[e]) : f1[e]));
      }
    }
    for (; r < r1; r += kColThreadsY) {
      float f[V];
      Vec<T>::to_f32(ld_policy_v4(col + r * ld, policy), f);
      const float sc = kScaled ? __ldg(row_scale + r) : 1.0f;
#pragma unroll
      for (int e = 0; e < V; ++e) m[e] = fmaxf(m[e], fabsf(kScaled ? __fmul_rn(sc, f[e]) : f[e]));
    }
  }
#pragma unroll
  for (int e = 0; e < V; ++e) red[threadIdx.y][threadIdx.x * V + e] = m[e];
  __syncthreads();
  // Threads of row lane 0 fold the 8 lanes and publish with an integer
  // atomicMax: for non-negative floats the bit patterns order as integers.
  if (threadIdx.y == 0 && v < nvec) {
#pragma unroll
    for (int e = 0; e < V; ++e) {
      float mm = red[0][threadIdx.x * V + e];
#pragma unroll
      for (int y = 1; y < kColThreadsY; ++y) mm = fmaxf(mm, red[y][threadIdx.x * V + e]);
      atomicMax(reinterpret_cast<int *>(amax + v * V + e), __float_as_int(mm));
    }
  }
}

// out[r] = max_c |x[r][c]|, one CTA per row.
template <typename T>
__global__ void __launch_bounds__(256) absmax_rows_kernel(const T *__restrict__ x, int64_t nvec, int64_t ld,
                                                          float *__restrict__ out) {
  pdl_wait();  // the previous kernel's results are visible from here on
  pdl_trigger();
  constexpr int V = Vec<T>::N;
  __shared__ float red[32];
  const T *row = x + (int64_t)blockIdx.x * ld;
  float m = 0.0f;
  for (int64_t v = threadIdx.x; v < nvec; v += blockDim.x) {
    float f[V];
    Vec<T>::to_f32(ld_stream_v4(row + v * V), f);
#pragma unroll
    for (int e = 0; e < V; e += 2) m = fmax3(m, fabsf(f[e]), fabsf(f[e + 1]));
  }
  m = block_max(m, red);
  if (threadIdx.x == 0) out[blockIdx.x] = m;
}

// s_j = a^alpha / w^(1-alpha) with a, w floored at 1e-5; IEEE sqrt for the
// quarter-step alphas, double pow (rounded once) otherwise.
__global__ void smooth_factor_kernel(const float *__restrict__ amax, float *__restrict__ s_inout,
                                     float *__restrict__ inv_s, int64_t K, float alpha) {
  pdl_wait();  // the previous kernel's results are visible from here on
  pdl_trigger();
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= K) return;
  const float a = fmaxf(amax[j], 1e-5f);
  const float w = fmaxf(s_inout[j], 1e-5f);
  float s;
  if (alpha == 1.0f) {
    s = a;
  } else if (alpha == 0.0f) {
    s = __fdiv_rn(1.0f, w);
  } else if (alpha == 0.5f) {
    s = __fdiv_rn(__fsqrt_rn(a), __fsqrt_rn(w));
  } else if (alpha == 0.25f) {
    const float a14 = __fsqrt_rn(__fsqrt_rn(a));
    const float w34 = __fmul_rn(__fsqrt_rn(w), __fsqrt_rn(__fsqrt_rn(w)));
    s = __fdiv_rn(a14, w34);
  } else if (alpha == 0.75f) {
    const float a34 = __fmul_rn(__fsqrt_rn(a), __fsqrt_rn(__fsqrt_rn(a)));
    const float w14 = __fsqrt_rn(__fsqrt_rn(w));
    s = __fdiv_rn(a34, w14);
  } else {
    const double num = pow((double)a, (double)alpha);
    const double den = pow((double)w, 1.0 - (double)alpha);
    s = __double2float_rn(__ddiv_rn(num, den));
  }
  s_inout[j] = s;
  inv_s[j] = __fdiv_rn(1.0f, s);
}

// Row quantizer (persistent): each CTA walks rows r = blockIdx.x,
// blockIdx.x + gridDim.x, ...; per row
//   v_c = x[r][c] * col_scale[c];  m = max_c |v_c|;
//   row_scale_out[r] = delta = m / Q;  q[r][c] = code(v_c / delta),
// Q = F::kMax (127 for INT8 codes, 448 for E4M3).
// Thread t owns the 16-byte vectors t + i*blockDim (i < kVPT) of every row:
// their column scales stay in registers for the CTA's lifetime, the next
// row's vectors are loaded before the current row is reduced, and the row
// maximum needs one barrier (two alternating reduction slots).
constexpr int kRowMaxThreads = 512;
template <typename T, int kVPT, typename F>
__global__ void __launch_bounds__(kRowMaxThreads)
    quant_rows_kernel(const T *__restrict__ x, int64_t rows, int64_t nvec, int64_t ld,
                      const float *__restrict__ col_scale, int8_t *__restrict__ q, float *__restrict__ row_scale_out) {
  pdl_wait();  // the previous kernel's results are visible from here on
  pdl_trigger();
  constexpr int V = Vec<T>::N;
  __shared__ float red[2][kRowMaxThreads / 32];
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
  const uint64_t policy = policy_evict_first();  // every row is read exactly once
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
    float m = 0.0f;
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
#pragma unroll
      for (int e = 0; e < V; e += 2) m = fmax3(m, fabsf(val[i][e]), fabsf(val[i][e + 1]));
    }
    m = warp_max(m);
    if (lane == 0) red[slot][warp] = m;
    __syncthreads();
    m = 0.0f;
    for (int w = 0; w < nwarps; ++w) m = fmaxf(m, red[slot][w]);
    slot ^= 1;
    // m == 0 (all-zero row): rcp = 0 gives codes 0 and scale 0
    // scale delta = m / Q; codes of fl(v / delta) (rcp = 0 for a zero row)
    const float delta = __fdiv_rn(m, F::kMax);
    const float rcp = m > 0.0f ? __frcp_rn(delta) : 0.0f;
    if (tid == 0) row_scale_out[r] = delta;
    int8_t *qrow = q + r * K;
#pragma unroll
    for (int i = 0; i < kVPT; ++i) {
      const int64_t v = tid + (int64_t)i * blockDim.x;
      if (v < nvec) {
        if constexpr (V == 8) {
          *reinterpret_cast<uint2 *>(qrow + v * V) = F::codes8(val[i], delta, rcp);
        } else {
          *reinterpret_cast<uint32_t *>(qrow + v * V) = F::codes4(val[i], delta, rcp);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kVPT; ++i) cur[i] = nxt[i];
  }
}

// The same row quantizer with its row loads staged in shared memory: each
// thread copies its own 16-byte vectors of the next D rows with cp.async
// (no registers held for them), so a CTA keeps D + 1 rows in flight; the
// copies are the thread's own, so reading them back needs no barrier.
// With eight vectors a thread holds 64 values and their column scales, so
// that form is launched with at most 256 threads (registers up to 255).
constexpr int kRowAsync8Threads = 256;
template <typename T, int kVPT, int D, typename F>
__global__ void __launch_bounds__(kVPT == 8 ? kRowAsync8Threads : kRowMaxThreads)
    quant_rows_async_kernel(const T *__restrict__ x, int64_t rows, int64_t nvec, int64_t ld,
                            const float *__restrict__ col_scale, int8_t *__restrict__ q,
                            float *__restrict__ row_scale_out) {
  pdl_wait();  // the previous kernel's results are visible from here on
  pdl_trigger();
  constexpr int V = Vec<T>::N;
  extern __shared__ uint4 stage[];  // [D][kVPT][blockDim]
  __shared__ float red[2][kRowMaxThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5, nt = blockDim.x;
  const int64_t K = nvec * V;

  float sc[kVPT][V];
#pragma unroll
  for (int i = 0; i < kVPT; ++i) {
    const int64_t v = tid + (int64_t)i * nt;
#pragma unroll
    for (int e = 0; e < V; ++e) sc[i][e] = v < nvec ? __ldg(col_scale + v * V + e) : 0.0f;
  }
  const uint64_t policy = policy_evict_first();  // every row is read exactly once
  auto issue = [&](int64_t rr, int slot) {
#pragma unroll
    for (int i = 0; i < kVPT; ++i) {
      const int64_t v = tid + (int64_t)i * nt;
      if (rr < rows && v < nvec) cp_async_16(&stage[(slot * kVPT + i) * nt + tid], x + rr * ld + v * V, policy);
    }
    cp_async_commit();  // one group per row, empty past the last row
  };
  int64_t r = blockIdx.x;
#pragma unroll
  for (int d = 0; d < D; ++d) issue(r + (int64_t)d * gridDim.x, d);
  int slot = 0, rslot = 0;
  for (; r < rows; r += gridDim.x) {
    cp_async_wait<D - 1>();  // this row's copies (the oldest group) have landed
    uint4 cur[kVPT];
#pragma unroll
    for (int i = 0; i < kVPT; ++i) cur[i] = stage[(slot * kVPT + i) * nt + tid];
    issue(r + (int64_t)D * gridDim.x, slot);  // the slot's next row
    slot = slot + 1 == D ? 0 : slot + 1;
    float val[kVPT][V];
    float m = 0.0f;
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
#pragma unroll
      for (int e = 0; e < V; e += 2) m = fmax3(m, fabsf(val[i][e]), fabsf(val[i][e + 1]));
    }
    m = warp_max(m);
    if (lane == 0) red[rslot][warp] = m;
    __syncthreads();
    m = 0.0f;
    for (int w = 0; w < nwarps; ++w) m = fmaxf(m, red[rslot][w]);
    rslot ^= 1;
    // scale delta = m / Q; codes of fl(v / delta) (rcp = 0 for a zero row)
    const float delta = __fdiv_rn(m, F::kMax);
    const float rcp = m > 0.0f ? __frcp_rn(delta) : 0.0f;
    if (tid == 0) row_scale_out[r] = delta;
    int8_t *qrow = q + r * K;
#pragma unroll
    for (int i = 0; i < kVPT; ++i) {
      const int64_t v = tid + (int64_t)i * nt;
      if (v < nvec) {
        if constexpr (V == 8) {
          *reinterpret_cast<uint2 *>(qrow + v * V) = F::codes8(val[i], delta, rcp);
        } else {
          *reinterpret_cast<uint32_t *>(qrow + v * V) = F::codes4(val[i], delta, rcp);
        }
      }
    }
  }
  cp_async_wait<0>();  // no copy may land after the CTA exits
}

// Row quantizer for long rows (persistent, one CTA of 512 threads per SM):
// whole rows are staged in shared memory by bulk async copies into
// kStages buffers (one mbarrier each), issued kStages rows ahead; the
// column scales stay in registers; each row is read from shared memory
// twice (maximum, then codes), so HBM sees every byte once.
constexpr int kSmemRowThreads = 512;
template <typename T, int kVPT, int kStages, typename F>
__global__ void __launch_bounds__(kSmemRowThreads, 1)
    quant_rows_smem_kernel(const T *__restrict__ x, int64_t rows, int64_t nvec, int64_t ld,
                           const float *__restrict__ col_scale, int8_t *__restrict__ q,
                           float *__restrict__ row_scale_out, uint32_t row_bytes, unsigned *err) {
  pdl_wait();  // the previous kernel's results are visible from here on
  pdl_trigger();
  constexpr int V = Vec<T>::N;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const uint32_t buf_bytes = (row_bytes + 127u) & ~127u;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * buf_bytes);
  float *red = reinterpret_cast<float *>(full + kStages);  // [2][16]
  volatile int *abort_flag = reinterpret_cast<volatile int *>(red + 32);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t K = nvec * V;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      const int64_t r = blockIdx.x + (int64_t)s * gridDim.x;
      if (r < rows) {
        mbar_arrive_expect_tx(&full[s], row_bytes);
        bulk_load(smem + s * buf_bytes, x + r * ld, row_bytes, &full[s]);
      }
    }
  }
  float sc[kVPT][V];
#pragma unroll
  for (int i = 0; i < kVPT; ++i) {
    const int64_t v = tid + (int64_t)i * kSmemRowThreads;
#pragma unroll
    for (int e = 0; e < V; ++e) sc[i][e] = v < nvec ? __ldg(col_scale + v * V + e) : 0.0f;
  }
  int slot = 0;
  int64_t it = 0;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x, ++it) {
    const int s = (int)(it % kStages);
    const uint32_t parity = (uint32_t)((it / kStages) & 1);
    const bool ok = mbar_wait(&full[s], parity, abort_flag, err);
    if (!__syncthreads_and(ok)) break;
    const uint4 *row = reinterpret_cast<const uint4 *>(smem + s * buf_bytes);
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < kVPT; ++i) {
      const int64_t v = tid + (int64_t)i * kSmemRowThreads;
      if (v < nvec) {
        float f[V];
        Vec<T>::to_f32(row[v], f);
#pragma unroll
        for (int e = 0; e < V; e += 2) {
          const float2 p = fmul2_rn(make_float2(f[e], f[e + 1]), make_float2(sc[i][e], sc[i][e + 1]));
          m = fmax3(m, fabsf(p.x), fabsf(p.y));
        }
      }
    }
    m = warp_max(m);
    if (lane == 0) red[slot * 16 + warp] = m;
    __syncthreads();
    m = 0.0f;
#pragma unroll
    for (int w = 0; w < kSmemRowThreads / 32; ++w) m = fmaxf(m, red[slot * 16 + w]);
    slot ^= 1;
    // scale delta = m / Q; codes of fl(v / delta) (rcp = 0 for a zero row)
    const float delta = __fdiv_rn(m, F::kMax);
    const float rcp = m > 0.0f ? __frcp_rn(delta) : 0.0f;
    if (tid == 0) row_scale_out[r] = delta;
    int8_t *qrow = q + r * K;
#pragma unroll
    for (int i = 0; i < kVPT; ++i) {
      const int64_t v = tid + (int64_t)i * kSmemRowThreads;
      if (v < nvec) {
        float f[V];
        Vec<T>::to_f32(row[v], f);
        float val[V];
#pragma unroll
        for (int e = 0; e < V; e += 2) {
          const float2 p = fmul2_rn(make_float2(f[e], f[e + 1]), make_float2(sc[i][e], sc[i][e + 1]));
          val[e] = p.x;
          val[e + 1] = p.y;
        }
        if constexpr (V == 8) {
          *reinterpret_cast<uint2 *>(qrow + v * V) = F::codes8(val, delta, rcp);
        } else {
          *reinterpret_cast<uint32_t *>(qrow + v * V) = F::codes4(val, delta, rcp);
        }
      }
    }
    __syncthreads();  // every thread is done with buffer s
    if (tid == 0) {
      const int64_t rn = r + (int64_t)kStages * gridDim.x;
      if (rn < rows) {
        mbar_arrive_expect_tx(&full[s], row_bytes);
        bulk_load(smem + s * buf_bytes, x + rn * ld, row_bytes, &full[s]);
      }
    }
  }
  // on an abort, copies already issued must land before the CTA exits
  if (tid == 0 && *abort_flag) {
    int64_t r = blockIdx.x + it * gridDim.x;
    for (int k = 0; k < kStages && r < rows; ++k, ++it, r += gridDim.x)
      mbar_wait(&full[it % kStages], (uint32_t)((it / kStages) & 1), nullptr, err);
  }
}

// Row quantizer for rows too long to hold in registers: one pass for the
// maximum, a second for the codes (the row is re-read, mostly from L2).
template <typename T, typename F>
__global__ void __launch_bounds__(1024) quant_rows_twopass_kernel(const T *__restrict__ x, int64_t nvec, int64_t ld,
                                                                  const float *__restrict__ col_scale,
                                                                  int8_t *__restrict__ q,
                                                                  float *__restrict__ row_scale_out) {
  pdl_wait();  // the previous kernel's results are visible from here on
  pdl_trigger();
  constexpr int V = Vec<T>::N;
  __shared__ float red[32];
  const int64_t r = blockIdx.x;
  const T *row = x + r * ld;
  const int64_t K = nvec * V;
  float m = 0.0f;
  for (int64_t v = threadIdx.x; v < nvec; v += blockDim.x) {
    float f[V];
    Vec<T>::to_f32(ld_nc_v4(row + v * V), f);
#pragma unroll
    for (int e = 0; e < V; ++e) m = fmaxf(m, fabsf(__fmul_rn(f[e], __ldg(col_scale + v * V + e))));
  }
  m = block_max(m, red);
  const float delta = __fdiv_rn(m, F::kMax);
  const float rcp = m > 0.0f ? __frcp_rn(delta) : 0.0f;
  if (threadIdx.x == 0) row_scale_out[r] = delta;
  int8_t *qrow = q + r * K;
  for (int64_t v = threadIdx.x; v < nvec; v += blockDim.x) {
    float f[V];
    Vec<T>::to_f32(ld_stream_v4(row + v * V), f);
    float val[V];
#pragma unroll
    for (int e = 0; e < V; ++e) val[e] = __fmul_rn(f[e], __ldg(col_scale + v * V + e));
    if constexpr (V == 8) {
      *reinterpret_cast<uint2 *>(qrow + v * V) = F::codes8(val, delta, rcp);
    } else {
      *reinterpret_cast<uint32_t *>(qrow + v * V) = F::codes4(val, delta, rcp);
    }
  }
}

// W[K][N] (row j = input channel) -> Wq[N][K]: a 64 x 64 tile is read with
// row-contiguous loads, quantized with its column's maximum, transposed in
// shared memory and written with row-contiguous stores.
constexpr int kTT = 64;
template <typename T, typename F>
__global__ void __launch_bounds__(256) quant_cols_transpose_kernel(const T *__restrict__ w, int64_t K, int64_t N,
                                                                   int64_t ld, const float *__restrict__ s,
                                                                   const float *__restrict__ colmax,
                                                                   int8_t *__restrict__ wq) {
  pdl_wait();  // the previous kernel's results are visible from here on
  pdl_trigger();
  __shared__ uint8_t tile[kTT][kTT + 4];  // [n][j] codes
  __shared__ float dlt[kTT], rcp[kTT];  // per column: scale, fl(1 / scale)
  const int64_t j0 = (int64_t)blockIdx.y * kTT, n0 = (int64_t)blockIdx.x * kTT;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;  // 16 x 16 threads
  if (threadIdx.x < kTT) {
    const int64_t n = n0 + threadIdx.x;
    const float cm = n < N ? __ldg(colmax + n) : 0.0f;
    // the scale finalize_scale_kernel stores: fl(colmax / Q)
    dlt[threadIdx.x] = __fdiv_rn(cm, F::kMax);
    rcp[threadIdx.x] = cm > 0.0f ? __frcp_rn(dlt[threadIdx.x]) : 0.0f;
  }
  __syncthreads();
  // each thread: 4 consecutive n of one j row, rows ty, ty+16, ...
#pragma unroll
  for (int jj = ty; jj < kTT; jj += 16) {
    const int64_t j = j0 + jj;
    const int64_t n = n0 + tx * 4;
    uint8_t c[4] = {0, 0, 0, 0};
    if (j < K && n < N) {  // N % 16 == 0: a group of 4 is all in or all out
      const float sj = __ldg(s + j);
      const T *p = w + j * ld + n;
#pragma unroll
      for (int e = 0; e < 4; ++e) c[e] = F::code1(__fmul_rn(sj, Vec<T>::one(p + e)), dlt[tx * 4 + e], rcp[tx * 4 + e]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) tile[tx * 4 + e][jj] = c[e];
  }
  __syncthreads();
  // write: row n of the tile, 64 bytes of j; each thread 4 bytes
#pragma unroll
  for (int nn = ty; nn < kTT; nn += 16) {
    const int64_t n = n0 + nn;
    const int64_t j = j0 + tx * 4;
    if (n < N && j < K) {
      const uint32_t packed = (uint32_t)tile[nn][tx * 4 + 0] | ((uint32_t)tile[nn][tx * 4 + 1] << 8) |
                              ((uint32_t)tile[nn][tx * 4 + 2] << 16) | ((uint32_t)tile[nn][tx * 4 + 3] << 24);
      *reinterpret_cast<uint32_t *>(wq + n * K + j) = packed;
    }
  }
}

template <typename F>
__global__ void finalize_scale_kernel(float *__restrict__ m_to_scale, int64_t n) {
  pdl_wait();  // the previous kernel's results are visible from here on
  pdl_trigger();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) m_to_scale[i] = __fdiv_rn(m_to_scale[i], F::kMax);
}

__global__ void zero_fill_kernel(float *__restrict__ p, int64_t n) {
  pdl_wait();  // the previous kernel's results are visible from here on
  pdl_trigger();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    p[i] = 0.0f;
}

// One thread waits on a barrier that nothing arrives at: the bounded wait
// gives up after limit_ns and records the timeout (self-test of the path
// every other kernel takes when a wait runs out).
__global__ void wait_timeout_selftest_kernel(unsigned long long limit_ns, unsigned *err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait(&bar, 0, nullptr, err, limit_ns);
  }
}

template <typename T>
cudaError_t absmax_cols_t(const void *x, int64_t rows, int64_t cols, int64_t ld, const float *row_scale,
                          float *amax, bool keep_in_l2, cudaStream_t st) {
  constexpr int V = Vec<T>::N;
  const int64_t nvec = cols / V;
  const int64_t slabs = (nvec + kColThreadsX - 1) / kColThreadsX;
  const int64_t want = (int64_t)num_sms() * 8;
  int64_t gy = (want + slabs - 1) / slabs;
  const int64_t max_gy = (rows + kColUnroll * kColThreadsY - 1) / (kColUnroll * kColThreadsY);
  gy = std::max<int64_t>(1, std::min<int64_t>(gy, std::min<int64_t>(max_gy, 65535)));
  dim3 grid((unsigned)slabs, (unsigned)gy), block(kColThreadsX, kColThreadsY);
  if (row_scale)
    return launch_pdl(absmax_cols_kernel<T, true>, grid, block, 0, st, 1, (const T *)x, rows, nvec, ld, row_scale,
                      amax, keep_in_l2);
  return launch_pdl(absmax_cols_kernel<T, false>, grid, block, 0, st, 1, (const T *)x, rows, nvec, ld,
                    (const float *)nullptr, amax, keep_in_l2);
}

template <typename T>
cudaError_t absmax_rows_t(const void *x, int64_t rows, int64_t cols, int64_t ld, float *out, cudaStream_t st) {
  constexpr int V = Vec<T>::N;
  return launch_pdl(absmax_rows_kernel<T>, dim3((unsigned)rows), dim3(256), 0, st, 1, (const T *)x, cols / V, ld, out);
}

template <typename T, int kVPT, typename F>
cudaError_t launch_quant_rows_persistent(const T *x, int64_t rows, int64_t nvec, int64_t ld, const float *col_scale,
                                         int8_t *q, float *row_scale_out, int threads, cudaStream_t st) {
  static int per_sm[64][kRowMaxThreads / 32 + 1] = {};  // [device][warps], per instantiation
  int dev = 0;
  cudaGetDevice(&dev);
  int &cached = per_sm[dev & 63][threads / 32];
  if (cached == 0) {
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, quant_rows_kernel<T, kVPT, F>, threads, 0);
    if (e != cudaSuccess) return e;
    cached = n > 0 ? n : 1;
  }
  const int64_t grid = std::min<int64_t>(rows, (int64_t)cached * num_sms());
  return launch_pdl(quant_rows_kernel<T, kVPT, F>, dim3((unsigned)grid), dim3(threads), 0, st, 1, x, rows, nvec, ld,
                    col_scale, q, row_scale_out);
}

// Sets the staged row kernel's shared-memory limit for `threads` and
// returns how many of its CTAs an SM holds (cached per device and warps).
template <typename T, int kVPT, int D, typename F>
cudaError_t quant_rows_async_occupancy(int threads, int *per_sm_out) {
  static int per_sm[64][kRowMaxThreads / 32 + 1] = {};  // [device][warps], per instantiation
  static int attr_bytes[64] = {};
  auto kern = quant_rows_async_kernel<T, kVPT, D, F>;
  const size_t smem = (size_t)D * kVPT * threads * 16;
  int dev = 0;
  cudaGetDevice(&dev);
  if (attr_bytes[dev & 63] < (int)smem) {
    // (the dynamic share plus the kernel's static reduction array may pass
    // the 48 KB available without opting in)
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_bytes[dev & 63] = (int)smem;
  }
  int &cached = per_sm[dev & 63][threads / 32];
  if (cached == 0) {
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem);
    if (e != cudaSuccess) return e;
    cached = n > 0 ? n : 1;
  }
  *per_sm_out = cached;
  return cudaSuccess;
}

template <typename T, int kVPT, int D, typename F>
cudaError_t launch_quant_rows_async(const T *x, int64_t rows, int64_t nvec, int64_t ld, const float *col_scale,
                                    int8_t *q, float *row_scale_out, int threads, cudaStream_t st) {
  int per_sm = 0;
  cudaError_t e = quant_rows_async_occupancy<T, kVPT, D, F>(threads, &per_sm);
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)D * kVPT * threads * 16;
  const int64_t grid = std::min<int64_t>(rows, (int64_t)per_sm * num_sms());
  return launch_pdl(quant_rows_async_kernel<T, kVPT, D, F>, dim3((unsigned)grid), dim3(threads), smem, st, 1, x, rows,
                    nvec, ld, col_scale, q, row_scale_out);
}

template <typename T, int kVPT, int kStages, typename F>
cudaError_t launch_quant_rows_smem(const T *x, int64_t rows, int64_t nvec, int64_t ld, const float *col_scale,
                                   int8_t *q, float *row_scale_out, uint32_t row_bytes, uint32_t smem_bytes,
                                   cudaStream_t st) {
  auto kern = quant_rows_smem_kernel<T, kVPT, kStages, F>;
  static int attr_bytes[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (attr_bytes[dev & 63] < (int)smem_bytes) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes);
    if (e != cudaSuccess) return e;
    attr_bytes[dev & 63] = (int)smem_bytes;
  }
  const int64_t grid = std::min<int64_t>(rows, (int64_t)num_sms());
  return launch_pdl(kern, dim3((unsigned)grid), dim3(kSmemRowThreads), smem_bytes, st, 1, x, rows, nvec, ld, col_scale,
                    q, row_scale_out, row_bytes, device_error_word());
}

// Which of the two register-row quantizers serves rows of 129..2048 16-byte
// vectors.  Long batches (8192 rows or more) stream best with the next three
// rows staged by cp.async (measured on 16384-token batches: 0.81 against
// 0.77 of HBM at K = 4096, 0.75 against 0.70 at K = 7168); shorter ones with
// the next row in registers, whose smaller shared-memory share lets the
// neighbouring kernels overlap it (at 2048 tokens: 8.0 against 9.1 us), but
// only while rows are short: 16-bit rows of 7168 values or more stage better
// from 2048 rows up (2048 x 11008: 18.2 against 20.5 us; 6144 x 7168: 28.9
// against 31.9; 4096 x 16384: 45.1 against 46.2).
inline bool quant_rows_async_enabled(int64_t rows, int64_t cols, int elem_bytes) {
  return rows >= 8192 || (elem_bytes == 2 && rows >= 2048 && cols >= 7168);
}

template <typename T, typename F>
cudaError_t quant_rows_t(const void *x, int64_t rows, int64_t cols, int64_t ld, const float *col_scale, int8_t *q,
                         float *row_scale_out, cudaStream_t st) {
  constexpr int V = Vec<T>::N;
  const int64_t nvec = cols / V;
  const T *xp = (const T *)x;
  auto threads_for = [&](int vpt) {
    int64_t t = (nvec + vpt - 1) / vpt;
    return (int)std::max<int64_t>(32, ((t + 31) / 32) * 32);
  };
  if (nvec <= 4 * 32) {
    return launch_quant_rows_persistent<T, 1, F>(xp, rows, nvec, ld, col_scale, q, row_scale_out, threads_for(1), st);
  }
  if (nvec <= 4 * kRowMaxThreads) {
    // the routing below was measured with INT8 codes; E4M3 codes keep the
    // 8192-row rule and four vectors per thread
    constexpr bool kI8 = std::is_same<F, FmtI8>::value;
    if (quant_rows_async_enabled(rows, kI8 ? cols : 0, (int)sizeof(T))) {
      // eight vectors per thread (half the threads per row) where that
      // still leaves two or more CTAs on an SM: more rows in flight per SM
      // at the same thread count (16384 tokens, bf16: K = 7168 0.76 -> 0.86
      // of HBM, K = 11008 0.67 -> 0.87); with one CTA per SM it loses
      if (kI8 && V == 8 && nvec >= 8 * 32 && nvec <= 8 * kRowAsync8Threads) {  // 16-bit rows, as measured
        int per_sm = 0;
        cudaError_t e = quant_rows_async_occupancy<T, 8, 3, F>(threads_for(8), &per_sm);
        if (e != cudaSuccess) return e;
        if (per_sm >= 2)
          return launch_quant_rows_async<T, 8, 3, F>(xp, rows, nvec, ld, col_scale, q, row_scale_out, threads_for(8),
                                                     st);
      }
      return launch_quant_rows_async<T, 4, 3, F>(xp, rows, nvec, ld, col_scale, q, row_scale_out, threads_for(4), st);
    }
    return launch_quant_rows_persistent<T, 4, F>(xp, rows, nvec, ld, col_scale, q, row_scale_out, threads_for(4), st);
  }
  const uint32_t row_bytes = (uint32_t)(cols * sizeof(T));
  const uint32_t buf = (row_bytes + 127u) & ~127u;
  const uint32_t extra = 128 + 8 * 3 + 2 * 16 * 4 + 16;
  if (nvec <= 8 * kSmemRowThreads && 3 * buf + extra <= 200 * 1024) {
    return launch_quant_rows_smem<T, 8, 3, F>(xp, rows, nvec, ld, col_scale, q, row_scale_out, row_bytes,
                                           3 * buf + extra, st);
  }
  if (nvec <= 8 * kSmemRowThreads && 2 * buf + extra <= 220 * 1024) {
    return launch_quant_rows_smem<T, 8, 2, F>(xp, rows, nvec, ld, col_scale, q, row_scale_out, row_bytes,
                                           2 * buf + extra, st);
  }
  return launch_pdl(quant_rows_twopass_kernel<T, F>, dim3((unsigned)rows), dim3(1024), 0, st, 1, xp, nvec, ld, col_scale,
                    q, row_scale_out);
}

template <typename T, typename F>
cudaError_t quant_cols_t(const void *w, int64_t K, int64_t N, int64_t ld, const float *s, float *colmax, int8_t *wq,
                         cudaStream_t st) {
  dim3 grid((unsigned)((N + kTT - 1) / kTT), (unsigned)((K + kTT - 1) / kTT));
  cudaError_t e = launch_pdl(quant_cols_transpose_kernel<T, F>, grid, dim3(256), 0, st, 1, (const T *)w, K, N, ld, s,
                             (const float *)colmax, wq);
  if (e != cudaSuccess) return e;
  return launch_pdl(finalize_scale_kernel<F>, dim3((unsigned)((N + 255) / 256)), dim3(256), 0, st, 1, colmax, N);
}

}  // namespace

cudaError_t launch_absmax_cols(const void *x, sq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                               const float *row_scale, float *amax, bool keep_in_l2, cudaStream_t st) {
  switch (xt) {
    case SQ_F32: return absmax_cols_t<float>(x, rows, cols, ld, row_scale, amax, keep_in_l2, st);
    case SQ_F16: return absmax_cols_t<__half>(x, rows, cols, ld, row_scale, amax, keep_in_l2, st);
    default: return absmax_cols_t<__nv_bfloat16>(x, rows, cols, ld, row_scale, amax, keep_in_l2, st);
  }
}

cudaError_t launch_absmax_rows(const void *x, sq_dtype xt, int64_t rows, int64_t cols, int64_t ld, float *out,
                               cudaStream_t st) {
  switch (xt) {
    case SQ_F32: return absmax_rows_t<float>(x, rows, cols, ld, out, st);
    case SQ_F16: return absmax_rows_t<__half>(x, rows, cols, ld, out, st);
    default: return absmax_rows_t<__nv_bfloat16>(x, rows, cols, ld, out, st);
  }
}

cudaError_t launch_wait_timeout_selftest(unsigned long long limit_ns, cudaStream_t st) {
  wait_timeout_selftest_kernel<<<1, 32, 0, st>>>(limit_ns, device_error_word());
  return cudaGetLastError();
}

cudaError_t launch_zero_fill(float *p, int64_t n, cudaStream_t st) {
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 4 * (int64_t)num_sms());
  return launch_pdl(zero_fill_kernel, dim3((unsigned)std::max<int64_t>(1, blocks)), dim3(256), 0, st, 1, p, n);
}

cudaError_t launch_smooth_factor(const float *amax, float *s_inout, float *inv_s, int64_t K, float alpha,
                                 cudaStream_t st) {
  return launch_pdl(smooth_factor_kernel, dim3((unsigned)((K + 255) / 256)), dim3(256), 0, st, 1, amax, s_inout, inv_s,
                    K, alpha);
}

template <typename F>
cudaError_t quant_rows_fmt(const void *x, sq_dtype xt, int64_t rows, int64_t cols, int64_t ld, const float *col_scale,
                           int8_t *q, float *row_scale_out, cudaStream_t st) {
  switch (xt) {
    case SQ_F32: return quant_rows_t<float, F>(x, rows, cols, ld, col_scale, q, row_scale_out, st);
    case SQ_F16: return quant_rows_t<__half, F>(x, rows, cols, ld, col_scale, q, row_scale_out, st);
    default: return quant_rows_t<__nv_bfloat16, F>(x, rows, cols, ld, col_scale, q, row_scale_out, st);
  }
}

cudaError_t launch_quant_rows(const void *x, sq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                              const float *col_scale, int8_t *q, float *row_scale_out, QFmt fmt, cudaStream_t st) {
  return fmt == QFmt::E4M3 ? quant_rows_fmt<FmtE4M3>(x, xt, rows, cols, ld, col_scale, q, row_scale_out, st)
                           : quant_rows_fmt<FmtI8>(x, xt, rows, cols, ld, col_scale, q, row_scale_out, st);
}

template <typename F>
cudaError_t quant_cols_fmt(const void *w, sq_dtype wt, int64_t K, int64_t N, int64_t ld, const float *s,
                           float *colmax_to_scale, int8_t *wq, cudaStream_t st) {
  switch (wt) {
    case SQ_F32: return quant_cols_t<float, F>(w, K, N, ld, s, colmax_to_scale, wq, st);
    case SQ_F16: return quant_cols_t<__half, F>(w, K, N, ld, s, colmax_to_scale, wq, st);
    default: return quant_cols_t<__nv_bfloat16, F>(w, K, N, ld, s, colmax_to_scale, wq, st);
  }
}

cudaError_t launch_quant_cols_transpose(const void *w, sq_dtype wt, int64_t K, int64_t N, int64_t ld,
                                        const float *s, float *colmax_to_scale, int8_t *wq, QFmt fmt,
                                        cudaStream_t st) {
  return fmt == QFmt::E4M3 ? quant_cols_fmt<FmtE4M3>(w, wt, K, N, ld, s, colmax_to_scale, wq, st)
                           : quant_cols_fmt<FmtI8>(w, wt, K, N, ld, s, colmax_to_scale, wq, st);
}

}  // namespace sq
