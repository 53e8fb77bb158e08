// sq_common.cuh -- device helpers shared by the libsq kernels (sm_100a).
//
// Element loads/conversions, the INT8 quantizer, block reductions, and thin
// inline-PTX wrappers for mbarriers (with bounded waits), TMA and tcgen05.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace sq {

// Device error word bits (see sq_check_device_error).
constexpr unsigned kDevErrTimeout = 1u;
// Every in-kernel wait gives up after this long.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  Every libsq kernel is launched so that it
// may start while the previous kernel on the stream is still finishing; it
// runs only its prologue (shared-memory barriers, TMEM allocation, tensor
// map prefetch) before pdl_wait(), which returns once the previous grid has
// completed and its memory is visible, and it touches global memory only
// after that.  pdl_trigger() lets the next kernel's blocks be scheduled as
// soon as this grid's blocks have all started.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              unsigned cluster_x, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Element types: 16-byte vectors converted exactly to fp32.
// ---------------------------------------------------------------------------
template <typename T>
struct Vec;
template <>
struct Vec<float> {
  static constexpr int N = 4;
  static __device__ __forceinline__ void to_f32(const uint4 &v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
  static __device__ __forceinline__ float one(const float *p) { return *p; }
};
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  // bf16 is the top half of an fp32: widening is a shift, exact.
  static __device__ __forceinline__ void to_f32(const uint4 &v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ float one(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
};
template <>
struct Vec<__half> {
  static constexpr int N = 8;
  static __device__ __forceinline__ void to_f32(const uint4 &v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h = *reinterpret_cast<const __half2 *>(&w[i]);
      float2 g = __half22float2(h);
      f[2 * i] = g.x;
      f[2 * i + 1] = g.y;
    }
  }
  static __device__ __forceinline__ float one(const __half *p) { return __half2float(*p); }
};

__device__ __forceinline__ uint4 ld_nc_v4(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Read-once data: same load; kept as a separate name for streaming inputs.
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) { return ld_nc_v4(p); }

// 16-byte load with an L2 eviction policy (from createpolicy below).
__device__ __forceinline__ uint4 ld_policy_v4(const void *p, uint64_t policy) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p), "l"(policy));
  return r;
}

// 16-byte asynchronous copy global -> this thread's shared memory (through
// L2 only), with an L2 eviction policy; completion in commit groups.
__device__ __forceinline__ void cp_async_16(void *smem_dst, const void *gsrc, uint64_t policy) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
               "l"(gsrc), "l"(policy)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Waits until at most n of this thread's most recent commit groups are pending.
template <int n>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(n) : "memory");
}

// ---------------------------------------------------------------------------
// The quantizer: code = rne(fl(v / delta)) for a row with scale delta =
// absmax / Q (Q = 127 for INT8, 448 for E4M3), clamped to [-127, 127] for
// INT8.  Every product and sum below is a separately rounded IEEE operation
// (explicit _rn intrinsics or .rn PTX), never contracted.
// ---------------------------------------------------------------------------
// Rounds u to the nearest integer, ties to even, with one exact IEEE
// addition: for |u| < 2^22, u + 1.5 * 2^23 lies in [2^23, 2^24), where
// adjacent floats are 1 apart, so the round-to-nearest-even sum equals
// 1.5 * 2^23 + rne(u) (the shift is even, so ties land on the even integer)
// and rne(u) sits in the low bits of the sum's encoding: its low byte is
// the two's-complement int8 code whenever |rne(u)| <= 127.  This keeps the
// conversion off the float-to-integer unit.
constexpr float kRneShift = 12582912.0f;  // 1.5 * 2^23

// A value's code is rne(fl(v / delta)) (IEEE division by the row's scale),
// formed here without a division per value.  With rcp = fl(1 / delta) the
// exact product P = v * rcp is within |v / delta| * 2^-24 <= 2^-17 of
// Q = v / delta (|Q| < 128), and fl(Q) within 2^-18 of Q, so fl(Q) and P
// differ by less than 2^-16.  fma(v, rcp, 1.5 * 2^23) rounds P to its
// nearest integer k (the code, in the low byte), and fma(v, rcp, -k) is
// P - k rounded once (error <= 2^-25).  When that is below 1/2 - 2^-15 in
// magnitude, P is farther than 2^-15 - 2^-25 from every half-integer, so
// fl(Q) lies on the same side and rounds to k too.  Otherwise -- a value
// within ~2^-15 of a rounding boundary -- the quotient is taken with an
// IEEE division.
constexpr float kNearTie = 0.5f - 0x1p-15f;

// Two IEEE fp32 products at once (sm_100 packed fp32 pipe), each rounded
// to nearest even exactly as a scalar __fmul_rn would be.
__device__ __forceinline__ float2 fmul2_rn(float2 a, float2 b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;"
      : "=l"(d)
      : "l"(*reinterpret_cast<const uint64_t *>(&a)), "l"(*reinterpret_cast<const uint64_t *>(&b)));
  return *reinterpret_cast<float2 *>(&d);
}

// max(a, b, c) in one instruction (sm_100 three-input max).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Two fused multiply-adds at once, each rounded once as __fmaf_rn.
__device__ __forceinline__ float2 ffma2_rn(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(d)
      : "l"(*reinterpret_cast<const uint64_t *>(&a)), "l"(*reinterpret_cast<const uint64_t *>(&b)),
        "l"(*reinterpret_cast<const uint64_t *>(&c)));
  return *reinterpret_cast<float2 *>(&d);
}

__device__ __forceinline__ float2 fsub2_rn(float2 a, float2 b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;"
      : "=l"(d)
      : "l"(*reinterpret_cast<const uint64_t *>(&a)), "l"(*reinterpret_cast<const uint64_t *>(&b)));
  return *reinterpret_cast<float2 *>(&d);
}

// Code words (low byte = code) of n values (n even) of one row with
// |v / delta| <= 127.5 -- every value bounded by the row's absmax m and
// delta = fl(m / 127).  delta == 0 (an all-zero row, rcp == 0) gives 0.
// All on the packed fp32 pipe: sh = fma(v, rcp, S) holds k, S - sh = -k
// exactly, fma(v, rcp, -k) = P - k; one compare of the largest distance
// per call decides whether any value needs the division.
template <int n>
__device__ __forceinline__ void code_words(const float *v, float delta, float rcp, uint32_t *w) {
  const float2 r2 = make_float2(rcp, rcp), s2 = make_float2(kRneShift, kRneShift);
  float dm = 0.0f;
#pragma unroll
  for (int e = 0; e < n; e += 2) {
    const float2 v2 = make_float2(v[e], v[e + 1]);
    const float2 sh = ffma2_rn(v2, r2, s2);
    w[e] = __float_as_uint(sh.x);
    w[e + 1] = __float_as_uint(sh.y);
    const float2 d = ffma2_rn(v2, r2, fsub2_rn(s2, sh));
    dm = fmax3(dm, fabsf(d.x), fabsf(d.y));
  }
  if (!(dm < kNearTie)) {  // rare: recompute the values next to a boundary exactly
#pragma unroll
    for (int e = 0; e < n; ++e) {
      const float k = __fsub_rn(__uint_as_float(w[e]), kRneShift);
      if (!(fabsf(__fmaf_rn(v[e], rcp, -k)) < kNearTie))
        w[e] = __float_as_uint(__fadd_rn(__fdiv_rn(v[e], delta), kRneShift));
    }
  }
}

// Clamped code for a finite v of any magnitude (static scales):
// clamp(rne(fl(v / delta)), -127, 127).  lim = fl(127 * delta) >=
// 127 * delta * (1 - 2^-24), so |v| >= lim means |v / delta| > 126.5 and a
// saturated code, which the clamped value lim also gives (lim / delta is
// within 2^-17 of 127); below lim, |v / delta| <= 127 * (1 + 2^-24).
__device__ __forceinline__ float clamp_to_range(float v, float lim) { return fminf(fmaxf(v, -lim), lim); }

__device__ __forceinline__ int quantize_div(float v, float delta, float rcp) {
  float vc[2] = {clamp_to_range(v, __fmul_rn(127.0f, delta)), 0.0f};
  uint32_t w[2];
  code_words<2>(vc, delta, rcp, w);
  return (int)(int8_t)(w[0] & 0xffu);
}

// Bytes 0..3 of the result are the low bytes of a, b, c, d.
__device__ __forceinline__ uint32_t pack4_low(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Eight codes of one 16-byte row vector, packed into 8 bytes (4 into 4).
__device__ __forceinline__ uint2 codes8(const float *v, float delta, float rcp) {
  uint32_t w[8];
  code_words<8>(v, delta, rcp, w);
  return make_uint2(pack4_low(w[0], w[1], w[2], w[3]), pack4_low(w[4], w[5], w[6], w[7]));
}
__device__ __forceinline__ uint32_t codes4(const float *v, float delta, float rcp) {
  uint32_t w[4];
  code_words<4>(v, delta, rcp, w);
  return pack4_low(w[0], w[1], w[2], w[3]);
}

// Two fp32 values to two E4M3 codes (round to nearest even, saturating at
// +-448): lo in bits 0-7, hi in bits 8-15.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}

// Code formats of the quantizers.  kMax is the code magnitude a row's
// absmax maps to: scale delta = absmax / kMax, codes of fl(v / delta).
//   FmtI8    symmetric INT8, codes in [-127, 127]
//   FmtE4M3  FP8 E4M3 codes, values in [-448, 448]
// codes8 / codes4 quantize one 16- or 8-byte vector of a dynamic row
// (scale delta, rcp = fl(1 / delta)); code1 one value of any magnitude
// (saturating).
struct FmtI8 {
  static constexpr float kMax = 127.0f;
  static __device__ __forceinline__ uint2 codes8(const float *v, float delta, float rcp) {
    return sq::codes8(v, delta, rcp);
  }
  static __device__ __forceinline__ uint32_t codes4(const float *v, float delta, float rcp) {
    return sq::codes4(v, delta, rcp);
  }
  static __device__ __forceinline__ uint8_t code1(float v, float delta, float rcp) {
    return (uint8_t)(int8_t)quantize_div(v, delta, rcp);
  }
};
struct FmtE4M3 {
  static constexpr float kMax = 448.0f;
  // Codes of fl(v / delta) without a division per value: y = fl(v * rcp)
  // is within |y| * 2^-22 of fl(v / delta) (two roundings of 2^-24 each,
  // plus rcp's).  y * (1 -+ 2^-21), each rounded once, bracket that
  // interval, and E4M3 rounding is monotone, so when both ends give the
  // same code every value between them -- fl(v / delta) included -- does
  // too.  Otherwise (a value next to an E4M3 midpoint) the quotient is taken
  // with an IEEE division.  An all-zero row (delta == 0) gets codes +0.
  static __device__ __forceinline__ void pairs(const float *v, float delta, float rcp, int n, uint32_t *out) {
    const float2 r2 = make_float2(rcp, rcp);
    const float2 lo2 = make_float2(1.0f - 0x1p-21f, 1.0f - 0x1p-21f), hi2 = make_float2(1.0f + 0x1p-21f, 1.0f + 0x1p-21f);
    uint32_t diff = 0;
    uint32_t hi[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      if (e < n) {
        const float2 y = fmul2_rn(make_float2(v[e], v[e + 1]), r2);
        const float2 yl = fmul2_rn(y, lo2), yh = fmul2_rn(y, hi2);
        out[e / 2] = e4m3x2(yl.x, yl.y);
        hi[e / 2] = e4m3x2(yh.x, yh.y);
        diff |= out[e / 2] ^ hi[e / 2];
      }
    }
    if (diff != 0u) {  // rare
#pragma unroll
      for (int e = 0; e < 8; e += 2)
        if (e < n && out[e / 2] != hi[e / 2]) out[e / 2] = e4m3x2(__fdiv_rn(v[e], delta), __fdiv_rn(v[e + 1], delta));
    }
  }
  static __device__ __forceinline__ uint2 codes8(const float *v, float delta, float rcp) {
    if (delta == 0.0f) return make_uint2(0u, 0u);
    uint32_t c[4];
    pairs(v, delta, rcp, 8, c);
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
  }
  static __device__ __forceinline__ uint32_t codes4(const float *v, float delta, float rcp) {
    if (delta == 0.0f) return 0u;
    uint32_t c[4];
    pairs(v, delta, rcp, 4, c);
    return c[0] | (c[1] << 16);
  }
  static __device__ __forceinline__ uint8_t code1(float v, float delta, float) {
    return delta == 0.0f ? (uint8_t)0 : (uint8_t)(e4m3x2(__fdiv_rn(v, delta), 0.0f) & 0xffu);
  }
};

// Max over a warp; values are non-negative floats.
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Max over the block; `red` holds >= 32 floats of shared memory.  All
// threads get the result.  Ends with a barrier so `red` can be reused.
__device__ __forceinline__ float block_max(float v, float *red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = (blockDim.x + 31) >> 5;
  v = warp_max(v);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = lane < nwarps ? red[lane] : 0.0f;
  r = warp_max(r);
  __syncthreads();
  return r;
}

// ---------------------------------------------------------------------------
// Shared-memory addresses, mbarriers (bounded waits), TMA, tcgen05.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits until the barrier phase of parity `parity` has completed.  Returns
// false, without waiting further, once *abort is set by another role or
// after kWaitLimitNs; on the timeout it records kDevErrTimeout in *err and
// raises *abort for the rest of the block.  `abort` may be null.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort, unsigned *err,
                                          unsigned long long limit_ns = kWaitLimitNs) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(a, parity)) return true;
    if ((it & 15u) == 0) {
      if (abort != nullptr && *abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        atomicOr(err, kDevErrTimeout);
        if (abort != nullptr) *abort = 1;
        return false;
      }
    }
  }
}

// Brings a 2-D tile of a tensor into L2 (no shared memory, no barrier).
// L2 is the device's point of coherence, so a prefetch issued before the
// previous kernel's results are visible reads no stale data later: a write
// that lands after it updates the same L2 lines.
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap *m, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(m)),
               "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// Contiguous bulk copy global -> this CTA's shared memory (both addresses
// 16-byte aligned, bytes a multiple of 16); completion counted on `bar`.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 2-D tiled TMA load into this CTA's shared memory; completion is counted
// in bytes on `bar`.  x is the innermost (contiguous) coordinate.
__device__ __forceinline__ void tma_load_2d(const CUtensorMap *m, uint64_t *bar, void *dst, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// Same, with an L2 eviction-priority hint (policy from createpolicy).
__device__ __forceinline__ void tma_load_2d_hint(const CUtensorMap *m, uint64_t *bar, void *dst, int x, int y,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// --- tcgen05 (5th-generation tensor cores, accumulators in TMEM) ----------
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, signed 8-bit operands, int32 accumulate.
__device__ __forceinline__ void umma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 op this thread issued so far ends.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i gets lane (base+i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
// Barrier among `count` threads (a multiple of 32) on hardware barrier `id`.
__device__ __forceinline__ void named_barrier(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Barrier among `count` threads that also ANDs a predicate over them, so
// every participant leaves with the same decision.
__device__ __forceinline__ bool named_barrier_and(int id, int count, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(out)
      : "r"((uint32_t)pred), "r"(id), "r"(count)
      : "memory");
  return out != 0;
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// --- CTA pairs (cluster of 2, tcgen05 cta_group::2) -----------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on an mbarrier given by its shared::cluster address (any CTA).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// 16-byte load (address 16-byte aligned) from shared memory of any CTA of
// the cluster.
__device__ __forceinline__ uint4 ld_shared_cluster_v4(uint32_t cluster_addr) {
  uint4 v;
  asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(cluster_addr)
               : "memory");
  return v;
}
// TMA load into this CTA's shared memory whose byte count completes on an
// mbarrier that may live in the peer CTA of the pair.
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap *m, uint32_t bar_cluster, void *dst, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D[tmem] (+)= A * B^T over the CTA pair: M = 256 (128 rows of A from each
// CTA's shared memory at the same offset), N columns of B split in halves.
__device__ __forceinline__ void umma_i8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the mbarrier at shared::cluster address `bar` when every
// pair MMA issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar_cluster) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster)
               : "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile written by TMA
// with 128-byte swizzling: rows of 128 bytes, 8-row groups 1024 bytes apart.
// Bits: [0,14) start>>4, [16,30) leading offset>>4 (unused for this
// layout), [32,46) stride offset>>4 = 1024>>4, [46,48) version 1,
// [61,64) layout 2 = 128-byte swizzle.
__device__ __forceinline__ uint64_t desc_sw128_kmajor(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor for kind::i8: D = s32 (bits 4-5 = 2), A and B
// signed 8-bit (bits 7-9, 10-12 = 1), both K-major, N>>3 at bits 17-22,
// M>>4 at bits 24-28.
__host__ __device__ constexpr uint32_t idesc_i8(int m, int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// Instruction descriptor for kind::f8f6f4 with E4M3 A and B (format code 0
// at bits 7-9 and 10-12) and an f32 accumulator (bits 4-5 = 1); the other
// fields as idesc_i8.
__host__ __device__ constexpr uint32_t idesc_e4m3(int m, int n) {
  return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// 8-bit operands: INT8 (s32 accumulator) or, with F8, E4M3 (f32 accumulator).
template <bool F8>
__host__ __device__ constexpr uint32_t idesc8(int m, int n) {
  return F8 ? idesc_e4m3(m, n) : idesc_i8(m, n);
}

template <bool F8>
__device__ __forceinline__ void umma8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                      uint32_t accumulate) {
  if constexpr (F8) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    umma_i8(d_tmem, adesc, bdesc, idesc, accumulate);
  }
}

template <bool F8>
__device__ __forceinline__ void umma8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  if constexpr (F8) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    umma_i8_pair(d_tmem, adesc, bdesc, idesc, accumulate);
  }
}

// The accumulator's 32 bits as a float: an int32 sum (INT8) converted with
// round to nearest even, or the f32 sum itself (E4M3).
template <bool F8>
__device__ __forceinline__ float acc_value(uint32_t bits) {
  if constexpr (F8) {
    return __uint_as_float(bits);
  } else {
    return __int2float_rn((int)bits);
  }
}

}  // namespace sq
