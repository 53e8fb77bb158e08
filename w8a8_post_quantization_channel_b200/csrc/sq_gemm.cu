// sq_gemm.cu -- W8A8 linear on the 5th-generation tensor cores (sm_100a).
//
// acc_tn = sum_j Xq_tj * Wq_nj (int32, exact), then
// y_tn = round(((float)acc_tn * dx_t) * dw_n).
// The page's comparison table puts W8A8's gain in running the product
// directly on INT8 tensor cores ("SmoothQuant (activation smoothing
// quantization)", jisaku.com glossary, comparison with GPTQ/AWQ).
//
// Kernel structure (one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: Xq and Wq tiles (K-major, 128-byte swizzle)
//               into a STAGES-deep shared-memory ring;
//   warp 1      allocates TMEM; one thread issues tcgen05.mma kind::i8
//               (M=128, N=BN, K=32 per instruction) into one of two TMEM
//               accumulators and signals the ring / epilogue with
//               tcgen05.commit;
//   warps 2-5   epilogue: tcgen05.ld of the finished accumulator (one TMEM
//               lane quarter per warp), fp32 dequant, rounding, stores;
//               the other accumulator is filled by the MMA meanwhile.
// Every mbarrier wait is bounded (see mbar_wait); on a timeout the roles
// stop, in-flight copies and MMAs are drained, TMEM is freed.
#include <cudaTypedefs.h>

#include <mutex>

#include "sq_common.cuh"
#include "sq_internal.h"

namespace sq {

namespace {

constexpr int kBM = 128;  // rows of Xq per tile (= TMEM lanes)
constexpr int kBK = 128;  // K bytes per stage (one 128-byte swizzle row)
constexpr int kThreads = 192;
constexpr int kDecodeMaxM = 64;  // token counts served by the weight-streaming kernel

// Workspace of the decode kernel: int32 partial sums [M][N], then one
// arrival counter per 128-row tile of Wq (each region 256-byte aligned).
inline int64_t decode_ws_elems(int64_t M, int64_t N) { return ((M * N * 4 + 255) / 256) * 64; }
inline int64_t decode_counter_bytes(int64_t N) { return (((N + 127) / 128) * 4 + 255) / 256 * 256; }

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr uint32_t kA = kBM * kBK;
  static constexpr uint32_t kB = BN * kBK;
  static constexpr uint32_t kRing = STAGES * (kA + kB);
  static constexpr uint32_t kBars = (2 * STAGES + 5) * 8 + 16;
  static constexpr uint32_t kTotal = kRing + kBars + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = 2 * BN;
};

template <OutKind KIND, bool F8>
__device__ __forceinline__ void store_chunk(const uint32_t (&r)[32], const YDest &dst, int64_t ldy, int row, int n0,
                                            int N, float dx, const float *__restrict__ w_scale) {
  // N % 16 == 0 and n0 % 32 == 0, so a chunk has 16 or 32 valid columns.
  const int groups16 = min(2, (N - n0) / 16);
  constexpr int kEsz = KIND == OutKind::F16 || KIND == OutKind::BF16 ? 2 : 4;
  constexpr int kVecs = 32 * kEsz / 16;  // 16-byte vectors of a 32-column chunk
  uint4 out[kVecs];
  if constexpr (KIND == OutKind::I32) {
#pragma unroll
    for (int g = 0; g < 8; ++g) out[g] = make_uint4(r[4 * g], r[4 * g + 1], r[4 * g + 2], r[4 * g + 3]);
  } else {
    float v[32];
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      if (g / 4 < groups16) {
        const float4 dw = __ldg(reinterpret_cast<const float4 *>(w_scale + n0) + g);
        v[4 * g + 0] = __fmul_rn(__fmul_rn(acc_value<F8>(r[4 * g + 0]), dx), dw.x);
        v[4 * g + 1] = __fmul_rn(__fmul_rn(acc_value<F8>(r[4 * g + 1]), dx), dw.y);
        v[4 * g + 2] = __fmul_rn(__fmul_rn(acc_value<F8>(r[4 * g + 2]), dx), dw.z);
        v[4 * g + 3] = __fmul_rn(__fmul_rn(acc_value<F8>(r[4 * g + 3]), dx), dw.w);
      } else {
        v[4 * g + 0] = v[4 * g + 1] = v[4 * g + 2] = v[4 * g + 3] = 0.0f;
      }
    }
    if constexpr (KIND == OutKind::F32) {
#pragma unroll
      for (int g = 0; g < 8; ++g)
        out[g] = make_uint4(__float_as_uint(v[4 * g]), __float_as_uint(v[4 * g + 1]), __float_as_uint(v[4 * g + 2]),
                            __float_as_uint(v[4 * g + 3]));
    } else {
      uint32_t p[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if constexpr (KIND == OutKind::BF16) {
          __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
          p[i] = *reinterpret_cast<uint32_t *>(&h);
        } else {
          __half2 h = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
          p[i] = *reinterpret_cast<uint32_t *>(&h);
        }
      }
#pragma unroll
      for (int g = 0; g < 4; ++g) out[g] = make_uint4(p[4 * g], p[4 * g + 1], p[4 * g + 2], p[4 * g + 3]);
    }
  }
  // the same words to every destination (this rank's Y, and peers' copies)
#pragma unroll 1
  for (int d = 0; d < dst.n; ++d) {
    uint4 *yr = reinterpret_cast<uint4 *>(static_cast<uint8_t *>(dst.p[d]) + ((int64_t)row * ldy + n0) * kEsz);
#pragma unroll
    for (int g = 0; g < kVecs; ++g)
      if (g * 2 / kVecs < groups16) yr[g] = out[g];
  }
}

template <int BN, int STAGES, OutKind KIND, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
    w8a8_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const float *__restrict__ x_scale, const float *__restrict__ w_scale, const YDest dst,
                        int64_t ldy, int M, int N, int K, unsigned *err) {
  using L = GemmSmem<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * L::kA;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kRing);
  uint64_t *empty = full + STAGES;
  uint64_t *tfull = empty + STAGES;
  uint64_t *tempty = tfull + 2;
  uint64_t *drain = tempty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m = (M + kBM - 1) / kBM;
  const int num_n = (N + BN - 1) / BN;
  const int tiles = num_m * num_n;
  const int nk = (K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // prologue done; the previous kernel's results are visible from here on
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      uint32_t stage = 0, phase = 0;
      uint32_t armed = 0, armed_parity = 0;  // per-stage bit masks
      bool ok = true;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        const int mb = tile % num_m, nb = tile / num_m;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], L::kA + L::kB);
          tma_load_2d(&tmA, &full[stage], sA + stage * L::kA, kb * kBK, mb * kBM);
          tma_load_2d(&tmB, &full[stage], sB + stage * L::kB, kb * kBK, nb * BN);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {  // let every issued copy land before the CTA may exit
        for (int s = 0; s < STAGES; ++s)
          if (armed & (1u << s)) mbar_wait(&full[s], (armed_parity >> s) & 1u, nullptr, err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = idesc8<F8>(kBM, BN);
      uint32_t stage = 0, phase = 0, ab = 0, aphase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(&tempty[ab], aphase ^ 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + ab * BN;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a0 = desc_sw128_kmajor(smem_u32(sA + stage * L::kA));
          const uint64_t b0 = desc_sw128_kmajor(smem_u32(sB + stage * L::kB));
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k)  // 32 int8 = 32 bytes = +2 in the >>4 address field
            umma8<F8>(d, a0 + 2 * k, b0 + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[ab]);
        ab ^= 1;
        if (ab == 0) aphase ^= 1;
      }
      // every MMA issued above must finish before TMEM is released
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, err);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint32_t ab = 0, aphase = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
      bool ok = mbar_wait(&tfull[ab], aphase, abort_flag, err);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int mb = tile % num_m, nb = tile / num_m;
      const int row = mb * kBM + q * 32 + lane;
      const bool row_ok = row < M;
      const float dx = (KIND != OutKind::I32 && row_ok) ? __ldg(x_scale + row) : 0.0f;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + ab * BN + c * 32, r);
        tmem_ld_wait();
        const int n0 = nb * BN + c * 32;
        if (row_ok && n0 < N) store_chunk<KIND, F8>(r, dst, ldy, row, n0, N, dx, w_scale);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[ab]);
      ab ^= 1;
      if (ab == 0) aphase ^= 1;
    }
  }

  // stores into other GPUs' memory (the column-parallel scatter) are made
  // visible system-wide before the kernel ends, so that the stream-ordered
  // collective that follows cannot overtake them
  if (dst.n > 1) __threadfence_system();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// CTA-pair kernel: a cluster of two CTAs computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 32 per instruction).
// CTA r of the pair loads rows [128 r, 128 r + 128) of the tile's Xq block
// and of its Wq block into its own shared memory; both loads count bytes on
// the leader CTA's (rank 0) full barrier.  The leader's single MMA thread
// drives the pair; its commits arrive on the matching barriers of both
// CTAs.  Each CTA's epilogue reads its own TMEM: 128 rows x BN columns.
// With BN = 256, per CTA and k-block this moves 32 KB for 128 x 256 x 128
// MACs, a third less operand traffic than the single-CTA 128 x 256 tile.
// (Narrower pair tiles, 160 or 224 wide, chosen to fill the last round of
// tiles, measured 15-37% slower per launch on every shape that took them;
// the library runs BN = 256.)
// ---------------------------------------------------------------------------
template <int BN, int STAGES>
struct PairSmem {
  static_assert(BN % 32 == 0 && BN >= 128 && BN <= 256, "pair tile width");
  static constexpr uint32_t kA = kBM * kBK;       // 16 KB: this CTA's 128 rows of Xq
  static constexpr uint32_t kB = (BN / 2) * kBK;  // this CTA's BN / 2 rows of Wq (a multiple of 1 KB)
  static constexpr uint32_t kRing = STAGES * (kA + kB);
  static constexpr uint32_t kBars = (2 * STAGES + 5) * 8 + 16;
  static constexpr uint32_t kTotal = kRing + kBars + 1024;
  static constexpr uint32_t kTmemCols = 512;  // two BN-column accumulators
};

template <int BN, int STAGES, OutKind KIND, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
    w8a8_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const float *__restrict__ x_scale, const float *__restrict__ w_scale,
                          const YDest dst, int64_t ldy, int M, int N, int K, unsigned *err) {
  using L = PairSmem<BN, STAGES>;
  constexpr int kPairBN = BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * L::kA;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kRing);
  uint64_t *empty = full + STAGES;
  uint64_t *tfull = empty + STAGES;
  uint64_t *tempty = tfull + 2;
  uint64_t *drain = tempty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int num_m = (M + 2 * kBM - 1) / (2 * kBM);
  const int num_n = (N + kPairBN - 1) / kPairBN;
  const int tiles = num_m * num_n;
  const int nk = (K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);  // 4 epilogue warps in each CTA of the pair
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, L::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // prologue done; the previous kernel's results are visible from here on
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      uint32_t stage = 0, phase = 0;
      uint32_t armed = 0, armed_parity = 0;
      bool ok = true;
      for (int tile = pair; tile < tiles && ok; tile += npairs) {
        const int mb = tile % num_m, nb = tile / num_m;
        const int row_a = mb * 2 * kBM + (int)rank * kBM;
        const int row_b = nb * kPairBN + (int)rank * (kPairBN / 2);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, err)) {
            ok = false;
            break;
          }
          if (leader) {
            mbar_arrive_expect_tx(&full[stage], 2 * (L::kA + L::kB));
            armed |= 1u << stage;
            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          }
          const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
          tma_load_2d_pair(&tmA, bar, sA + stage * L::kA, kb * kBK, row_a);
          tma_load_2d_pair(&tmB, bar, sB + stage * L::kB, kb * kBK, row_b);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok && leader) {  // the leader's barriers count both CTAs' copies
        for (int s = 0; s < STAGES; ++s)
          if (armed & (1u << s)) mbar_wait(&full[s], (armed_parity >> s) & 1u, nullptr, err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (leader CTA) ----------------
      constexpr uint32_t idesc = idesc8<F8>(2 * kBM, kPairBN);
      uint32_t stage = 0, phase = 0, ab = 0, aphase = 0;
      bool ok = true;
      for (int tile = pair; tile < tiles && ok; tile += npairs) {
        if (!mbar_wait(&tempty[ab], aphase ^ 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + ab * 256;  // accumulators at columns 0 and 256
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a0 = desc_sw128_kmajor(smem_u32(sA + stage * L::kA));
          const uint64_t b0 = desc_sw128_kmajor(smem_u32(sB + stage * L::kB));
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k) umma8_pair<F8>(d, a0 + 2 * k, b0 + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          const uint32_t e = smem_u32(&empty[stage]);
          umma_commit_pair(mapa_shared(e, 0));
          umma_commit_pair(mapa_shared(e, 1));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        const uint32_t t = smem_u32(&tfull[ab]);
        umma_commit_pair(mapa_shared(t, 0));
        umma_commit_pair(mapa_shared(t, 1));
        ab ^= 1;
        if (ab == 0) aphase ^= 1;
      }
      umma_commit_pair(mapa_shared(smem_u32(drain), 0));
      mbar_wait(drain, 0, nullptr, err);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..5 of both CTAs) ----------------
    const int q = warp & 3;
    const uint32_t tempty_leader = mapa_shared(smem_u32(&tempty[0]), 0);
    uint32_t ab = 0, aphase = 0;
    for (int tile = pair; tile < tiles; tile += npairs) {
      bool ok = mbar_wait(&tfull[ab], aphase, abort_flag, err);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int mb = tile % num_m, nb = tile / num_m;
      const int row = mb * 2 * kBM + (int)rank * kBM + q * 32 + lane;
      const bool row_ok = row < M;
      const float dx = (KIND != OutKind::I32 && row_ok) ? __ldg(x_scale + row) : 0.0f;
#pragma unroll 1
      for (int c = 0; c < kPairBN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + ab * 256 + c * 32, r);
        tmem_ld_wait();
        const int n0 = nb * kPairBN + c * 32;
        if (row_ok && n0 < N) store_chunk<KIND, F8>(r, dst, ldy, row, n0, N, dx, w_scale);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader + ab * 8);
      ab ^= 1;
      if (ab == 0) aphase ^= 1;
    }
  }

  // stores into other GPUs' memory (the column-parallel scatter) are made
  // visible system-wide before the kernel ends, so that the stream-ordered
  // collective that follows cannot overtake them
  if (dst.n > 1) __threadfence_system();
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's shared memory and TMEM stay live until the leader is done
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Decode-shaped linear (M <= 64 tokens): bound by streaming Wq from HBM.
// The roles of the operands swap: 128 rows of Wq sit on the MMA's M side
// and the (padded) MP tokens on its N side, so D^T[n][t] accumulates in
// TMEM lanes n, columns t.  The N/128 x K/128 (tile, k-block) items are
// split evenly over the CTAs (each streams the same number of Wq bytes);
// a CTA's share may cover parts of two tiles.  A CTA that covers a whole
// tile dequantizes it straight from TMEM.  Otherwise it adds its int32
// partial sums into the workspace (exact, order-free), counts the k-blocks
// it contributed on the tile's counter, and the CTA whose count completes
// the tile dequantizes it from the workspace and leaves the workspace and
// the counter zero again.  No CTA waits for another.
// ---------------------------------------------------------------------------
constexpr int kDecRows = 128;  // Wq rows per tile (MMA M)

template <int MP>
struct DecSmem {
  static constexpr uint32_t kW = kDecRows * kBK;  // 16 KB of Wq per stage
  static constexpr uint32_t kX = MP * kBK;        // MP token rows of Xq per stage
  static constexpr uint32_t kStage = kW + kX;
  // Under full HBM load a request takes ~3-4 us to return, so each SM keeps
  // as many stages in flight as ~216 KB of shared memory holds.
  static constexpr int kStages = (216 * 1024) / kStage;
  static constexpr uint32_t kRing = kStages * kStage;
  static constexpr uint32_t kBars = (2 * kStages + 5) * 8 + 32;
  static constexpr uint32_t kTotal = kRing + kBars + 1024;
  static constexpr uint32_t kTmemCols = (2 * MP <= 32) ? 32 : (2 * MP <= 64) ? 64 : 128;
};

template <OutKind KIND, bool F8>
__device__ __forceinline__ void store_one(const YDest &dst, int64_t ldy, int t, int n, uint32_t acc, float dx,
                                          float dw) {
  const int64_t i = (int64_t)t * ldy + n;
  if constexpr (KIND == OutKind::I32) {
#pragma unroll 1
    for (int d = 0; d < dst.n; ++d) static_cast<uint32_t *>(dst.p[d])[i] = acc;  // the raw accumulator
  } else {
    const float v = __fmul_rn(__fmul_rn(acc_value<F8>(acc), dx), dw);
    if constexpr (KIND == OutKind::F32) {
#pragma unroll 1
      for (int d = 0; d < dst.n; ++d) static_cast<float *>(dst.p[d])[i] = v;
    } else if constexpr (KIND == OutKind::BF16) {
      const __nv_bfloat16 h = __float2bfloat16_rn(v);
#pragma unroll 1
      for (int d = 0; d < dst.n; ++d) static_cast<__nv_bfloat16 *>(dst.p[d])[i] = h;
    } else {
      const __half h = __float2half_rn(v);
#pragma unroll 1
      for (int d = 0; d < dst.n; ++d) static_cast<__half *>(dst.p[d])[i] = h;
    }
  }
}

template <int MP, OutKind KIND, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
    w8a8_gemm_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                            const float *__restrict__ x_scale, const float *__restrict__ w_scale,
                            const YDest dst, int64_t ldy, int M, int N, int K, int32_t *__restrict__ ws,
                            unsigned *__restrict__ tile_count, unsigned *err) {
  using L = DecSmem<MP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kRing);
  uint64_t *empty = full + L::kStages;
  uint64_t *tfull = empty + L::kStages;
  uint64_t *tempty = tfull + 2;
  uint64_t *drain = tempty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *last_flag = reinterpret_cast<volatile int *>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = (N + kDecRows - 1) / kDecRows;
  const int nk = (K + kBK - 1) / kBK;
  const int64_t items = (int64_t)ntiles * nk;
  const int64_t w0 = items * blockIdx.x / gridDim.x;
  const int64_t w1 = items * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmX);
    // the first ring's worth of this CTA's Wq boxes, into L2 while the
    // previous kernel may still run (L2 stays coherent if it writes them)
    for (int64_t w = w0; w < w1 && w < w0 + L::kStages; ++w)
      tma_prefetch_l2_2d(&tmW, (int)(w % nk) * kBK, (int)(w / nk) * kDecRows);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // prologue done; the previous kernel's results are visible from here on
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      uint32_t stage = 0, phase = 0, armed = 0, armed_parity = 0;
      bool ok = true;
      for (int64_t w = w0; w < w1 && ok; ++w) {
        const int tile = (int)(w / nk), kb = (int)(w % nk);
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, err)) {
          ok = false;
          break;
        }
        uint8_t *st = smem + stage * L::kStage;
        mbar_arrive_expect_tx(&full[stage], L::kStage);
        tma_load_2d(&tmW, &full[stage], st, kb * kBK, tile * kDecRows);
        tma_load_2d(&tmX, &full[stage], st + L::kW, kb * kBK, 0);
        armed |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == L::kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) {
        for (int s = 0; s < L::kStages; ++s)
          if (armed & (1u << s)) mbar_wait(&full[s], (armed_parity >> s) & 1u, nullptr, err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: one accumulation per segment ----------------
      constexpr uint32_t idesc = idesc8<F8>(kDecRows, MP);
      uint32_t stage = 0, phase = 0, ab = 0, aphase = 0;
      bool ok = true;
      for (int64_t w = w0; w < w1 && ok;) {
        const int tile = (int)(w / nk);
        const int64_t seg_end = w1 < (int64_t)(tile + 1) * nk ? w1 : (int64_t)(tile + 1) * nk;
        if (!mbar_wait(&tempty[ab], aphase ^ 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + ab * MP;
        for (int64_t i = w; i < seg_end; ++i) {
          if (!mbar_wait(&full[stage], phase, abort_flag, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t *st = smem + stage * L::kStage;
          const uint64_t a0 = desc_sw128_kmajor(smem_u32(st));
          const uint64_t b0 = desc_sw128_kmajor(smem_u32(st + L::kW));
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k)
            umma8<F8>(d, a0 + 2 * k, b0 + 2 * k, idesc, (i != w || k != 0) ? 1u : 0u);
          umma_commit(&empty[stage]);
          if (++stage == L::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[ab]);
        ab ^= 1;
        if (ab == 0) aphase ^= 1;
        w = seg_end;
      }
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, err);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..5: 128 threads, one Wq row each) ----------------
    const int q = warp & 3;
    const int et = threadIdx.x - 64;  // 0..127
    uint32_t ab = 0, aphase = 0;
    for (int64_t w = w0; w < w1;) {
      const int tile = (int)(w / nk);
      const int64_t seg_end = w1 < (int64_t)(tile + 1) * nk ? w1 : (int64_t)(tile + 1) * nk;
      const int seg_len = (int)(seg_end - w);
      // one decision for all four warps: they share named barriers below
      const bool ok = mbar_wait(&tfull[ab], aphase, abort_flag, err);
      if (!named_barrier_and(1, 128, ok)) break;
      tc_fence_after();
      const int n = tile * kDecRows + q * 32 + lane;
      const bool n_ok = n < N;
      const float dw = (KIND != OutKind::I32 && n_ok) ? __ldg(w_scale + n) : 0.0f;
      const bool whole = seg_len == nk;
#pragma unroll
      for (int c = 0; c < MP / 16; ++c) {
        uint32_t r[16];
        tmem_ld16(tmem_base + ((uint32_t)(q * 32) << 16) + ab * MP + c * 16, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int t = c * 16 + j;
          if (t < M && n_ok) {
            if (whole) {
              const float dx = KIND != OutKind::I32 ? __ldg(x_scale + t) : 0.0f;
              store_one<KIND, F8>(dst, ldy, t, n, r[j], dx, dw);
            } else if (r[j] != 0u) {
              // int32 sums are exact in any order; an f32 tile here has at
              // most two contributors (each CTA's share spans >= one tile's
              // k-blocks when tiles outnumber CTAs), and 0 + a + b rounds
              // the same in either order
              if constexpr (F8) {
                atomicAdd(reinterpret_cast<float *>(ws) + (int64_t)t * N + n, __uint_as_float(r[j]));
              } else {
                atomicAdd(ws + (int64_t)t * N + n, (int32_t)r[j]);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[ab]);
      if (!whole) {
        // publish this CTA's partial sums, then count its k-blocks
        __threadfence();
        named_barrier(1, 128);
        if (et == 0) {
          const unsigned before = atomicAdd(tile_count + tile, (unsigned)seg_len);
          *last_flag = (before + (unsigned)seg_len == (unsigned)nk) ? 1 : 0;
        }
        named_barrier(1, 128);
        if (*last_flag) {
          __threadfence();
          if (n_ok) {
            // 16 tokens at a time: their partial sums as independent L2
            // loads, then dequantize, store, and leave the workspace zero
#pragma unroll 1
            for (int t0 = 0; t0 < M; t0 += 16) {
              uint32_t acc[16];
#pragma unroll
              for (int j = 0; j < 16; ++j)
                acc[j] = t0 + j < M ? (uint32_t)__ldcg(ws + (int64_t)(t0 + j) * N + n) : 0u;
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const int t = t0 + j;
                if (t < M) {
                  const float dx = KIND != OutKind::I32 ? __ldg(x_scale + t) : 0.0f;
                  store_one<KIND, F8>(dst, ldy, t, n, acc[j], dx, dw);
                  __stcg(ws + (int64_t)t * N + n, 0);
                }
              }
            }
          }
          if (et == 0) tile_count[tile] = 0u;
        }
        named_barrier(1, 128);
      }
      ab ^= 1;
      if (ab == 0) aphase ^= 1;
      w = seg_end;
    }
  }

  // stores into other GPUs' memory (the column-parallel scatter) are made
  // visible system-wide before the kernel ends, so that the stream-ordered
  // collective that follows cannot overtake them
  if (dst.n > 1) __threadfence_system();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Decode-shaped linear, cluster split.  C clusters of S CTAs.  Cluster c
// owns the 128-row Wq tiles [nt c / C, nt (c+1) / C); its (tile, k-block)
// items, in tile-major order, are split evenly over its S CTAs.  A CTA's
// share is thus one or more segments: runs of k-blocks of one tile.  Each
// segment accumulates in its own TMEM columns (Wq rows on the MMA's M side,
// tokens on N, as in the stream-K kernel).  A segment that covers a whole
// tile is dequantized straight from TMEM.  A partial segment is parked in
// shared memory; after a cluster barrier, every CTA that contributed to a
// split tile sums its share of that tile's rows over all contributors'
// partials through distributed shared memory (int32 sums: exact; E4M3: f32
// sums taken in rank order) and dequantizes them.  No workspace, no global
// atomics.  The scales are read into shared memory while the weights stream.
// ---------------------------------------------------------------------------
constexpr int kDecMaxSegs = 16;   // segments per CTA (scale slots in shared memory)
constexpr int kDecMaxPeers = 8;   // CTAs per cluster

// A split tile's reduction, worked out once per CTA while the weights
// stream: the tile's contributors (ranks ra .. ra + cnt - 1), this CTA's
// share of its rows (4-row units [u0, u1) of 32), and where in each
// contributor's parked partials the tile's segment lies (word offsets).
struct DecSplit {
  int g, ra, cnt, u0, u1;
  uint32_t off[kDecMaxPeers];
};

// Segments that fit one CTA: TMEM columns (MP each, 512 in all), parking
// space in the drained ring (MP x 128 int32 each) and the scale slots.
template <int MP>
constexpr int dec_max_segs() {
  constexpr int by_tmem = 512 / MP;
  constexpr int by_smem = (int)(DecSmem<MP>::kRing / (MP * kDecRows * 4));
  constexpr int m = by_tmem < by_smem ? by_tmem : by_smem;
  return m < kDecMaxSegs ? m : kDecMaxSegs;
}

template <int MP>
struct DecClusterSmem {
  static constexpr uint32_t kRing = DecSmem<MP>::kRing;
  static constexpr uint32_t kBars = DecSmem<MP>::kBars;
  static constexpr uint32_t kScales = (kDecMaxSegs * kDecRows + MP) * 4;  // dw per segment row, dx per token
  static constexpr uint32_t kSplits = 2 * sizeof(DecSplit) + 16;           // at most two split tiles per CTA
  static constexpr uint32_t kTotal = kRing + kBars + kScales + kSplits + 1024;
};

// Item range [i0, i1) of CTA `rank` among S sharing I items.
__device__ __forceinline__ void dec_share(int I, int S, int rank, int &i0, int &i1) {
  i0 = (int)((int64_t)I * rank / S);
  i1 = (int)((int64_t)I * (rank + 1) / S);
}

template <OutKind KIND, bool F8>
__device__ __forceinline__ void store_four(const YDest &dst, int64_t ldy, int t, int n, const uint32_t (&acc)[4],
                                           float dx, const float *dw) {
  // four consecutive columns n..n+3 of row t (n % 4 == 0, so 8- or 16-byte aligned)
  const int64_t i = (int64_t)t * ldy + n;
  if constexpr (KIND == OutKind::I32) {
    const uint4 v = make_uint4(acc[0], acc[1], acc[2], acc[3]);
#pragma unroll 1
    for (int d = 0; d < dst.n; ++d) *reinterpret_cast<uint4 *>(static_cast<uint32_t *>(dst.p[d]) + i) = v;
  } else {
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = __fmul_rn(__fmul_rn(acc_value<F8>(acc[k]), dx), dw[k]);
    if constexpr (KIND == OutKind::F32) {
      const float4 f = make_float4(v[0], v[1], v[2], v[3]);
#pragma unroll 1
      for (int d = 0; d < dst.n; ++d) *reinterpret_cast<float4 *>(static_cast<float *>(dst.p[d]) + i) = f;
    } else {
      uint2 u;
      if constexpr (KIND == OutKind::BF16) {
        __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
        u = make_uint2(*reinterpret_cast<uint32_t *>(&a), *reinterpret_cast<uint32_t *>(&b));
      } else {
        __half2 a = __floats2half2_rn(v[0], v[1]), b = __floats2half2_rn(v[2], v[3]);
        u = make_uint2(*reinterpret_cast<uint32_t *>(&a), *reinterpret_cast<uint32_t *>(&b));
      }
#pragma unroll 1
      for (int d = 0; d < dst.n; ++d) *reinterpret_cast<uint2 *>(static_cast<uint16_t *>(dst.p[d]) + i) = u;
    }
  }
}

template <int MP, OutKind KIND, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
    w8a8_gemm_decode_cluster_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                                    const float *__restrict__ x_scale, const float *__restrict__ w_scale,
                                    const YDest dst, int64_t ldy, int M, int N, int K, int S, int C, uint32_t tcols,
                                    unsigned *err) {
  using L = DecClusterSmem<MP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kRing);
  uint64_t *empty = full + DecSmem<MP>::kStages;
  uint64_t *tfull = empty + DecSmem<MP>::kStages;
  uint64_t *drain = tfull + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  float *dws = reinterpret_cast<float *>(smem + L::kRing + L::kBars);  // [segment][128]
  float *dxs = dws + kDecMaxSegs * kDecRows;                            // [MP]
  DecSplit *splits = reinterpret_cast<DecSplit *>(dxs + MP);            // [2]
  int *nsplit = reinterpret_cast<int *>(splits + 2);
  // after the MMAs have drained the ring, it holds this CTA's partial
  // segments as part[segment][t][row] (t < MP, row < 128)
  uint32_t *part = reinterpret_cast<uint32_t *>(smem);
  constexpr int kStages = DecSmem<MP>::kStages;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = S > 1 ? (int)cluster_ctarank() : 0;
  const int cid = blockIdx.x / S;
  const int nt = (N + kDecRows - 1) / kDecRows;
  const int nk = (K + kBK - 1) / kBK;
  const int tile0 = (int)((int64_t)nt * cid / C);  // the cluster's first tile
  const int I = ((int)((int64_t)nt * (cid + 1) / C) - tile0) * nk;
  int i0, i1;
  dec_share(I, S, rank, i0, i1);
  const int lt_first = i0 / nk;  // local index of the first tile this CTA touches
  const int nseg = i1 > i0 ? (i1 - 1) / nk - lt_first + 1 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmX);
    // the first ring's worth of this CTA's Wq boxes, into L2 while the
    // previous kernel may still run (weights do not depend on it, and L2
    // stays coherent if it does write them)
    int n = 0;
    for (int g = 0; g < nseg && n < kStages; ++g) {
      const int lt = lt_first + g;
      const int a = max(i0, lt * nk) - lt * nk, b = min(i1, (lt + 1) * nk) - lt * nk;
      const int len = b - a, rot = (tile0 + lt) % len;
      for (int j = 0; j < len && n < kStages; ++j, ++n)
        tma_prefetch_l2_2d(&tmW, (a + (j + rot) % len) * kBK, (tile0 + lt) * kDecRows);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // prologue done; the previous kernel's results are visible from here on
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      uint32_t stage = 0, phase = 0, armed = 0, armed_parity = 0;
      bool ok = true;
      for (int g = 0; g < nseg && ok; ++g) {
        const int lt = lt_first + g;
        const int a = max(i0, lt * nk) - lt * nk, b = min(i1, (lt + 1) * nk) - lt * nk;  // k-blocks [a, b)
        const int len = b - a;
        // tiles start their k-walk at different k-blocks so that the CTAs
        // of the grid do not all fetch the same Xq tile from L2 at once
        // (the segment's sum does not depend on the order)
        const int rot = (tile0 + lt) % len;
        for (int j = 0; j < len; ++j) {
          const int kb = a + (j + rot) % len;
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, err)) {
            ok = false;
            break;
          }
          uint8_t *st = smem + stage * DecSmem<MP>::kStage;
          mbar_arrive_expect_tx(&full[stage], DecSmem<MP>::kStage);
          tma_load_2d(&tmW, &full[stage], st, kb * kBK, (tile0 + lt) * kDecRows);
          tma_load_2d(&tmX, &full[stage], st + DecSmem<MP>::kW, kb * kBK, 0);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        for (int s = 0; s < kStages; ++s)
          if (armed & (1u << s)) mbar_wait(&full[s], (armed_parity >> s) & 1u, nullptr, err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: one accumulator per segment ----------------
      constexpr uint32_t idesc = idesc8<F8>(kDecRows, MP);
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (int g = 0; g < nseg && ok; ++g) {
        const int lt = lt_first + g;
        const int len = min(i1, (lt + 1) * nk) - max(i0, lt * nk);
        const uint32_t d = tmem_base + (uint32_t)(g * MP);
        for (int j = 0; j < len; ++j) {
          if (!mbar_wait(&full[stage], phase, abort_flag, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t *st = smem + stage * DecSmem<MP>::kStage;
          const uint64_t a0 = desc_sw128_kmajor(smem_u32(st));
          const uint64_t b0 = desc_sw128_kmajor(smem_u32(st + DecSmem<MP>::kW));
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k)
            umma8<F8>(d, a0 + 2 * k, b0 + 2 * k, idesc, (j != 0 || k != 0) ? 1u : 0u);
          umma_commit(&empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      umma_commit(tfull);  // also arrives when no MMA was issued
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, err);
    }
    __syncwarp();
  } else {
    // ---- epilogue warps, while the weights stream: the scales this CTA
    // will need, into shared memory, and the layout of its split tiles ----
    const int e = threadIdx.x - 64;  // 0..127
    if (KIND != OutKind::I32) {
      for (int g = 0; g < nseg; ++g) {
        const int n = (tile0 + lt_first + g) * kDecRows + e;
        dws[g * kDecRows + e] = n < N ? __ldg(w_scale + n) : 0.0f;
      }
      if (e < M) dxs[e] = __ldg(x_scale + e);
    }
    if (e == 0) {
      // only a CTA's first and last segments can be parts of a tile
      int ns = 0;
      for (int g = 0; g < nseg; g += (nseg > 1 ? nseg - 1 : 1)) {
        const int lt = lt_first + g;
        if (min(i1, (lt + 1) * nk) - max(i0, lt * nk) == nk) continue;  // a whole tile
        DecSplit &sp = splits[ns++];
        sp.g = g;
        sp.ra = -1;
        int rb = -1;
        for (int r = 0; r < S; ++r) {  // the CTAs whose item ranges meet the tile
          int a, b;
          dec_share(I, S, r, a, b);
          if (a < b && a < (lt + 1) * nk && b > lt * nk) {
            if (sp.ra < 0) sp.ra = r;
            rb = r;
            sp.off[rb - sp.ra] = (uint32_t)((lt - a / nk) * MP * kDecRows);
          }
        }
        sp.cnt = rb - sp.ra + 1;
        sp.u0 = (rank - sp.ra) * (kDecRows / 4) / sp.cnt;
        sp.u1 = (rank - sp.ra + 1) * (kDecRows / 4) / sp.cnt;
      }
      *nsplit = ns;
    }
  }

  // ---- epilogue: accumulators -> output (whole tiles) or shared memory ----
  const bool epi = warp >= 2;
  const int q = warp & 3;
  const int row = q * 32 + lane;  // 0..127 for the epilogue warps
  bool ok = true;
  if (epi) ok = mbar_wait(tfull, 0, abort_flag, err);
  ok = __syncthreads_and(ok);  // every thread of the CTA takes the same path; scales visible
  if (ok && epi) {
    tc_fence_after();
    for (int g = 0; g < nseg; ++g) {
      const int lt = lt_first + g;
      const bool whole = min(i1, (lt + 1) * nk) - max(i0, lt * nk) == nk;
      const int n = (tile0 + lt) * kDecRows + row;
      const float dw = dws[g * kDecRows + row];
#pragma unroll
      for (int c = 0; c < MP / 16; ++c) {
        uint32_t r[16];
        tmem_ld16(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(g * MP + c * 16), r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int t = c * 16 + j;
          if (whole) {
            if (t < M && n < N) store_one<KIND, F8>(dst, ldy, t, n, r[j], dxs[t], dw);
          } else if (t < M) {
            part[(g * MP + t) * kDecRows + row] = r[j];
          }
        }
      }
    }
  }
  if (S > 1) {
    // every CTA's partials in place (and visible cluster-wide)
    cluster_sync();
    if (ok && epi) {
      const int e = threadIdx.x - 64;
      const uint32_t part_addr = smem_u32(part);
      for (int si = 0; si < *nsplit; ++si) {
        const DecSplit &sp = splits[si];
        const int lt = lt_first + sp.g, units = sp.u1 - sp.u0, total = units * M;
        // two (token, 4-row) items per thread and round: all their
        // contributors' partials are requested before any is summed
        for (int i0r = e; i0r < total; i0r += 256) {
          uint4 v[2][kDecMaxPeers];
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            const int idx = i0r + b * 128;
            if (idx < total) {
              const int t = idx / units, rr = (sp.u0 + idx % units) * 4;
#pragma unroll
              for (int p = 0; p < kDecMaxPeers; ++p)
                if (p < sp.cnt)
                  v[b][p] = ld_shared_cluster_v4(
                      mapa_shared(part_addr + (sp.off[p] + (uint32_t)(t * kDecRows + rr)) * 4u, (uint32_t)(sp.ra + p)));
            }
          }
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            const int idx = i0r + b * 128;
            if (idx < total) {
              const int t = idx / units, rr = (sp.u0 + idx % units) * 4;
              // int32 sums, or (E4M3) f32 sums taken in rank order
              uint32_t sum[4] = {0u, 0u, 0u, 0u};
#pragma unroll
              for (int p = 0; p < kDecMaxPeers; ++p)
                if (p < sp.cnt) {
                  const uint32_t w4[4] = {v[b][p].x, v[b][p].y, v[b][p].z, v[b][p].w};
#pragma unroll
                  for (int k = 0; k < 4; ++k) {
                    if constexpr (F8) {
                      sum[k] = __float_as_uint(__fadd_rn(__uint_as_float(sum[k]), __uint_as_float(w4[k])));
                    } else {
                      sum[k] += w4[k];
                    }
                  }
                }
              const int n = (tile0 + lt) * kDecRows + rr;
              if (n < N) store_four<KIND, F8>(dst, ldy, t, n, sum, dxs[t], dws + sp.g * kDecRows + rr);
            }
          }
        }
      }
    }
    cluster_sync();  // no CTA leaves while a peer still reads its partials
  }
  // stores into other GPUs' memory (the column-parallel scatter) are made
  // visible system-wide before the kernel ends, so that the stream-ordered
  // collective that follows cannot overtake them
  if (dst.n > 1) __threadfence_system();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tcols);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D int8 tensor map over a [rows][cols] row-major matrix (row stride
// `cols` bytes), box of box_rows x 128 bytes with 128-byte swizzling.
bool make_tmap_i8(CUtensorMap *m, const int8_t *base, int64_t rows, int64_t cols, int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols};
  cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, int STAGES, OutKind KIND, bool F8>
cudaError_t launch_tc(const CUtensorMap &tmA, const CUtensorMap &tmB, const float *x_scale, const float *w_scale,
                      const YDest &dst, int64_t ldy, int M, int N, int K, cudaStream_t st) {
  using L = GemmSmem<BN, STAGES>;
  auto kern = w8a8_gemm_tc_kernel<BN, STAGES, KIND, F8>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kTotal);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int tiles = ((M + kBM - 1) / kBM) * ((N + BN - 1) / BN);
  const int grid = tiles < num_sms() ? tiles : num_sms();
  return launch_pdl(kern, dim3(grid), dim3(kThreads), L::kTotal, st, 1, tmA, tmB, x_scale, w_scale, dst, ldy, M, N, K,
                    device_error_word());
}

template <int BN, int STAGES, OutKind KIND, bool F8>
cudaError_t launch_pair(const CUtensorMap &tmA, const CUtensorMap &tmB, const float *x_scale, const float *w_scale,
                        const YDest &dst, int64_t ldy, int M, int N, int K, int max_clusters, cudaStream_t st) {
  using L = PairSmem<BN, STAGES>;
  auto kern = w8a8_gemm_pair_kernel<BN, STAGES, KIND, F8>;
  const int tiles = ((M + 2 * kBM - 1) / (2 * kBM)) * ((N + BN - 1) / BN);
  const int clusters = tiles < max_clusters ? tiles : max_clusters;
  return launch_pdl(kern, dim3(2 * clusters), dim3(kThreads), L::kTotal, st, 2, tmA, tmB, x_scale, w_scale, dst, ldy, M,
                    N, K, device_error_word());
}

// Clusters of two 1-CTA-per-SM blocks that fit on the device at once.
template <int BN, int STAGES, OutKind KIND, bool F8>
int pair_capacity() {
  using L = PairSmem<BN, STAGES>;
  static int cache[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  int &c = cache[dev & 63];
  if (c == 0) {
    auto kern = w8a8_gemm_pair_kernel<BN, STAGES, KIND, F8>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kTotal) != cudaSuccess)
      return -1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = L::kTotal;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) return -1;
    c = n;
  }
  return c;
}

// Ring depths that fill ~224 KB of shared memory at each tile width.
template <int BN>
constexpr int pair_stages() {
  return (int)((224u * 1024u) / PairSmem<BN, 1>::kRing);
}

template <int BN, OutKind KIND, bool F8>
cudaError_t run_pair(const int8_t *xq, const float *x_scale, const int8_t *wq, const float *w_scale, int M, int N,
                     int K, const YDest &dst, int64_t ldy, int pairs, cudaStream_t st) {
  CUtensorMap tmA, tmB;
  if (!make_tmap_i8(&tmA, xq, M, K, kBM)) return cudaErrorInvalidValue;
  if (!make_tmap_i8(&tmB, wq, N, K, BN / 2)) return cudaErrorInvalidValue;
  constexpr int S = pair_stages<BN>();
  const int cap = pair_capacity<BN, S, KIND, F8>();
  if (cap <= 0) return cudaErrorLaunchOutOfResources;
  return launch_pair<BN, S, KIND, F8>(tmA, tmB, x_scale, w_scale, dst, ldy, M, N, K, cap < pairs ? cap : pairs, st);
}

template <int MP, OutKind KIND, bool F8>
void prepare_decode_cluster_kernel() {
  using L = DecClusterSmem<MP>;
  static bool done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!done[dev & 63]) {
    auto kern = w8a8_gemm_decode_cluster_kernel<MP, KIND, F8>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kTotal);
    cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    done[dev & 63] = true;
  }
}

// Clusters of S one-CTA-per-SM blocks of the decode cluster kernel that can
// be resident at once (0 if none or the query fails).
template <int MP, OutKind KIND, bool F8>
int cluster_capacity(int S) {
  using L = DecClusterSmem<MP>;
  if (S == 1) return num_sms();
  static int cache[64][kDecMaxPeers + 1] = {};  // [device][S]
  int dev = 0;
  cudaGetDevice(&dev);
  int &c = cache[dev & 63][S];
  if (c == 0) {
    prepare_decode_cluster_kernel<MP, KIND, F8>();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(S, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = L::kTotal;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, w8a8_gemm_decode_cluster_kernel<MP, KIND, F8>, &cfg) != cudaSuccess) {
      cudaGetLastError();  // clear the query's error
      n = -1;
    }
    c = n > 0 ? n : -1;
  }
  return c > 0 ? c : 0;
}

// How a decode-shaped product is laid over the SMs: C clusters of S CTAs
// (cluster split, no workspace), or the stream-K kernel over the workspace.
struct DecodePlan {
  bool cluster = false;
  int S = 1, C = 0;
  uint32_t tcols = 32;  // TMEM columns per CTA of the cluster kernel
};

// Extra cost of splitting tiles across a cluster (two cluster barriers, and
// partial sums of M tokens through distributed shared memory), in k-blocks
// streamed by one CTA: 6 + M / 4, fitted to timed launches of the Llama-2
// decode shapes (M = 1 .. 64).
inline int dec_split_cost(int M) { return 6 + M / 4; }

// The plan for a decode-shaped product of M tokens on the current device.
//  - More tiles than SMs and at most 32 tokens: the stream-K kernel.  Every
//    CTA's share then spans at least one tile's k-blocks, so a split tile
//    has at most two contributors: their int32 partials, and E4M3 (f32)
//    ones too, add to the same value in either order.
//  - Otherwise the cluster split with the least cost: the k-blocks its
//    busiest CTA streams, plus dec_split_cost(M) when tiles are split (ties:
//    fewer CTAs per cluster), among the splits whose segments fit one CTA;
//    the stream-K kernel if none fits and tiles outnumber the SMs.
// Residency is taken from one instantiation of the cluster kernel: all of
// them use the same shared memory and one CTA per SM, and a plan that named
// more clusters than fit would still be correct (clusters do not wait for
// one another), only slower.
template <int MP>
DecodePlan plan_decode(int M, int N, int K) {
  const int nt = (N + kDecRows - 1) / kDecRows, nk = (K + kBK - 1) / kBK, sms = num_sms();
  DecodePlan best;
  if (nt > sms && M <= 32) return best;
  int64_t best_cost = INT64_MAX;
  for (int S = 1; S <= kDecMaxPeers; ++S) {
    const int cap = cluster_capacity<MP, OutKind::BF16, false>(S);
    int C = nt < sms / S ? nt : sms / S;
    if (cap < C) C = cap;
    if (C <= 0) continue;
    const int64_t tmax = (nt + C - 1) / C;              // tiles of the largest cluster
    // every CTA of the smallest cluster gets items, so that a split tile's
    // contributors are consecutive ranks (the split cost keeps such plans
    // out anyway; this states it)
    if (S > 1 && (nt / C) * nk < S) continue;
    const int64_t items = (tmax * nk + S - 1) / S;       // k-blocks of its busiest CTA
    int64_t segs = items == 0 ? 0 : (items + nk - 1) / nk + 1;
    if (segs > tmax) segs = tmax;
    if (segs > dec_max_segs<MP>()) continue;
    const int64_t cost = items + (S > 1 ? dec_split_cost(M) : 0);
    if (cost < best_cost) {
      best_cost = cost;
      best.cluster = true;
      best.S = S;
      best.C = C;
      uint32_t need = (uint32_t)(segs * MP), cols = 32;
      while (cols < need) cols *= 2;
      best.tcols = cols;
    }
  }
  // (with no fitting split and no more tiles than SMs, S = 1 always fits:
  // one tile per CTA is one segment)
  return best;
}

// Whether the decode-shaped product takes the stream-K kernel (and so the
// workspace) on the current device.
bool decode_plan_uses_workspace(int M, int N, int K) {
  if (M <= 16) return !plan_decode<16>(M, N, K).cluster;
  if (M <= 32) return !plan_decode<32>(M, N, K).cluster;
  if (M <= 48) return !plan_decode<48>(M, N, K).cluster;
  return !plan_decode<64>(M, N, K).cluster;
}

template <int MP, OutKind KIND, bool F8>
cudaError_t launch_decode(const int8_t *xq, const float *x_scale, const int8_t *wq, const float *w_scale, int M,
                          int N, int K, const YDest &dst, int64_t ldy, void *workspace, cudaStream_t st) {
  CUtensorMap tmW, tmX;
  if (!make_tmap_i8(&tmW, wq, N, K, kDecRows)) return cudaErrorInvalidValue;
  if (!make_tmap_i8(&tmX, xq, M, K, MP)) return cudaErrorInvalidValue;
  const DecodePlan plan = plan_decode<MP>(M, N, K);
  if (plan.cluster) {
    prepare_decode_cluster_kernel<MP, KIND, F8>();
    return launch_pdl(w8a8_gemm_decode_cluster_kernel<MP, KIND, F8>, dim3(plan.C * plan.S), dim3(kThreads),
                      DecClusterSmem<MP>::kTotal, st, (unsigned)plan.S, tmW, tmX, x_scale, w_scale, dst, ldy, M, N,
                      K, plan.S, plan.C, plan.tcols, device_error_word());
  }
  using L = DecSmem<MP>;
  auto kern = w8a8_gemm_decode_kernel<MP, KIND, F8>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr_set[dev & 63]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kTotal);
    if (e != cudaSuccess) return e;
    attr_set[dev & 63] = true;
  }
  const int nt = (N + kDecRows - 1) / kDecRows, nk = (K + kBK - 1) / kBK;
  const int64_t items = (int64_t)nt * nk;
  const int grid = (int)(items < num_sms() ? items : num_sms());
  int32_t *ws = static_cast<int32_t *>(workspace);
  unsigned *counts = reinterpret_cast<unsigned *>(static_cast<uint8_t *>(workspace) + decode_ws_elems(M, N) * 4);
  return launch_pdl(kern, dim3(grid), dim3(kThreads), L::kTotal, st, 1, tmW, tmX, x_scale, w_scale, dst, ldy, M, N, K,
                    ws, counts, device_error_word());
}

template <OutKind KIND, bool F8>
cudaError_t gemm_dispatch(const int8_t *xq, const float *x_scale, const int8_t *wq, const float *w_scale, int M,
                          int N, int K, const YDest &dst, int64_t ldy, void *workspace, cudaStream_t st) {
  if (M <= kDecodeMaxM) {  // weight-streaming regime
    if (M <= 16) return launch_decode<16, KIND, F8>(xq, x_scale, wq, w_scale, M, N, K, dst, ldy, workspace, st);
    if (M <= 32) return launch_decode<32, KIND, F8>(xq, x_scale, wq, w_scale, M, N, K, dst, ldy, workspace, st);
    if (M <= 48) return launch_decode<48, KIND, F8>(xq, x_scale, wq, w_scale, M, N, K, dst, ldy, workspace, st);
    return launch_decode<64, KIND, F8>(xq, x_scale, wq, w_scale, M, N, K, dst, ldy, workspace, st);
  }
  const int sms = num_sms();
  CUtensorMap tmA, tmB;
  // CTA pairs once there are enough 256 x 256 tiles to occupy every pair
  const int tiles_pair = ((M + 255) / 256) * ((N + 255) / 256);
  const int cap = pair_capacity<256, pair_stages<256>(), KIND, F8>();
  if (cap > 0 && tiles_pair >= cap) {
    return run_pair<256, KIND, F8>(xq, x_scale, wq, w_scale, M, N, K, dst, ldy, cap, st);
  }
  const int tiles256 = ((M + kBM - 1) / kBM) * ((N + 255) / 256);
  const bool wide = tiles256 >= sms || (N % 256 == 0 && tiles256 * 2 > sms);
  if (!make_tmap_i8(&tmA, xq, M, K, kBM)) return cudaErrorInvalidValue;
  if (wide) {
    if (!make_tmap_i8(&tmB, wq, N, K, 256)) return cudaErrorInvalidValue;
    return launch_tc<256, 4, KIND, F8>(tmA, tmB, x_scale, w_scale, dst, ldy, M, N, K, st);
  }
  if (!make_tmap_i8(&tmB, wq, N, K, 128)) return cudaErrorInvalidValue;
  return launch_tc<128, 6, KIND, F8>(tmA, tmB, x_scale, w_scale, dst, ldy, M, N, K, st);
}

}  // namespace

bool w8a8_decode_uses_workspace(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || M > kDecodeMaxM) return false;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return true;  // no device to plan for: assume the workspace path
  }
  return decode_plan_uses_workspace((int)M, (int)N, (int)K);
}

size_t w8a8_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (!w8a8_decode_uses_workspace(M, N, K)) return 0;
  return decode_ws_elems(M, N) * 4 + decode_counter_bytes(N);
}

template <bool F8>
cudaError_t gemm_kind(const int8_t *xq, const float *x_scale, const int8_t *wq, const float *w_scale, int m, int n,
                      int k, const YDest &dst, OutKind kind, int64_t ldy, void *ws, cudaStream_t st) {
  switch (kind) {
    case OutKind::F32: return gemm_dispatch<OutKind::F32, F8>(xq, x_scale, wq, w_scale, m, n, k, dst, ldy, ws, st);
    case OutKind::F16: return gemm_dispatch<OutKind::F16, F8>(xq, x_scale, wq, w_scale, m, n, k, dst, ldy, ws, st);
    case OutKind::BF16: return gemm_dispatch<OutKind::BF16, F8>(xq, x_scale, wq, w_scale, m, n, k, dst, ldy, ws, st);
    default: return gemm_dispatch<OutKind::I32, F8>(xq, nullptr, wq, nullptr, m, n, k, dst, ldy, ws, st);
  }
}

cudaError_t launch_w8a8_gemm_dest(const int8_t *xq, const float *x_scale, const int8_t *wq, const float *w_scale,
                                  int64_t M, int64_t N, int64_t K, const YDest &dst, OutKind kind, int64_t ldy,
                                  void *ws, cudaStream_t st, QFmt fmt) {
  const int m = (int)M, n = (int)N, k = (int)K;
  if (fmt == QFmt::E4M3) return gemm_kind<true>(xq, x_scale, wq, w_scale, m, n, k, dst, kind, ldy, ws, st);
  return gemm_kind<false>(xq, x_scale, wq, w_scale, m, n, k, dst, kind, ldy, ws, st);
}

cudaError_t launch_w8a8_gemm(const int8_t *xq, const float *x_scale, const int8_t *wq, const float *w_scale,
                             int64_t M, int64_t N, int64_t K, void *y, OutKind kind, int64_t ldy, void *ws, size_t,
                             cudaStream_t st, QFmt fmt) {
  YDest dst{};
  dst.p[0] = y;
  dst.n = 1;
  return launch_w8a8_gemm_dest(xq, x_scale, wq, w_scale, M, N, K, dst, kind, ldy, ws, st, fmt);
}

}  // namespace sq

// ---------------------------------------------------------------------------
// Allocation-free decode entry point: the decode kernel's workspace comes
// from a scratch array compiled into this library instead of from the
// caller.  Its host-side name is not a device address, so the address is
// looked up once per device (cudaGetSymbolAddress, that device current).
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t sq_decode_scratch[SQ_DECODE_STATIC_SCRATCH_BYTES];

namespace {

// Device address of sq_decode_scratch on the current device, looked up on
// the first call per device; nullptr (and *err set) if the lookup fails.
void *decode_scratch_address(cudaError_t *err) {
  static void *addr[64] = {};
  static std::mutex mu;
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void *p = nullptr;
    *err = cudaGetSymbolAddress(&p, sq_decode_scratch);
    if (*err != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

bool is_aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" size_t sq_decode_static_scratch_bytes(void) { return SQ_DECODE_STATIC_SCRATCH_BYTES; }

extern "C" sq_status sq_w8a8_linear_decode_noalloc(const int8_t *xq, const float *x_scale, const int8_t *wq,
                                                   const float *w_scale, int64_t M, int64_t N, int64_t K, void *y,
                                                   sq_dtype yt, int64_t ldy, sq_stream_t stream) {
  SQ_TRACE_CALL();
  if (yt != SQ_F32 && yt != SQ_F16 && yt != SQ_BF16) return SQ_ERR_INVALID_ARG;
  const int64_t ysize = yt == SQ_F32 ? 4 : 2;
  if (M < 0 || N <= 0 || K <= 0 || N % 16 != 0 || K % 16 != 0 || N >= ((int64_t)1 << 31) ||
      K >= ((int64_t)1 << 31))
    return SQ_ERR_INVALID_ARG;
  if (ldy < N || (ldy * ysize) % 16 != 0) return SQ_ERR_INVALID_ARG;
  if (wq == nullptr || w_scale == nullptr || !is_aligned16(wq) || !is_aligned16(w_scale)) return SQ_ERR_INVALID_ARG;
  if (M == 0) return SQ_OK;
  if (xq == nullptr || x_scale == nullptr || y == nullptr || !is_aligned16(xq) || !is_aligned16(x_scale) ||
      !is_aligned16(y))
    return SQ_ERR_INVALID_ARG;
  if (M > sq::kDecodeMaxM) return SQ_ERR_UNSUPPORTED;
  const size_t need = sq::w8a8_workspace_bytes(M, N, K);
  if (need > SQ_DECODE_STATIC_SCRATCH_BYTES) return SQ_ERR_UNSUPPORTED;
  cudaError_t e = cudaSuccess;
  void *scratch = nullptr;
  if (need > 0) {  // a shape on the cluster split uses no scratch at all
    scratch = decode_scratch_address(&e);
    if (scratch == nullptr) return SQ_ERR_CUDA;
  }
  cudaStream_t st = (cudaStream_t)stream;
  const sq::OutKind kind = yt == SQ_F32 ? sq::OutKind::F32 : yt == SQ_F16 ? sq::OutKind::F16 : sq::OutKind::BF16;
  // the stream-K decode kernel expects zero partial sums and zero tile
  // counters (cleared on every call: a call that timed out may have left
  // them dirty)
  if (need > 0 && cudaMemsetAsync(scratch, 0, need, st) != cudaSuccess) return SQ_ERR_CUDA;
  e = sq::launch_w8a8_gemm(xq, x_scale, wq, w_scale, M, N, K, y, kind, ldy, scratch, need, st, sq::QFmt::I8);
  return e == cudaSuccess ? SQ_OK : SQ_ERR_CUDA;
}
