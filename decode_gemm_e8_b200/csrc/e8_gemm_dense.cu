// Dense bf16 GEMM on the 5th-generation tensor cores: Y = X * W^T.
//
// Used for large batches after the weights were decoded to bf16 (the full-row
// inverse Hadamard transform mixes every K tile, so for prefill-sized M the
// weights are reconstructed once into a workspace and read by this kernel).
//
// Persistent, warp specialised, one CTA per SM:
//   warp 0      TMA producer: X tile 128x64 and W tile 256x64 (128-byte
//               swizzle) into a 4-stage shared-memory ring
//   warp 1      allocates tensor memory, one thread issues tcgen05.mma
//               (M=128, N=256, K=16) into a double-buffered fp32 accumulator
//               (2 x 256 TMEM columns) and commits stages back to the producer
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//               lanes 32*(w%4)...), fp32 stores to Y, then frees the buffer
// Every wait is bounded; a wait that gives up marks the device status word and
// all roles leave their loops.
#include "e8_common.cuh"
#include "e8_internal.h"
#include "e8_tmap.h"

namespace e8 {

namespace dg {
constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 512;
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + 256;
}  // namespace dg

// Wait used only while shutting down after another role gave up: ignores the
// abort flag but still ends after `limit_ns`.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

__global__ void __launch_bounds__(dg::THREADS, 1)
    k_dense_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 float* __restrict__ Y, int M, int N, int K, uint32_t* status) {
  using namespace dg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = (M + BM - 1) / BM, tiles_n = (N + BN - 1) / BN;
  const int tiles = tiles_m * tiles_n;
  const int kblocks = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      int s = 0;
      uint32_t ph = 0;
      uint32_t issued = 0;
      for (int tile = blockIdx.x; tile < tiles && !*abort_flag; tile += gridDim.x) {
        const int tm = tile % tiles_m, tn = tile / tiles_m;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, status, kDevTimeoutEmpty)) break;
          uint8_t* st = smem + s * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          tma_load_2d(st, &tmA, &full[s], kb * BK, tm * BM);
          tma_load_2d(st + A_BYTES, &tmB, &full[s], kb * BK, tn * BN);
          ++issued;
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      if (*abort_flag) {
        // let copies already in flight land before the CTA can exit
        for (uint32_t j = 0; j < STAGES && j < issued; ++j) {
          uint32_t idx = issued - 1 - j;
          mbar_wait_drain(&full[idx % STAGES], (idx / STAGES) & 1u, 100000000ull);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BM, BN);
      int s = 0;
      uint32_t ph = 0;
      int local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++local) {
        const int buf = local & 1;
        const uint32_t aph = (uint32_t)(local >> 1) & 1u;
        if (!mbar_wait_bounded(&acc_empty[buf], aph ^ 1u, abort_flag, status, kDevTimeoutMma)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_bounded(&full[s], ph, abort_flag, status, kDevTimeoutFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = smem_desc(a_addr + k * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(b_addr + k * 32, 16, 1024, 2);
            mma_ss(d_tmem, ad, bd, idesc, (kb > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit(&empty[s]);
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
        if (ok) mma_commit(&acc_full[buf]);
      }
      // all MMAs issued by this thread have finished once `drain` flips
      mma_commit(drain);
      mbar_wait_drain(drain, 0, 200000000ull);
    }
  } else {
    const int quarter = warp & 3;
    const int row_in_tile = quarter * 32 + lane;
    const bool vec4 = (N & 3) == 0;
    int local = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++local) {
      const int buf = local & 1;
      const uint32_t aph = (uint32_t)(local >> 1) & 1u;
      if (!mbar_wait_bounded(&acc_full[buf], aph, abort_flag, status, kDevTimeoutMma)) break;
      tc_fence_after();
      const int tm = tile % tiles_m, tn = tile / tiles_m;
      const int row = tm * BM + row_in_tile;
      float* yrow = Y + (size_t)row * N;
      for (int c = 0; c < BN; c += 16) {
        uint32_t r[16];
        tmem_ld16(tmem_base + (uint32_t)(buf * BN + c) + ((uint32_t)(quarter * 32) << 16), r);
        tmem_ld_wait();
        const int col = tn * BN + c;
        if (row < M) {
          if (vec4 && col + 16 <= N) {
#pragma unroll
            for (int j = 0; j < 16; j += 4)
              *reinterpret_cast<float4*>(yrow + col + j) =
                  make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                              __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (col + j < N) yrow[col + j] = __uint_as_float(r[j]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Two-SM variant: a cluster of two CTAs computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16).  CTA r of the pair holds
// rows r*128.. of the X tile and rows r*128.. of the W tile in its shared
// memory and rows r*128.. of the accumulator in its tensor memory; the even
// CTA (the leader) issues the MMAs for both.  Per 64-deep K step each SM now
// loads 32 KB for 128 x 256 x 64 products, two thirds of the one-SM tile's
// 48 KB, so six stages in flight cover the load latency.
//   warp 0      TMA producer of both CTAs: its halves of the X and W tiles;
//               the copies of both CTAs complete on the leader's barrier
//   warp 1      tensor-memory allocation (both CTAs, cta_group::2); in the
//               leader one thread issues the MMAs and the commits, which
//               arrive on the barriers of both CTAs
//   warps 2-5   epilogue of each CTA: its 128 accumulator rows -> Y, then a
//               release of the buffer on the leader's barrier
// No TMA multicast: every copy reads global memory into its own CTA.
namespace dg2 {
constexpr int BM = 256, BN = 256, BK = 64, STAGES = 6;
constexpr int HALF_BYTES = 128 * BK * 2;            // 128 rows of a 64-wide bf16 K step
constexpr int STAGE_BYTES = 2 * HALF_BYTES;         // X half + W half, per CTA
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 512;                      // two 256-column fp32 accumulators
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + 256;
constexpr uint32_t kPeerBitMask = 0xFEFFFFFFu;      // shared::cluster address -> the even CTA
}  // namespace dg2

__device__ __forceinline__ void tmem_alloc_2sm(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_2sm() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_2sm(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void mma_ss_2sm(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives, when this thread's MMAs are complete, on the barrier at the same
// shared-memory offset in each CTA of `mask` (a commit, not a data copy).
__device__ __forceinline__ void mma_commit_2sm_mc(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(mask)
      : "memory");
}
__device__ __forceinline__ void mma_commit_2sm(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// 2-D tile load into this CTA's shared memory whose completion is counted on
// the barrier at shared::cluster address `bar` (the leader's).
__device__ __forceinline__ void tma_load_2d_2sm(void* smem_dst, const CUtensorMap* map,
                                                uint32_t bar, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

__global__ void __launch_bounds__(dg2::THREADS, 1)
    k_dense_gemm2(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  float* __restrict__ Y, int M, int N, int K, uint32_t* status) {
  using namespace dg2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = (int)blockIdx.x >> 1, npairs = (int)gridDim.x >> 1;
  const int tiles_m = (M + BM - 1) / BM, tiles_n = (N + BN - 1) / BN;
  const int tiles = tiles_m * tiles_n;
  const int kblocks = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);    // the leader's producer; both CTAs' copies add bytes
      mbar_init(&empty[s], 1);   // the leader's commit, multicast to both CTAs
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 8);   // four epilogue warps of each CTA (used in the leader)
    }
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_2sm(tmem_slot, TMEM_COLS);
    tmem_relinquish_2sm();
  }
  // both CTAs' barriers are initialised before any copy or commit reaches them
  tc_fence_before();
  cluster_arrive();
  cluster_wait();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      int s = 0;
      uint32_t ph = 0;
      for (int tile = pair; tile < tiles && !*abort_flag; tile += npairs) {
        const int tm = tile % tiles_m, tn = tile / tiles_m;
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, status, kDevTimeoutEmpty)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * STAGE_BYTES;
          if (leader) mbar_arrive_expect_tx(&full[s], 2u * STAGE_BYTES);
          const uint32_t bar = smem_u32(&full[s]) & kPeerBitMask;
          tma_load_2d_2sm(st, &tmA, bar, kb * BK, tm * BM + (int)rank * 128);
          tma_load_2d_2sm(st + HALF_BYTES, &tmB, bar, kb * BK, tn * BN + (int)rank * 128);
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        // copies in flight may still land: give them time before the CTA exits
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 1000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BM, BN);
      int s = 0;
      uint32_t ph = 0;
      int local = 0;
      bool ok = true;
      for (int tile = pair; tile < tiles && ok; tile += npairs, ++local) {
        const int buf = local & 1;
        const uint32_t aph = (uint32_t)(local >> 1) & 1u;
        if (!mbar_wait_bounded(&acc_empty[buf], aph ^ 1u, abort_flag, status, kDevTimeoutMma)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_bounded(&full[s], ph, abort_flag, status, kDevTimeoutFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t b_addr = a_addr + HALF_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = smem_desc(a_addr + k * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(b_addr + k * 32, 16, 1024, 2);
            mma_ss_2sm(d_tmem, ad, bd, idesc, (kb > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit_2sm_mc(&empty[s], 0x3);
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
        if (ok) mma_commit_2sm_mc(&acc_full[buf], 0x3);
      }
      // every MMA of this thread has finished once `drain` flips
      mma_commit_2sm(drain);
      mbar_wait_drain(drain, 0, 200000000ull);
    }
  } else {
    const int quarter = warp & 3;
    const int row_in_tile = (int)rank * 128 + quarter * 32 + lane;
    const bool vec4 = (N & 3) == 0;
    const uint32_t leader_acc_empty0 = mapa_shared(smem_u32(&acc_empty[0]), 0);
    int local = 0;
    for (int tile = pair; tile < tiles; tile += npairs, ++local) {
      const int buf = local & 1;
      const uint32_t aph = (uint32_t)(local >> 1) & 1u;
      if (!mbar_wait_bounded(&acc_full[buf], aph, abort_flag, status, kDevTimeoutMma)) break;
      tc_fence_after();
      const int tm = tile % tiles_m, tn = tile / tiles_m;
      const int row = tm * BM + row_in_tile;
      float* yrow = Y + (size_t)row * N;
      for (int c = 0; c < BN; c += 16) {
        uint32_t r[16];
        tmem_ld16(tmem_base + (uint32_t)(buf * BN + c) + ((uint32_t)(quarter * 32) << 16), r);
        tmem_ld_wait();
        const int col = tn * BN + c;
        if (row < M) {
          if (vec4 && col + 16 <= N) {
#pragma unroll
            for (int j = 0; j < 16; j += 4)
              *reinterpret_cast<float4*>(yrow + col + j) =
                  make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                              __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (col + j < N) yrow[col + j] = __uint_as_float(r[j]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      // the buffer is free again: the leader's barrier counts both CTAs' warps
      if (lane == 0) mbar_arrive_cluster(leader_acc_empty0 + (uint32_t)(buf * 8));
    }
  }
  // neither CTA frees its tensor memory while the pair's MMAs or the other
  // CTA's epilogue may still use it
  __syncwarp();
  tc_fence_before();
  cluster_arrive();
  cluster_wait();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_2sm(tmem_base, TMEM_COLS);
  }
}

static int active_pairs(int sm_count) {
  // clusters of two that can be resident at once (cached per device)
  constexpr int kMaxDev = 64;
  static int cache[kMaxDev];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 0;
  if (cache[dev] > 0) return cache[dev];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(sm_count & ~1));
  cfg.blockDim = dim3(dg2::THREADS);
  cfg.dynamicSmemBytes = dg2::SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, k_dense_gemm2, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  cache[dev] = n;
  return n;
}

cudaError_t launch_dense_gemm(const uint16_t* X, int64_t M, const uint16_t* W, int64_t N,
                              int64_t K, float* Y, uint32_t* status, int sm_count,
                              cudaStream_t st) {
  using namespace dg;
  // the two-SM kernel where a 256 x 256 tile fits the problem
  if (M >= 256 && N >= 256) {
    CUtensorMap ta, tb;
    if (!make_tmap_2d(&ta, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)M, (uint64_t)K, 128,
                      BK, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    if (!make_tmap_2d(&tb, W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)N, (uint64_t)K, 128,
                      BK, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem_limit(k_dense_gemm2, kMaxDynSmem);
    if (e != cudaSuccess) return e;
    const int pairs_max = active_pairs(sm_count);
    if (pairs_max > 0) {
      const int64_t tiles = ((M + dg2::BM - 1) / dg2::BM) * ((N + dg2::BN - 1) / dg2::BN);
      const int pairs = (int)(tiles < pairs_max ? tiles : pairs_max);
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)(2 * pairs));
      cfg.blockDim = dim3(dg2::THREADS);
      cfg.dynamicSmemBytes = dg2::SMEM_BYTES;
      cfg.stream = st;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      e = cudaLaunchKernelEx(&cfg, k_dense_gemm2, ta, tb, Y, (int)M, (int)N, (int)K, status);
      if (e != cudaSuccess) return e;
      return cudaGetLastError();
    }
  }

  CUtensorMap ta, tb;
  if (!make_tmap_2d(&ta, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)M, (uint64_t)K, BM, BK,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tb, W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)N, (uint64_t)K, BN, BK,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_limit(k_dense_gemm, kMaxDynSmem);
  if (e != cudaSuccess) return e;
  const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = (int)(tiles < sm_count ? tiles : sm_count);
  k_dense_gemm<<<grid, THREADS, SMEM_BYTES, st>>>(ta, tb, Y, (int)M, (int)N, (int)K, status);
  return cudaGetLastError();
}

// ------------------------------------------------------- CUDA-core GEMM ---
// Plain tiled fp32 GEMM on CUDA cores (diagnostic mode and cross-check).
__global__ void k_simt_gemm(const uint16_t* __restrict__ X, int M, const uint16_t* __restrict__ W,
                            int N, int K, float* __restrict__ Y) {
  __shared__ float xs[16][33], ws[16][33];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m = blockIdx.y * 16 + ty, n = blockIdx.x * 16 + tx;
  float acc = 0.0f;
  for (int k0 = 0; k0 < K; k0 += 32) {
    for (int j = tx; j < 32; j += 16) {
      int mm = blockIdx.y * 16 + ty, nn = blockIdx.x * 16 + ty, kk = k0 + j;
      xs[ty][j] = (mm < M && kk < K) ? __uint_as_float((uint32_t)X[(size_t)mm * K + kk] << 16) : 0.f;
      ws[ty][j] = (nn < N && kk < K) ? __uint_as_float((uint32_t)W[(size_t)nn * K + kk] << 16) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int j = 0; j < 32; ++j) acc = fmaf(xs[ty][j], ws[tx][j], acc);
    __syncthreads();
  }
  if (m < M && n < N) Y[(size_t)m * N + n] = acc;
}

cudaError_t launch_simt_gemm(const uint16_t* X, int64_t M, const uint16_t* W, int64_t N,
                             int64_t K, float* Y, cudaStream_t st) {
  dim3 grid((unsigned)((N + 15) / 16), (unsigned)((M + 15) / 16));
  k_simt_gemm<<<grid, 256, 0, st>>>(X, (int)M, W, (int)N, (int)K, Y);
  return cudaGetLastError();
}

}  // namespace e8
