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

cudaError_t launch_dense_gemm(const uint16_t* X, int64_t M, const uint16_t* W, int64_t N,
                              int64_t K, float* Y, uint32_t* status, int sm_count,
                              cudaStream_t st) {
  using namespace dg;
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
