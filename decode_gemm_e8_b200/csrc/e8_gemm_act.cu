// Fused decode + GEMM for small batches (tokens M <= 64).
//
//   Y[m][n] = alpha * sum_k (FWHT D x_m)_k z_nk                  (activation-side RHT)
//
// z_n = m (c1 + beta c2) is the integer codebook vector of each group of row
// n ("glq 0.1.1", "How it works", item 1); |z| <= 30 is exact in bf16.  The
// transformed activations arrive as bf16 hi/lo row pairs (Xt rows 2m and
// 2m + 1, built by k_act_rht), so one MMA with N = 2M columns computes both
// parts at once and the epilogue adds adjacent columns.
//
// One CTA owns 128 weight rows and a contiguous range of K; the CTAs of a
// thread-block cluster split K and reduce their partial tiles through
// distributed shared memory in a fixed order (deterministic result).
//   warp 0      TMA producer: index tiles (16 groups x 128 rows) and the Xt
//               tile (128 x rows_b, 128-byte swizzle) per K step of 128
//   warp 1      allocates tensor memory; one thread issues tcgen05.mma
//               (M = 128 weight rows, N = rows_b, K = 16)
//   warps 2-9   decode: each thread owns one weight row (TMEM lane) and 8 of the
//               16 groups of a K step: codebook gather, combine, bf16 convert,
//               then writes the A operand either to shared memory (128-byte
//               swizzled K-major layout) or to tensor memory (tcgen05.st)
// The tensor cores are used only for the X W^T contraction.
#include "e8_common.cuh"
#include "e8_codebook.cuh"
#include "e8_internal.h"
#include "e8_tmap.h"

namespace e8 {

namespace ag {
constexpr int BN_ROWS = 128;     // weight rows per CTA (MMA M)
constexpr int KSTEP = 128;       // K per pipeline step (16 groups)
constexpr int GROUPS = KSTEP / 8;
constexpr int THREADS = 320;
constexpr int DECODE_WARPS = 8;
constexpr int A_BYTES = BN_ROWS * KSTEP * 2;  // shared-memory A operand (SS variant)
constexpr int I1_BYTES = BN_ROWS * GROUPS * 2;
constexpr int TABLE_BYTES = 131088;           // 32769 entries padded to 16 bytes
}  // namespace ag

struct ActSmemPlan {
  int stages, rows_b, a_bytes, b_bytes, i2_bytes, stage_bytes, table_off, bar_off, total;
};

__host__ __device__ inline ActSmemPlan act_plan(int rows_b, int bpw, bool a_in_tmem) {
  using namespace ag;
  ActSmemPlan p;
  p.rows_b = rows_b;
  p.a_bytes = a_in_tmem ? 0 : A_BYTES;
  p.b_bytes = rows_b * KSTEP * 2;
  p.i2_bytes = bpw == 2 ? 0 : (bpw == 3 ? BN_ROWS * GROUPS : BN_ROWS * GROUPS * 2);
  int raw = p.a_bytes + p.b_bytes + I1_BYTES + p.i2_bytes;
  p.stage_bytes = (raw + 1023) & ~1023;
  // 227 KB of shared memory per CTA, minus 2 KB for alignment slack and barriers
  const int budget = 225 * 1024 - (a_in_tmem ? TABLE_BYTES : 0);
  p.stages = budget / p.stage_bytes;
  if (p.stages > 4) p.stages = 4;
  p.table_off = p.stages * p.stage_bytes;
  int after = p.table_off + (a_in_tmem ? TABLE_BYTES : 0);
  // the epilogue's partial tile [128][rows_b + 1] fp32 reuses the stage area
  int part = BN_ROWS * (rows_b + 1) * 4;
  if (part > p.table_off) after = part > after ? part : after;
  p.bar_off = (after + 15) & ~15;
  p.total = 1024 + p.bar_off + 256;
  return p;
}

template <bool A_IN_TMEM>
__global__ void __launch_bounds__(ag::THREADS, 1)
    k_act_gemm(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmI1,
               const __grid_constant__ CUtensorMap tmI2, DeviceCodebook cb, int M, int N, int K,
               int rows_b, int bpw, float alpha, float* __restrict__ Y) {
  using namespace ag;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const ActSmemPlan plan = act_plan(rows_b, bpw, A_IN_TMEM);
  const int S = plan.stages;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + plan.bar_off);
  uint64_t* full_load = bars;          // [S]
  uint64_t* full_a = bars + 4;         // [S]
  uint64_t* empty = bars + 8;          // [S]
  uint64_t* acc_full = bars + 12;
  uint64_t* table_full = bars + 13;
  uint64_t* drain = bars + 14;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  const uint32_t* s_table = reinterpret_cast<const uint32_t*>(smem + plan.table_off);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  uint32_t ncl;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(ncl));
  const int tile = (int)(blockIdx.x / ncl);
  const int n0 = tile * BN_ROWS;
  const int ksteps = K / KSTEP;
  const int ks_begin = (int)((int64_t)crank * ksteps / ncl);
  const int ks_end = (int)((int64_t)(crank + 1) * ksteps / ncl);
  const int nks = ks_end - ks_begin;
  const uint32_t tmem_cols = A_IN_TMEM ? 512u : (rows_b <= 32 ? 32u : (rows_b <= 64 ? 64u : 128u));
  const uint32_t a_col0 = 128;  // A stages at columns 128 + 64 s (tensor-memory variant)

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_load[s], 1);
      mbar_init(&full_a[s], DECODE_WARPS);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(table_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  uint32_t* status = cb.status;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmB);
      tma_prefetch_desc(&tmI1);
      if (bpw > 2) tma_prefetch_desc(&tmI2);
      if (A_IN_TMEM) {
        mbar_arrive_expect_tx(table_full, TABLE_BYTES);
        bulk_load(smem + plan.table_off, cb.table, TABLE_BYTES, table_full);
      }
      const uint32_t tx = (uint32_t)(plan.b_bytes + I1_BYTES + plan.i2_bytes);
      int s = 0;
      uint32_t ph = 0, issued = 0;
      for (int i = 0; i < nks; ++i) {
        if (!mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, status, kDevTimeoutEmpty)) break;
        uint8_t* st = smem + s * plan.stage_bytes;
        uint8_t* sb = st + plan.a_bytes;
        uint8_t* si1 = sb + plan.b_bytes;
        uint8_t* si2 = si1 + I1_BYTES;
        const int k0 = (ks_begin + i) * KSTEP;
        mbar_arrive_expect_tx(&full_load[s], tx);
        tma_load_2d(sb, &tmB, &full_load[s], k0, 0);
        tma_load_2d(sb + rows_b * 128, &tmB, &full_load[s], k0 + 64, 0);
        tma_load_2d(si1, &tmI1, &full_load[s], k0 / 8, n0);
        if (bpw > 2) tma_load_2d(si2, &tmI2, &full_load[s], k0 / 8, n0);
        ++issued;
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      if (*abort_flag) {
        for (uint32_t j = 0; j < (uint32_t)S && j < issued; ++j) {
          uint32_t idx = issued - 1 - j;
          uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(&full_load[idx % S], (idx / S) & 1u))
            if (global_timer_ns() - t0 > 100000000ull) break;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BN_ROWS, (uint32_t)rows_b);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int i = 0; i < nks && ok; ++i) {
        if (!mbar_wait_bounded(&full_a[s], ph, abort_flag, status, kDevTimeoutFull) ||
            !mbar_wait_bounded(&full_load[s], ph, abort_flag, status, kDevTimeoutFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(smem + s * plan.stage_bytes);
        const uint32_t sb = st + plan.a_bytes;
#pragma unroll
        for (int j = 0; j < KSTEP / 16; ++j) {
          const uint32_t sub = (uint32_t)(j >> 2), koff = (uint32_t)(j & 3) * 32u;
          const uint64_t bd = smem_desc(sb + sub * (uint32_t)(rows_b * 128) + koff, 16, 1024, 2);
          const uint32_t acc = (i > 0 || j > 0) ? 1u : 0u;
          if (A_IN_TMEM) {
            mma_ts(tmem_base, tmem_base + a_col0 + (uint32_t)(s * 64 + j * 8), bd, idesc, acc);
          } else {
            const uint64_t ad = smem_desc(st + sub * 16384u + koff, 16, 1024, 2);
            mma_ss(tmem_base, ad, bd, idesc, acc);
          }
        }
        mma_commit(&empty[s]);
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      if (ok) mma_commit(acc_full);
      mma_commit(drain);
      uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0))
        if (global_timer_ns() - t0 > 200000000ull) break;
    }
  } else {
    // ---------------------------------------------------------- decoders --
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int half = (warp - 2) >> 2;       // which 8 of the 16 groups of a step
    const int r = q * 32 + lane;            // weight row within the tile
    const int mul = bpw == 3 ? 2 : 4;
    const uint32_t* table = A_IN_TMEM ? s_table : cb.table;
    bool ok = true;
    if (A_IN_TMEM) ok = mbar_wait_bounded(table_full, 0, abort_flag, status, kDevTimeoutFull);
    int s = 0;
    uint32_t ph = 0;
    for (int i = 0; i < nks && ok; ++i) {
      if (!mbar_wait_bounded(&full_load[s], ph, abort_flag, status, kDevTimeoutFull)) break;
      tc_fence_after();
      uint8_t* st = smem + s * plan.stage_bytes;
      const uint8_t* si1 = st + plan.a_bytes + plan.b_bytes;
      const uint8_t* si2 = si1 + I1_BYTES;
      const uint4 c1 = *reinterpret_cast<const uint4*>(si1 + r * 32 + half * 16);
      uint32_t i1w[4] = {c1.x, c1.y, c1.z, c1.w};
      uint32_t i2w[4] = {0, 0, 0, 0};
      if (bpw == 4) {
        const uint4 c2 = *reinterpret_cast<const uint4*>(si2 + r * 32 + half * 16);
        i2w[0] = c2.x; i2w[1] = c2.y; i2w[2] = c2.z; i2w[3] = c2.w;
      } else if (bpw == 3) {
        const uint2 c2 = *reinterpret_cast<const uint2*>(si2 + r * 16 + half * 8);
        // widen 8 bytes to 8 halfwords
        i2w[0] = (c2.x & 0xFFu) | ((c2.x & 0xFF00u) << 8);
        i2w[1] = ((c2.x >> 16) & 0xFFu) | ((c2.x >> 8) & 0xFF0000u);
        i2w[2] = (c2.y & 0xFFu) | ((c2.y & 0xFF00u) << 8);
        i2w[3] = ((c2.y >> 16) & 0xFFu) | ((c2.y >> 8) & 0xFF0000u);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t a = (i1w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
        const uint32_t ea = table[(a + 1u) >> 1];
        const bool na = a != 0u && (a & 1u) == 0u;
        int z[8];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          int v0 = (int)((ea >> (8 * t)) & 0xFu) - 8, v4 = (int)((ea >> (8 * t + 4)) & 0xFu) - 8;
          z[t] = na ? -v0 : v0;
          z[t + 4] = na ? -v4 : v4;
        }
        if (bpw > 2) {
          const uint32_t b = (i2w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
          const uint32_t eb = table[(b + 1u) >> 1];
          const bool nb = b != 0u && (b & 1u) == 0u;
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            int v0 = (int)((eb >> (8 * t)) & 0xFu) - 8, v4 = (int)((eb >> (8 * t + 4)) & 0xFu) - 8;
            z[t] = mul * z[t] + (nb ? -v0 : v0);
            z[t + 4] = mul * z[t + 4] + (nb ? -v4 : v4);
          }
        }
        uint32_t w0 = pack_bf16x2((float)z[0], (float)z[1]);
        uint32_t w1 = pack_bf16x2((float)z[2], (float)z[3]);
        uint32_t w2 = pack_bf16x2((float)z[4], (float)z[5]);
        uint32_t w3 = pack_bf16x2((float)z[6], (float)z[7]);
        const int gl = half * 8 + j;
        if (A_IN_TMEM) {
          tmem_st4(tmem_base + ((uint32_t)(q * 32) << 16) + a_col0 + (uint32_t)(s * 64 + gl * 4),
                   w0, w1, w2, w3);
        } else {
          uint8_t* dst = st + half * 16384 + (r >> 3) * 1024 + (r & 7) * 128 +
                         (((gl & 7) ^ (r & 7)) << 4);
          *reinterpret_cast<uint4*>(dst) = make_uint4(w0, w1, w2, w3);
        }
      }
      if (A_IN_TMEM) {
        tmem_st_wait();
        tc_fence_before();
      } else {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&full_a[s]);
      if (++s == S) { s = 0; ph ^= 1u; }
    }
    // ---------------------------------------------------------- epilogue --
    if (warp < 6) {
      float* part = reinterpret_cast<float*>(smem);
      const int ld = rows_b + 1;
      bool have = nks > 0 && mbar_wait_bounded(acc_full, 0, abort_flag, status, kDevTimeoutMma);
      tc_fence_after();
      for (int c = 0; c < rows_b; c += 16) {
        uint32_t v[16];
        tmem_ld16(tmem_base + (uint32_t)c + ((uint32_t)(q * 32) << 16), v);
        tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < 16; ++t) part[r * ld + c + t] = have ? __uint_as_float(v[t]) : 0.0f;
      }
    }
  }
  // ------------------------------------------------ cluster reduction ----
  tc_fence_before();
  __syncthreads();
  cluster_arrive();
  cluster_wait();
  {
    const int R = BN_ROWS / (int)ncl;
    const int r0 = (int)crank * R;
    const int ld = rows_b + 1;
    const uint32_t part_addr = smem_u32(smem);
    for (int e = threadIdx.x; e < R * M; e += blockDim.x) {
      const int row = e % R, m = e / R;
      const int n = n0 + r0 + row;
      float acc = 0.0f;
      for (uint32_t src = 0; src < ncl; ++src) {
        const uint32_t base = mapa_shared(part_addr, src);
        const uint32_t off = (uint32_t)(((r0 + row) * ld + 2 * m) * 4);
        const uint32_t off2 = off + 4u;
        acc += ld_shared_cluster_f32(base + off) + ld_shared_cluster_f32(base + off2);
      }
      if (n < N) Y[(size_t)m * N + n] = alpha * acc;
    }
  }
  cluster_arrive();
  cluster_wait();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

static cudaError_t launch_act_gemm_generic(const DeviceCodebook& cb, const ActGemmArgs& a,
                                           int sm_count, cudaStream_t st) {
  using namespace ag;
  const bool tm = a.variant == 1;
  CUtensorMap tb, ti1, ti2;
  if (!make_tmap_2d(&tb, a.Xt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.rows_b,
                    (uint64_t)a.K, (uint32_t)a.rows_b, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&ti1, a.idx1, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, (uint64_t)a.N,
                    (uint64_t)(a.K / 8), BN_ROWS, GROUPS, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (a.bpw == 4) {
    if (!make_tmap_2d(&ti2, a.idx2, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, (uint64_t)a.N,
                      (uint64_t)(a.K / 8), BN_ROWS, GROUPS, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  } else if (a.bpw == 3) {
    if (!make_tmap_2d(&ti2, a.idx2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.N,
                      (uint64_t)(a.K / 8), BN_ROWS, GROUPS, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  } else {
    ti2 = ti1;
  }
  const ActSmemPlan plan = act_plan(a.rows_b, a.bpw, tm);
  if (plan.stages < 2) return cudaErrorInvalidValue;
  const int tiles = (int)((a.N + BN_ROWS - 1) / BN_ROWS);
  const int ksteps = (int)(a.K / KSTEP);
  int csize = 1;
  while (csize < 8 && tiles * csize * 2 <= sm_count && csize * 2 <= ksteps) csize *= 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(tiles * csize));
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = (size_t)plan.total;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (tm) {
    e = ensure_smem_limit(k_act_gemm<true>, kMaxDynSmem);
    if (e != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, k_act_gemm<true>, tb, ti1, ti2, cb, (int)a.M, (int)a.N, (int)a.K,
                           a.rows_b, a.bpw, a.alpha, a.Y);
  } else {
    e = ensure_smem_limit(k_act_gemm<false>, kMaxDynSmem);
    if (e != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, k_act_gemm<false>, tb, ti1, ti2, cb, (int)a.M, (int)a.N,
                           (int)a.K, a.rows_b, a.bpw, a.alpha, a.Y);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_act_gemm(const DeviceCodebook& cb, const ActGemmArgs& a, int sm_count,
                            cudaStream_t st) {
  return launch_act_gemm_generic(cb, a, sm_count, st);
}

}  // namespace e8
