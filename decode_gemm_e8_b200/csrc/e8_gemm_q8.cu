// Fused decode + GEMM for small batches (up to 32 tokens), int8 tensor cores.
//
//   Y[m][n] = alpha * sum_k (FWHT D x_m)_k z_nk                 (activation-side RHT)
//
// z_n = m (c1 + beta c2) is the integer codebook vector of each 8-weight group
// of row n ("glq 0.1.1", "How it works", item 1, and the "Bit widths" table),
// |z| <= 30.  The transformed activations arrive as two int8 pieces per token
// (rows 2m and 2m + 1 of Xq, written by k_act_q8) with a per-token step s_m:
//   xt_m = s_m (q0_m + q1_m / 128).
// The weight operand is z + 128 as unsigned bytes, decoded on chip straight
// into tensor memory; tcgen05.mma kind::i8 accumulates exactly in int32.  The
// +128 bias is removed by the tensor cores too: every K step is followed by a
// second product of the same Xq tile with a constant signed operand of -128,
// accumulating -128 sum_k Xq into the same accumulator, so D = Xq . z exactly
// and no partial sum carries the bias:
//   y[m][n] = alpha s_m (D[n][2m] + D[n][2m+1] / 128).
//
// Work split (stream-K): the (128-row tile, 128-wide K unit) pairs are laid out
// tile by tile and every CTA of a one-per-SM grid takes a contiguous run of
// them, so all SMs get the same number of units within one.  A launch may
// serve a group of up to four weight matrices with the same K and rate (for
// instance q, k and v, which read the same tokens): their tiles are
// concatenated, each with its own activation pieces, alpha and output, so the
// pair table, the grid boundaries and the tail are paid once per group.  A
// run covers at most a few tiles; the partial tile of each is added into Y
// (zeroed by the transform kernel that precedes this one) by a TMA bulk
// reduce-add, so the order of the few partial sums of an output is not fixed.
//
// Roles (one CTA per SM):
//   warp 0      TMA producer: the codebook pair table (once) and the index
//               tiles (a ring released by the decoders as soon as they hold
//               the indices in registers), without waiting for the transform
//               kernel
//   warp 23     TMA producer of the Xq tiles (a ring released by the MMA),
//               after the transform kernel
//   warps 1, 22 tensor-memory allocation (warp 1); one elected lane of each
//               issues tcgen05.mma (M = 128 weight rows, N = rows_b, K = 32)
//               and the commits for the even / odd units
//   warps 2-17  decoders, four groups of four (one warp per TMEM lane
//               quarter) taking units in turn: each thread owns one weight
//               row (its TMEM lane) and the 16 groups of the unit: index
//               loads, pair-table gathers, combine, two tcgen05.st of 16
//               columns into the unit's operand stage
//   warps 18-21 epilogue, one per TMEM lane quarter: accumulator -> shared
//               memory -> bulk reduce-add into Y
// The tensor cores are used only for the X W^T contraction.
#include "e8_common.cuh"
#include "e8_codebook.cuh"
#include "e8_internal.h"
#include "e8_tmap.h"

namespace e8 {

namespace sk {
constexpr int ROWS = 128;                 // weight rows per tile (MMA M)
constexpr int KU = 128;                   // K of one work unit
constexpr int GROUPS = KU / 8;            // groups of a row in one unit
constexpr int DEC_GROUPS = 4;
constexpr int DEC_WARPS = 4 * DEC_GROUPS;
constexpr int EPI_WARP0 = 2 + DEC_WARPS;
constexpr int MMA2_WARP = EPI_WARP0 + 4;  // issuer of the odd units
constexpr int XQ_WARP = MMA2_WARP + 1;    // producer of the Xq tiles
constexpr int THREADS = 32 * (XQ_WARP + 1);
constexpr int TABLE_BYTES = 131088;       // 32769 u32 entries, padded to 16 bytes
constexpr int I1_BYTES = ROWS * GROUPS * 2;
constexpr uint32_t ACC_COLS = 64;         // int32 accumulator columns per buffer
// tensor memory: accumulators [issuer parity][segment buffer], then the operand ring
constexpr uint32_t ACC_TOTAL = 4 * ACC_COLS;
constexpr uint32_t A_COLS = KU / 4;       // 4 int8 weights per TMEM column
constexpr int MAX_STAGES = 8;
static_assert(MAX_STAGES % DEC_GROUPS == 0 && MAX_STAGES % 2 == 0,
              "each operand stage serves one decoder group and one issuer");
constexpr int AUX_BYTES = 128 * kMaxGroup;   // per matrix: alpha times the per-token steps [32]
// The constant -128 operand (128 rows x 32 bytes, every byte 0x80 read as
// signed): up to 16 tokens it sits in tensor-memory columns that the
// accumulators of buffer 0 leave unused; above, in this shared-memory tile.
constexpr int CONST_A_BYTES = 4096;
constexpr uint32_t CONST_A_COL = 32;
constexpr int BAR_BYTES = 512;
// shared memory left free on the SM for a CTA of the activation transform
// (K = 4096: 16 KB), so that it can run next to this kernel's CTA
constexpr int CORESIDENT_RESERVE = 18 * 1024;
}  // namespace sk

// Shared memory: the pair table at offset 0 of the dynamic window (so its
// address folds into the gather instructions), then, from the next 1 KB
// boundary: the Xq ring (sx stages), the index-tile ring (sc stages), the
// staging tile of the output (16 or 32 tokens x 128 fp32), the per-token steps
// and row sums, and the barriers.  Offsets below are relative to that
// boundary.  The decoded operands live in a ring of sa tensor-memory stages.
struct SkPlan {
  int sa, sx, sc, b_bytes, code_bytes, i2_bytes, code_off, y_off, aux_off, const_off, bar_off,
      total;
  uint32_t tmem_cols;
};

__host__ __device__ inline SkPlan sk_plan(int rows_b, int bpw) {
  using namespace sk;
  SkPlan p;
  p.b_bytes = rows_b * KU;                                  // multiple of 2 KB
  p.i2_bytes = bpw == 2 ? 0 : (bpw == 3 ? ROWS * GROUPS : ROWS * GROUPS * 2);
  p.code_bytes = I1_BYTES + p.i2_bytes;                     // multiple of 1 KB
  const int y_bytes = (rows_b <= 32 ? 16 : 32) * ROWS * 4;
  const int budget = kMaxDynSmem - TABLE_BYTES - 1024 - AUX_BYTES - CONST_A_BYTES - BAR_BYTES -
                     CORESIDENT_RESERVE - y_bytes;
  p.sa = MAX_STAGES;                                        // 4 x 64 + 8 x 32 TMEM columns
  // Xq tiles are requested after the transform kernel ends and take ~1 us to
  // land, so the Xq ring holds a CTA's whole run where it can (7 units of
  // 128 at 4096 x 4096); the index ring gets the rest, at least 4 stages
  for (p.sx = 7; p.sx > 2; --p.sx)
    if (budget - p.sx * p.b_bytes >= 4 * p.code_bytes) break;
  p.sc = (budget - p.sx * p.b_bytes) / p.code_bytes;
  if (p.sc > MAX_STAGES) p.sc = MAX_STAGES;
  // A multiple of four index stages keeps each stage with one decoder group
  // (the four groups take units in turn).  Bulk copies may land out of order: were a
  // stage shared, a group could reach its next use of it while the other
  // group's copy into it was still in flight, and the parity wait would take
  // the barrier two phases behind for the phase it waits for.
  p.sc &= ~3;
  p.code_off = p.sx * p.b_bytes;
  p.y_off = p.code_off + p.sc * p.code_bytes;
  p.aux_off = p.y_off + y_bytes;
  p.const_off = p.aux_off + AUX_BYTES;      // multiple of 512 bytes
  p.bar_off = p.const_off + CONST_A_BYTES;
  p.total = TABLE_BYTES + 1024 + p.bar_off + BAR_BYTES;
  p.tmem_cols = 512u;
  return p;
}

// Byte offset, inside the pair table, of the entry of codebook index i
// (slot (i + 1) >> 1), for the index in the low / high 16 bits of w.
__device__ __forceinline__ uint32_t sk_off_lo(uint32_t w) {
  return (((w & 0xFFFFu) << 1) + 2u) & 0x3FFFCu;
}
__device__ __forceinline__ uint32_t sk_off_hi(uint32_t w) { return ((w >> 15) + 2u) & 0x3FFFCu; }
__device__ __forceinline__ uint32_t sk_entry(const uint8_t* table, uint32_t off) {
  return *reinterpret_cast<const uint32_t*>(table + off);
}

// Tensor maps of a group (kernel parameter space): per matrix the Xq pieces
// (box rows_b x 128), the index arrays (box 128 rows x 16 groups) and Y.
struct SkMaps {
  CUtensorMap B[kMaxGroup], I1[kMaxGroup], I2[kMaxGroup], Y[kMaxGroup];
};
struct SkMat {
  int tile0;             // first tile of the matrix in the concatenation
  int N;
  float alpha;
  int use_tma_y;         // Y by bulk reduce-add (else fp32 atomics)
  const float* tok_scale;
  float* Y;
};
struct SkGroup {
  int count;
  int tiles;             // tiles of all matrices
  SkMat mat[kMaxGroup];
};

// Matrix of a tile of the concatenation.
__device__ __forceinline__ int sk_mat_of(const SkGroup& g, int tile) {
  int j = 0;
#pragma unroll
  for (int q = 1; q < kMaxGroup; ++q)
    if (q < g.count && tile >= g.mat[q].tile0) j = q;
  return j;
}

// Offset of the 16-byte half `h` of row r in a 32-byte-swizzled index tile.
__device__ __forceinline__ uint32_t sw32_off(int r, int h) {
  return (uint32_t)(r * 32 + ((h ^ ((r >> 2) & 1)) << 4));
}

__device__ __forceinline__ void sk_mma_i8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// kind::i8 instruction descriptor: A unsigned 8-bit, B signed 8-bit, D int32,
// both operands K-major.
__host__ __device__ constexpr uint32_t sk_idesc(uint32_t M, uint32_t N) {
  return (2u << 4) | (0u << 7) | (1u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}
// The same with a signed A operand (the constant -128 bias product).
__host__ __device__ constexpr uint32_t sk_idesc_sa(uint32_t M, uint32_t N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// kind::i8 with both operands from shared memory (descriptors).
__device__ __forceinline__ void sk_mma_i8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void sk_tmem_st8(uint32_t taddr, uint32_t v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr),
      "r"(v)
      : "memory");
}

__device__ __forceinline__ void sk_tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}

// 32 lanes x 32 bit, 8 consecutive columns per thread.
__device__ __forceinline__ void sk_tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}

// No memory clobber: nothing later in the thread depends on the sum, and the
// shared-memory loads feeding the next adds may then be hoisted past it.
__device__ __forceinline__ void red_add_f32(float* p, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v));
}

// Element-wise fp32 add of a shared-memory tile into global memory by the TMA
// unit (box of the tensor map; elements outside the tensor are skipped).
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, uint32_t smem_src,
                                                  int32_t x, int32_t y) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2}], [%3];"
      ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_src)
      : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Units [begin, end) of CTA c when U units are spread over G CTAs.
__device__ __forceinline__ int sk_unit_begin(int c, int U, int G) {
  return (int)(((int64_t)c * U) / G);
}

// CW: accumulator columns read by the epilogue (32 for up to 16 tokens, else 64).
// maps.Y[j]: Y [M][N] fp32 of matrix j, box 128 x M (valid when its
// use_tma_y; else fp32 atomics).
// At most 64 registers, so that a CTA of the activation transform (512
// threads x 32 registers) fits on the SM next to it.
template <int BPW, int CW>
__global__ void __maxnreg__(64)
    k_gemm_q8(const __grid_constant__ SkMaps maps, const SkGroup grp, DeviceCodebook cb, int M,
              int K, int rows_b, int early_codes) {
  using namespace sk;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint8_t* table = smem_raw;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + TABLE_BYTES + 1023) & ~uintptr_t(1023));
  const SkPlan plan = sk_plan(rows_b, BPW);
  const int SA = plan.sa, SX = plan.sx, SC = plan.sc;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + plan.bar_off);
  uint64_t* full_code = bars;                     // [SC] index tiles landed
  uint64_t* code_empty = bars + MAX_STAGES;       // [SC] decoders hold the indices
  uint64_t* full_a = bars + 2 * MAX_STAGES;       // [SA] operand decoded + Xq landed
  uint64_t* a_empty = bars + 3 * MAX_STAGES;      // [SA] MMAs of the stage done
  uint64_t* acc_full = bars + 4 * MAX_STAGES;     // [2] both issuers done with a segment
  uint64_t* acc_empty = acc_full + 2;             // [2]
  uint64_t* table_full = acc_full + 4;
  uint64_t* drain = acc_full + 5;                 // [2] one per issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 7);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  float* s_sc = reinterpret_cast<float*>(smem + plan.aux_off);   // [G][32]
  float* s_y = reinterpret_cast<float*>(smem + plan.y_off);                // [M][128]
  uint8_t* xq_ring = smem;
  uint8_t* code_ring = smem + plan.code_off;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kunits = K / KU;
  const int U = grp.tiles * kunits;
  const int u_begin = sk_unit_begin((int)blockIdx.x, U, (int)gridDim.x);
  const int nu = sk_unit_begin((int)blockIdx.x + 1, U, (int)gridDim.x) - u_begin;
  const int first_tile = u_begin / kunits;
  const uint32_t code_tx = (uint32_t)plan.code_bytes;
  uint32_t* status = cb.status;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SC; ++s) {
      mbar_init(&full_code[s], 1);
      mbar_init(&code_empty[s], 4);
    }
    for (int s = 0; s < SA; ++s) {
      mbar_init(&full_a[s], 5);   // four decoder warps + the Xq tile
      mbar_init(&a_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 2);
      mbar_init(&acc_empty[b], 4);
      mbar_init(&drain[b], 1);
    }
    mbar_init(table_full, 1);
    fence_mbar_init();
    *abort_flag = 0u;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, plan.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tmem_a = tmem_base + ACC_TOTAL;
  // the constant -128 operand: with up to 16 tokens (CW == 32) columns 32..39
  // of accumulator buffer 0, which its MMAs (N <= 32) never write; else a
  // shared-memory tile (K-major, no swizzle: every byte is the same)
  const uint32_t const_a_tmem = tmem_base + CONST_A_COL;
  if (CW == 32) {
    if (warp >= 2 && warp < 6) {   // one warp per TMEM lane quarter
      sk_tmem_st8(const_a_tmem + ((uint32_t)((warp & 3) * 32) << 16), 0x80808080u);
      tmem_st_wait();
    }
  } else {
    uint4* ca = reinterpret_cast<uint4*>(smem + plan.const_off);
    for (int i = threadIdx.x; i < CONST_A_BYTES / 16; i += THREADS)
      ca[i] = make_uint4(0x80808080u, 0x80808080u, 0x80808080u, 0x80808080u);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int nseg = nu > 0 ? (u_begin + nu - 1) / kunits - first_tile + 1 : 0;
  const int ku_first = u_begin - first_tile * kunits;   // K unit of the run's first unit
  // the next kernel of the stream may be launched now: it waits for this grid
  // before it touches anything this grid reads or writes
  if (threadIdx.x == 0) grid_dep_launch();

  if (warp == 0) {
    if (lane == 0) {
      for (int j = 0; j < grp.count; ++j) {
        tma_prefetch_desc(&maps.B[j]);
        tma_prefetch_desc(&maps.I1[j]);
        if (BPW > 2) tma_prefetch_desc(&maps.I2[j]);
        if (grp.mat[j].use_tma_y) tma_prefetch_desc(&maps.Y[j]);
      }
      // the pair table in eight 16 KB pieces plus the last entry, starting at a
      // CTA-dependent piece so that the SMs do not all read the same L2 lines
      mbar_arrive_expect_tx(table_full, TABLE_BYTES);
      for (int j = 0; j < 8; ++j) {
        const int c = (j + (int)blockIdx.x) & 7;
        bulk_load(smem_raw + c * 16384, reinterpret_cast<const uint8_t*>(cb.table) + c * 16384,
                  16384, table_full);
      }
      bulk_load(smem_raw + 8 * 16384, reinterpret_cast<const uint8_t*>(cb.table) + 8 * 16384, 16,
                table_full);
      // m1 / m2: the index maps of the unit's matrix, tile0 its first tile
      auto load_codes = [&](int i, int s, const CUtensorMap* m1, const CUtensorMap* m2,
                            int tile0) {
        const int u = u_begin + i;
        const int lt = u / kunits - tile0;
        uint8_t* dst = code_ring + s * plan.code_bytes;
        mbar_arrive_expect_tx(&full_code[s], code_tx);
        tma_load_2d(dst, m1, &full_code[s], (u % kunits) * GROUPS, lt * ROWS);
        if (BPW > 2)
          tma_load_2d(dst + I1_BYTES, m2, &full_code[s], (u % kunits) * GROUPS, lt * ROWS);
      };
      // Index tiles do not depend on the preceding kernel: before waiting for
      // it, load those of the first SC + SA units (the decoders of units
      // below SA wait for nothing but their tiles, so the waits for free
      // stages here cannot depend on the MMAs).
      int cn = 0;                    // next unit whose index tiles to load
      int cs = 0;
      uint32_t cph = 0;
      bool ok = true;
      auto next_codes = [&](int limit, const CUtensorMap* m1, const CUtensorMap* m2,
                            int tile0) {
        while (ok && cn < limit) {
          if (cn >= SC &&
              !mbar_wait_sleep(&code_empty[cs], cph ^ 1u, abort_flag, status, kDevTimeoutEmpty)) {
            ok = false;
            break;
          }
          load_codes(cn, cs, m1, m2, tile0);
          ++cn;
          if (++cs == SC) {
            cs = 0;
            cph ^= 1u;
          }
        }
      };
      // every index tile, as the decoders free stages; the Xq tiles, which
      // come from the preceding kernel, have a producer of their own.  The
      // run is walked matrix by matrix with constant indices into the maps:
      // a TMA given a tensor map at a run-time offset into the parameters is
      // markedly slower per copy.
      if (!early_codes) grid_dep_wait();
#pragma unroll
      for (int jj = 0; jj < kMaxGroup; ++jj) {
        if (jj < grp.count) {
          const int end_tile = jj + 1 < grp.count ? grp.mat[jj + 1 < kMaxGroup ? jj + 1 : jj].tile0
                                                  : grp.tiles;
          const int64_t lim = (int64_t)end_tile * kunits - u_begin;
          next_codes(lim < nu ? (int)lim : nu, &maps.I1[jj], &maps.I2[jj], grp.mat[jj].tile0);
        }
      }
      if (ld_shared_volatile(abort_flag)) {
        // let the copies in flight land before the CTA exits (bounded waits:
        // a stage's barrier may never complete once the other roles stopped)
        uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(table_full, 0))
          if (global_timer_ns() - t0 > 100000000ull) break;
        t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 1000000ull) {
        }
      }
    }
  } else if (warp == 1 || warp == MMA2_WARP) {
    // Two issuers, one per decoder group: the even units accumulate into the
    // parity-0 buffers, the odd units into the parity-1 buffers (the epilogue
    // adds the two).  The whole warp runs the loop (warp-uniform operands);
    // the elected lane issues the MMAs and the commits, so that every commit
    // tracks all MMAs before it.  A stage is released only when the producer
    // or a decoder will reuse it.
    const int par = warp == 1 ? 0 : 1;
    const uint32_t idesc = sk_idesc(ROWS, (uint32_t)rows_b);
    const uint32_t idesc_bias = sk_idesc_sa(ROWS, (uint32_t)rows_b);
    const uint64_t bd0 = smem_desc(smem_u32(xq_ring), 16, 1024, 2);
    const uint64_t const_desc = smem_desc(smem_u32(smem + plan.const_off), 128, 256, 0);
    const uint32_t stage16 = (uint32_t)plan.b_bytes >> 4;
    int s = par, sxi = par % SX;   // operand and Xq stages of the issuer's unit
    uint32_t ph = 0;
    bool ok = true;
    int lo = 0;                    // first local unit of the segment
    for (int seg = 0; seg < nseg && ok; ++seg) {
      const int len = kunits - (seg == 0 ? ku_first : 0);
      const int hi = lo + len < nu ? lo + len : nu;
      const int b = seg & 1;
      if (seg >= 2 && !warp_wait(&acc_empty[b], (uint32_t)((seg - 2) >> 1) & 1u, abort_flag,
                                 status, kDevTimeoutMma)) {
        ok = false;
        break;
      }
      const int i0 = lo + (((lo & 1) != par) ? 1 : 0);
      if (i0 >= hi) {
        // no unit of this parity in the segment
        if (elect_one()) mbar_arrive(&acc_full[b]);
        __syncwarp();
        lo = hi;
        continue;
      }
      const uint32_t d = tmem_base + (uint32_t)(par * 2 + b) * ACC_COLS;
      for (int i = i0; i < hi; i += 2) {
        if (!warp_wait(&full_a[s], ph, abort_flag, status, kDevTimeoutFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = tmem_a + (uint32_t)s * A_COLS;
        const uint64_t bds = bd0 + (uint64_t)((uint32_t)sxi * stage16);
        if (elect_one()) {
#pragma unroll
          for (int j = 0; j < KU / 32; ++j) {
            sk_mma_i8(d, a0 + (uint32_t)(j * 8), bds + (uint64_t)(j * 2), idesc,
                      (i == i0 && j == 0) ? 0u : 1u);
            // minus 128 times the same Xq columns: removes the weight bias
            if (CW == 32)
              sk_mma_i8(d, const_a_tmem, bds + (uint64_t)(j * 2), idesc_bias, 1u);
            else
              sk_mma_i8_ss(d, const_desc, bds + (uint64_t)(j * 2), idesc_bias, 1u);
          }
          // the stage is reused by unit i + SX (Xq) and unit i + SA (operand)
          if (i + SX < nu) mma_commit(&a_empty[s]);
        }
        __syncwarp();
        s += 2;
        if (s >= SA) {
          s -= SA;
          ph ^= 1u;
        }
        sxi += 2;
        if (sxi >= SX) sxi -= SX;
      }
      if (!ok) break;
      if (elect_one()) mma_commit(&acc_full[b]);
      __syncwarp();
      lo = hi;
    }
    if (elect_one()) {
      mma_commit(&drain[par]);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(&drain[par], 0))
        if (global_timer_ns() - t0 > 200000000ull) break;
    }
    __syncwarp();
  } else if (warp == XQ_WARP) {
    // ------------------------------------------------------------ Xq tiles
    if (lane == 0) {
      grid_dep_wait();
      int sa = 0;                    // operand stage of unit i
      int i = 0;
#pragma unroll
      for (int jj = 0; jj < kMaxGroup; ++jj) {
        if (jj >= grp.count) break;
        // the units of matrix jj, with its map at a constant index (see the
        // index producer)
        const int end_tile = jj + 1 < grp.count ? grp.mat[jj + 1 < kMaxGroup ? jj + 1 : jj].tile0
                                                : grp.tiles;
        const int64_t lim64 = (int64_t)end_tile * kunits - u_begin;
        const int lim = lim64 < nu ? (int)lim64 : nu;
        const CUtensorMap* mb = &maps.B[jj];
        for (; i < lim; ++i) {
          // the Xq stage of unit i was last read by the MMAs of unit i - SX, and
          // the operand stage's barrier must have completed the phase of unit
          // i - SA before this unit's arrival (the two issuers' MMAs, of
          // alternate units, complete in no fixed order)
          if (i >= SX && !mbar_wait_sleep(&a_empty[(i - SX) % SA], (uint32_t)((i - SX) / SA) & 1u,
                                          abort_flag, status, kDevTimeoutEmpty))
            break;
          if (i >= SA && !mbar_wait_sleep(&a_empty[(i - SA) % SA], (uint32_t)((i - SA) / SA) & 1u,
                                          abort_flag, status, kDevTimeoutEmpty))
            break;
          const int u = u_begin + i;
          mbar_arrive_expect_tx(&full_a[sa], (uint32_t)plan.b_bytes);
          tma_load_2d(xq_ring + (i % SX) * plan.b_bytes, mb, &full_a[sa], (u % kunits) * KU, 0);
          if (++sa == SA) sa = 0;
        }
        if (i < lim) break;   // a wait gave up
      }
      if (ld_shared_volatile(abort_flag)) {
        // let the copies in flight land before the CTA exits
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 1000000ull) {
        }
      }
    }
  } else if (warp < EPI_WARP0) {
    // ------------------------------------------------------------ decoders
    const int dw = warp - 2;
    const int q = warp & 3;
    const int dg = dw >> 2;
    const int r = q * 32 + lane;
    const uint32_t lane_bits = (uint32_t)(q * 32) << 16;
    bool ok = mbar_wait_sleep(table_full, 0, abort_flag, status, kDevTimeoutFull);
    int cs = dg % SC, as = dg % SA;
    uint32_t cph = 0, aph = 0;
    for (int i = dg; i < nu && ok; i += DEC_GROUPS) {
      if (!mbar_wait_sleep(&full_code[cs], cph, abort_flag, status, kDevTimeoutFull)) break;
      const uint8_t* si1 = code_ring + cs * plan.code_bytes;
      uint4 c1h[2], c2h[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        c1h[h] = *reinterpret_cast<const uint4*>(si1 + sw32_off(r, h));
        c2h[h] = make_uint4(0u, 0u, 0u, 0u);
        if (BPW == 4) {
          c2h[h] = *reinterpret_cast<const uint4*>(si1 + I1_BYTES + sw32_off(r, h));
        } else if (BPW == 3) {
          const uint2 c = *reinterpret_cast<const uint2*>(si1 + I1_BYTES + r * 16 + h * 8);
          c2h[h] = make_uint4(__byte_perm(c.x, 0u, 0x4140), __byte_perm(c.x, 0u, 0x4342),
                              __byte_perm(c.y, 0u, 0x4140), __byte_perm(c.y, 0u, 0x4342));
        }
      }
      // the indices are in registers: the index-tile stage can be refilled
      // once these shared-memory reads are ordered before the next bulk copy
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&code_empty[cs]);
      // the operand stage must have been read by the MMAs of unit i - SA
      if (i >= SA &&
          !mbar_wait_sleep(&a_empty[as], aph ^ 1u, abort_flag, status, kDevTimeoutMma))
        break;
      tc_fence_after();
      // the two halves of the row's 16 groups, 16 TMEM columns each
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t w1[4] = {c1h[h].x, c1h[h].y, c1h[h].z, c1h[h].w};
        const uint32_t w2[4] = {c2h[h].x, c2h[h].y, c2h[h].z, c2h[h].w};
        uint32_t v[16];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t ea0 = sk_entry(table, sk_off_lo(w1[k]));
          const uint32_t ea1 = sk_entry(table, sk_off_hi(w1[k]));
          const uint32_t eb0 = BPW > 2 ? sk_entry(table, sk_off_lo(w2[k])) : 0u;
          const uint32_t eb1 = BPW > 2 ? sk_entry(table, sk_off_hi(w2[k])) : 0u;
          decode_group_q8<BPW>(w1[k] & 0xFFFFu, w2[k] & 0xFFFFu, ea0, eb0, v[4 * k],
                               v[4 * k + 1]);
          decode_group_q8<BPW>(w1[k] >> 16, w2[k] >> 16, ea1, eb1, v[4 * k + 2], v[4 * k + 3]);
        }
        sk_tmem_st16(tmem_a + lane_bits + (uint32_t)as * A_COLS + (uint32_t)(h * 16), v);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full_a[as]);
      cs += DEC_GROUPS;
      if (cs >= SC) {
        cs -= SC;
        cph ^= 1u;
      }
      as += DEC_GROUPS;
      if (as >= SA) {
        as -= SA;
        aph ^= 1u;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const bool issuer = warp == EPI_WARP0 && lane == 0;
    grid_dep_wait();   // steps and the zeroed Y come from the transform
    if (warp == EPI_WARP0) {
      for (int j = 0; j < grp.count; ++j) {
        const SkMat& mt = grp.mat[j];
        s_sc[32 * j + lane] = lane < M ? mt.alpha * __ldg(mt.tok_scale + lane) : 0.0f;
      }
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");   // the steps
    // every epilogue thread runs the same sequence of named barriers, also
    // after a failed wait (it then only skips the work)
    bool ok = true;
    int lo = 0;                      // first local unit of the segment
    for (int seg = 0; seg < nseg; ++seg) {
      const int b = seg & 1;
      const int len = kunits - (seg == 0 ? ku_first : 0);
      const int hi = lo + len < nu ? lo + len : nu;
      // which issuers accumulated into the segment (units of parity 0 / 1)
      const bool has0 = hi - lo >= 2 || (lo & 1) == 0;
      const bool has1 = hi - lo >= 2 || (lo & 1) == 1;
      const int tile = first_tile + seg;
      const int mj = sk_mat_of(grp, tile);
      lo = hi;
      ok = ok && mbar_wait_sleep(&acc_full[b], (uint32_t)(seg >> 1) & 1u, abort_flag, status,
                                 kDevTimeoutMma);
      tc_fence_after();
      const int N = grp.mat[mj].N;
      float* __restrict__ Y = grp.mat[mj].Y;
      const int use_tma_y = grp.mat[mj].use_tma_y;
      const float* sc = s_sc + 32 * mj;
      const int n = (tile - grp.mat[mj].tile0) * ROWS + r;
      const uint32_t lane_off = (uint32_t)(q * 32) << 16;
      const uint32_t t0a = tmem_base + (uint32_t)b * ACC_COLS + lane_off;         // parity 0
      const uint32_t t1a = tmem_base + (uint32_t)(2 + b) * ACC_COLS + lane_off;   // parity 1
      // 8 accumulator columns (4 tokens) per pass
#pragma unroll
      for (int c0 = 0; c0 < CW; c0 += 8) {
        if (!ok) break;
        uint32_t dv[8], dw[8];
        if (c0 < rows_b) {
          if (has0) sk_tmem_ld8(t0a + (uint32_t)c0, dv);
          if (has1) sk_tmem_ld8(t1a + (uint32_t)c0, dw);
          tmem_ld_wait();
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t x0 = (c0 < rows_b && has0) ? dv[j] : 0u;
          const uint32_t x1 = (c0 < rows_b && has1) ? dw[j] : 0u;
          dv[j] = x0 + x1;
        }
        if (use_tma_y) {
          // tokens past M have zero steps: staged as zeros (the
          // bulk reduce covers only M rows), no branch in the loop
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int m = (c0 >> 1) + j;
            s_y[m * ROWS + r] = sc[m] * ((float)(int)dv[2 * j] + (float)(int)dv[2 * j + 1] *
                                                                     (1.0f / 128.0f));
          }
        } else if (n < N) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int m = (c0 >> 1) + j;
            if (m < M)
              red_add_f32(Y + (size_t)m * N + n,
                          sc[m] * ((float)(int)dv[2 * j] + (float)(int)dv[2 * j + 1] *
                                                               (1.0f / 128.0f)));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(&acc_empty[b]);
      if (use_tma_y) {
        // the staged tile [M][128] goes to Y[0..M)[tile * 128 ..) by one bulk
        // reduce-add; the stage is reused only after the unit has read it
        fence_proxy_async_smem();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (issuer && ok) {
          const int ty = (tile - grp.mat[mj].tile0) * ROWS;
          // constant map indices (see the index producer)
          if (mj == 0) tma_reduce_add_2d(&maps.Y[0], smem_u32(s_y), ty, 0);
          else if (mj == 1) tma_reduce_add_2d(&maps.Y[1], smem_u32(s_y), ty, 0);
          else if (mj == 2) tma_reduce_add_2d(&maps.Y[2], smem_u32(s_y), ty, 0);
          else tma_reduce_add_2d(&maps.Y[3], smem_u32(s_y), ty, 0);
          bulk_wait_read_all();
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
      }
    }
    if (issuer) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, plan.tmem_cols);
  }
}

template <int BPW>
static cudaError_t launch_gemm_q8(const DeviceCodebook& cb, const Q8Item* items, int count,
                                  int64_t M, int64_t K, int rows_b, int pdl, int early_codes,
                                  int sm_count, cudaStream_t st) {
  using namespace sk;
  if (rows_b < 16 || rows_b > 64 || (rows_b % 16) != 0 || M < 1 || M > 32 || 2 * M > rows_b ||
      (K % KU) != 0 || K > INT32_MAX || count < 1 || count > kMaxGroup)
    return cudaErrorInvalidValue;
  SkMaps maps;
  SkGroup grp = {};
  grp.count = count;
  int64_t tiles = 0;
  for (int g = 0; g < count; ++g) {
    const Q8Item& a = items[g];
    if (a.N < 1 || a.N > INT32_MAX) return cudaErrorInvalidValue;
    if (!make_tmap_2d(&maps.B[g], a.Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)rows_b,
                      (uint64_t)K, (uint32_t)rows_b, KU, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    if (!make_tmap_2d(&maps.I1[g], a.idx1, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, (uint64_t)a.N,
                      (uint64_t)(K / 8), ROWS, GROUPS, CU_TENSOR_MAP_SWIZZLE_32B))
      return cudaErrorInvalidValue;
    if (BPW == 4) {
      if (!make_tmap_2d(&maps.I2[g], a.idx2, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, (uint64_t)a.N,
                        (uint64_t)(K / 8), ROWS, GROUPS, CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;
    } else if (BPW == 3) {
      if (!make_tmap_2d(&maps.I2[g], a.idx2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.N,
                        (uint64_t)(K / 8), ROWS, GROUPS, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    } else {
      maps.I2[g] = maps.I1[g];
    }
    // Y by bulk reduce-add when its rows are 16-byte multiples (else fp32 atomics)
    int use_tma_y = (a.N % 4) == 0 &&
                    make_tmap_2d(&maps.Y[g], a.Y, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)M,
                                 (uint64_t)a.N, (uint32_t)M, ROWS, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!use_tma_y) maps.Y[g] = maps.B[g];
    SkMat& mt = grp.mat[g];
    mt.tile0 = (int)tiles;
    mt.N = (int)a.N;
    mt.alpha = a.alpha;
    mt.use_tma_y = use_tma_y;
    mt.tok_scale = a.scales;
    mt.Y = a.Y;
    tiles += (a.N + ROWS - 1) / ROWS;
  }
  for (int g = count; g < kMaxGroup; ++g) {
    maps.B[g] = maps.B[0];
    maps.I1[g] = maps.I1[0];
    maps.I2[g] = maps.I2[0];
    maps.Y[g] = maps.Y[0];
  }
  const SkPlan plan = sk_plan(rows_b, BPW);
  if (plan.sa < 2 || plan.sc < 2 || plan.total > kMaxDynSmem) return cudaErrorInvalidValue;
  const int64_t units = tiles * (K / KU);
  if (units > INT32_MAX) return cudaErrorInvalidValue;
  grp.tiles = (int)tiles;
  const int grid = (int)(units < sm_count ? units : sm_count);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = (size_t)plan.total;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  auto kern = rows_b <= 32 ? k_gemm_q8<BPW, 32> : k_gemm_q8<BPW, 64>;
  // the largest carveout, as the transform kernel has: CTAs of the two can share an SM
  cudaError_t e = ensure_smem_limit(kern, kMaxDynSmem, true);
  if (e != cudaSuccess) return e;
  e = cudaLaunchKernelEx(&cfg, kern, maps, grp, cb, (int)M, (int)K, rows_b, early_codes);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_gemm_q8_group(const DeviceCodebook& cb, const Q8Item* items, int count,
                                 int64_t M, int64_t K, int rows_b, int bpw, int pdl,
                                 int early_codes, int sm_count, cudaStream_t st) {
  if (bpw == 2) return launch_gemm_q8<2>(cb, items, count, M, K, rows_b, pdl, early_codes,
                                         sm_count, st);
  if (bpw == 3) return launch_gemm_q8<3>(cb, items, count, M, K, rows_b, pdl, early_codes,
                                         sm_count, st);
  return launch_gemm_q8<4>(cb, items, count, M, K, rows_b, pdl, early_codes, sm_count, st);
}

cudaError_t launch_act_gemm_q8(const DeviceCodebook& cb, const ActQ8Args& a, int sm_count,
                               cudaStream_t st) {
  Q8Item it;
  it.idx1 = a.idx1;
  it.idx2 = a.idx2;
  it.N = a.N;
  it.alpha = a.alpha;
  it.Xq = a.Xq;
  it.scales = a.scales;
  it.Y = a.Y;
  return launch_gemm_q8_group(cb, &it, 1, a.M, a.K, a.rows_b, a.bpw, a.pdl, a.early_codes,
                              sm_count, st);
}

}  // namespace e8
