// Decoder on the tensor cores: codebook indices -> bf16 weights for Hadamard
// blocks of n_h = 1024, 2048 or 4096 ("glq 0.1.1", "How it works", items
// 1-2: the inverse of the randomized Hadamard transform of the encoder).
//
//   z = m (c1 + beta c2)   integer 8-vector per group
//   t = FWHT_nh(z)         exact on integers
//   w = bf16_rne(d * fl32(t * alpha))
//
// With n_h = 64 R and a block read as R rows of 64 (position 64 a + b), the
// natural-order Sylvester matrix factors as H_nh = H_R (x) H_8 (x) H_8:
//   * H_8 inside each group of 8: the decoders gather from the transformed
//     pair table, which holds H_8 v / 4, so one group decodes straight to
//     H_8 z / 4 (integers, |.| <= 20);
//   * H_8 across the 8 groups of a row of 64: three butterfly stages in the
//     decoder thread that owns the row, in fp16 (exact: |U / 4| <= 160), give
//     U / 4 with U = Z H_64 (H_64 = H_8 (x) H_8);
//   * H_R across the R rows of a block: one tensor-core product per slab of
//     8192 weights (128 rows of 64), kind::f16 with fp32 accumulation,
//     T / 4 = diag(H_R, ..., H_R) (U / 4): A = the 128 / R copies of H_R on
//     the diagonal (tensor memory), B = the slab's U / 4 as written by the
//     decoders, row after row (shared memory, N-major); |T / 4| <= 10240,
//     exact in fp32.
// Lane m of the accumulator owns slab weights 64 m .. 64 m + 63, and
// fl32((T / 4) (4 alpha)) = fl32(t alpha) exactly, so the result equals the
// sequential definition bit for bit (the only roundings are the two of w).
// Each warp of the readout stages its 32 x 32 bf16 piece of the slab in a
// 64-byte-swizzled tile and writes it with one TMA store.
//
// Roles (one CTA per SM, persistent over slabs):
//   warp 0      producer: table, then bulk copies of each slab's index words
//   warp 1      tensor-memory allocation; one elected lane issues the product
//   warps 2-9   decoders, two groups of four taking alternate slabs; thread r
//               of a group decodes row r of the slab
//   warps 10-17 readout: T -> scale, sign, bf16, TMA store
// The product of slab i waits on one barrier: the decoder warps that wrote
// its operand stage and the readout warps that emptied its accumulator
// buffer (slab i - 4) arrive on the same one.
#include <cuda_fp16.h>

#include "e8_common.cuh"
#include "e8_codebook.cuh"
#include "e8_internal.h"
#include "e8_tmap.h"

namespace e8 {

namespace dtc {
constexpr int SLAB = 8192;                  // weights per slab
constexpr int GROUPS = SLAB / 8;
constexpr int TABLE_BYTES = 131088;
constexpr int STAGES = 4;                   // operand and accumulator rings
// Index-word ring: an even number of stages, so that each stage serves one
// decoder group only.  Bulk copies may land out of order; were a stage shared
// by both groups, a group could reach its next use of the stage while the
// other group's copy into it was still in flight, and the parity wait would
// take the barrier two phases behind for the phase it waits for.
constexpr int CSTAGES = 2;
constexpr int CODE_BYTES = GROUPS * 4;      // idx1 (2 KB) + idx2 (up to 2 KB)
constexpr int B_BYTES = 128 * 128;          // 128 rows x 64 fp16, 128-byte swizzled
constexpr int YW_BYTES = 32 * 64;           // one readout warp's 32 x 32 bf16 tile
constexpr int SIGN_CHUNKS = 256;            // sign words kept in shared memory (K <= 16384)
constexpr int DEC_WARP0 = 2;
constexpr int DEC_WARPS = 8;                // two groups of four
constexpr int RD_WARP0 = DEC_WARP0 + DEC_WARPS;
constexpr int RD_WARPS = 8;
constexpr int THREADS = 32 * (RD_WARP0 + RD_WARPS);
// tensor memory columns
constexpr uint32_t A_COL = 0;               // diag(H_R ...), f16: 64 columns
constexpr uint32_t D_COL = 64;              // four buffers of 64
constexpr uint32_t TMEM_COLS = 512;
// shared memory (after the table, from the next 1 KB boundary)
constexpr int CODE_OFF = 0;
constexpr int B_OFF = CODE_OFF + CSTAGES * CODE_BYTES;        // 8 KB
constexpr int Y_OFF = B_OFF + STAGES * B_BYTES;               // 72 KB
constexpr int SIGN_OFF = Y_OFF + RD_WARPS * YW_BYTES;         // 88 KB
constexpr int BAR_OFF = SIGN_OFF + SIGN_CHUNKS * 8;           // 96 KB
constexpr int SMEM_TOTAL = TABLE_BYTES + 1024 + BAR_OFF + 256;
static_assert(SMEM_TOTAL <= kMaxDynSmem, "shared memory budget");
static_assert(B_OFF % 1024 == 0 && Y_OFF % 1024 == 0, "swizzled tiles sit on 1 KB boundaries");
}  // namespace dtc

__device__ __forceinline__ void dtc_mma_f16_ts(uint32_t d, uint32_t a, uint64_t b,
                                               uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// kind::f16: A, B fp16, D fp32; A K-major, B N-major (bit 16).
__host__ __device__ constexpr uint32_t dtc_idesc_f16_bn(uint32_t M, uint32_t N) {
  return (1u << 4) | (0u << 7) | (0u << 10) | (1u << 16) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

__device__ __forceinline__ void dtc_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void dtc_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

// Sylvester-Hadamard entry H[i][j] = (-1)^popcount(i & j).
__device__ __forceinline__ bool had_neg(uint32_t i, uint32_t j) { return __popc(i & j) & 1; }

// Byte address, in a 128-byte-swizzled K-major tile, of byte `col` of row `row`.
__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t col) {
  return row * 128u + ((((col >> 4) ^ (row & 7u)) << 4) | (col & 15u));
}

// The 32 sign bits v of 32 consecutive weights, rearranged for pairs: bit
// 15 - j holds v bit 2 j and bit 31 - j holds v bit 2 j + 1, so that
// (W << j) & 0x80008000 is the sign mask of the bf16 pair j.  Even bits are
// gathered into the low half and odd bits into the high half by four
// delta swaps, then the word is bit-reversed and its halves exchanged.
__device__ __forceinline__ uint32_t pair_sign_word(uint32_t v) {
  uint32_t t;
  t = (v ^ (v >> 1)) & 0x22222222u;
  v ^= t ^ (t << 1);
  t = (v ^ (v >> 2)) & 0x0C0C0C0Cu;
  v ^= t ^ (t << 2);
  t = (v ^ (v >> 4)) & 0x00F000F0u;
  v ^= t ^ (t << 4);
  t = (v ^ (v >> 8)) & 0x0000FF00u;
  v ^= t ^ (t << 8);
  const uint32_t b = __brev(v);
  return (b >> 16) | (b << 16);
}

struct DecodeTcParams {
  const uint16_t* idx1;
  const void* idx2;
  int64_t slabs;          // N * K / 8192
  int K, log2R;           // R = n_h / 64
  uint64_t seed;
  float alpha;
  const uint32_t* table;  // transformed pair table H_8 v / 4 (global)
  uint32_t* status;
};

// Bulk copies of one slab's index words into a stage of the ring.
template <int BPW>
__device__ __forceinline__ void load_codes(const DecodeTcParams& p, uint8_t* dst, uint64_t* bar,
                                           int64_t slab) {
  constexpr uint32_t i2b = BPW == 4 ? 2048u : (BPW == 3 ? 1024u : 0u);
  mbar_arrive_expect_tx(bar, 2048u + i2b);
  bulk_load(dst, p.idx1 + slab * dtc::GROUPS, 2048u, bar);
  if (BPW > 2)
    bulk_load(dst + 2048, static_cast<const uint8_t*>(p.idx2) + slab * (int64_t)i2b, i2b, bar);
}

// L2 prefetch of one slab's index words (no shared memory, no completion).
template <int BPW>
__device__ __forceinline__ void prefetch_codes_l2(const DecodeTcParams& p, int64_t slab) {
  constexpr uint32_t i2b = BPW == 4 ? 2048u : (BPW == 3 ? 1024u : 0u);
  bulk_prefetch_l2(p.idx1 + slab * dtc::GROUPS, 2048u);
  if (BPW > 2) bulk_prefetch_l2(static_cast<const uint8_t*>(p.idx2) + slab * (int64_t)i2b, i2b);
}

template <int BPW>
__global__ void __launch_bounds__(dtc::THREADS, 1)
    k_decode_tc(const DecodeTcParams p, const __grid_constant__ CUtensorMap tmOut) {
  using namespace dtc;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint8_t* table = smem_raw;   // transformed pair table: H_8 v / 4
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + TABLE_BYTES + 1023) & ~uintptr_t(1023));
  uint8_t* codes = smem + CODE_OFF;
  uint8_t* bst = smem + B_OFF;
  uint8_t* ytile = smem + Y_OFF;
  uint32_t* sgn = reinterpret_cast<uint32_t*>(smem + SIGN_OFF);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* code_full = bars;                 // [2] index words landed
  uint64_t* code_empty = bars + CSTAGES;      // [2] decoders hold them in registers
  uint64_t* b_full = bars + 2 * CSTAGES;      // [4] operand written + accumulator buffer free
  uint64_t* b_empty = b_full + STAGES;        // [4] product done with the operand
  uint64_t* d_full = b_empty + STAGES;        // [4] product in tensor memory
  uint64_t* table_full = d_full + STAGES;
  uint64_t* drain = table_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  uint32_t* status = p.status;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nsl = (p.slabs - (int64_t)blockIdx.x + gridDim.x - 1) / gridDim.x;
  const int chunks = p.K >> 6;
  const bool sgn_in_smem = chunks <= SIGN_CHUNKS;

  if (threadIdx.x == 0) {
    for (int s = 0; s < CSTAGES; ++s) {
      mbar_init(&code_full[s], 1);
      mbar_init(&code_empty[s], DEC_WARPS / 2);
    }
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&b_full[s], DEC_WARPS / 2 + RD_WARPS);
      mbar_init(&b_empty[s], 1);
      mbar_init(&d_full[s], 1);
      // the accumulator buffers start free
      for (int w = 0; w < RD_WARPS; ++w) mbar_arrive(&b_full[s]);
    }
    mbar_init(table_full, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
    *abort_flag = 0u;
    // the 128 KB table and the first index words stream in while the
    // constants are built
    mbar_arrive_expect_tx(table_full, TABLE_BYTES);
    for (int j = 0; j < 8; ++j) {
      const int c = (j + (int)blockIdx.x) & 7;
      bulk_load(smem_raw + c * 16384, reinterpret_cast<const uint8_t*>(p.table) + c * 16384,
                16384, table_full);
    }
    bulk_load(smem_raw + 8 * 16384, reinterpret_cast<const uint8_t*>(p.table) + 8 * 16384, 16,
              table_full);
    for (int64_t i = 0; i < nsl && i < CSTAGES; ++i)
      load_codes<BPW>(p, codes + i * CODE_BYTES, &code_full[i], (int64_t)blockIdx.x + i * gridDim.x);
    tma_prefetch_desc(&tmOut);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp >= RD_WARP0) {
    // diag(H_R, ...) as fp16, one row per tensor-memory lane: columns 0-31
    // (k = 0..63) by warps 10-13, 32-63 by warps 14-17.  H[d][a0 | b] =
    // H[d][a0] H[d][b] for b < 2 <= lowest set bit of a0: each word is the
    // row's first two entries, negated by H[d][a0].
    const uint32_t q = warp & 3, m = q * 32 + lane;
    const uint32_t lane_bits = (q * 32) << 16;
    const int part = (warp - RD_WARP0) >> 2;
    const uint32_t lr = (uint32_t)p.log2R, d = m & ((1u << lr) - 1u);
    const uint32_t base2 = 0x3C00u | ((d & 1u) ? 0xBC000000u : 0x3C000000u);
    uint32_t v[32];
#pragma unroll
    for (int w = 0; w < 32; ++w) {
      const uint32_t k0 = 64u * part + 2u * w;
      v[w] = (k0 >> lr) != (m >> lr) ? 0u : (had_neg(d, k0) ? base2 ^ 0x80008000u : base2);
    }
    dtc_st32(tmem_base + lane_bits + A_COL + 32 * part, v);
    tmem_st_wait();
    if (sgn_in_smem) {
      // the sign words of every 64-column chunk of a row, in pair form
      for (int g = threadIdx.x - 32 * RD_WARP0; g < chunks; g += 32 * RD_WARPS) {
        const uint64_t word = splitmix64_output(p.seed, (uint64_t)g);
        sgn[2 * g] = pair_sign_word((uint32_t)word);
        sgn[2 * g + 1] = pair_sign_word((uint32_t)(word >> 32));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // slabs 0 .. CSTAGES - 1 were issued before the role split
      int s = 0;
      uint32_t ph = 1;
      int64_t issued = nsl < CSTAGES ? nsl : CSTAGES;
      for (int64_t i = CSTAGES; i < nsl; ++i) {
        if (!mbar_wait_sleep(&code_empty[s], ph ^ 1u, abort_flag, status, kDevTimeoutEmpty))
          break;
        load_codes<BPW>(p, codes + s * CODE_BYTES, &code_full[s],
                        (int64_t)blockIdx.x + i * gridDim.x);
        ++issued;
        // the ring holds two slabs, less than the latency of a copy from
        // HBM; bring the index words of slabs i + 3 and i + 4 into L2 now
        for (int64_t f = i + 3; f < i + 5 && f < nsl; ++f)
          prefetch_codes_l2<BPW>(p, (int64_t)blockIdx.x + f * gridDim.x);
        if (++s == CSTAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (ld_shared_volatile(abort_flag)) {
        // let the copies in flight land before the CTA exits
        uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(table_full, 0))
          if (global_timer_ns() - t0 > 100000000ull) break;
        for (int64_t j = issued > CSTAGES ? issued - CSTAGES : 0; j < issued; ++j) {
          t0 = global_timer_ns();
          while (!mbar_try_wait(&code_full[j % CSTAGES], (uint32_t)(j / CSTAGES) & 1u))
            if (global_timer_ns() - t0 > 100000000ull) break;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (warp-uniform operands); one elected lane
    // issues.  K = 128 slab rows: eight steps of 16 rows = 2 KB of the
    // operand stage each.
    const uint32_t idesc = dtc_idesc_f16_bn(128, 64);
    const uint64_t bd0 = smem_desc(smem_u32(bst), 16, 1024, 2);
    int s = 0;
    uint32_t ph = 0;
    for (int64_t i = 0; i < nsl; ++i) {
      if (!warp_wait(&b_full[s], ph, abort_flag, status, kDevTimeoutFull)) break;
      tc_fence_after();
      const uint32_t d = tmem_base + D_COL + 64u * (uint32_t)s;
      const uint64_t bd = bd0 + (uint64_t)(((uint32_t)s * B_BYTES) >> 4);
      if (elect_one()) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          dtc_mma_f16_ts(d, tmem_base + A_COL + 8u * j, bd + (uint64_t)(j * (2048 >> 4)), idesc,
                         j > 0 ? 1u : 0u);
        mma_commit(&b_empty[s]);
        mma_commit(&d_full[s]);
      }
      __syncwarp();
      if (++s == STAGES) {
        s = 0;
        ph ^= 1u;
      }
    }
    if (elect_one()) {
      mma_commit(drain);
      const uint64_t t1 = global_timer_ns();
      while (!mbar_try_wait(drain, 0))
        if (global_timer_ns() - t1 > 200000000ull) break;
    }
    __syncwarp();
  } else if (warp < RD_WARP0) {
    // ------------------------------------------------------------ decoders
    // group `grp` takes slabs grp, grp + 2, ...; thread r decodes slab row r
    // (groups 8 r .. 8 r + 7) and finishes its 64-point transform
    const int grp = (warp - DEC_WARP0) >> 2;
    const uint32_t r = (uint32_t)(threadIdx.x - 32 * DEC_WARP0) & 127u;
    const __half2 bias2 = __half2half2(__ushort_as_half((unsigned short)0x6880u));   // 2304
    bool ok = warp_wait(table_full, 0, abort_flag, status, kDevTimeoutFull);
    for (int64_t i = grp; i < nsl && ok; i += 2) {
      const int cs = (int)(i % CSTAGES);
      if (!warp_wait(&code_full[cs], (uint32_t)(i / CSTAGES) & 1u, abort_flag, status,
                     kDevTimeoutFull))
        break;
      const uint8_t* cw = codes + cs * CODE_BYTES;
      const uint4 c1 = *reinterpret_cast<const uint4*>(cw + 16 * r);
      uint4 c2 = make_uint4(0u, 0u, 0u, 0u);
      if (BPW == 4) {
        c2 = *reinterpret_cast<const uint4*>(cw + 2048 + 16 * r);
      } else if (BPW == 3) {
        const uint2 c = *reinterpret_cast<const uint2*>(cw + 2048 + 8 * r);
        c2 = make_uint4(__byte_perm(c.x, 0u, 0x4140), __byte_perm(c.x, 0u, 0x4342),
                        __byte_perm(c.y, 0u, 0x4140), __byte_perm(c.y, 0u, 0x4342));
      }
      // the index words are in registers; order these shared-memory reads
      // before the producer's next bulk-copy write into the stage
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&code_empty[cs]);
      const int s = (int)(i % STAGES);
      const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
      // decode: group g -> four fp16 pairs 1024 + (H_8 z / 4 + 128), in
      // coordinate order
      __half2 x[8][4];
      const uint32_t w1[4] = {c1.x, c1.y, c1.z, c1.w}, w2[4] = {c2.x, c2.y, c2.z, c2.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t ea0 = *reinterpret_cast<const uint32_t*>(table + ((((w1[k] & 0xFFFFu) << 1) + 2u) & 0x3FFFCu));
        const uint32_t ea1 = *reinterpret_cast<const uint32_t*>(table + (((w1[k] >> 15) + 2u) & 0x3FFFCu));
        const uint32_t eb0 = BPW > 2 ? *reinterpret_cast<const uint32_t*>(table + ((((w2[k] & 0xFFFFu) << 1) + 2u) & 0x3FFFCu)) : 0u;
        const uint32_t eb1 = BPW > 2 ? *reinterpret_cast<const uint32_t*>(table + (((w2[k] >> 15) + 2u) & 0x3FFFCu)) : 0u;
        uint32_t lo0, hi0, lo1, hi1;
        decode_group_q8<BPW>(w1[k] & 0xFFFFu, w2[k] & 0xFFFFu, ea0, eb0, lo0, hi0);
        decode_group_q8<BPW>(w1[k] >> 16, w2[k] >> 16, ea1, eb1, lo1, hi1);
        const uint32_t wd[4] = {lo0, hi0, lo1, hi1};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t a = __byte_perm(wd[e], 0x64646464u, 0x4140);
          const uint32_t b = __byte_perm(wd[e], 0x64646464u, 0x4342);
          x[2 * k + (e >> 1)][2 * (e & 1)] = *reinterpret_cast<const __half2*>(&a);
          x[2 * k + (e >> 1)][2 * (e & 1) + 1] = *reinterpret_cast<const __half2*>(&b);
        }
      }
      // H_8 across the groups, natural order, exact in fp16.  First stage
      // with the bias 2 x 1152 removed: (A + (B - 2304)) and (A - B), both
      // intermediates integers below 2048 in magnitude.
#pragma unroll
      for (int g = 0; g < 8; g += 2)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __half2 a = x[g][e], b = x[g + 1][e];
          x[g][e] = __hadd2(a, __hsub2(b, bias2));
          x[g + 1][e] = __hsub2(a, b);
        }
#pragma unroll
      for (int h = 2; h < 8; h <<= 1)
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          if (g & h) continue;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __half2 a = x[g][e], b = x[g + h][e];
            x[g][e] = __hadd2(a, b);
            x[g + h][e] = __hsub2(a, b);
          }
        }
      // the product of slab i - 4 has read this operand stage
      if (i >= STAGES && !warp_wait(&b_empty[s], ph ^ 1u, abort_flag, status, kDevTimeoutMma))
        break;
      // row r of the N-major operand: U[r][8 g' + k'] for g' = 0..7, one
      // 16-byte chunk per g', 128-byte swizzled
      uint8_t* brow = bst + s * B_BYTES + r * 128u;
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        uint4 v;
        v.x = *reinterpret_cast<const uint32_t*>(&x[g][0]);
        v.y = *reinterpret_cast<const uint32_t*>(&x[g][1]);
        v.z = *reinterpret_cast<const uint32_t*>(&x[g][2]);
        v.w = *reinterpret_cast<const uint32_t*>(&x[g][3]);
        *reinterpret_cast<uint4*>(brow + (((uint32_t)g ^ (r & 7u)) << 4)) = v;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b_full[s]);
    }
  } else {
    // ------------------------------------------------------------ readout
    // lane m of the accumulator, columns 32 hh .. 32 hh + 31: slab weights
    // 64 m + 32 hh .., staged as row `lane` of this warp's 32 x 32 tile
    // (64-byte swizzled: chunk j of row l at ((j ^ ((l >> 1) & 3)) << 4))
    const uint32_t q = warp & 3, wi = (uint32_t)(warp - RD_WARP0), hh = wi >> 2;
    const uint32_t m = q * 32 + lane;
    const uint32_t lane_bits = (q * 32) << 16;
    const uint32_t K = (uint32_t)p.K;
    const float alpha4 = 4.0f * p.alpha;
    // column of the slab's first weight, advanced by grid * 8192 mod K
    const uint32_t step = (uint32_t)(((uint64_t)gridDim.x * SLAB) % K);
    uint32_t base = (uint32_t)(((uint64_t)blockIdx.x * SLAB) % K);
    const uint32_t offm = (64u * m) % K;
    uint8_t* yt = ytile + wi * YW_BYTES;
    uint32_t yoff[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) yoff[j] = lane * 64u + ((j ^ ((lane >> 1) & 3u)) << 4);
    int s = 0;
    uint32_t ph = 0;
    for (int64_t i = 0; i < nsl; ++i) {
      if (!warp_wait(&d_full[s], ph, abort_flag, status, kDevTimeoutMma)) break;
      tc_fence_after();
      uint32_t y[32];
      dtc_ld32(tmem_base + lane_bits + D_COL + 64u * (uint32_t)s + 32u * hh, y);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b_full[s]);   // accumulator buffer free for slab i + 4
      uint32_t pos = base + offm;
      if (pos >= K) pos -= K;
      uint32_t W;
      if (sgn_in_smem) {
        W = sgn[2 * (pos >> 6) + hh];
      } else {
        const uint64_t word = splitmix64_output(p.seed, (uint64_t)(pos >> 6));
        W = pair_sign_word((uint32_t)(word >> (32 * hh)));
      }
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float a = __fmul_rn(__uint_as_float(y[2 * e]), alpha4);
        const float b = __fmul_rn(__uint_as_float(y[2 * e + 1]), alpha4);
        pk[e] = pack_bf16x2(a, b) ^ ((W << e) & 0x80008000u);
      }
      // the store of slab i - 1 has read the tile
      if (i >= 1 && lane == 0) bulk_wait_read_all();
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4*>(yt + yoff[j]) =
            make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const int64_t slab = (int64_t)blockIdx.x + i * gridDim.x;
        tma_store_2d(&tmOut, smem_u32(yt), (int32_t)(32 * hh), (int32_t)(slab * 128 + 32 * q));
      }
      base += step;
      if (base >= K) base -= K;
      if (++s == STAGES) {
        s = 0;
        ph ^= 1u;
      }
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <int BPW>
static cudaError_t launch_decode_tc_t(const DecodeTcParams& p, const CUtensorMap& tm, int grid,
                                      cudaStream_t st) {
  cudaError_t e = ensure_smem_limit(k_decode_tc<BPW>, kMaxDynSmem);
  if (e != cudaSuccess) return e;
  k_decode_tc<BPW><<<grid, dtc::THREADS, dtc::SMEM_TOTAL, st>>>(p, tm);
  return cudaGetLastError();
}

// Shapes served: n_h in {1024, 2048, 4096}, N K a multiple of 8192 with
// N K / 64 rows addressable by the store, 16-byte aligned buffers.
bool decode_tc_eligible(int64_t N, int64_t K, const void* idx1, const void* idx2,
                        const void* out, int64_t nh_arg) {
  const int64_t nh = resolve_nh(K, nh_arg);
  auto al = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
  return N > 0 && (nh == 1024 || nh == 2048 || nh == 4096) && ((N * K) % dtc::SLAB) == 0 &&
         K <= ((int64_t)1 << 30) && N * K / 64 < ((int64_t)1 << 31) && al(idx1) &&
         (idx2 == nullptr || al(idx2)) && al(out);
}

cudaError_t launch_decode_tc(const DeviceCodebook& cb, const uint16_t* idx1, const void* idx2,
                             int64_t N, int64_t K, int bpw, uint64_t seed, float alpha,
                             uint16_t* Wdec, int sm_count, cudaStream_t st, int64_t nh_arg) {
  if (!decode_tc_eligible(N, K, idx1, bpw > 2 ? idx2 : nullptr, Wdec, nh_arg))
    return cudaErrorNotSupported;
  CUtensorMap tm;
  if (!make_tmap_2d(&tm, Wdec, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)(N * K / 64), 64,
                    32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorNotSupported;
  DecodeTcParams p;
  p.idx1 = idx1;
  p.idx2 = idx2;
  p.slabs = N * K / dtc::SLAB;
  p.K = (int)K;
  const int64_t nh = resolve_nh(K, nh_arg);
  p.log2R = 0;
  while ((int64_t(64) << p.log2R) < nh) ++p.log2R;
  p.seed = seed;
  p.alpha = alpha;
  p.table = cb.h8table;
  p.status = cb.status;
  const int grid = (int)(p.slabs < sm_count ? p.slabs : sm_count);
  if (bpw == 2) return launch_decode_tc_t<2>(p, tm, grid, st);
  if (bpw == 3) return launch_decode_tc_t<3>(p, tm, grid, st);
  return launch_decode_tc_t<4>(p, tm, grid, st);
}

}  // namespace e8
