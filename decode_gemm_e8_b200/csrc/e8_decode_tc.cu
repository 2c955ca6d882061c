// Decoder on the tensor cores: codebook indices -> bf16 weights for Hadamard
// blocks of n_h = 1024, 2048 or 4096 ("glq 0.1.1", "How it works", items
// 1-2: the inverse of the randomized Hadamard transform of the encoder).
//
//   z = m (c1 + beta c2)   integer 8-vector per group, |z| <= 30
//   t = FWHT_nh(z)         exact on integers
//   w = bf16_rne(d * fl32(t * alpha))
//
// With n_h = 64 R and a block read as R rows of 64 (position 64 a + b), the
// Sylvester matrix factors as H_nh = H_R (x) H_64, so t = H_R Z H_64.  Work
// unit: a slab of 8192 consecutive weights = 128 rows of 64 (8192 / n_h whole
// blocks).  Two products per slab, both exact:
//   GEMM 1 (kind::i8):  U^T = diag(H_64, H_64) [Z rows r and r + 64 side by
//     side], A = the block-diagonal H_64 pair (signed, tensor memory), B = the
//     decoded bytes z + 128 (unsigned, shared memory, 64 rows of 128): the
//     accumulator lane c + 64 h holds row c of U^T for slab rows 64 h .. 64 h
//     + 63, i.e. U[r][c] = sum_b z[r][b] H_64[c][b] (plus 128 * 64 on c = 0,
//     removed exactly); |U| <= 64 * 30 = 1920, exact in fp16.
//   GEMM 2 (kind::f16):  T = diag(H_R, ..., H_R) [U^T rows], A = the 128/R
//     copies of H_R on the diagonal (tensor memory), B = U^T in fp16 (shared
//     memory, 64 rows of 128): lane d + R t holds row d of block t,
//     T[d][c] = sum_a H_R[d][a] U_t[a][c], |T| <= 122880 < 2^24, exact in fp32.
// So each lane of the second accumulator owns 64 consecutive weights: scaled,
// signed, rounded and stored as 128 contiguous bytes.  The result equals the
// sequential definition bit for bit (the only roundings are the two of w).
//
// Roles (one CTA per SM, persistent over slabs):
//   warp 0      producer: bulk copies of the slab's index words (ring of 4)
//   warp 1      tensor-memory allocation; one thread issues both GEMMs
//   warps 2-9   decoders: pair-table gathers -> z + 128 bytes (ring of 2)
//   warps 10-13 first readout: U^T -> fp16 operand of GEMM 2 (ring of 2)
//   warps 14-17 second readout: T -> scale, sign, bf16, global stores
#include <cuda_fp16.h>

#include "e8_common.cuh"
#include "e8_codebook.cuh"
#include "e8_internal.h"

namespace e8 {

namespace dtc {
constexpr int SLAB = 8192;                  // weights per slab
constexpr int GROUPS = SLAB / 8;
constexpr int TABLE_BYTES = 131088;
constexpr int CODE_STAGES = 4;
constexpr int CODE_BYTES = GROUPS * 4;      // idx1 (2 KB) + idx2 (up to 2 KB)
constexpr int B1_BYTES = 64 * 128;          // 64 rows x 128 bytes (u8)
constexpr int B2_BYTES = 64 * 256;          // 64 rows x 128 fp16, two 128-byte panels
constexpr int DEC_WARPS = 8;
constexpr int THREADS = 32 * 18;
// tensor memory columns
constexpr uint32_t A1_COL = 0;              // diag(H64, H64), s8: 32 columns
constexpr uint32_t A2_COL = 32;             // diag(H_R ...), f16: 64 columns
constexpr uint32_t D1_COL = 128;            // two buffers of 64
constexpr uint32_t D2_COL = 256;            // two buffers of 64
// shared memory (after the table, from the next 1 KB boundary)
constexpr int CODE_OFF = 0;
constexpr int B1_OFF = CODE_OFF + CODE_STAGES * CODE_BYTES;   // 16 KB
constexpr int B2_OFF = B1_OFF + 2 * B1_BYTES;                 // 32 KB
constexpr int BAR_OFF = B2_OFF + 2 * B2_BYTES;                // 64 KB
constexpr int SMEM_TOTAL = TABLE_BYTES + 1024 + BAR_OFF + 256;
}  // namespace dtc

__device__ __forceinline__ void dtc_mma_i8_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc,
                                              uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void dtc_mma_f16_ts(uint32_t d, uint32_t a, uint64_t b,
                                               uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// kind::i8: A signed, B unsigned, D int32, K-major; kind::f16: A, B fp16, D fp32.
__host__ __device__ constexpr uint32_t dtc_idesc_i8(uint32_t M, uint32_t N) {
  return (2u << 4) | (1u << 7) | (0u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}
__host__ __device__ constexpr uint32_t dtc_idesc_f16(uint32_t M, uint32_t N) {
  return (1u << 4) | (0u << 7) | (0u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
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

struct DecodeTcParams {
  const uint16_t* idx1;
  const void* idx2;
  int64_t slabs;          // N * K / 8192
  int K, nh, R;           // R = nh / 64
  uint64_t seed;
  float alpha;
  uint16_t* out;
  const uint32_t* table;  // pair table (global)
  uint32_t* status;
};

template <int BPW>
__global__ void __launch_bounds__(dtc::THREADS, 1) k_decode_tc(DecodeTcParams p) {
  using namespace dtc;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint8_t* table = smem_raw;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + TABLE_BYTES + 1023) & ~uintptr_t(1023));
  uint8_t* codes = smem + CODE_OFF;
  uint8_t* b1 = smem + B1_OFF;
  uint8_t* b2 = smem + B2_OFF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* code_full = bars;         // [4] index words landed
  uint64_t* code_empty = bars + 4;    // [4] decoders hold them in registers
  uint64_t* b1_full = bars + 8;       // [2] z + 128 bytes of the slab written
  uint64_t* b1_empty = bars + 10;     // [2] GEMM 1 done with them
  uint64_t* d1_full = bars + 12;      // [2] U^T in tensor memory
  uint64_t* d1_empty = bars + 14;     // [2] U^T read out
  uint64_t* b2_full = bars + 16;      // [2] fp16 U^T written
  uint64_t* b2_empty = bars + 18;     // [2] GEMM 2 done with it
  uint64_t* d2_full = bars + 20;      // [2] T in tensor memory
  uint64_t* d2_empty = bars + 22;     // [2] T read out
  uint64_t* table_full = bars + 24;
  uint64_t* drain = bars + 25;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 26);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  uint32_t* status = p.status;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nsl = (p.slabs - (int64_t)blockIdx.x + gridDim.x - 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < CODE_STAGES; ++s) {
      mbar_init(&code_full[s], 1);
      mbar_init(&code_empty[s], DEC_WARPS);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&b1_full[s], DEC_WARPS);
      mbar_init(&b1_empty[s], 1);
      mbar_init(&d1_full[s], 1);
      mbar_init(&d1_empty[s], 4);
      mbar_init(&b2_full[s], 4);
      mbar_init(&b2_empty[s], 1);
      mbar_init(&d2_full[s], 1);
      mbar_init(&d2_empty[s], 4);
    }
    mbar_init(table_full, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
    *abort_flag = 0u;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // the constant operands: diag(H64, H64) as s8 and diag(H_R, ...) as fp16,
  // one row per tensor-memory lane
  if (warp >= 10 && warp < 14) {
    const uint32_t q = warp & 3, m = q * 32 + lane;
    const uint32_t lane_bits = (q * 32) << 16;
    uint32_t v[32];
#pragma unroll
    for (int w = 0; w < 32; ++w) {
      uint32_t x = 0u;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint32_t k = 4 * w + b;
        const uint32_t e = (m >> 6) == (k >> 6) ? (had_neg(m & 63, k & 63) ? 0xFFu : 0x01u) : 0u;
        x |= e << (8 * b);
      }
      v[w] = x;
    }
    dtc_st32(tmem_base + lane_bits + A1_COL, v);
    const uint32_t R = (uint32_t)p.R;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
#pragma unroll
      for (int w = 0; w < 32; ++w) {
        uint32_t x = 0u;
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const uint32_t k = 64 * half + 2 * w + b;
          const uint32_t e =
              m / R == k / R ? (had_neg(m % R, k % R) ? 0xBC00u : 0x3C00u) : 0u;
          x |= e << (16 * b);
        }
        v[w] = x;
      }
      dtc_st32(tmem_base + lane_bits + A2_COL + 32 * half, v);
    }
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(table_full, TABLE_BYTES);
      for (int j = 0; j < 8; ++j) {
        const int c = (j + (int)blockIdx.x) & 7;
        bulk_load(smem_raw + c * 16384, reinterpret_cast<const uint8_t*>(p.table) + c * 16384,
                  16384, table_full);
      }
      bulk_load(smem_raw + 8 * 16384, reinterpret_cast<const uint8_t*>(p.table) + 8 * 16384, 16,
                table_full);
      const uint32_t i2b = BPW == 4 ? 2048u : (BPW == 3 ? 1024u : 0u);
      int s = 0;
      uint32_t ph = 0;
      int64_t issued = 0;
      for (int64_t i = 0; i < nsl; ++i) {
        if (i >= CODE_STAGES &&
            !mbar_wait_sleep(&code_empty[s], ph ^ 1u, abort_flag, status, kDevTimeoutEmpty))
          break;
        const int64_t slab = (int64_t)blockIdx.x + i * gridDim.x;
        uint8_t* dst = codes + s * CODE_BYTES;
        mbar_arrive_expect_tx(&code_full[s], 2048u + i2b);
        bulk_load(dst, p.idx1 + slab * GROUPS, 2048u, &code_full[s]);
        if (BPW > 2)
          bulk_load(dst + 2048, static_cast<const uint8_t*>(p.idx2) + slab * (int64_t)i2b, i2b,
                    &code_full[s]);
        ++issued;
        if (++s == CODE_STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (ld_shared_volatile(abort_flag)) {
        // let the copies in flight land before the CTA exits
        uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(table_full, 0))
          if (global_timer_ns() - t0 > 100000000ull) break;
        for (int64_t j = issued > CODE_STAGES ? issued - CODE_STAGES : 0; j < issued; ++j) {
          t0 = global_timer_ns();
          while (!mbar_try_wait(&code_full[j % CODE_STAGES], (uint32_t)(j / CODE_STAGES) & 1u))
            if (global_timer_ns() - t0 > 100000000ull) break;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc1 = dtc_idesc_i8(128, 64);
      const uint32_t idesc2 = dtc_idesc_f16(128, 64);
      const uint64_t bd1 = smem_desc(smem_u32(b1), 16, 1024, 2);
      const uint64_t bd2 = smem_desc(smem_u32(b2), 16, 1024, 2);
      bool ok = true;
      for (int64_t i = 0; i <= nsl && ok; ++i) {
        if (i < nsl) {
          // GEMM 1 of slab i
          const int s = (int)(i & 1);
          const uint32_t ph = (uint32_t)(i >> 1) & 1u;
          if (!mbar_wait_sleep(&b1_full[s], ph, abort_flag, status, kDevTimeoutFull) ||
              (i >= 2 &&
               !mbar_wait_sleep(&d1_empty[s], ph ^ 1u, abort_flag, status, kDevTimeoutMma))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + D1_COL + 64u * (uint32_t)s;
          const uint64_t bd = bd1 + (uint64_t)((uint32_t)(s * B1_BYTES) >> 4);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dtc_mma_i8_ts(d, tmem_base + A1_COL + 8u * j, bd + (uint64_t)(2 * j), idesc1,
                          j > 0 ? 1u : 0u);
          mma_commit(&b1_empty[s]);
          mma_commit(&d1_full[s]);
        }
        if (i >= 1) {
          // GEMM 2 of slab i - 1
          const int64_t k = i - 1;
          const int s = (int)(k & 1);
          const uint32_t ph = (uint32_t)(k >> 1) & 1u;
          if (!mbar_wait_sleep(&b2_full[s], ph, abort_flag, status, kDevTimeoutFull) ||
              (k >= 2 &&
               !mbar_wait_sleep(&d2_empty[s], ph ^ 1u, abort_flag, status, kDevTimeoutMma))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + D2_COL + 64u * (uint32_t)s;
          const uint64_t bd = bd2 + (uint64_t)((uint32_t)(s * B2_BYTES) >> 4);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            dtc_mma_f16_ts(d, tmem_base + A2_COL + 8u * j,
                           bd + (uint64_t)((j >> 2) * (8192 >> 4) + (j & 3) * 2), idesc2,
                           j > 0 ? 1u : 0u);
          mma_commit(&b2_empty[s]);
          mma_commit(&d2_full[s]);
        }
      }
      mma_commit(drain);
      uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0))
        if (global_timer_ns() - t0 > 200000000ull) break;
    }
  } else if (warp < 2 + DEC_WARPS) {
    // ------------------------------------------------------------ decoders
    const int t = threadIdx.x - 64;     // 0 .. 255: groups 4t .. 4t + 3 of the slab
    const uint32_t r = (uint32_t)t >> 1;               // slab row (64 weights)
    const uint32_t rb = r & 63u, hcol = (r >> 6) * 64u;
    bool ok = mbar_wait_sleep(table_full, 0, abort_flag, status, kDevTimeoutFull);
    int cs = 0;
    uint32_t cph = 0;
    for (int64_t i = 0; i < nsl && ok; ++i) {
      if (!mbar_wait_sleep(&code_full[cs], cph, abort_flag, status, kDevTimeoutFull)) break;
      const uint8_t* cw = codes + cs * CODE_BYTES;
      const uint2 w1 = *reinterpret_cast<const uint2*>(cw + 8 * t);
      uint2 w2 = make_uint2(0u, 0u);
      if (BPW == 4) {
        w2 = *reinterpret_cast<const uint2*>(cw + 2048 + 8 * t);
      } else if (BPW == 3) {
        const uint32_t c = *reinterpret_cast<const uint32_t*>(cw + 2048 + 4 * t);
        w2 = make_uint2(__byte_perm(c, 0u, 0x4140), __byte_perm(c, 0u, 0x4342));
      }
      // the index words are in registers; order these shared-memory reads
      // before the producer's next bulk-copy write into the stage
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&code_empty[cs]);
      const int s = (int)(i & 1);
      if (i >= 2) {
        if (!mbar_wait_sleep(&b1_empty[s], ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_flag, status,
                             kDevTimeoutMma))
          break;
        // the tensor cores' reads of the stage (async proxy) before these writes
        fence_proxy_async_smem();
      }
      uint8_t* bt = b1 + s * B1_BYTES;
      const uint32_t ww1[2] = {w1.x, w1.y}, ww2[2] = {w2.x, w2.y};
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const uint32_t ea0 = *reinterpret_cast<const uint32_t*>(table + ((((ww1[k] & 0xFFFFu) << 1) + 2u) & 0x3FFFCu));
        const uint32_t ea1 = *reinterpret_cast<const uint32_t*>(table + (((ww1[k] >> 15) + 2u) & 0x3FFFCu));
        const uint32_t eb0 = BPW > 2 ? *reinterpret_cast<const uint32_t*>(table + ((((ww2[k] & 0xFFFFu) << 1) + 2u) & 0x3FFFCu)) : 0u;
        const uint32_t eb1 = BPW > 2 ? *reinterpret_cast<const uint32_t*>(table + (((ww2[k] >> 15) + 2u) & 0x3FFFCu)) : 0u;
        uint32_t lo0, hi0, lo1, hi1;
        decode_group_q8<BPW>(ww1[k] & 0xFFFFu, ww2[k] & 0xFFFFu, ea0, eb0, lo0, hi0);
        decode_group_q8<BPW>(ww1[k] >> 16, ww2[k] >> 16, ea1, eb1, lo1, hi1);
        // groups 4t + 2k and 4t + 2k + 1: bytes 8 ((t & 1) * 4 + 2k) .. of row r
        const uint32_t col = hcol + 8u * (((uint32_t)t & 1u) * 4u + 2u * k);
        *reinterpret_cast<uint2*>(bt + sw128(rb, col)) = make_uint2(lo0, hi0);
        *reinterpret_cast<uint2*>(bt + sw128(rb, col + 8u)) = make_uint2(lo1, hi1);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b1_full[s]);
      if (++cs == CODE_STAGES) {
        cs = 0;
        cph ^= 1u;
      }
    }
  } else if (warp < 14) {
    // ------------------------------------------------------------ readout 1
    const uint32_t q = warp & 3, m = q * 32 + lane;
    const uint32_t c = m & 63u, h = m >> 6;
    const uint32_t lane_bits = (q * 32) << 16;
    const int bias = c == 0 ? 128 * 64 : 0;
    for (int64_t i = 0; i < nsl; ++i) {
      const int s = (int)(i & 1);
      const uint32_t ph = (uint32_t)(i >> 1) & 1u;
      if (!mbar_wait_sleep(&d1_full[s], ph, abort_flag, status, kDevTimeoutMma)) break;
      if (i >= 2) {
        if (!mbar_wait_sleep(&b2_empty[s], ph ^ 1u, abort_flag, status, kDevTimeoutMma)) break;
        fence_proxy_async_smem();
      }
      tc_fence_after();
      uint32_t u[32], u2[32];
      dtc_ld32(tmem_base + lane_bits + D1_COL + 64u * (uint32_t)s, u);
      dtc_ld32(tmem_base + lane_bits + D1_COL + 64u * (uint32_t)s + 32u, u2);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&d1_empty[s]);
      // row c of panel h of the fp16 operand: 64 values, 128 bytes
      uint8_t* row = b2 + s * B2_BYTES + h * 8192u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int x = 8 * j + 2 * e;
          const int a = (int)(x < 32 ? u[x] : u2[x - 32]) - bias;
          const int b = (int)(x + 1 < 32 ? u[x + 1] : u2[x - 31]) - bias;
          __half2 hv = __floats2half2_rn((float)a, (float)b);
          pk[e] = *reinterpret_cast<uint32_t*>(&hv);
        }
        *reinterpret_cast<uint4*>(row + sw128(c, 16u * j)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b2_full[s]);
    }
  } else {
    // ------------------------------------------------------------ readout 2
    const uint32_t q = warp & 3, m = q * 32 + lane;
    const uint32_t lane_bits = (q * 32) << 16;
    const int R = p.R;
    const int tb = (int)m / R, d = (int)m % R;
    for (int64_t i = 0; i < nsl; ++i) {
      const int s = (int)(i & 1);
      const uint32_t ph = (uint32_t)(i >> 1) & 1u;
      if (!mbar_wait_sleep(&d2_full[s], ph, abort_flag, status, kDevTimeoutMma)) break;
      tc_fence_after();
      uint32_t y[32], y2[32];
      dtc_ld32(tmem_base + lane_bits + D2_COL + 64u * (uint32_t)s, y);
      dtc_ld32(tmem_base + lane_bits + D2_COL + 64u * (uint32_t)s + 32u, y2);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&d2_empty[s]);
      const int64_t slab = (int64_t)blockIdx.x + i * gridDim.x;
      const int64_t e0 = slab * SLAB + (int64_t)tb * p.nh + 64 * d;
      const int64_t col = e0 % p.K;
      const uint64_t word = splitmix64_output(p.seed, (uint64_t)(col >> 6));
      uint4* dst = reinterpret_cast<uint4*>(p.out + e0);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int x = 8 * j + 2 * e;
          float a = __fmul_rn(__uint_as_float(x < 32 ? y[x] : y2[x - 32]), p.alpha);
          float b = __fmul_rn(__uint_as_float(x + 1 < 32 ? y[x + 1] : y2[x - 31]), p.alpha);
          a = __uint_as_float(__float_as_uint(a) ^ ((uint32_t)(word >> x) & 1u) << 31);
          b = __uint_as_float(__float_as_uint(b) ^ ((uint32_t)(word >> (x + 1)) & 1u) << 31);
          pk[e] = pack_bf16x2(a, b);
        }
        dst[j] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int BPW>
static cudaError_t launch_decode_tc_t(const DecodeTcParams& p, int grid, cudaStream_t st) {
  cudaError_t e = ensure_smem_limit(k_decode_tc<BPW>, kMaxDynSmem);
  if (e != cudaSuccess) return e;
  k_decode_tc<BPW><<<grid, dtc::THREADS, dtc::SMEM_TOTAL, st>>>(p);
  return cudaGetLastError();
}

// Shapes served: n_h in {1024, 2048, 4096} and N K a multiple of 8192.
bool decode_tc_eligible(int64_t N, int64_t K) {
  const int64_t nh = hadamard_block(K);
  return N > 0 && (nh == 1024 || nh == 2048 || nh == 4096) && ((N * K) % dtc::SLAB) == 0 &&
         K <= (int64_t)1 << 30;
}

cudaError_t launch_decode_tc(const DeviceCodebook& cb, const uint16_t* idx1, const void* idx2,
                             int64_t N, int64_t K, int bpw, uint64_t seed, float alpha,
                             uint16_t* Wdec, int sm_count, cudaStream_t st) {
  if (!decode_tc_eligible(N, K)) return cudaErrorInvalidValue;
  DecodeTcParams p;
  p.idx1 = idx1;
  p.idx2 = idx2;
  p.slabs = N * K / dtc::SLAB;
  p.K = (int)K;
  p.nh = (int)hadamard_block(K);
  p.R = p.nh / 64;
  p.seed = seed;
  p.alpha = alpha;
  p.out = Wdec;
  p.table = cb.table;
  p.status = cb.status;
  const int grid = (int)(p.slabs < sm_count ? p.slabs : sm_count);
  if (bpw == 2) return launch_decode_tc_t<2>(p, grid, st);
  if (bpw == 3) return launch_decode_tc_t<3>(p, grid, st);
  return launch_decode_tc_t<4>(p, grid, st);
}

}  // namespace e8
