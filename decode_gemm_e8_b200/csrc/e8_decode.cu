// Decoder: codebook indices -> bf16 weights (inverse of the encoder's
// randomized Hadamard transform, "glq 0.1.1", "How it works", items 1-2).
//
//   z   = m (c1 + beta c2)  integer 8-vector per group (m = 2, 4, 8 for 2, 3, 4 bpw)
//   t   = FWHT_nh(z)        exact: |t| <= nh * 30 < 2^24 fits fp32 integers
//   w_k = bf16_rne(d_k * fl32(t_k * alpha)),  alpha = fl32(s / (m sqrt(nh)))
//
// Because the transform on integers is exact, its evaluation order is free;
// the two roundings (fp32 product, then bf16) are the only ones, so the
// result is bit-identical to any exact evaluation.
#include "e8_common.cuh"
#include "e8_codebook.cuh"
#include "e8_internal.h"

namespace e8 {

__device__ __forceinline__ void unpack_entry(uint32_t e, bool neg, int (&v)[8]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    int a = (int)((e >> (8 * j)) & 0xFu) - 8;
    int b = (int)((e >> (8 * j + 4)) & 0xFu) - 8;
    v[j] = neg ? -a : a;
    v[j + 4] = neg ? -b : b;
  }
}

// Codebook vector (doubled coordinates) of index i.
__device__ __forceinline__ void lookup(const uint32_t* table, uint32_t i, int (&v)[8]) {
  uint32_t e = __ldg(table + ((i + 1u) >> 1));
  unpack_entry(e, i != 0u && (i & 1u) == 0u, v);
}

struct DecodeParams {
  const uint16_t* idx1;
  const void* idx2;
  int64_t N, K;
  int nh, elems_per_cta, bpw;
  uint64_t seed;
  float alpha;
  uint16_t* out;
};

__global__ void __launch_bounds__(256) k_decode(DecodeParams p, DeviceCodebook cb) {
  extern __shared__ __align__(16) float s_t[];
  const int64_t total = p.N * p.K;
  const int64_t base = (int64_t)blockIdx.x * p.elems_per_cta;
  const int E = (int)(int64_t)min((long long)p.elems_per_cta, (long long)(total - base));
  const int ngroups = E >> 3;
  const int64_t g0 = base >> 3;
  for (int g = threadIdx.x; g < ngroups; g += blockDim.x) {
    int v1[8], z[8];
    lookup(cb.table, p.idx1[g0 + g], v1);
    if (p.bpw == 2) {
#pragma unroll
      for (int i = 0; i < 8; ++i) z[i] = v1[i];
    } else {
      uint32_t i2 = p.bpw == 3 ? (uint32_t)reinterpret_cast<const uint8_t*>(p.idx2)[g0 + g]
                               : (uint32_t)reinterpret_cast<const uint16_t*>(p.idx2)[g0 + g];
      int v2[8];
      lookup(cb.table, i2, v2);
      const int mul = p.bpw == 3 ? 2 : 4;
#pragma unroll
      for (int i = 0; i < 8; ++i) z[i] = mul * v1[i] + v2[i];
    }
    float y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = (float)z[i];
    // stages h = 1, 2, 4 inside the group
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if ((i & h) == 0) {
          float a = y[i], c = y[i + h];
          y[i] = a + c;
          y[i + h] = a - c;
        }
      }
    }
    float4* dst = reinterpret_cast<float4*>(s_t + 8 * g);
    dst[0] = make_float4(y[0], y[1], y[2], y[3]);
    dst[1] = make_float4(y[4], y[5], y[6], y[7]);
  }
  // remaining stages across groups (exact on integers, any order)
  const int half = E >> 1;
  for (int h = 8; h < p.nh; h <<= 1) {
    __syncthreads();
    for (int b = threadIdx.x; b < half; b += blockDim.x) {
      int i = (b / h) * (2 * h) + (b % h);
      float a = s_t[i], c = s_t[i + h];
      s_t[i] = a + c;
      s_t[i + h] = a - c;
    }
  }
  __syncthreads();
  for (int g = threadIdx.x; g < ngroups; g += blockDim.x) {
    int64_t e0 = base + 8 * (int64_t)g;
    int64_t k0 = e0 % p.K;
    uint64_t word = splitmix64_output(p.seed, (uint64_t)(k0 >> 6));
    uint32_t bits = (uint32_t)(word >> (k0 & 63));
    const float4* src = reinterpret_cast<const float4*>(s_t + 8 * g);
    float4 lo = src[0], hi = src[1];
    float t[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      float a = __fmul_rn(t[i], p.alpha);
      float b = __fmul_rn(t[i + 1], p.alpha);
      a = __uint_as_float(__float_as_uint(a) ^ (((bits >> i) & 1u) << 31));
      b = __uint_as_float(__float_as_uint(b) ^ (((bits >> (i + 1)) & 1u) << 31));
      w[i >> 1] = pack_bf16x2(a, b);
    }
    *reinterpret_cast<uint4*>(p.out + e0) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// ---------------------------------------------------------------------------
// Fast decoder for Hadamard blocks of 256..4096 (K a multiple of 128).
//
// One warp turns a tile of 4096 consecutive weights (row-major [N][K]) into
// bf16.  The 8-point transform inside a group is taken from the transformed
// pair table (H8 v / 4), so only the stages across groups are computed, on
// exact small integers in fp32, and the factor 4 is folded into alpha:
//   w = bf16(d * fl32(t'' * 4 alpha)),  t'' = FWHT over groups of H8 z / 4.
// Layout 1: lane l holds tile elements 128 l .. 128 l + 127 (16 groups), so
// the stages on element bits 3..6 run in registers.  The tile is then
// transposed through shared memory, half at a time (element bit 1), to layout
// 2, where lane u holds elements 128 L + 4 u + {bit 1, bit 0} for L = 0..31:
// the stages on bits 7..11 run in registers and the stores of each L cover
// 256 contiguous bytes.  Signs come from a table of bf16-pair XOR masks per
// column pair, extended periodically to K + 4096 columns so that a tile never
// wraps it.
// ---------------------------------------------------------------------------
namespace dq {
constexpr int TILE = 4096;
constexpr int TABLE_BYTES = 131088;
constexpr int XBUF_OFF = 131328;     // table rounded up to 256 bytes
constexpr int XBUF_BYTES = 8192;     // per warp: half a tile, fp32
constexpr int MAX_WARPS = 8;
}  // namespace dq

struct DecodeFastParams {
  const uint16_t* idx1;
  const void* idx2;
  int64_t total;     // N * K
  int K, log_nh, warps, mask_off, bar_off;
  uint64_t seed;
  float alpha4;      // 4 alpha (exact)
  uint16_t* out;
  uint32_t* status;
  const uint32_t* h8table;
};

__device__ __forceinline__ void sts128f(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}
__device__ __forceinline__ float2 lds64f(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr) : "memory");
  return v;
}

// 2^23 + (byte c of w), an exact float.
__device__ __forceinline__ float magic_byte(uint32_t w, uint32_t c) {
  return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7440u | c));
}

template <int BPW>
__device__ __forceinline__ void load_tile_codes(const DecodeFastParams& p, int64_t tile, int lane,
                                                uint4& c1a, uint4& c1b, uint4& c2a, uint4& c2b) {
  c1a = c1b = c2a = c2b = make_uint4(0u, 0u, 0u, 0u);
  const int64_t e = tile * dq::TILE + 128 * (int64_t)lane;
  if (e >= p.total) return;
  const int64_t g = e >> 3;
  const uint4* s1 = reinterpret_cast<const uint4*>(p.idx1 + g);
  c1a = __ldg(s1);
  c1b = __ldg(s1 + 1);
  if (BPW == 4) {
    const uint4* s2 = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.idx2) + g);
    c2a = __ldg(s2);
    c2b = __ldg(s2 + 1);
  } else if (BPW == 3) {
    c2a = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.idx2) + g));
  }
}

template <int BPW>
__global__ void __launch_bounds__(dq::MAX_WARPS * 32, 1) k_decode_fast(DecodeFastParams p) {
  using namespace dq;
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(smem + p.mask_off);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + p.bar_off);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(bar + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = p.K;
  if (threadIdx.x == 0) {
    *abort_flag = 0u;
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, TABLE_BYTES);
    bulk_load(smem, p.h8table, TABLE_BYTES, bar);
  }
  // XOR masks of the column pairs (2q, 2q + 1): bit 15 / bit 31 when the sign
  // of the even / odd column is negative (word j of the sign stream holds
  // columns 64 j .. 64 j + 63, bit set = negative)
  for (int w = threadIdx.x; w < K / 64; w += blockDim.x) {
    const uint64_t bits = splitmix64_output(p.seed, (uint64_t)w);
#pragma unroll 4
    for (int j = 0; j < 32; ++j)
      s_mask[32 * w + j] = ((uint32_t)(bits >> (2 * j)) & 1u) << 15 |
                           ((uint32_t)(bits >> (2 * j + 1)) & 1u) << 31;
  }
  __syncthreads();
  const int half_k = K / 2, nmask = (K + TILE) / 2;
  for (int q = half_k + threadIdx.x; q < nmask; q += blockDim.x) s_mask[q] = s_mask[q % half_k];
  __syncthreads();
  const bool have_table = mbar_wait_sleep(bar, 0, abort_flag, p.status, kDevTimeoutFull);
  if (!have_table) return;

  const uint32_t tbl = smem_u32(smem);
  const uint32_t xb = smem_u32(smem + XBUF_OFF + warp * XBUF_BYTES);
  const uint32_t mk = smem_u32(s_mask);
  const int64_t ntiles = (p.total + TILE - 1) / TILE;
  const int64_t stride = (int64_t)gridDim.x * p.warps;
  const int l2stages = p.log_nh - 7;   // stages on element bits 7 .. log_nh - 1
  const float two_m = 16777472.0f;     // 2 (2^23 + 128), exact
  int64_t tile = (int64_t)blockIdx.x * p.warps + warp;
  uint4 n1a, n1b, n2a, n2b;
  if (tile < ntiles) load_tile_codes<BPW>(p, tile, lane, n1a, n1b, n2a, n2b);
  for (; tile < ntiles; tile += stride) {
    const uint32_t w1[8] = {n1a.x, n1a.y, n1a.z, n1a.w, n1b.x, n1b.y, n1b.z, n1b.w};
    const uint32_t w2[8] = {n2a.x, n2a.y, n2a.z, n2a.w, n2b.x, n2b.y, n2b.z, n2b.w};
    if (tile + stride < ntiles) load_tile_codes<BPW>(p, tile + stride, lane, n1a, n1b, n2a, n2b);
    const int64_t e0 = tile * TILE;

    // ---- layout 1: decode 16 groups, stages on element bits 3..6
    float x[16][8];
#pragma unroll
    for (int gp = 0; gp < 8; ++gp) {
      uint32_t lo[2], hi[2];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int g = 2 * gp + t;
        const uint32_t i1 = (w1[g >> 1] >> (16 * (g & 1))) & 0xFFFFu;
        uint32_t i2 = 0u;
        if (BPW == 4) i2 = (w2[g >> 1] >> (16 * (g & 1))) & 0xFFFFu;
        if (BPW == 3) i2 = (w2[g >> 2] >> (8 * (g & 3))) & 0xFFu;
        const uint32_t ea = lds32(tbl + (((i1 + 1u) >> 1) << 2));
        const uint32_t eb = BPW > 2 ? lds32(tbl + (((i2 + 1u) >> 1) << 2)) : 0u;
        decode_group_q8<BPW>(i1, i2, ea, eb, lo[t], hi[t]);
      }
      // first stage (groups 2gp, 2gp + 1) with the byte bias removed exactly:
      // a + b = ((2^23 + 128 + a) - 2 (2^23 + 128)) + (2^23 + 128 + b)
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t wa = c < 4 ? lo[0] : hi[0], wb = c < 4 ? lo[1] : hi[1];
        const float A = magic_byte(wa, (uint32_t)(c & 3));
        const float B = magic_byte(wb, (uint32_t)(c & 3));
        x[2 * gp][c] = __fadd_rn(__fadd_rn(A, -two_m), B);
        x[2 * gp + 1][c] = __fsub_rn(A, B);
      }
    }
#pragma unroll
    for (int s = 1; s < 4; ++s) {
#pragma unroll
      for (int g = 0; g < 16; ++g) {
        if (g & (1 << s)) continue;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float a = x[g][c], b = x[g | (1 << s)][c];
          x[g][c] = __fadd_rn(a, b);
          x[g | (1 << s)][c] = __fsub_rn(a, b);
        }
      }
    }

    // ---- layout 2, half by half (element bit 1 = h)
    const int valid_l = (int)min((int64_t)32, (p.total - e0) >> 7);
    const int col0 = (int)(e0 % K);
    const uint32_t mrow = mk + 4u * (uint32_t)(col0 / 2 + 2 * lane);
    uint16_t* orow = p.out + e0 + 4 * lane;
    uint32_t pk0[32];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      __syncwarp();
#pragma unroll
      for (int g = 0; g < 16; ++g)
        sts128f(xb + (uint32_t)(lane * 256 + ((g ^ (lane & 7)) << 4)), x[g][2 * h],
                x[g][2 * h + 1], x[g][4 + 2 * h], x[g][5 + 2 * h]);
      __syncwarp();
      float y[32][2];
#pragma unroll
      for (int L = 0; L < 32; ++L) {
        const float2 v =
            lds64f(xb + (uint32_t)(L * 256 + (((lane >> 1) ^ (L & 7)) << 4) + (lane & 1) * 8));
        y[L][0] = v.x;
        y[L][1] = v.y;
      }
#pragma unroll
      for (int s = 0; s < 5; ++s) {
        if (s < l2stages) {
#pragma unroll
          for (int L = 0; L < 32; ++L) {
            if (L & (1 << s)) continue;
#pragma unroll
            for (int b = 0; b < 2; ++b) {
              const float a = y[L][b], c = y[L | (1 << s)][b];
              y[L][b] = __fadd_rn(a, c);
              y[L | (1 << s)][b] = __fsub_rn(a, c);
            }
          }
        }
      }
#pragma unroll
      for (int L = 0; L < 32; ++L) {
        const uint32_t m = lds32(mrow + (uint32_t)(256 * L + 4 * h));
        const uint32_t pk =
            pack_bf16x2(__fmul_rn(y[L][0], p.alpha4), __fmul_rn(y[L][1], p.alpha4)) ^ m;
        if (h == 0) {
          pk0[L] = pk;
        } else if (L < valid_l) {
          asm volatile("st.global.v2.u32 [%0], {%1, %2};" ::"l"(orow + 128 * L), "r"(pk0[L]),
                       "r"(pk)
                       : "memory");
        }
      }
    }
  }
}

template <int BPW>
static cudaError_t launch_decode_fast_t(const DecodeFastParams& p, int grid, size_t smem,
                                        cudaStream_t st) {
  cudaError_t e = ensure_smem_limit(k_decode_fast<BPW>, kMaxDynSmem);
  if (e != cudaSuccess) return e;
  k_decode_fast<BPW><<<grid, p.warps * 32, smem, st>>>(p);
  return cudaGetLastError();
}

// Shared-memory plan of the fast decoder: warps that fit next to the table and
// the mask table (0 if fewer than 2 fit).
static int decode_fast_plan(int64_t K, int* mask_off, int* bar_off, size_t* smem) {
  using namespace dq;
  const int mask_bytes = (int)(((K + TILE) / 2) * 4);
  int warps = MAX_WARPS;
  while (warps >= 2) {
    const int moff = XBUF_OFF + warps * XBUF_BYTES;
    const int boff = (moff + mask_bytes + 15) & ~15;
    if (boff + 16 <= kMaxDynSmem) {
      *mask_off = moff;
      *bar_off = boff;
      *smem = (size_t)(boff + 16);
      return warps;
    }
    --warps;
  }
  return 0;
}

cudaError_t launch_decode(const DeviceCodebook& cb, const uint16_t* idx1, const void* idx2,
                          int64_t N, int64_t K, int bpw, uint64_t seed, float alpha,
                          uint16_t* Wdec, int sm_count, cudaStream_t st, int64_t nh_arg) {
  {
    const cudaError_t e =
        launch_decode_tc(cb, idx1, idx2, N, K, bpw, seed, alpha, Wdec, sm_count, st, nh_arg);
    if (e != cudaErrorNotSupported) return e;
  }
  const int64_t nh = resolve_nh(K, nh_arg);
  if ((K % 128) == 0 && nh >= 256 && nh <= 4096 && K <= 32768 && N > 0) {
    DecodeFastParams f;
    size_t smem = 0;
    const int warps = decode_fast_plan(K, &f.mask_off, &f.bar_off, &smem);
    if (warps >= 2) {
      f.idx1 = idx1;
      f.idx2 = idx2;
      f.total = N * K;
      f.K = (int)K;
      f.log_nh = 0;
      while ((int64_t(1) << f.log_nh) < nh) ++f.log_nh;
      f.warps = warps;
      f.seed = seed;
      f.alpha4 = 4.0f * alpha;
      f.out = Wdec;
      f.status = cb.status;
      f.h8table = cb.h8table;
      const int64_t tiles = (f.total + dq::TILE - 1) / dq::TILE;
      const int64_t ctas = (tiles + warps - 1) / warps;
      const int grid = (int)(ctas < sm_count ? ctas : sm_count);
      if (bpw == 2) return launch_decode_fast_t<2>(f, grid, smem, st);
      if (bpw == 3) return launch_decode_fast_t<3>(f, grid, smem, st);
      return launch_decode_fast_t<4>(f, grid, smem, st);
    }
  }
  DecodeParams p;
  p.idx1 = idx1;
  p.idx2 = idx2;
  p.N = N;
  p.K = K;
  p.nh = (int)nh;
  p.elems_per_cta = p.nh < 2048 ? 2048 : p.nh;
  p.bpw = bpw;
  p.seed = seed;
  p.alpha = alpha;
  p.out = Wdec;
  const int64_t total = N * K;
  const int64_t ctas = (total + p.elems_per_cta - 1) / p.elems_per_cta;
  const size_t smem = (size_t)p.elems_per_cta * sizeof(float);
  cudaError_t e = ensure_smem_limit(k_decode, kMaxDynSmem);
  if (e != cudaSuccess) return e;
  k_decode<<<(unsigned)ctas, 256, smem, st>>>(p, cb);
  return cudaGetLastError();
}

}  // namespace e8
