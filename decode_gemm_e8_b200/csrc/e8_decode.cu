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

cudaError_t launch_decode(const DeviceCodebook& cb, const uint16_t* idx1, const void* idx2,
                          int64_t N, int64_t K, int bpw, uint64_t seed, float alpha,
                          uint16_t* Wdec, cudaStream_t st) {
  DecodeParams p;
  p.idx1 = idx1;
  p.idx2 = idx2;
  p.N = N;
  p.K = K;
  p.nh = (int)hadamard_block(K);
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
