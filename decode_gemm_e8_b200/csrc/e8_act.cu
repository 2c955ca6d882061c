// Activation-side transform for the small-batch GEMM.
//
// With w_n = alpha D H z_n per Hadamard block (H symmetric, "glq 0.1.1",
// "How it works", item 2), every output is
//     y[m][n] = sum_k x_mk w_nk = alpha * sum_k (H D x_m)_k z_nk,
// so the GEMM can run on the integer codebook vectors z (exact in bf16) once
// the activations are transformed.  The transformed row xt = FWHT(D x) is
// split into two bf16 parts, hi = bf16(xt) and lo = bf16(xt - hi), stored as
// rows 2m and 2m + 1, so that the bf16 tensor-core product keeps about 16
// significant bits of xt and the two parts of a token sit in adjacent
// accumulator columns.
#include "e8_common.cuh"
#include "e8_internal.h"

namespace e8 {

__global__ void __launch_bounds__(256) k_act_rht(const uint16_t* __restrict__ X, int64_t M,
                                                 int64_t K, int nh, int elems_per_cta,
                                                 uint64_t seed, uint16_t* __restrict__ Xt,
                                                 int64_t data_ctas, int64_t pad_elems) {
  extern __shared__ __align__(16) float s_x[];
  if ((int64_t)blockIdx.x >= data_ctas) {
    // trailing CTAs zero the padding rows 2M..rows-1 (16-byte stores)
    uint4* pad = reinterpret_cast<uint4*>(Xt + 2 * M * K);
    const int64_t n16 = pad_elems / 8;
    const int64_t nct = (int64_t)gridDim.x - data_ctas;
    for (int64_t i = ((int64_t)blockIdx.x - data_ctas) * blockDim.x + threadIdx.x; i < n16;
         i += nct * blockDim.x)
      pad[i] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const int64_t total = M * K;
  const int64_t base = (int64_t)blockIdx.x * elems_per_cta;
  const int E = (int)(int64_t)min((long long)elems_per_cta, (long long)(total - base));
  const int ngroups = E >> 3;
  for (int g = threadIdx.x; g < ngroups; g += blockDim.x) {
    int64_t e0 = base + 8 * (int64_t)g;
    int64_t k0 = e0 % K;
    uint4 raw = __ldg(reinterpret_cast<const uint4*>(X + e0));
    uint32_t r[4] = {raw.x, raw.y, raw.z, raw.w};
    float y[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      y[2 * i] = bf16_lo_to_f32(r[i]);
      y[2 * i + 1] = bf16_hi_to_f32(r[i]);
    }
    uint64_t word = splitmix64_output(seed, (uint64_t)(k0 >> 6));
    uint32_t bits = (uint32_t)(word >> (k0 & 63));
#pragma unroll
    for (int i = 0; i < 8; ++i)
      y[i] = __uint_as_float(__float_as_uint(y[i]) ^ (((bits >> i) & 1u) << 31));
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
    float4* dst = reinterpret_cast<float4*>(s_x + 8 * g);
    dst[0] = make_float4(y[0], y[1], y[2], y[3]);
    dst[1] = make_float4(y[4], y[5], y[6], y[7]);
  }
  const int half = E >> 1;
  for (int h = 8; h < nh; h <<= 1) {
    __syncthreads();
    for (int b = threadIdx.x; b < half; b += blockDim.x) {
      int i = (b / h) * (2 * h) + (b % h);
      float a = s_x[i], c = s_x[i + h];
      s_x[i] = a + c;
      s_x[i + h] = a - c;
    }
  }
  __syncthreads();
  for (int g = threadIdx.x; g < ngroups; g += blockDim.x) {
    int64_t e0 = base + 8 * (int64_t)g;
    int64_t m = e0 / K, k0 = e0 % K;
    const float4* src = reinterpret_cast<const float4*>(s_x + 8 * g);
    float4 lo4 = src[0], hi4 = src[1];
    float y[8] = {lo4.x, lo4.y, lo4.z, lo4.w, hi4.x, hi4.y, hi4.z, hi4.w};
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      hw[i] = pack_bf16x2(y[2 * i], y[2 * i + 1]);
      float r0 = y[2 * i] - bf16_lo_to_f32(hw[i]);
      float r1 = y[2 * i + 1] - bf16_hi_to_f32(hw[i]);
      lw[i] = pack_bf16x2(r0, r1);
    }
    *reinterpret_cast<uint4*>(Xt + (2 * m) * K + k0) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(Xt + (2 * m + 1) * K + k0) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
}

// Fast path for Hadamard blocks of 256..4096 (others use k_act_rht): one CTA of nh/8 threads per
// (row, block).  Stages h = 1, 2, 4 inside a thread's group of 8, stages
// 8..128 by warp shuffles, stages 256..nh/2 after one transpose through shared
// memory, where 256 threads hold nh/256 elements 256 apart.  Launched with
// programmatic serialization: it waits for the previous kernel before reading
// X (and before overwriting Xt, which that kernel may still read), then lets
// the GEMM that follows start its prologue.
__global__ void __launch_bounds__(512) k_act_rht_fast(const uint16_t* __restrict__ X, int64_t M,
                                                      int64_t K, int nh, uint64_t seed,
                                                      uint16_t* __restrict__ Xt,
                                                      int64_t data_ctas, int64_t pad_elems) {
  __shared__ __align__(16) float s_x[4096];
  grid_dep_wait();
  grid_dep_launch();
  if ((int64_t)blockIdx.x >= data_ctas) {
    uint4* pad = reinterpret_cast<uint4*>(Xt + 2 * M * K);
    const int64_t n16 = pad_elems / 8;
    const int64_t nct = (int64_t)gridDim.x - data_ctas;
    for (int64_t i = ((int64_t)blockIdx.x - data_ctas) * blockDim.x + threadIdx.x; i < n16;
         i += nct * blockDim.x)
      pad[i] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const int t = threadIdx.x, lane = t & 31;
  const int64_t base = (int64_t)blockIdx.x * nh;   // first element of this block
  const int64_t m = base / K, kb = base % K;
  // blocks of 512..1024 run 256 threads for the second phase; only nh/8 of
  // them (whole warps) own a group in the first phase
  const bool owner = t < (nh >> 3);
  const int64_t e0 = base + 8 * t;
  const int64_t k0 = kb + 8 * t;
  uint4 raw = owner ? __ldg(reinterpret_cast<const uint4*>(X + e0)) : make_uint4(0u, 0u, 0u, 0u);
  const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
  float y[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    y[2 * i] = bf16_lo_to_f32(rw[i]);
    y[2 * i + 1] = bf16_hi_to_f32(rw[i]);
  }
  const uint64_t word = splitmix64_output(seed, (uint64_t)(k0 >> 6));
  const uint32_t bits = (uint32_t)(word >> (k0 & 63));
#pragma unroll
  for (int i = 0; i < 8; ++i)
    y[i] = __uint_as_float(__float_as_uint(y[i]) ^ (((bits >> i) & 1u) << 31));
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
#pragma unroll
  for (int h = 8; h < 256; h <<= 1) {
    const int lm = h >> 3;
    const bool upper = (lane & lm) != 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, y[i], lm);
      y[i] = upper ? o - y[i] : y[i] + o;
    }
  }
  if (nh <= 256) {
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      hw[i] = pack_bf16x2(y[2 * i], y[2 * i + 1]);
      lw[i] = pack_bf16x2(y[2 * i] - bf16_lo_to_f32(hw[i]), y[2 * i + 1] - bf16_hi_to_f32(hw[i]));
    }
    *reinterpret_cast<uint4*>(Xt + (2 * m) * K + k0) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(Xt + (2 * m + 1) * K + k0) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    return;
  }
  if (owner) {
    float4* dst = reinterpret_cast<float4*>(s_x + 8 * t);
    dst[0] = make_float4(y[0], y[1], y[2], y[3]);
    dst[1] = make_float4(y[4], y[5], y[6], y[7]);
  }
  __syncthreads();
  if (t >= 256) return;
  const int per = nh >> 8;   // elements per thread, 256 apart
  float z[16];
#pragma unroll
  for (int j = 0; j < 16; ++j)
    if (j < per) z[j] = s_x[t + 256 * j];
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
    if (h >= per) break;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (j < per && (j & h) == 0) {
        float a = z[j], c = z[j + h];
        z[j] = a + c;
        z[j + h] = a - c;
      }
    }
  }
  uint16_t* hi_row = Xt + (2 * m) * K + kb;
  uint16_t* lo_row = Xt + (2 * m + 1) * K + kb;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    if (j < per) {
      const uint32_t hb = f32_to_bf16_rne(z[j]);
      const float rest = z[j] - __uint_as_float(hb << 16);
      hi_row[t + 256 * j] = (uint16_t)hb;
      lo_row[t + 256 * j] = (uint16_t)f32_to_bf16_rne(rest);
    }
  }
}

cudaError_t launch_act_rht(const uint16_t* X, int64_t M, int64_t K, uint64_t seed, uint16_t* Xt,
                           int64_t rows, cudaStream_t st, int pdl, int64_t nh_arg) {
  {
    const int nh = (int)resolve_nh(K, nh_arg);
    if (nh >= 256 && nh <= 4096) {
      const int64_t data = M * K / nh;
      const int64_t pad_elems = (rows - 2 * M) * K;
      const int64_t pad_ctas = pad_elems > 0 ? (pad_elems / 8 + 4095) / 4096 : 0;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)(data + pad_ctas));
      cfg.blockDim = dim3((unsigned)(nh <= 256 ? 32 : (nh / 8 < 256 ? 256 : nh / 8)));
      cfg.dynamicSmemBytes = 0;
      cfg.stream = st;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      cudaError_t e = cudaLaunchKernelEx(&cfg, k_act_rht_fast, X, M, K, nh, seed, Xt, data,
                                         pad_elems);
      if (e != cudaSuccess) return e;
      return cudaGetLastError();
    }
  }
  const int nh = (int)resolve_nh(K, nh_arg);
  const int epc = nh < 2048 ? 2048 : nh;
  const int64_t total = M * K;
  const int64_t ctas = (total + epc - 1) / epc;
  const size_t smem = (size_t)epc * sizeof(float);
  cudaError_t e = ensure_smem_limit(k_act_rht, kMaxDynSmem);
  if (e != cudaSuccess) return e;
  const int64_t pad_elems = (rows - 2 * M) * K;  // multiple of 8 since K is
  const int64_t pad_ctas = pad_elems > 0 ? (pad_elems / 8 + 2047) / 2048 : 0;
  k_act_rht<<<(unsigned)(ctas + pad_ctas), 256, smem, st>>>(X, M, K, nh, epc, seed, Xt, ctas,
                                                            pad_elems);
  return cudaGetLastError();
}

}  // namespace e8

namespace e8 {


// Activation transform for the int8 tensor-core path.  A token row is cut
// into chunks of up to 4096 positions, one CTA of 512 threads per chunk and
// one thread-block cluster per row (at most 8 CTAs: K <= 32768).  A Hadamard
// block (n_h a power of two, 256 <= n_h <= 4096, dividing K) never straddles
// a chunk.  Inside a chunk, position p = 256 w + 8 l + e (warp w, lane l,
// register e): the stages of the three low bits run in registers, the next
// five by warp shuffles, and the stages across warps (n_h > 256) after one
// exchange through shared memory, where thread t takes the 8 positions
// g + 256 (8 (t & 1) + j), g = t >> 1, three stages in registers and the last
// by a shuffle with its neighbour.
// The row's largest magnitude (the chunks' maxima, exchanged through
// distributed shared memory) fixes the token's step s_m = max / 127, and the
// row is written as two int8 pieces
//   q0 = rint(x / s_m),  q1 = rint((x - q0 s_m) * 128 / s_m),  |q1| <= 64,
// so x = s_m (q0 + q1 / 128) + e with |e| <= s_m / 256.  Piece rows are
// interleaved (row 2m = q0, row 2m + 1 = q1).
// Kept small (32 registers, at most 16 KB of shared memory) so that a CTA can
// share an SM with a CTA of the GEMM that follows it; the transform runs
// before the wait for the preceding kernel, and only the stores wait for it.
// Several seeds (a grouped call: one set of outputs per weight matrix) run in
// one launch: CTA b serves output set b / (M nc), token row (b mod M nc) / nc.
struct ActQ8Group {
  int count;
  uint64_t seed[kMaxGroup];
  int8_t* Xq[kMaxGroup];
  float* scales[kMaxGroup];
  float* Yz[kMaxGroup];
  int64_t yz_elems[kMaxGroup];
};

// a[g] for a runtime g without dynamic indexing of the parameter array
template <typename T>
__device__ __forceinline__ T pick_group(const T (&a)[kMaxGroup], int g) {
  T r = a[0];
#pragma unroll
  for (int j = 1; j < kMaxGroup; ++j)
    if (g == j) r = a[j];
  return r;
}

__global__ void __launch_bounds__(512, 4) k_act_q8(const uint16_t* __restrict__ X, int M, int K,
                                                   int nh, const ActQ8Group grp, int rows) {
  extern __shared__ __align__(16) float chunk[];   // the chunk's positions
  __shared__ float s_max[16];
  __shared__ float s_cmax;     // the chunk's largest magnitude, read by the cluster
  __shared__ float s_amax;     // the row's largest magnitude
  // the GEMM that follows may start at once: it touches nothing that this
  // kernel or its predecessor writes until its own wait for this grid.  A
  // kernel that releases its dependents early writes nothing that this one
  // reads (X comes from a finished kernel), so everything up to the stores
  // overlaps the tail of the preceding kernel.
  grid_dep_launch();
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int nc = (K + 4095) >> 12;                          // chunks of the row
  const int per_set = M * nc;                              // CTAs of one output set
  const int g = (int)blockIdx.x / per_set;
  const int rem = (int)blockIdx.x - g * per_set;
  const int m = rem / nc, c = rem % nc;                     // c: rank in the cluster
  const uint64_t seed = pick_group(grp.seed, g);
  int8_t* __restrict__ Xq = pick_group(grp.Xq, g);
  float* __restrict__ scales = pick_group(grp.scales, g);
  float* __restrict__ Yz = pick_group(grp.Yz, g);
  const int64_t yz_elems = pick_group(grp.yz_elems, g);
  const int kb = c << 12;
  const int C = K - kb < 4096 ? K - kb : 4096;              // a multiple of n_h
  const uint16_t* xrow = X + (size_t)m * K;
  float mx = 0.0f;
  if (8 * t < C) {
    const int k0 = kb + 8 * t;
    float y[8];
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(xrow + k0));
    const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      y[2 * i] = bf16_lo_to_f32(rw[i]);
      y[2 * i + 1] = bf16_hi_to_f32(rw[i]);
    }
    const uint32_t bits = (uint32_t)(splitmix64_output(seed, (uint64_t)(k0 >> 6)) >> (k0 & 63));
#pragma unroll
    for (int i = 0; i < 8; ++i)
      y[i] = __uint_as_float(__float_as_uint(y[i]) ^ (((bits >> i) & 1u) << 31));
    // butterflies (a, b) -> (a + b, a - b), a the lower position
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if ((i & h) == 0) {
          const float a = y[i], d = y[i + h];
          y[i] = a + d;
          y[i + h] = a - d;
        }
      }
    }
#pragma unroll
    for (int lm = 1; lm < 32; lm <<= 1) {
      const bool upper = (lane & lm) != 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float o = __shfl_xor_sync(0xffffffffu, y[i], lm);
        y[i] = upper ? o - y[i] : y[i] + o;
      }
    }
    *reinterpret_cast<float4*>(chunk + 8 * t) = make_float4(y[0], y[1], y[2], y[3]);
    *reinterpret_cast<float4*>(chunk + 8 * t + 4) = make_float4(y[4], y[5], y[6], y[7]);
    if (nh <= 256) {
#pragma unroll
      for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(y[i]));
    }
  }
  if (nh > 256) {
    __syncthreads();
    // stages across warps: h = 256 .. nh/2 on the positions g + 256 i
    const int g = t >> 1, half = t & 1;
    const int nw = C >> 8;                 // 256-position slices in the chunk
    float y[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = 8 * half + j;
      y[j] = i < nw ? chunk[g + 256 * i] : 0.0f;
    }
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {
      if (256 * h < nh) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if ((j & h) == 0) {
            const float a = y[j], d = y[j + h];
            y[j] = a + d;
            y[j + h] = a - d;
          }
        }
      }
    }
    if (nh > 2048) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float o = __shfl_xor_sync(0xffffffffu, y[j], 1);
        y[j] = half ? o - y[j] : y[j] + o;
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = 8 * half + j;
      if (i < nw) {
        chunk[g + 256 * i] = y[j];
        mx = fmaxf(mx, fabsf(y[j]));
      }
    }
  }
  // largest magnitude of the chunk, then of the row
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) s_max[warp] = mx;
  __syncthreads();
  if (t == 0) {
    float a = 0.0f;
#pragma unroll
    for (int w = 0; w < 16; ++w) a = fmaxf(a, s_max[w]);
    s_cmax = a;
    if (nc == 1) s_amax = a;
  }
  if (nc > 1) {
    // every CTA of the row publishes its maximum before any reads one
    cluster_arrive();
    cluster_wait();
    if (warp == 0) {
      float a = lane < nc ? ld_shared_cluster_f32(mapa_shared(smem_u32(&s_cmax), (uint32_t)lane))
                          : 0.0f;
#pragma unroll
      for (int off = 4; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
      if (lane == 0) s_amax = a;
    }
    // no CTA of the row leaves while another may still read its maximum
    cluster_arrive();
    cluster_wait();
  }
  __syncthreads();
  const float amax = s_amax;
  const float step = amax > 0.0f ? amax / 127.0f : 1.0f;
  const float inv = 1.0f / step;
  uint2 e0 = make_uint2(0u, 0u), e1 = make_uint2(0u, 0u);   // this thread's bytes
  if (8 * t < C) {
    const float4 xa = *reinterpret_cast<const float4*>(chunk + 8 * t);
    const float4 xb = *reinterpret_cast<const float4*>(chunk + 8 * t + 4);
    const float xs[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
    uint32_t p0[2] = {0u, 0u}, p1[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float a = fminf(fmaxf(rintf(xs[i] * inv), -127.0f), 127.0f);
      const float r = xs[i] - a * step;
      const float b = fminf(fmaxf(rintf(r * inv * 128.0f), -127.0f), 127.0f);
      const int ia = (int)a, ib = (int)b;
      p0[i >> 2] |= (uint32_t)(ia & 0xFF) << (8 * (i & 3));
      p1[i >> 2] |= (uint32_t)(ib & 0xFF) << (8 * (i & 3));
    }
    e0 = make_uint2(p0[0], p0[1]);
    e1 = make_uint2(p1[0], p1[1]);
  }
  // the stores wait for the preceding kernel, which may still read Xq, the
  // steps and Y
  grid_dep_wait();
  if (8 * t < C) {
    *reinterpret_cast<uint2*>(Xq + (size_t)(2 * m) * K + kb + 8 * t) = e0;
    *reinterpret_cast<uint2*>(Xq + (size_t)(2 * m + 1) * K + kb + 8 * t) = e1;
  }
  if (c == 0 && t == 0) scales[m] = step;
  if (Yz) {
    // the output that the following GEMM accumulates into starts at zero
    const int64_t nb = per_set;
    const int64_t per = ((yz_elems + nb - 1) / nb + 3) & ~int64_t(3);
    const int64_t z0 = (int64_t)rem * per, z1 = z0 + per < yz_elems ? z0 + per : yz_elems;
    for (int64_t i = z0 + 4 * t; i < z1; i += 4 * blockDim.x) {
      if (i + 4 <= z1) {
        *reinterpret_cast<float4*>(Yz + i) = make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        for (int64_t j = i; j < z1; ++j) Yz[j] = 0.0f;
      }
    }
  }
  // padding rows 2M .. rows-1: zero bytes
  for (int pr = 2 * M + m; pr < rows; pr += M) {
    for (int k = 16 * t; k < C; k += 16 * 512)
      *reinterpret_cast<uint4*>(Xq + (size_t)pr * K + kb + k) = make_uint4(0u, 0u, 0u, 0u);
  }
}

cudaError_t launch_act_q8_group(const uint16_t* X, int64_t M, int64_t K, const ActQ8Out* outs,
                                int count, int64_t rows, cudaStream_t st, int pdl,
                                int64_t nh_arg) {
  const int nh = (int)resolve_nh(K, nh_arg);
  if (nh < 256 || nh > 4096 || K > 32768 || M < 1 || M > 32 || rows < 2 * M || rows > 64 ||
      count < 1 || count > kMaxGroup)
    return cudaErrorInvalidValue;
  ActQ8Group grp = {};
  grp.count = count;
  for (int g = 0; g < count; ++g) {
    grp.seed[g] = outs[g].seed;
    grp.Xq[g] = outs[g].Xq;
    grp.scales[g] = outs[g].scales;
    grp.Yz[g] = outs[g].Yz;
    grp.yz_elems[g] = outs[g].Yz ? outs[g].yz_elems : 0;
  }
  const int nc = (int)((K + 4095) / 4096);
  const size_t smem = (size_t)(K < 4096 ? K : 4096) * sizeof(float);
  // the same shared-memory carveout as the GEMM that follows, so that the two
  // can share an SM (an SM runs CTAs of one carveout at a time)
  cudaError_t e = ensure_smem_limit(k_act_q8, kMaxDynSmem, true);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(M * nc * count));
  cfg.blockDim = dim3(512);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)nc;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = nc > 1 ? 2 : 1;
  e = cudaLaunchKernelEx(&cfg, k_act_q8, X, (int)M, (int)K, nh, grp, (int)rows);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_act_q8(const uint16_t* X, int64_t M, int64_t K, uint64_t seed, int8_t* Xq,
                          float* scales, int64_t rows, cudaStream_t st, int pdl, float* Yz,
                          int64_t yz_elems, int64_t nh) {
  ActQ8Out o;
  o.seed = seed;
  o.Xq = Xq;
  o.scales = scales;
  o.Yz = Yz;
  o.yz_elems = yz_elems;
  return launch_act_q8_group(X, M, K, &o, 1, rows, st, pdl, nh);
}

}  // namespace e8
