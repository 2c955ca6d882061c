// Entropy-coded E8 variant ("Transformers Proposes EntroPack Integration for
// Configurable Non-Integer-Bit-Rate Weight Compression", second paragraph:
// per-row normalised E8 lattice quantisation, a conditional probability model
// and entropy coding, the coded coordinates in independently decodable blocks,
// symbol decoding and weight reconstruction fused on the GPU; third paragraph:
// the actual rate counts the metadata).  The page fixes no detail; the format
// below is this library's reading of it:
//
//   t_n = fl32(max_k |w_nk| * delta), g_n = fl32(1 / t_n) (0 below FLT_MIN)
//   u   = fl32(w * g_n) per group of 8
//   V   = E8 point (doubled coordinates) by Conway & Sloane ("Sphere Packings,
//         Lattices and Groups", ch. 20) in fp32 with fixed tie rules:
//         D8: rint, parity repair at the first coordinate farthest from its
//         rounding, one step towards u (up when u_j >= f_j); D8 + 1/2: floor
//         + 1/2, repair likewise; squared distances summed in coordinate order
//         without fused operations; D8 wins ties
//   w'  = bf16_rne(fl32(V * fl32(t_n / 2)))
//   symbols per group: c = V mod 2, m_i = (V_i - c) / 2 (i < 7), q = floor(m_7 / 2)
//         (sum m even fixes m_7 mod 2); models P(c), P(m | c), P(q | c) with
//         12-bit frequencies counted over the matrix
//   rANS (Duda, 2013): 32-bit state in [2^16, 2^32), 16-bit words; one stream
//         per 64 consecutive groups: [x >> 16, x & 0xFFFF] of the final encoder
//         state, then the emitted words, last emitted first.
//
// Kernels: k_ep_rowscale (per-row maximum), k_ep_quant (lattice point, symbols,
// histogram), k_ep_rans (sizes, then words, one thread per block), k_ep_decode
// (one thread per block: symbols -> bf16 weights).
#include <cfloat>
#include <cmath>
#include <vector>

#include <cuda_bf16.h>

#include "e8.h"
#include "e8_common.cuh"
#include "e8_internal.h"

namespace e8 {
namespace ep {
constexpr int SCALE_BITS = 12;
constexpr uint32_t M_TOTAL = 1u << SCALE_BITS;
constexpr uint32_t RANS_L = 1u << 16;
constexpr int M_OFF = 128, M_SIZE = 256, Q_OFF = 64, Q_SIZE = 128;
constexpr int T_C = 0, T_M0 = 2, T_M1 = T_M0 + M_SIZE, T_Q0 = T_M1 + M_SIZE, T_Q1 = T_Q0 + Q_SIZE;
static_assert(T_Q1 + Q_SIZE == kEpTableWords, "table layout");
constexpr int kModelStart[5] = {T_C, T_M0, T_M1, T_Q0, T_Q1};
constexpr int kModelSize[5] = {2, M_SIZE, M_SIZE, Q_SIZE, Q_SIZE};
__device__ __forceinline__ int model_start(int i) {
  return i == 0 ? T_C : (i == 1 ? T_M0 : (i == 2 ? T_M1 : (i == 3 ? T_Q0 : T_Q1)));
}
__device__ __forceinline__ int model_size(int i) {
  return i == 0 ? 2 : (i < 3 ? M_SIZE : Q_SIZE);
}
}  // namespace ep

// ------------------------------------------------------------ row scales --
// One CTA per row: t_n = fl32(max |w| * delta), g_n = fl32(1 / t_n).
__global__ void __launch_bounds__(256) k_ep_rowscale(const float* __restrict__ W, int64_t K,
                                                     float delta, float* t, float* g) {
  const int64_t n = blockIdx.x;
  const float* row = W + n * K;
  float m = 0.0f;
  for (int64_t k = threadIdx.x; k < K; k += blockDim.x) m = fmaxf(m, fabsf(__ldg(row + k)));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  __shared__ float s_m[8];
  if ((threadIdx.x & 31) == 0) s_m[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, s_m[w]);
    float tn = __fmul_rn(m, delta);
    float gn = 0.0f;
    if (tn >= FLT_MIN) gn = __fdiv_rn(1.0f, tn);
    else tn = 0.0f;
    t[n] = tn;
    g[n] = gn;
  }
}

// ------------------------------------------------------- lattice point ----
// The quantiser's E8 point of u (doubled coordinates), rules as above.
__device__ __forceinline__ void ep_nearest(const float (&u)[8], int (&V)[8]) {
  float f[8], b[8];
  int sf = 0, sb = 0, jf = 0, jb = 0;
  float af = -1.0f, ab = -1.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f[i] = rintf(u[i]);
    b[i] = floorf(u[i]);
    sf += (int)f[i];
    sb += (int)b[i];
    const float ef = fabsf(__fsub_rn(u[i], f[i]));
    const float eb = fabsf(__fsub_rn(u[i], __fadd_rn(b[i], 0.5f)));
    if (ef > af) { af = ef; jf = i; }
    if (eb > ab) { ab = eb; jb = i; }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if ((sf & 1) && i == jf) f[i] = __fadd_rn(f[i], u[i] >= f[i] ? 1.0f : -1.0f);
    if ((sb & 1) && i == jb) b[i] = __fadd_rn(b[i], u[i] >= __fadd_rn(b[i], 0.5f) ? 1.0f : -1.0f);
  }
  float dD = 0.0f, dH = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float e = __fsub_rn(u[i], f[i]);
    dD = __fadd_rn(dD, __fmul_rn(e, e));
    const float h = __fsub_rn(u[i], __fadd_rn(b[i], 0.5f));
    dH = __fadd_rn(dH, __fmul_rn(h, h));
  }
  const bool d8 = dD <= dH;
#pragma unroll
  for (int i = 0; i < 8; ++i) V[i] = d8 ? 2 * (int)f[i] : 2 * (int)b[i] + 1;
}

// One thread per group (grid-stride): symbols packed in three words and the
// per-model histogram (shared-memory counts, then one global add per bin).
__global__ void __launch_bounds__(256) k_ep_quant(const float* __restrict__ W, int64_t G,
                                                  int64_t gpr, const float* __restrict__ g,
                                                  uint32_t* __restrict__ sym,
                                                  unsigned long long* hist, uint32_t* status) {
  using namespace ep;
  __shared__ uint32_t h[kEpTableWords];
  for (int i = threadIdx.x; i < kEpTableWords; i += blockDim.x) h[i] = 0u;
  __syncthreads();
  bool bad = false;
  for (int64_t gi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; gi < G;
       gi += (int64_t)gridDim.x * blockDim.x) {
    const float4* src = reinterpret_cast<const float4*>(W + 8 * gi);
    const float4 lo = __ldg(src), hi = __ldg(src + 1);
    const float gn = __ldg(g + gi / gpr);
    const float u[8] = {__fmul_rn(lo.x, gn), __fmul_rn(lo.y, gn), __fmul_rn(lo.z, gn),
                        __fmul_rn(lo.w, gn), __fmul_rn(hi.x, gn), __fmul_rn(hi.y, gn),
                        __fmul_rn(hi.z, gn), __fmul_rn(hi.w, gn)};
    int V[8];
    ep_nearest(u, V);
    const int c = V[0] & 1;
    int m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      m[i] = (V[i] - c) >> 1;
      if (m[i] < -128 || m[i] > 127) {   // only for non-finite weights or a smaller step
        bad = true;
        m[i] = m[i] < -128 ? -128 : 127;
      }
    }
    const int q = m[7] >> 1;
    const uint32_t w0 = (uint32_t)c | ((uint32_t)(m[0] + M_OFF) << 8) |
                        ((uint32_t)(m[1] + M_OFF) << 16) | ((uint32_t)(m[2] + M_OFF) << 24);
    const uint32_t w1 = (uint32_t)(m[3] + M_OFF) | ((uint32_t)(m[4] + M_OFF) << 8) |
                        ((uint32_t)(m[5] + M_OFF) << 16) | ((uint32_t)(m[6] + M_OFF) << 24);
    sym[3 * gi] = w0;
    sym[3 * gi + 1] = w1;
    sym[3 * gi + 2] = (uint32_t)(q + Q_OFF);
    atomicAdd(&h[T_C + c], 1u);
    const int tm = c ? T_M1 : T_M0;
#pragma unroll
    for (int i = 0; i < 7; ++i) atomicAdd(&h[tm + m[i] + M_OFF], 1u);
    atomicAdd(&h[(c ? T_Q1 : T_Q0) + q + Q_OFF], 1u);
  }
  if (bad) atomicOr(status, kDevBadInput);
  __syncthreads();
  for (int i = threadIdx.x; i < kEpTableWords; i += blockDim.x)
    if (h[i]) atomicAdd(hist + i, (unsigned long long)h[i]);
}

// ------------------------------------------------------------------- rANS --
// Frequencies and cumulative frequencies of the five models in shared memory
// (fc[i] = f | cum << 16).  Returns false when a model does not sum to 4096.
__device__ bool ep_load_tables(const uint16_t* __restrict__ tables, uint32_t* fc) {
  using namespace ep;
  __shared__ int s_ok;
  if (threadIdx.x == 0) s_ok = 1;
  __syncthreads();
  if (threadIdx.x < 5) {
    const int st = model_start((int)threadIdx.x), sz = model_size((int)threadIdx.x);
    uint32_t cum = 0;
    for (int s = 0; s < sz; ++s) {
      const uint32_t f = __ldg(tables + st + s);
      fc[st + s] = f | ((cum & 0xFFFFu) << 16);
      cum += f;
    }
    if (cum != M_TOTAL) atomicAnd(&s_ok, 0);
  }
  __syncthreads();
  return s_ok != 0;
}

// Encodes block b (groups [64 b, 64 b + n)) last symbol first.  Pass 0 writes
// the block's size in words; pass 1 writes its stream at offsets[b].
__global__ void __launch_bounds__(128) k_ep_rans(const uint32_t* __restrict__ sym, int64_t G,
                                                 int64_t nblocks,
                                                 const uint16_t* __restrict__ tables, int pass,
                                                 uint32_t* sizes, const uint32_t* offsets,
                                                 uint16_t* words, uint32_t* status) {
  using namespace ep;
  __shared__ uint32_t fc[kEpTableWords];
  if (!ep_load_tables(tables, fc)) {
    if (threadIdx.x == 0) atomicOr(status, kDevBadInput);
    return;
  }
  const int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= nblocks) return;
  const int64_t g0 = b * kEpBlockGroups;
  const int64_t g1 = g0 + kEpBlockGroups < G ? g0 + kEpBlockGroups : G;
  uint32_t x = RANS_L;
  uint32_t emitted = 0;
  uint16_t* out = nullptr;
  if (pass == 1) out = words + offsets[b + 1];   // emitted words fill backwards from the end
  auto put = [&](int idx, bool& ok) {
    const uint32_t e = fc[idx];
    const uint32_t f = e & 0xFFFFu, cum = e >> 16;
    if (f == 0u) {
      ok = false;
      return;
    }
    if ((uint64_t)x >= ((uint64_t)f << (32 - SCALE_BITS))) {   // f = 4096 reaches 2^32
      if (pass == 1) *--out = (uint16_t)(x & 0xFFFFu);
      ++emitted;
      x >>= 16;
    }
    x = ((x / f) << SCALE_BITS) + (x % f) + cum;
  };
  bool ok = true;
  for (int64_t gi = g1 - 1; gi >= g0 && ok; --gi) {
    const uint32_t w0 = __ldg(sym + 3 * gi), w1 = __ldg(sym + 3 * gi + 1);
    const uint32_t q = __ldg(sym + 3 * gi + 2);
    const uint32_t c = w0 & 1u;
    put((c ? T_Q1 : T_Q0) + (int)q, ok);
    const int tm = c ? T_M1 : T_M0;
    put(tm + (int)(w1 >> 24), ok);
    put(tm + (int)((w1 >> 16) & 0xFFu), ok);
    put(tm + (int)((w1 >> 8) & 0xFFu), ok);
    put(tm + (int)(w1 & 0xFFu), ok);
    put(tm + (int)(w0 >> 24), ok);
    put(tm + (int)((w0 >> 16) & 0xFFu), ok);
    put(tm + (int)((w0 >> 8) & 0xFFu), ok);
    put(T_C + (int)c, ok);
  }
  if (!ok) atomicOr(status, kDevBadInput);
  if (pass == 0) {
    sizes[b] = 2u + emitted;
  } else {
    words[offsets[b]] = (uint16_t)(x >> 16);
    words[offsets[b] + 1] = (uint16_t)(x & 0xFFFFu);
  }
}

// One thread per block: its stream -> symbols -> bf16 weights.  A stream that
// runs past its end or does not return to the initial state sets
// kDevBadStream; the weights it wrote are then unspecified.  With stage_cap >
// 0 the streams of the CTA's 128 blocks are first copied, coalesced, into
// shared memory (when they fit), so that the serial decode of each block waits
// on shared-memory rather than global-memory latency for every word; the
// launcher stages only when all CTAs fit on the GPU at once (the 48 KB stage
// costs occupancy, which a grid of several waves needs more).
constexpr int kEpStageWords = 24576;   // 48 KB
__global__ void __launch_bounds__(128) k_ep_decode(const uint16_t* __restrict__ words,
                                                   const uint32_t* __restrict__ offsets,
                                                   const float* __restrict__ t,
                                                   const uint16_t* __restrict__ tables, int64_t G,
                                                   int64_t gpr, int64_t nblocks, uint32_t n_words,
                                                   uint32_t stage_cap, uint16_t* out,
                                                   uint32_t* status) {
  using namespace ep;
  extern __shared__ uint16_t s_words[];    // the CTA's streams, stage_cap words at most
  __shared__ uint32_t fc[kEpTableWords];
  __shared__ uint8_t sym_of[4][M_TOTAL];   // slot -> symbol of m|0, m|1, q|0, q|1
  const int64_t b0 = (int64_t)blockIdx.x * blockDim.x;
  const int64_t b1 = b0 + (int64_t)blockDim.x < nblocks ? b0 + (int64_t)blockDim.x : nblocks;
  const uint32_t base = __ldg(offsets + b0), top = __ldg(offsets + b1);
  const bool staged = top >= base && top <= n_words && top - base <= stage_cap;
  if (staged)
    for (uint32_t i = threadIdx.x; i < top - base; i += blockDim.x) s_words[i] = __ldg(words + base + i);
  if (!ep_load_tables(tables, fc)) {
    if (threadIdx.x == 0) atomicOr(status, kDevBadStream);
    return;
  }
  {
    // each thread a run of consecutive slots: the last symbol whose cum is at
    // most the slot, found once by bisection and then walked forward
    const uint32_t per = M_TOTAL / blockDim.x, j0 = threadIdx.x * per;
#pragma unroll
    for (int mdl = 0; mdl < 4; ++mdl) {
      const int st = model_start(mdl + 1), sz = model_size(mdl + 1);
      int lo = 0, hi = sz - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((fc[st + mid] >> 16) <= j0) lo = mid;
        else hi = mid - 1;
      }
      for (uint32_t j = j0; j < j0 + per; ++j) {
        while (lo + 1 < sz && (fc[st + lo + 1] >> 16) <= j) ++lo;
        sym_of[mdl][j] = (uint8_t)lo;
      }
    }
  }
  __syncthreads();
  const int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= nblocks) return;
  const uint32_t off = __ldg(offsets + b), end = __ldg(offsets + b + 1);
  const uint32_t len = end - off;
  if (end < off || len < 2u || end > n_words || (staged && (off < base || end > top))) {
    atomicOr(status, kDevBadStream);
    return;
  }
  const uint16_t* w = staged ? s_words + (off - base) : words + off;
  uint32_t x = ((uint32_t)w[0] << 16) | (uint32_t)w[1];
  uint32_t p = 2;
  bool ok = true;
  const uint32_t fc0 = fc[T_C] & 0xFFFFu;
  auto step = [&](uint32_t e, uint32_t slot) {
    x = (e & 0xFFFFu) * (x >> SCALE_BITS) + slot - (e >> 16);
    if (x < RANS_L) {
      if (p < len) x = (x << 16) | (uint32_t)w[p];
      else ok = false;
      ++p;
    }
  };
  const int64_t g0 = b * kEpBlockGroups;
  const int64_t g1 = g0 + kEpBlockGroups < G ? g0 + kEpBlockGroups : G;
  // row of the current group, advanced without a division per group
  int64_t row = g0 / gpr, col = g0 - row * gpr;
  float a = __fmul_rn(__ldg(t + row), 0.5f);
  for (int64_t gi = g0; gi < g1 && ok; ++gi) {
    if (col == gpr) {
      col = 0;
      a = __fmul_rn(__ldg(t + ++row), 0.5f);
    }
    ++col;
    uint32_t slot = x & (M_TOTAL - 1u);
    const int c = slot >= fc0 ? 1 : 0;
    step(fc[T_C + c], slot);
    const uint8_t* sm = sym_of[c];
    const int tm = c ? T_M1 : T_M0;
    int m[8];
    int par = 0;
#pragma unroll
    for (int i = 0; i < 7; ++i) {
      slot = x & (M_TOTAL - 1u);
      const int s = sm[slot];
      step(fc[tm + s], slot);
      m[i] = s - M_OFF;
      par += m[i];
    }
    slot = x & (M_TOTAL - 1u);
    const int sq = sym_of[2 + c][slot];
    step(fc[(c ? T_Q1 : T_Q0) + sq], slot);
    m[7] = 2 * (sq - Q_OFF) + (par & 1);
    uint32_t pk[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float v0 = __fmul_rn((float)(2 * m[2 * i] + c), a);
      const float v1 = __fmul_rn((float)(2 * m[2 * i + 1] + c), a);
      pk[i] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v0)) |
              ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v1)) << 16);
    }
    *reinterpret_cast<uint4*>(out + 8 * gi) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
  if (!ok || x != RANS_L || p != len) atomicOr(status, kDevBadStream);
}

// ------------------------------------------------------------------- host --
// Frequencies summing to 4096 from counts (the rule of the format: floor
// scaling with at least 1 for a symbol that occurs, the difference to the most
// frequent symbol, smallest index on ties, while it stays >= 1; any rest one
// unit at a time from the largest frequencies; an empty model puts 4096 on
// symbol 0).
static bool ep_normalise(const unsigned long long* counts, int n, uint16_t* f) {
  unsigned long long total = 0;
  for (int s = 0; s < n; ++s) total += counts[s];
  std::vector<long long> fr(n, 0);
  if (total == 0) {
    fr[0] = ep::M_TOTAL;
  } else {
    long long sum = 0;
    int big = 0;
    for (int s = 0; s < n; ++s) {
      if (counts[s]) {
        const long long v = (long long)((counts[s] * (unsigned long long)ep::M_TOTAL) / total);
        fr[s] = v < 1 ? 1 : v;
      }
      sum += fr[s];
      if (counts[s] > counts[big]) big = s;
    }
    long long diff = (long long)ep::M_TOTAL - sum;
    if (fr[big] + diff >= 1) {
      fr[big] += diff;
    } else {
      diff += fr[big] - 1;
      fr[big] = 1;
      while (diff < 0) {
        int s = 0;
        for (int r = 1; r < n; ++r)
          if (fr[r] > fr[s]) s = r;
        if (fr[s] <= 1) return false;
        --fr[s];
        ++diff;
      }
    }
  }
  for (int s = 0; s < n; ++s) f[s] = (uint16_t)fr[s];
  return true;
}

int64_t ep_num_blocks(int64_t N, int64_t K) {
  const int64_t G = N * (K / 8);
  return (G + kEpBlockGroups - 1) / kEpBlockGroups;
}

int64_t ep_max_words(int64_t N, int64_t K) {
  return 9 * N * (K / 8) + 2 * ep_num_blocks(N, K);
}

size_t ep_encode_workspace_bytes(int64_t N, int64_t K) {
  const int64_t G = N * (K / 8);
  auto r256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  return r256((size_t)G * 12) + r256((size_t)ep_num_blocks(N, K) * 4) +
         2 * r256((size_t)N * 4) + r256(kEpTableWords * 8);
}

namespace {
struct EpScratch {
  uint32_t* sym;
  uint32_t* sizes;
  float* g;
  float* t;   // row scales of the rate estimate
  unsigned long long* hist;
};
EpScratch ep_scratch(void* ws, int64_t N, int64_t K) {
  auto r256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  const int64_t G = N * (K / 8);
  uint8_t* p = static_cast<uint8_t*>(ws);
  EpScratch s;
  s.sym = reinterpret_cast<uint32_t*>(p);
  p += r256((size_t)G * 12);
  s.sizes = reinterpret_cast<uint32_t*>(p);
  p += r256((size_t)ep_num_blocks(N, K) * 4);
  s.g = reinterpret_cast<float*>(p);
  p += r256((size_t)N * 4);
  s.t = reinterpret_cast<float*>(p);
  p += r256((size_t)N * 4);
  s.hist = reinterpret_cast<unsigned long long*>(p);
  return s;
}

int quant_grid(int64_t G, int sm_count) {
  const int64_t want = (G + 255) / 256;
  const int64_t cap = (int64_t)sm_count * 8;
  return (int)(want < cap ? (want < 1 ? 1 : want) : cap);
}

// Row scales, lattice points, symbols and the histogram at step delta; the
// histogram is copied to `hist_host` (the call synchronises the stream).
cudaError_t ep_quantise_and_count(const float* W, int64_t N, int64_t K, float delta, float* t,
                                  const EpScratch& s, uint32_t* status, int sm_count,
                                  cudaStream_t st, unsigned long long* hist_host) {
  const int64_t G = N * (K / 8);
  cudaError_t e = cudaMemsetAsync(s.hist, 0, kEpTableWords * 8, st);
  if (e != cudaSuccess) return e;
  k_ep_rowscale<<<(unsigned)N, 256, 0, st>>>(W, K, delta, t, s.g);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  k_ep_quant<<<quant_grid(G, sm_count), 256, 0, st>>>(W, G, K / 8, s.g, s.sym, s.hist, status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  e = cudaMemcpyAsync(hist_host, s.hist, kEpTableWords * 8, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(st);
}

bool ep_tables_from_hist(const unsigned long long* hist, uint16_t* tables) {
  for (int mdl = 0; mdl < 5; ++mdl)
    if (!ep_normalise(hist + ep::kModelStart[mdl], ep::kModelSize[mdl],
                      tables + ep::kModelStart[mdl]))
      return false;
  return true;
}
}  // namespace

int ep_encode(const float* W, int64_t N, int64_t K, float delta, uint16_t* words,
              int64_t max_words, uint32_t* offsets, float* t, uint16_t* tables, void* ws,
              uint32_t* status, int sm_count, cudaStream_t st, int64_t* total_words) {
  const int64_t G = N * (K / 8);
  const int64_t nb = ep_num_blocks(N, K);
  const EpScratch s = ep_scratch(ws, N, K);
  std::vector<unsigned long long> hist(kEpTableWords);
  cudaError_t e = ep_quantise_and_count(W, N, K, delta, t, s, status, sm_count, st, hist.data());
  if (e != cudaSuccess) return 1;
  uint16_t tb[kEpTableWords];
  if (!ep_tables_from_hist(hist.data(), tb)) return 2;
  if (cudaMemcpyAsync(tables, tb, sizeof(tb), cudaMemcpyHostToDevice, st) != cudaSuccess) return 1;
  const unsigned grid = (unsigned)((nb + 127) / 128);
  k_ep_rans<<<grid, 128, 0, st>>>(s.sym, G, nb, tables, 0, s.sizes, nullptr, nullptr, status);
  if (cudaGetLastError() != cudaSuccess) return 1;
  std::vector<uint32_t> sizes(nb), offs(nb + 1);
  if (cudaMemcpyAsync(sizes.data(), s.sizes, nb * 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return 1;
  uint64_t acc = 0;
  for (int64_t b = 0; b < nb; ++b) {
    offs[b] = (uint32_t)acc;
    acc += sizes[b];
  }
  if (acc > (uint64_t)max_words || acc >= (1ull << 32)) return 3;
  offs[nb] = (uint32_t)acc;
  if (cudaMemcpyAsync(offsets, offs.data(), (nb + 1) * 4, cudaMemcpyHostToDevice, st) !=
      cudaSuccess)
    return 1;
  k_ep_rans<<<grid, 128, 0, st>>>(s.sym, G, nb, tables, 1, nullptr, offsets, words, status);
  if (cudaGetLastError() != cudaSuccess) return 1;
  if (cudaStreamSynchronize(st) != cudaSuccess) return 1;
  *total_words = (int64_t)acc;
  return 0;
}

int ep_estimate_bpp(const float* W, int64_t N, int64_t K, float delta, void* ws,
                    uint32_t* status, int sm_count, cudaStream_t st, double* bpp) {
  const EpScratch s = ep_scratch(ws, N, K);
  std::vector<unsigned long long> hist(kEpTableWords);
  if (ep_quantise_and_count(W, N, K, delta, s.t, s, status, sm_count, st, hist.data()) !=
      cudaSuccess)
    return 1;
  uint16_t tb[kEpTableWords];
  if (!ep_tables_from_hist(hist.data(), tb)) return 2;
  double bits = 0.0;
  for (int i = 0; i < kEpTableWords; ++i)
    if (hist[i]) bits += (double)hist[i] * (ep::SCALE_BITS - std::log2((double)tb[i]));
  const int64_t nb = ep_num_blocks(N, K);
  bits += 32.0 * nb + 32.0 * (nb + 1) + 32.0 * N + 16.0 * kEpTableWords + 32.0;
  *bpp = bits / ((double)N * (double)K);
  return 0;
}

cudaError_t launch_ep_decode(const uint16_t* words, int64_t n_words, const uint32_t* offsets,
                             const float* t, const uint16_t* tables, int64_t N, int64_t K,
                             uint16_t* out, uint32_t* status, int sm_count, cudaStream_t st) {
  const int64_t G = N * (K / 8);
  const int64_t nb = ep_num_blocks(N, K);
  if (nb == 0) return cudaSuccess;
  cudaError_t e = ensure_smem_limit(k_ep_decode, kEpStageWords * 2);
  if (e != cudaSuccess) return e;
  static int per_sm = -1;   // CTAs per SM with the stage (same on every B200)
  if (per_sm < 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_ep_decode, 128, kEpStageWords * 2) !=
        cudaSuccess)
      n = 0;
    per_sm = n;
  }
  const int64_t ctas = (nb + 127) / 128;
  const bool stage = ctas <= (int64_t)per_sm * sm_count;
  k_ep_decode<<<(unsigned)ctas, 128, stage ? kEpStageWords * 2 : 0, st>>>(
      words, offsets, t, tables, G, K / 8, nb, (uint32_t)n_words,
      stage ? (uint32_t)kEpStageWords : 0u, out, status);
  return cudaGetLastError();
}

}  // namespace e8

// ------------------------------------------------------------------ C ABI --
namespace {
int ep_check(const e8_codebook* cb) {
  if (!cb) return E8_EINVAL;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return E8_ECUDA;
  return dev == cb->device ? E8_OK : E8_EDEVICE;
}
bool ep_shape_ok(int64_t N, int64_t K) {
  return N >= 0 && K >= 8 && (K % 8) == 0 && N <= (int64_t)1 << 31 &&
         N * (K / 8) <= ((int64_t)1 << 31);
}
bool ep_delta_ok(float d) { return std::isfinite(d) && d >= 1.0f / 120.0f; }
bool al(const void* p, unsigned a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
}  // namespace

extern "C" {

int64_t e8_ep_num_blocks(int64_t N, int64_t K) {
  return ep_shape_ok(N, K) ? e8::ep_num_blocks(N, K) : -1;
}

int64_t e8_ep_max_words(int64_t N, int64_t K) {
  return ep_shape_ok(N, K) ? e8::ep_max_words(N, K) : -1;
}

size_t e8_ep_encode_workspace_bytes(int64_t N, int64_t K) {
  return ep_shape_ok(N, K) ? e8::ep_encode_workspace_bytes(N, K) : 0;
}

double e8_ep_actual_bpp(int64_t N, int64_t K, int64_t total_words) {
  if (!ep_shape_ok(N, K) || N == 0 || total_words < 0) return -1.0;
  const double bits = 16.0 * (double)total_words + 32.0 * (double)(e8::ep_num_blocks(N, K) + 1) +
                      32.0 * (double)N + 16.0 * e8::kEpTableWords + 32.0;
  return bits / ((double)N * (double)K);
}

size_t e8_ep_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || !ep_shape_ok(N, K)) return 0;
  return ((size_t)N * (size_t)K * 2 + 255) & ~size_t(255);
}

int e8_ep_encode(const e8_codebook* cb, const float* W, int64_t N, int64_t K, float delta,
                 uint16_t* words, int64_t max_words, uint32_t* offsets, float* t,
                 uint16_t* tables, int64_t* total_words, void* workspace, size_t ws_bytes,
                 void* stream) {
  (void)cudaGetLastError();  // a failed earlier launch must not be reported here
  int rc = ep_check(cb);
  if (rc != E8_OK) return rc;
  if (!ep_shape_ok(N, K) || !ep_delta_ok(delta) || !total_words) return E8_EINVAL;
  *total_words = 0;
  if (!offsets || !tables || !al(offsets, 4) || !al(tables, 2)) return E8_EINVAL;
  cudaStream_t st = (cudaStream_t)stream;
  if (N == 0) {
    // no groups: an empty stream and the tables of empty models
    uint16_t tb[e8::kEpTableWords] = {};
    for (int mdl = 0; mdl < 5; ++mdl) tb[e8::ep::kModelStart[mdl]] = (uint16_t)e8::ep::M_TOTAL;
    const uint32_t zero = 0;
    if (cudaMemcpyAsync(tables, tb, sizeof(tb), cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(offsets, &zero, 4, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return E8_ECUDA;
    return E8_OK;
  }
  if (!W || !words || !t || !al(W, 16) || !al(words, 2) || !al(t, 4)) return E8_EINVAL;
  if (!workspace || !al(workspace, 256) ||
      ws_bytes < e8::ep_encode_workspace_bytes(N, K))
    return E8_EWORKSPACE;
  int64_t total = 0;
  const int r = e8::ep_encode(W, N, K, delta, words, max_words, offsets, t, tables, workspace,
                              cb->status, cb->sm_count, st, &total);
  if (r == 1) return E8_ECUDA;
  if (r == 2) return E8_EINVAL;
  if (r == 3) return E8_EWORKSPACE;
  *total_words = total;
  return E8_OK;
}

int e8_ep_estimate_bpp(const e8_codebook* cb, const float* W, int64_t N, int64_t K, float delta,
                       double* bpp, void* workspace, size_t ws_bytes, void* stream) {
  (void)cudaGetLastError();
  int rc = ep_check(cb);
  if (rc != E8_OK) return rc;
  if (!ep_shape_ok(N, K) || N == 0 || !ep_delta_ok(delta) || !bpp || !W || !al(W, 16))
    return E8_EINVAL;
  if (!workspace || !al(workspace, 256) || ws_bytes < e8::ep_encode_workspace_bytes(N, K))
    return E8_EWORKSPACE;
  const int r = e8::ep_estimate_bpp(W, N, K, delta, workspace, cb->status, cb->sm_count,
                                    (cudaStream_t)stream, bpp);
  return r == 0 ? E8_OK : (r == 1 ? E8_ECUDA : E8_EINVAL);
}

int e8_ep_choose_delta(const e8_codebook* cb, const float* W, int64_t N, int64_t K,
                       double target_bpp, float* delta, void* workspace, size_t ws_bytes,
                       void* stream) {
  if (!delta || !(target_bpp > 0.0) || !std::isfinite(target_bpp)) return E8_EINVAL;
  // the estimate falls as the step grows: bisection on log(delta) between
  // 1/120 and 16 for the smallest step whose estimate is at most the target
  float lo = 1.0f / 120.0f, hi = 16.0f;
  double b = 0.0;
  int rc = e8_ep_estimate_bpp(cb, W, N, K, lo, &b, workspace, ws_bytes, stream);
  if (rc != E8_OK) return rc;
  if (b <= target_bpp) {
    *delta = lo;
    return E8_OK;
  }
  for (int it = 0; it < 40; ++it) {
    const float mid = (float)std::sqrt((double)lo * (double)hi);
    if (!(mid > lo && mid < hi)) break;
    rc = e8_ep_estimate_bpp(cb, W, N, K, mid, &b, workspace, ws_bytes, stream);
    if (rc != E8_OK) return rc;
    if (b <= target_bpp) hi = mid;
    else lo = mid;
  }
  *delta = hi;
  return E8_OK;
}

int e8_ep_decode_to_bf16(const e8_codebook* cb, const uint16_t* words, int64_t n_words,
                         const uint32_t* offsets, const float* t, const uint16_t* tables,
                         int64_t N, int64_t K, uint16_t* out, void* stream) {
  (void)cudaGetLastError();
  int rc = ep_check(cb);
  if (rc != E8_OK) return rc;
  if (!ep_shape_ok(N, K) || n_words < 0 || n_words >= ((int64_t)1 << 32)) return E8_EINVAL;
  if (N == 0) return E8_OK;
  if (!words || !offsets || !t || !tables || !out || !al(words, 2) || !al(offsets, 4) ||
      !al(t, 4) || !al(tables, 2) || !al(out, 16))
    return E8_EINVAL;
  return e8::launch_ep_decode(words, n_words, offsets, t, tables, N, K, out, cb->status,
                              cb->sm_count, (cudaStream_t)stream) == cudaSuccess
             ? E8_OK
             : E8_ECUDA;
}

int e8_ep_gemm(const e8_codebook* cb, const uint16_t* X, int64_t M, const uint16_t* words,
               int64_t n_words, const uint32_t* offsets, const float* t, const uint16_t* tables,
               int64_t N, int64_t K, float* Y, void* workspace, size_t ws_bytes, void* stream) {
  (void)cudaGetLastError();
  int rc = ep_check(cb);
  if (rc != E8_OK) return rc;
  if (M < 0 || !ep_shape_ok(N, K)) return E8_EINVAL;
  if (M == 0 || N == 0) return E8_OK;
  if (!X || !Y || !al(X, 16) || !al(Y, 16)) return E8_EINVAL;
  if (!workspace || !al(workspace, 256) || ws_bytes < e8_ep_gemm_workspace_bytes(M, N, K))
    return E8_EWORKSPACE;
  uint16_t* Wd = static_cast<uint16_t*>(workspace);
  rc = e8_ep_decode_to_bf16(cb, words, n_words, offsets, t, tables, N, K, Wd, stream);
  if (rc != E8_OK) return rc;
  return e8::launch_dense_gemm(X, M, Wd, N, K, Y, cb->status, cb->sm_count,
                               (cudaStream_t)stream) == cudaSuccess
             ? E8_OK
             : E8_ECUDA;
}

}  // extern "C"

