// Encoder: randomized Hadamard transform, then nearest E8 codebook point per
// group of 8 weights ("glq 0.1.1", "How it works", items 1 and 2).
//
//   u = fl32(FWHT_nh(D w) * gamma),  gamma = fl32(1 / (s sqrt(nh)))
//   idx1 = argmin_{c in C} |u - c|^2                       (ties: smallest index)
//   idx2 = argmin_{c2 in C2} |u - c1 - beta c2|^2          (3 bpw: C2 = first 256
//          entries, beta = 1/2; 4 bpw: C2 = C, beta = 1/4)
//
// The forward transform runs in fp32 with the butterflies of stage h pairing
// elements i and i + h, (a, b) -> (a + b, a - b), stages h = 1, 2, 4, ... in
// that order, so every element sees exactly the same rounding sequence as in a
// plain sequential loop.
//
// Nearest point, fast path (Conway & Sloane, "Sphere Packings, Lattices and
// Groups", ch. 20: E8 = D8 u (D8 + 1/2)): round every coordinate, repair the
// coordinate sum parity at the coordinate with the largest rounding error, do
// the same for the half-integer coset, keep the nearer of the two.  All
// rounding decisions are exact in fp32; the coset comparison is linear in the
// rounding errors.  Any decision that is a tie, or closer than a safe margin to
// one, and any lattice point that is not in the codebook, sends the group to
// the exact slow path: a brute force over the codebook whose comparisons are
// exact (floating-point expansions), smallest index on ties.
#include "e8_common.cuh"
#include "e8_codebook.cuh"
#include "e8_internal.h"

namespace e8 {

// ------------------------------------------------------------ FWHT in SMEM --
// Elements [0, E) of smem hold E / nh independent blocks; performs the stages
// h = from_h, 2 from_h, ..., nh / 2 on every block.  Called by all threads.
__device__ __forceinline__ void smem_fwht_stages(float* s, int E, int nh, int from_h) {
  const int half = E >> 1;
  for (int h = from_h; h < nh; h <<= 1) {
    __syncthreads();
    for (int b = threadIdx.x; b < half; b += blockDim.x) {
      int i = (b / h) * (2 * h) + (b % h);
      float a = s[i], c = s[i + h];
      s[i] = a + c;
      s[i + h] = a - c;
    }
  }
  __syncthreads();
}

// In-register stages h = 1, 2, 4 on one group of 8 consecutive elements.
__device__ __forceinline__ void group_fwht8(float (&y)[8]) {
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
}

// ----------------------------------------------------- Conway-Sloane step --
// Lattice point nearest to x = y - o, with y fp32 (exact input) and o an
// integer vector; the result is written in doubled coordinates V.  Returns
// false when the answer is not certain (a rounding tie, a parity repair tie, a
// coset comparison within the safety margin, or coordinates too large).
__device__ bool cs_nearest(const float (&y)[8], const int (&o)[8], int (&V)[8]) {
  float a[8], d[8];
  int r[8], fl[8];
  int sumD = 0, sumH = 0;
  bool tieD = false, tieH = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (!(fabsf(y[i]) < 1048576.0f)) return false;
    float ri = rintf(y[i]);
    d[i] = y[i] - ri;  // exact
    a[i] = fabsf(d[i]);
    r[i] = (int)ri - o[i];
    fl[i] = (int)floorf(y[i]) - o[i];
    sumD += r[i];
    sumH += fl[i];
    tieD |= (a[i] == 0.5f);
    tieH |= (a[i] == 0.0f);
  }
  // D8: repair parity at the coordinate farthest from its rounding
  bool flipD = (sumD & 1) != 0;
  int jD = 0;
  float aD = -1.0f;
  bool tieFD = false;
  if (flipD) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (a[i] > aD) { aD = a[i]; jD = i; tieFD = false; }
      else if (a[i] == aD) tieFD = true;
    }
    if (aD == 0.0f) tieFD = true;
  }
  // D8 + 1/2: nearest half-integer is floor(y) + 1/2 at distance 1/2 - a_i;
  // repair parity at the coordinate farthest from it, i.e. smallest a_i
  bool flipH = (sumH & 1) != 0;
  int jH = 0;
  float aH = 2.0f;
  bool tieFH = false;
  if (flipH) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (a[i] < aH) { aH = a[i]; jH = i; tieFH = false; }
      else if (a[i] == aH) tieFH = true;
    }
    if (aH == 0.5f) tieFH = true;
  }
  // |y - D8 point|^2 - |y - half point|^2 = sum a_i - 2 + corrections
  float sa = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) sa += a[i];
  float diff = sa - 2.0f;
  if (flipD) diff += 1.0f - 2.0f * aD;
  if (flipH) diff -= 2.0f * aH;
  if (fabsf(diff) <= 0x1p-16f) return false;
  if (diff < 0.0f) {
    if (tieD || (flipD && tieFD)) return false;
#pragma unroll
    for (int i = 0; i < 8; ++i) V[i] = 2 * r[i];
    if (flipD) V[jD] += d[jD] > 0.0f ? 2 : -2;
  } else {
    if (tieH || (flipH && tieFH)) return false;
#pragma unroll
    for (int i = 0; i < 8; ++i) V[i] = 2 * fl[i] + 1;
    if (flipH) {
      // move to the other side of y: up when y is above the half-integer
      float frac = y[jH] - floorf(y[jH]);
      V[jH] += frac > 0.5f ? 2 : -2;
    }
  }
  return true;
}

// Index of V inside the candidate set (C, or its first 256 entries), or -1.
__device__ __forceinline__ int member_index(const DeviceCodebook& cb, const int (&V)[8],
                                            int set_size) {
  int n4 = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (V[i] < -6 || V[i] > 6) return -1;
    n4 += V[i] * V[i];
  }
  if (n4 > 48) return -1;
  int idx = rank_vector(cb, V);
  return (idx >= 0 && idx < set_size) ? idx : -1;
}

struct EncodeParams {
  const float* W;
  int64_t N, K;
  int nh, elems_per_cta, bpw;
  uint64_t seed;
  float gamma;
  uint16_t* idx1;
  void* idx2;
  WorkItem* work;
  uint32_t* work_count;
  uint64_t work_cap;
  float* U;  // optional: transformed weights out (nullptr: not written)
  int do_quantise;
};

__device__ __forceinline__ void push_work(const EncodeParams& p, const DeviceCodebook& cb,
                                          const float (&u)[8], int64_t g, uint32_t mask) {
  uint32_t slot = atomicAdd(p.work_count, 1u);
  if (slot >= p.work_cap) {
    atomicOr(cb.status, kDevWorklistOverflow);
    return;
  }
  WorkItem& w = p.work[slot];
#pragma unroll
  for (int i = 0; i < 8; ++i) w.u[i] = u[i];
  w.group = g;
  w.mask = mask;
  w.cand = 0u;
}

__global__ void __launch_bounds__(256) k_encode(EncodeParams p, DeviceCodebook cb) {
  extern __shared__ __align__(16) float s_y[];
  const int64_t total = p.N * p.K;
  const int64_t base = (int64_t)blockIdx.x * p.elems_per_cta;
  const int E = (int)(int64_t)min((long long)p.elems_per_cta, (long long)(total - base));  // multiple of nh
  const int ngroups = E >> 3;
  // load, sign, in-register stages h = 1, 2, 4, store to shared memory
  for (int g = threadIdx.x; g < ngroups; g += blockDim.x) {
    int64_t e0 = base + 8 * (int64_t)g;
    int64_t k0 = e0 % p.K;
    const float4* src = reinterpret_cast<const float4*>(p.W + e0);
    float4 lo = __ldg(src), hi = __ldg(src + 1);
    float y[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    uint64_t word = splitmix64_output(p.seed, (uint64_t)(k0 >> 6));
    uint32_t bits = (uint32_t)(word >> (k0 & 63));
#pragma unroll
    for (int i = 0; i < 8; ++i)
      y[i] = __uint_as_float(__float_as_uint(y[i]) ^ (((bits >> i) & 1u) << 31));
    group_fwht8(y);
    float4* dst = reinterpret_cast<float4*>(s_y + 8 * g);
    dst[0] = make_float4(y[0], y[1], y[2], y[3]);
    dst[1] = make_float4(y[4], y[5], y[6], y[7]);
  }
  if (p.nh > 8) smem_fwht_stages(s_y, E, p.nh, 8);
  else __syncthreads();
  // scale, then quantise group by group
  for (int g = threadIdx.x; g < ngroups; g += blockDim.x) {
    const float4* src = reinterpret_cast<const float4*>(s_y + 8 * g);
    float4 lo = src[0], hi = src[1];
    float u[8] = {lo.x * p.gamma, lo.y * p.gamma, lo.z * p.gamma, lo.w * p.gamma,
                  hi.x * p.gamma, hi.y * p.gamma, hi.z * p.gamma, hi.w * p.gamma};
    int64_t gg = (base >> 3) + g;
    if (p.U) {
      float4* o = reinterpret_cast<float4*>(p.U + 8 * gg);
      o[0] = make_float4(u[0], u[1], u[2], u[3]);
      o[1] = make_float4(u[4], u[5], u[6], u[7]);
    }
    if (!p.do_quantise) continue;
    bool finite = true;
#pragma unroll
    for (int i = 0; i < 8; ++i) finite &= isfinite(u[i]);
    int i1 = 0, i2 = 0;
    uint32_t mask = 0;
    if (finite) {
      int V[8], o[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      i1 = cs_nearest(u, o, V) ? member_index(cb, V, kCbSize) : -1;
      if (i1 < 0) {
        mask = 3u;  // stage 1 (and hence stage 2) need the exact path
        i1 = 0;
      } else if (p.bpw > 2) {
        // stage 2: x = (u - c1) / beta; work on y = u / beta (exact) with the
        // integer offset o = c1 / beta
        const float inv_beta = p.bpw == 3 ? 2.0f : 4.0f;
        const int omul = p.bpw == 3 ? 1 : 2;  // c1/beta = omul * v1 (v1 doubled)
        float y[8];
        const int8_t* v1 = cb.vecs + 8 * i1;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          y[i] = u[i] * inv_beta;
          o[i] = omul * (int)v1[i];
        }
        i2 = cs_nearest(y, o, V) ? member_index(cb, V, p.bpw == 3 ? 256 : kCbSize) : -1;
        if (i2 < 0) {
          mask = 2u;
          i2 = 0;
        }
      }
    }
    p.idx1[gg] = (uint16_t)i1;
    if (p.bpw == 3) reinterpret_cast<uint8_t*>(p.idx2)[gg] = (uint8_t)i2;
    if (p.bpw == 4) reinterpret_cast<uint16_t*>(p.idx2)[gg] = (uint16_t)i2;
    if (mask) push_work(p, cb, u, gg, mask);
  }
}

// --------------------------------------------------------- exact slow path --
// Sign of sum t[0..n), each t exactly representable, by a nonoverlapping
// floating-point expansion (Shewchuk, "Adaptive Precision Floating-Point
// Arithmetic and Fast Robust Geometric Predicates", 1997: Two-Sum and
// Grow-Expansion with zero elimination).  The sign of an expansion is the sign
// of its largest (last nonzero) component.
__device__ int exact_sign_sum(const double* t, int n) {
  double e[12];
  int len = 0;
  for (int k = 0; k < n; ++k) {
    double q = t[k];
    int nl = 0;
    for (int i = 0; i < len; ++i) {
      double s = __dadd_rn(q, e[i]);
      double bv = __dsub_rn(s, q);
      double av = __dsub_rn(s, bv);
      double err = __dadd_rn(__dsub_rn(q, av), __dsub_rn(e[i], bv));
      q = s;
      if (err != 0.0) e[nl++] = err;
    }
    e[nl++] = q;
    len = nl;
  }
  for (int i = len - 1; i >= 0; --i)
    if (e[i] != 0.0) return e[i] > 0.0 ? 1 : -1;
  return 0;
}

// +1 if candidate b is strictly closer to u than candidate a, -1 if a is, 0 on
// an exact tie.  Candidates are Z / den with integer Z.
__device__ int exact_cmp(const float (&u)[8], const int (&Za)[8], const int (&Zb)[8], int den) {
  double t[9];
  long long na = 0, nb = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    t[i] = __dmul_rn((double)u[i], (double)(2 * den * (Zb[i] - Za[i])));
    na += (long long)Za[i] * Za[i];
    nb += (long long)Zb[i] * Zb[i];
  }
  t[8] = (double)(na - nb);
  return exact_sign_sum(t, 9);
}

// Exact argmin of |u - (base + v_c)/den|^2 by one warp over the listed
// norm-12 points (all of squared norm 12, doubled 48) plus `extra` when >= 0;
// smallest index on ties.  On the list |base + v|^2 - 2 den <u, base + v>
// differs from -2 <den u - base, v> by a constant, so each lane ranks its
// candidates by the fp32 score <T, v>, T = den u - base, read from the
// shared-memory copy sl of the list (eight fp32 coordinates per point), and
// compares two candidates exactly whenever their scores are within tol of
// each other: every decision of the lane scan and of the warp tournament is
// then the exact one, so the winner is the exact argmin.
// Bound: t_k = fl32(T_k) within 2^-24 |T_k|; the fused chain of eight
// products with |v_k| <= 6 adds at most 8 roundings of 2^-24 6 S, S = sum
// |t_k|; a score is within 54 2^-24 S (1 + 2^-20) < 2^-18 S of <T, v>, the
// difference of two within 2^-17 S; tol = 2^-15 (S + 1) covers it.
__device__ int warp_list_argmin(const DeviceCodebook& cb, const float4* sl, const float (&u)[8],
                                const int (&base)[8], int den, int extra) {
  const int lane = threadIdx.x & 31;
  float t[8];
  float S = 0.0f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    t[k] = __fsub_rn(__fmul_rn((float)den, u[k]), (float)base[k]);
    S += fabsf(t[k]);
  }
  const float tol = 0x1p-15f * (S * 1.0001f + 1.0f);
  auto z_of = [&](int c, int (&Z)[8]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) Z[k] = base[k] + (int)cb.vecs[8 * c + k];
  };
  // true when candidate list[j] (score sj) beats list[i] (score si)
  auto beats = [&](int j, float sj, int i, float si) -> bool {
    if (i < 0) return j >= 0;
    if (j < 0) return false;
    if (sj > si + tol) return true;
    if (sj < si - tol) return false;
    const int cj = __ldg(cb.clist + j), ci = __ldg(cb.clist + i);
    int Zi[8], Zj[8];
    z_of(ci, Zi);
    z_of(cj, Zj);
    const int cmp = exact_cmp(u, Zi, Zj, den);
    return cmp > 0 || (cmp == 0 && cj < ci);
  };
  float bs = -INFINITY;
  int bi = -1;
  for (int i = lane; i < cb.clist_len; i += 32) {
    const float4 a = sl[2 * i], b = sl[2 * i + 1];
    float sc = __fmul_rn(t[0], a.x);
    sc = __fmaf_rn(t[1], a.y, sc);
    sc = __fmaf_rn(t[2], a.z, sc);
    sc = __fmaf_rn(t[3], a.w, sc);
    sc = __fmaf_rn(t[4], b.x, sc);
    sc = __fmaf_rn(t[5], b.y, sc);
    sc = __fmaf_rn(t[6], b.z, sc);
    sc = __fmaf_rn(t[7], b.w, sc);
    if (beats(i, sc, bi, bs)) {
      bi = i;
      bs = sc;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
    const float os = __shfl_xor_sync(0xffffffffu, bs, off);
    if (beats(oi, os, bi, bs)) {
      bi = oi;
      bs = os;
    }
  }
  int best = bi < 0 ? -1 : __ldg(cb.clist + bi);
  if (extra >= 0) {
    if (best < 0) {
      best = extra;
    } else {
      int Zb[8], Ze[8];
      z_of(best, Zb);
      z_of(extra, Ze);
      const int cmp = exact_cmp(u, Zb, Ze, den);
      if (cmp > 0 || (cmp == 0 && extra < best)) best = extra;
    }
  }
  return best < 0 ? 0 : best;
}

// Exact argmin of |u - (base + v_c)/den|^2 by one warp over c = 0 .. n - 1,
// smallest index on ties.  Each lane ranks its candidates by the fp32 score
// q_c - 2 <T, v_c>, q_c = |v_c|^2 (exact), T = den u - base, which differs
// from den^2 |u - (base + v_c)/den|^2 by a constant; two scores within tol
// of each other are compared exactly.  Bound: <T, v> is within 2^-18 S of
// its value (as in warp_list_argmin, S = sum |t_k|), the subtraction adds
// 2^-24 (48 + 12 S), so a score is within 2^-17 S + 2^-19 and a difference
// within 2^-16 S + 2^-18; tol = 2^-14 (S + 1).  Out of line: few items take
// it, and its eight loads in flight would crowd the registers of the list
// search beside it.
__device__ __noinline__ int warp_full_argmin(const DeviceCodebook& cb, const float (&u)[8],
                                const int (&base)[8], int den, int n) {
  const int lane = threadIdx.x & 31;
  float t[8];
  float S = 0.0f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    t[k] = __fsub_rn(__fmul_rn((float)den, u[k]), (float)base[k]);
    S += fabsf(t[k]);
  }
  const float tol = 0x1p-14f * (S * 1.0001f + 1.0f);
  auto z_of = [&](int c, int (&Z)[8]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) Z[k] = base[k] + (int)cb.vecs[8 * c + k];
  };
  // true when candidate cj (score sj) beats ci (score si)
  auto beats = [&](int cj, float sj, int ci, float si) -> bool {
    if (ci < 0) return cj >= 0;
    if (cj < 0) return false;
    if (sj < si - tol) return true;
    if (sj > si + tol) return false;
    int Zi[8], Zj[8];
    z_of(ci, Zi);
    z_of(cj, Zj);
    const int cmp = exact_cmp(u, Zi, Zj, den);
    return cmp > 0 || (cmp == 0 && cj < ci);
  };
  // eight candidates per lane and step, their loads issued together (a lone
  // warp scans up to 65536 entries: one load at a time would leave it bound
  // by the L2 latency)
  const uint2* vv = reinterpret_cast<const uint2*>(cb.vecs);
  float bs = INFINITY;
  int bc = -1;
  for (int c0 = lane; c0 < n; c0 += 32 * 8) {
    uint2 w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      w[j] = c0 + 32 * j < n ? __ldg(vv + c0 + 32 * j) : make_uint2(0u, 0u);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = c0 + 32 * j;
      if (c >= n) break;
      float v[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v[k] = (float)(int8_t)(w[j].x >> (8 * k));
        v[k + 4] = (float)(int8_t)(w[j].y >> (8 * k));
      }
      float q = 0.0f, d = 0.0f;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        q = __fmaf_rn(v[k], v[k], q);
        d = __fmaf_rn(t[k], v[k], d);
      }
      const float sc = __fsub_rn(q, 2.0f * d);
      if (beats(c, sc, bc, bs)) {
        bc = c;
        bs = sc;
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const int oc = __shfl_xor_sync(0xffffffffu, bc, off);
    const float os = __shfl_xor_sync(0xffffffffu, bs, off);
    if (beats(oc, os, bc, bs)) {
      bc = oc;
      bs = os;
    }
  }
  return bc < 0 ? 0 : bc;
}

// One warp per work item: exact brute force over the whole candidate set, or
// over the listed norm-12 points plus the item's best other candidate.  A
// stage 1 settled here sends its stage 2 back (to `out`) for the class search.
__global__ void __launch_bounds__(256, 4) k_encode_slow(const WorkItem* in, const uint32_t* in_count,
                                                     uint64_t cap, WorkItem* out,
                                                     uint32_t* out_count, int bpw,
                                                     uint16_t* idx1, void* idx2,
                                                     DeviceCodebook cb) {
  // the listed norm-12 points as fp32 coordinates (exact small integers)
  extern __shared__ float4 s_list[];
  for (int i = threadIdx.x; i < cb.clist_len; i += blockDim.x) {
    const int8_t* v = cb.vecs + 8 * __ldg(cb.clist + i);
    s_list[2 * i] = make_float4(v[0], v[1], v[2], v[3]);
    s_list[2 * i + 1] = make_float4(v[4], v[5], v[6], v[7]);
  }
  __syncthreads();
  const uint64_t n = (uint64_t)min((unsigned long long)*in_count, (unsigned long long)cap);
  const uint64_t warp = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint64_t nwarps = ((uint64_t)gridDim.x * blockDim.x) >> 5;
  const int lane = threadIdx.x & 31;
  for (uint64_t w = warp; w < n; w += nwarps) {
    const WorkItem& it = in[w];
    float u[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) u[i] = it.u[i];
    const int64_t g = it.group;
    const uint32_t mask = it.mask;
    if (mask & kWorkStage1) {
      int zero[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      const int i1 = (mask & kWorkStage1List)
                         ? warp_list_argmin(cb, s_list, u, zero, 2, (int)it.cand)
                         : warp_full_argmin(cb, u, zero, 2, kCbSize);
      if (lane == 0) {
        idx1[g] = (uint16_t)i1;
        if (bpw > 2) {
          const uint32_t slot = out ? atomicAdd(out_count, 1u) : 0xFFFFFFFFu;
          if (slot < cap) {
            WorkItem& o = out[slot];
#pragma unroll
            for (int i = 0; i < 8; ++i) o.u[i] = u[i];
            o.group = g;
            o.mask = kWorkStage2;
            o.cand = 0u;
          } else {
            atomicOr(cb.status, kDevWorklistOverflow);
          }
        }
      }
      continue;
    }
    if (bpw > 2 && (mask & kWorkStage2)) {
      const int i1 = idx1[g];
      const int m = bpw == 3 ? 4 : 8;
      int base[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) base[i] = (m / 2) * (int)cb.vecs[8 * i1 + i];
      const int i2 = (mask & kWorkStage2List)
                         ? warp_list_argmin(cb, s_list, u, base, m, (int)it.cand)
                         : warp_full_argmin(cb, u, base, m, bpw == 3 ? 256 : kCbSize);
      if (lane == 0) {
        if (bpw == 3) reinterpret_cast<uint8_t*>(idx2)[g] = (uint8_t)i2;
        else reinterpret_cast<uint16_t*>(idx2)[g] = (uint16_t)i2;
      }
    }
  }
}

// ------------------------------------------------------------------ host --
int encode_elems_per_cta(int nh) { return nh < 2048 ? 2048 : nh; }

cudaError_t launch_encode(const DeviceCodebook& cb, const float* W, int64_t N, int64_t K, int bpw,
                          uint64_t seed, float gamma, uint16_t* idx1, void* idx2,
                          WorkItem* work, uint32_t* work_count, uint64_t work_cap, float* U,
                          int do_quantise, int sm_count, cudaStream_t st, int64_t nh) {
  EncodeParams p;
  p.W = W;
  p.N = N;
  p.K = K;
  p.nh = (int)resolve_nh(K, nh);
  p.elems_per_cta = encode_elems_per_cta(p.nh);
  p.bpw = bpw;
  p.seed = seed;
  p.gamma = gamma;
  p.idx1 = idx1;
  p.idx2 = idx2;
  p.work = work;
  p.work_count = work_count;
  p.work_cap = work_cap;
  p.U = U;
  p.do_quantise = do_quantise;
  const int64_t total = N * K;
  const int64_t ctas = (total + p.elems_per_cta - 1) / p.elems_per_cta;
  const size_t smem = (size_t)p.elems_per_cta * sizeof(float);
  cudaError_t e = ensure_smem_limit(k_encode, kMaxDynSmem);
  if (e != cudaSuccess) return e;
  if (do_quantise) {
    e = cudaMemsetAsync(work_count, 0, 4 * sizeof(uint32_t), st);
    if (e != cudaSuccess) return e;
  }
  k_encode<<<(unsigned)ctas, 256, smem, st>>>(p, cb);
  e = cudaGetLastError();
  if (e != cudaSuccess || !do_quantise) return e;
  // undecided groups: class search (thread per group), then the warp brute
  // force for what stays open; stage 2 of a group whose stage 1 needed the
  // brute force takes a second round
  WorkItem* r1 = work;
  WorkItem* r2 = work + work_cap;
  const size_t slow_smem = (size_t)(cb.clist_len > 0 ? cb.clist_len : 0) * 2 * sizeof(float4);
  if ((e = ensure_smem_limit(k_encode_slow, kMaxDynSmem, true)) != cudaSuccess) return e;
  e = launch_encode_leader(cb, r1, work_count, work_cap, r2, work_count + 1, bpw, idx1, idx2,
                           sm_count, st);
  if (e != cudaSuccess) return e;
  k_encode_slow<<<sm_count * 4, 256, slow_smem, st>>>(r2, work_count + 1, work_cap, r1, work_count + 2,
                                              bpw, idx1, idx2, cb);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (bpw == 2) return cudaSuccess;
  e = launch_encode_leader(cb, r1, work_count + 2, work_cap, r2, work_count + 3, bpw, idx1, idx2,
                           sm_count, st);
  if (e != cudaSuccess) return e;
  k_encode_slow<<<sm_count * 4, 256, slow_smem, st>>>(r2, work_count + 3, work_cap, nullptr, nullptr, bpw,
                                              idx1, idx2, cb);
  return cudaGetLastError();
}

}  // namespace e8
