// Exact nearest codebook point for groups that the Conway-Sloane fast path did
// not settle ("glq 0.1.1", "How it works", item 1: nearest of 65536 E8 points;
// Conway & Sloane, "Sphere Packings, Lattices and Groups": E8 shells).
//
// Every full shell of E8 (squared norm 2..10) is a union of classes: vectors
// with a fixed multiset of absolute coordinates (the class leader), all
// permutations, and all sign patterns (integer vectors) or the sign patterns
// with a fixed parity of the number of minus signs (half-integer vectors, whose
// coordinate sum must stay even).  Over one class the inner product with a
// target T is largest when the leader's values, in decreasing order, sit on
// the coordinates of T in decreasing order of |T_i|, with the signs of T; under
// the parity rule, if the signs of T have the wrong parity, the sign on the
// smallest |T_i| flips.  So one sort of |T| gives the best point of every class,
// and the nearest codebook point is the best of the classes' best points.
//
// The codebook keeps only 8655 of the 60480 points of squared norm 12: every
// kept point has x1 = 0, and they are, exactly, all such points with x2 = 0
// (class search over coordinates 3..8), all with |x2| = 1 (same), and a
// lexicographic prefix of those with |x2| = 2.  For the last set the best point
// of the two classes containing it is taken when it is a codebook member;
// otherwise the group goes to the brute force over that set.
//
// Distances are compared through scores |V|^2 - 2 <T, V> (doubled coordinates)
// in binary64; any two scores closer than a bound on their rounding error, and
// any tie in |T_i| (or a zero coordinate), send the group to the exact brute
// force instead.  Results are therefore exact: the unique nearest point, or the
// brute force's smallest-index rule when distances tie.
#include "e8_common.cuh"
#include "e8_codebook.cuh"
#include "e8_internal.h"

namespace e8 {

namespace ls {
// Class leaders in doubled coordinates (decreasing), parity type and norm.
// odd = 1: half-integer vectors; need_odd: the number of minus signs must be odd.
struct Cls8 {
  int8_t l[8];
  int8_t odd, need_odd, norm;
};
struct Cls6 {
  int8_t l[6];
  int8_t norm;
};
constexpr int kFull = 18;
__constant__ Cls8 kFullCls[kFull] = {
    {{1, 1, 1, 1, 1, 1, 1, 1}, 1, 0, 8},  {{2, 2, 0, 0, 0, 0, 0, 0}, 0, 0, 8},
    {{2, 2, 2, 2, 0, 0, 0, 0}, 0, 0, 16}, {{3, 1, 1, 1, 1, 1, 1, 1}, 1, 1, 16},
    {{4, 0, 0, 0, 0, 0, 0, 0}, 0, 0, 16}, {{2, 2, 2, 2, 2, 2, 0, 0}, 0, 0, 24},
    {{3, 3, 1, 1, 1, 1, 1, 1}, 1, 0, 24}, {{4, 2, 2, 0, 0, 0, 0, 0}, 0, 0, 24},
    {{2, 2, 2, 2, 2, 2, 2, 2}, 0, 0, 32}, {{3, 3, 3, 1, 1, 1, 1, 1}, 1, 1, 32},
    {{4, 2, 2, 2, 2, 0, 0, 0}, 0, 0, 32}, {{4, 4, 0, 0, 0, 0, 0, 0}, 0, 0, 32},
    {{5, 1, 1, 1, 1, 1, 1, 1}, 1, 0, 32}, {{3, 3, 3, 3, 1, 1, 1, 1}, 1, 0, 40},
    {{4, 2, 2, 2, 2, 2, 2, 0}, 0, 0, 40}, {{4, 4, 2, 2, 0, 0, 0, 0}, 0, 0, 40},
    {{5, 3, 1, 1, 1, 1, 1, 1}, 1, 1, 40}, {{6, 2, 0, 0, 0, 0, 0, 0}, 0, 0, 40}};
constexpr int kS12 = 5;
__constant__ Cls8 kS12Cls[kS12] = {{{4, 4, 2, 2, 2, 2, 0, 0}, 0, 0, 48},
                                   {{4, 4, 4, 0, 0, 0, 0, 0}, 0, 0, 48},
                                   {{6, 2, 2, 2, 0, 0, 0, 0}, 0, 0, 48},
                                   {{3, 3, 3, 3, 3, 1, 1, 1}, 1, 1, 48},
                                   {{5, 3, 3, 1, 1, 1, 1, 1}, 1, 0, 48}};
// x1 = x2 = 0: coordinates 3..8 of squared norm 12 (doubled 48), even sum
constexpr int kA = 3;
__constant__ Cls6 kACls[kA] = {{{4, 4, 2, 2, 2, 2}, 48}, {{4, 4, 4, 0, 0, 0}, 48},
                               {{6, 2, 2, 2, 0, 0}, 48}};
// x1 = 0, |x2| = 1: coordinates 3..8 of squared norm 11 (doubled 44), odd sum
constexpr int kB = 2;
__constant__ Cls6 kBCls[kB] = {{{4, 4, 2, 2, 2, 0}, 44}, {{6, 2, 2, 0, 0, 0}, 44}};
// x1 = 0, |x2| = 2: coordinates 3..8 of squared norm 8 (doubled 32), even sum
constexpr int kC = 2;
__constant__ Cls6 kCCls[kC] = {{{4, 2, 2, 2, 2, 0}, 32}, {{4, 4, 0, 0, 0, 0}, 32}};
}  // namespace ls

// Sorts |t| decreasingly: b = sorted magnitudes, p = their coordinates.
// Returns false on a tie or a zero (the class optimum would not be unique).
template <int N>
__device__ __forceinline__ void cmpx(double (&b)[N], int (&p)[N], int i, int j) {
  if (b[i] < b[j]) {
    const double tb = b[i];
    b[i] = b[j];
    b[j] = tb;
    const int tp = p[i];
    p[i] = p[j];
    p[j] = tp;
  }
}
__device__ __forceinline__ bool sort8(const double (&t)[8], double (&b)[8], int (&p)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    b[i] = fabs(t[i]);
    p[i] = i;
  }
  cmpx(b, p, 0, 1); cmpx(b, p, 2, 3); cmpx(b, p, 4, 5); cmpx(b, p, 6, 7);
  cmpx(b, p, 0, 2); cmpx(b, p, 1, 3); cmpx(b, p, 4, 6); cmpx(b, p, 5, 7);
  cmpx(b, p, 1, 2); cmpx(b, p, 5, 6); cmpx(b, p, 0, 4); cmpx(b, p, 3, 7);
  cmpx(b, p, 1, 5); cmpx(b, p, 2, 6); cmpx(b, p, 1, 4); cmpx(b, p, 3, 6);
  cmpx(b, p, 2, 4); cmpx(b, p, 3, 5); cmpx(b, p, 3, 4);
  bool ok = b[7] > 0.0;
#pragma unroll
  for (int i = 0; i < 7; ++i) ok = ok && (b[i] > b[i + 1]);
  return ok;
}
// Sorts |t[2..7]| decreasingly (positions returned as 2..7).
__device__ __forceinline__ void sort6_tail(const double (&t)[8], double (&b)[6], int (&p)[6]) {
#pragma unroll
  for (int i = 0; i < 6; ++i) {
    b[i] = fabs(t[i + 2]);
    p[i] = i + 2;
  }
  cmpx(b, p, 1, 2); cmpx(b, p, 4, 5); cmpx(b, p, 0, 2); cmpx(b, p, 3, 5);
  cmpx(b, p, 0, 1); cmpx(b, p, 3, 4); cmpx(b, p, 2, 5); cmpx(b, p, 0, 3);
  cmpx(b, p, 1, 4); cmpx(b, p, 2, 4); cmpx(b, p, 1, 3); cmpx(b, p, 2, 3);
}

__device__ __forceinline__ int sgn_of(double x) { return x < 0.0 ? -1 : 1; }

// Best point of an 8-dimensional class: returns max <T, V>, fills V.
__device__ __forceinline__ double class8_best(const ls::Cls8& c, const double (&t)[8],
                                              const double (&b)[8], const int (&p)[8],
                                              int nneg, int (&V)[8]) {
  double s = 0.0;
#pragma unroll
  for (int k = 0; k < 8; ++k) s = __dadd_rn(s, __dmul_rn((double)c.l[k], b[k]));
#pragma unroll
  for (int k = 0; k < 8; ++k) V[p[k]] = sgn_of(t[p[k]]) * (int)c.l[k];
  if (c.odd && ((nneg & 1) != c.need_odd)) {
    s = __dsub_rn(s, __dmul_rn(2.0 * (double)c.l[7], b[7]));
    V[p[7]] = -V[p[7]];
  }
  return s;
}
__device__ __forceinline__ double class8_score(const ls::Cls8& c, const double (&b)[8], int nneg) {
  double s = 0.0;
#pragma unroll
  for (int k = 0; k < 8; ++k) s = __dadd_rn(s, __dmul_rn((double)c.l[k], b[k]));
  if (c.odd && ((nneg & 1) != c.need_odd)) s = __dsub_rn(s, __dmul_rn(2.0 * (double)c.l[7], b[7]));
  return __dsub_rn((double)c.norm, 2.0 * s);
}
__device__ __forceinline__ double class6_dot(const ls::Cls6& c, const double (&b)[6]) {
  double s = 0.0;
#pragma unroll
  for (int k = 0; k < 6; ++k) s = __dadd_rn(s, __dmul_rn((double)c.l[k], b[k]));
  return s;
}

// Tracks the best valid candidate and the closest other score.
struct Best {
  double score, second;
  int idx;
  __device__ void init() {
    score = INFINITY;
    second = INFINITY;
    idx = -1;
  }
  // a valid candidate (codebook index known)
  __device__ void offer(double s, int i) {
    if (s < score) {
      second = fmin(second, score);
      score = s;
      idx = i;
    } else {
      second = fmin(second, s);
    }
  }
  // a score that only competes in the margin test
  __device__ void shadow(double s) { second = fmin(second, s); }
};

enum { kLsOk = 0, kLsNeedC = 1, kLsFallback = 2 };

// The tables the class search reads, passed by value so that the searches
// below can stay out of line: one copy of their code serves both stages and
// every call site (the kernel is bound by instruction fetch and divergence
// when each call site inlines its own copy).
struct LsTabs {
  const uint32_t* hkeys;
  const uint32_t* hvals;
  const int8_t* vecs;
};

__device__ __noinline__ int ls_rank(const LsTabs& tb, const int (&v)[8]) {
  return rank_vector(tb.hkeys, tb.hvals, v);
}

// Nearest point of the whole codebook to T (doubled coordinates, binary64,
// exactly the target).  kLsOk: *idx is the answer.  kLsNeedC: the answer is
// *idx unless a point of the x1 = 0, |x2| = 2 part of the norm-12 shell is
// nearer.  kLsFallback: undecided.
__device__ __noinline__ int leader_search(const LsTabs tb, const double (&t)[8], int* idx) {
  using namespace ls;
  double b[8];
  int p[8];
  if (!sort8(t, b, p)) return kLsFallback;
  int nneg = 0;
  double sum_abs = 0.0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    nneg += t[i] < 0.0 ? 1 : 0;
    sum_abs += b[i];
  }
  Best best;
  best.init();
  best.offer(0.0, 0);  // origin
  int bestcls = -1;
  double bscore = INFINITY;
  for (int c = 0; c < kFull; ++c) {
    const double s = class8_score(kFullCls[c], b, nneg);
    if (s < bscore) {
      if (bscore < INFINITY) best.shadow(bscore);
      bscore = s;
      bestcls = c;
    } else {
      best.shadow(s);
    }
  }
  {
    int V[8];
    class8_best(kFullCls[bestcls], t, b, p, nneg, V);
    const int r = ls_rank(tb, V);
    if (r < 0) return kLsFallback;  // full shells are always members
    best.offer(bscore, r);
  }
  // norm 12: the best of the whole shell, when it is a member
  int c12 = 0;
  double s12 = INFINITY, s12b = INFINITY;
  for (int c = 0; c < kS12; ++c) {
    const double s = class8_score(kS12Cls[c], b, nneg);
    if (s < s12) {
      s12b = s12;
      s12 = s;
      c12 = c;
    } else {
      s12b = fmin(s12b, s);
    }
  }
  bool need_c = false;
  int V[8];
  class8_best(kS12Cls[c12], t, b, p, nneg, V);
  int r12 = ls_rank(tb, V);
  if (r12 >= 0) {
    best.offer(s12, r12);
    best.shadow(s12b);
  } else {
    // kept part of the shell: x1 = 0 with x2 = 0, |x2| = 1, |x2| = 2
    double b6[6];
    int p6[6];
    sort6_tail(t, b6, p6);
    const double a1 = fabs(t[1]);
    const int s1 = sgn_of(t[1]);
    for (int part = 0; part < 3; ++part) {
      const int n = part == 0 ? kA : (part == 1 ? kB : kC);
      int cb6 = 0;
      double sb = INFINITY, sb2 = INFINITY;
      for (int c = 0; c < n; ++c) {
        const Cls6& cl = part == 0 ? kACls[c] : (part == 1 ? kBCls[c] : kCCls[c]);
        const double x2 = part == 0 ? 0.0 : (part == 1 ? 2.0 * a1 : 4.0 * a1);
        const double s = __dsub_rn(48.0, 2.0 * __dadd_rn(x2, class6_dot(cl, b6)));
        if (s < sb) {
          sb2 = sb;
          sb = s;
          cb6 = c;
        } else {
          sb2 = fmin(sb2, s);
        }
      }
      const Cls6& cl = part == 0 ? kACls[cb6] : (part == 1 ? kBCls[cb6] : kCCls[cb6]);
      int W[8];
      W[0] = 0;
      W[1] = part == 0 ? 0 : s1 * (part == 1 ? 2 : 4);
#pragma unroll
      for (int k = 0; k < 6; ++k) W[p6[k]] = sgn_of(t[p6[k]]) * (int)cl.l[k];
      const int r = ls_rank(tb, W);
      if (part < 2) {
        if (r < 0) return kLsFallback;  // these parts are kept whole
        best.offer(sb, r);
        best.shadow(sb2);
      } else if (r >= 0) {
        best.offer(sb, r);
        best.shadow(sb2);
      } else {
        need_c = true;
      }
    }
  }
  // rounding bound of the scores: products are exact, sums of at most ten
  // terms of magnitude <= 6 sum |T| + 48
  const double tol = 0x1p-40 * (64.0 + 16.0 * sum_abs);
  if (!(best.second - best.score > tol)) return kLsFallback;
  *idx = best.idx;
  return need_c ? kLsNeedC : kLsOk;
}

// Nearest of the first 256 codebook entries (origin, the 240 points of norm 2,
// 15 points of norm 4) to T (doubled coordinates).
__device__ __noinline__ int c28_search(const LsTabs tb, const double (&t)[8], int* idx) {
  using namespace ls;
  double b[8];
  int p[8];
  if (!sort8(t, b, p)) return kLsFallback;
  int nneg = 0;
  double sum_abs = 0.0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    nneg += t[i] < 0.0 ? 1 : 0;
    sum_abs += b[i];
  }
  Best best;
  best.init();
  best.offer(0.0, 0);
  for (int c = 0; c < 2; ++c) {  // the two classes of norm 2 (doubled 8)
    int V[8];
    const double s = class8_best(kFullCls[c], t, b, p, nneg, V);
    const int r = ls_rank(tb, V);
    if (r < 0 || r >= 241) return kLsFallback;
    best.offer(__dsub_rn(8.0, 2.0 * s), r);
  }
  for (int i = 241; i < 256; ++i) {
    const int8_t* v = tb.vecs + 8 * i;
    double s = 0.0;
#pragma unroll
    for (int k = 0; k < 8; ++k) s = __dadd_rn(s, __dmul_rn((double)v[k], t[k]));
    best.offer(__dsub_rn(16.0, 2.0 * s), i);
  }
  const double tol = 0x1p-40 * (64.0 + 16.0 * sum_abs);
  if (!(best.second - best.score > tol)) return kLsFallback;
  *idx = best.idx;
  return kLsOk;
}

__device__ __forceinline__ void push_item(WorkItem* list, uint32_t* count, uint64_t cap,
                                          uint32_t* status, const float (&u)[8], int64_t g,
                                          uint32_t mask, uint32_t cand) {
  const uint32_t slot = atomicAdd(count, 1u);
  if (slot >= cap) {
    atomicOr(status, kDevWorklistOverflow);
    return;
  }
  WorkItem& w = list[slot];
#pragma unroll
  for (int i = 0; i < 8; ++i) w.u[i] = u[i];
  w.group = g;
  w.mask = mask;
  w.cand = cand;
}

// One thread per work item: class search for the undecided stages; what stays
// undecided goes to `out` for the warp brute force.  Both stages go through
// one call site of the (out-of-line) search.  Four blocks per SM (64
// registers): the search is latency-bound and gains more from warps in
// flight than it loses to the few spilled values.
__global__ void __launch_bounds__(256, 4) k_encode_leader(const WorkItem* in, const uint32_t* in_count,
                                                       uint64_t cap, WorkItem* out,
                                                       uint32_t* out_count, int bpw,
                                                       uint16_t* idx1, void* idx2,
                                                       DeviceCodebook cb) {
  const LsTabs tb{cb.hkeys, cb.hvals, cb.vecs};
  const uint64_t n = (uint64_t)min((unsigned long long)*in_count, (unsigned long long)cap);
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t w = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; w < n; w += stride) {
    const WorkItem& it = in[w];
    float u[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) u[i] = it.u[i];
    const int64_t g = it.group;
    const uint32_t mask = it.mask;
    if (!(mask & kWorkStage1) && (bpw == 2 || !(mask & kWorkStage2))) continue;
    // stage 1 target 2u; stage 2 target (2u - V1) / beta (doubled coordinates)
    int stage = (mask & kWorkStage1) ? 1 : 2;
    int i1 = stage == 1 ? -1 : (int)idx1[g];
    for (;;) {
      double t[8];
      if (stage == 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) t[i] = 2.0 * (double)u[i];
      } else {
        const int8_t* v1 = cb.vecs + 8 * i1;
        const double k = bpw == 3 ? 2.0 : 4.0;
#pragma unroll
        for (int i = 0; i < 8; ++i) t[i] = k * __dsub_rn(2.0 * (double)u[i], (double)v1[i]);
      }
      int r = 0;
      const int st = (stage == 2 && bpw == 3) ? c28_search(tb, t, &r) : leader_search(tb, t, &r);
      if (st != kLsOk) {
        uint32_t m;
        if (stage == 1)
          m = kWorkStage1 | (bpw > 2 ? kWorkStage2 : 0u) | (st == kLsNeedC ? kWorkStage1List : 0u);
        else
          m = kWorkStage2 | (st == kLsNeedC ? kWorkStage2List : 0u);
        push_item(out, out_count, cap, cb.status, u, g, m, (uint32_t)r);
        break;
      }
      if (stage == 1) {
        idx1[g] = (uint16_t)r;
        if (bpw == 2) break;
        i1 = r;
        stage = 2;
        continue;
      }
      if (bpw == 3) reinterpret_cast<uint8_t*>(idx2)[g] = (uint8_t)r;
      else reinterpret_cast<uint16_t*>(idx2)[g] = (uint16_t)r;
      break;
    }
  }
}

cudaError_t launch_encode_leader(const DeviceCodebook& cb, const WorkItem* in,
                                 const uint32_t* in_count, uint64_t cap, WorkItem* out,
                                 uint32_t* out_count, int bpw, uint16_t* idx1, void* idx2,
                                 int sm_count, cudaStream_t st) {
  k_encode_leader<<<sm_count * 8, 256, 0, st>>>(in, in_count, cap, out, out_count, bpw, idx1,
                                                idx2, cb);
  return cudaGetLastError();
}

}  // namespace e8
