/*
 * E8 lattice-codebook weight quantisation -- plain CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  This file defines, slowly and literally, what the
 * GPU library computes, so that the GPU results can be checked against it.
 * Nothing in the product path may load it: only tests/, the smoke check in
 * __graft_entry__.py and the cpu_baseline / --impl reference legs of bench.py
 * call it.  It shares no code, header, table or constant with the CUDA path.
 *
 * What it follows (page "glq 0.1.1" on PyPI):
 *   - "How it works", item 1: a codebook of 65536 vectors taken from the first
 *     7 shells of the E8 lattice; one 16-bit index per group of 8 weights
 *     (2 bits per weight); for 3 and 4 bits per weight a second-stage residual
 *     codebook adds 8 or 16 bits per group.
 *   - "How it works", item 2: a randomized Hadamard transform -- random sign
 *     flips followed by a fast Walsh-Hadamard transform -- is applied to the
 *     weights, after which each group is mapped to its Euclidean nearest
 *     codebook vector.
 *   - "Bit widths" table and "Results" note: one global scale per layer, no
 *     per-group scale, so the effective rate equals the nominal rate.
 *   - "Acknowledgments": E8 geometry per Conway & Sloane (the lattice is the set
 *     of vectors whose coordinates are all integers or all half-integers and
 *     whose coordinate sum is even).
 *
 * Readings where the page is silent:
 *   - the 7 shells are the squared norms 0,2,...,12 (the origin counts);
 *   - canonical order: origin first, then shells by increasing norm; inside a
 *     shell the vectors whose first nonzero coordinate is positive are sorted
 *     lexicographically ascending on doubled coordinates and each is emitted as
 *     p then -p; the list is cut at 65536 entries;
 *   - residual codebook: the first 256 entries at scale 1/2 (3 bpw) or the whole
 *     codebook at scale 1/4 (4 bpw), greedy second stage after the first;
 *   - exact Euclidean distances on the fp32 transformed weights, ties to the
 *     smallest index;
 *   - Hadamard block = largest power of two dividing K (the *_nh entry points
 *     take any power-of-two block dividing K instead); sign vector from a
 *     SplitMix64 stream; forward transform in fp32 with stages h = 1,2,4,...
 *     and butterfly (a+b, a-b); decoded weight = bf16_rne(d * fl32(t * alpha)).
 *
 * Every floating point operation here is IEEE binary32/binary64 with round to
 * nearest even; build with -ffp-contract=off and without -ffast-math.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_CB_SIZE 65536
#define ORC_MAX_NH 32768

/* ------------------------------------------------------------------------- */
/* Codebook: the E8 points of squared norm <= 12 in canonical order.          */
/* Coordinates are stored doubled (2x), so every entry is an int8 in [-6,6].  */
/* ------------------------------------------------------------------------- */

typedef struct { int8_t v[8]; int norm4; } orc_vec;   /* norm4 = sum (2x)^2 = 4|x|^2 */

static int orc_lex_cmp(const void* pa, const void* pb) {
  const orc_vec* a = (const orc_vec*)pa;
  const orc_vec* b = (const orc_vec*)pb;
  if (a->norm4 != b->norm4) return a->norm4 < b->norm4 ? -1 : 1;
  for (int i = 0; i < 8; ++i)
    if (a->v[i] != b->v[i]) return a->v[i] < b->v[i] ? -1 : 1;
  return 0;
}

static int orc_first_nonzero_positive(const int8_t* v) {
  for (int i = 0; i < 8; ++i) {
    if (v[i] > 0) return 1;
    if (v[i] < 0) return 0;
  }
  return 0; /* the origin */
}

/* Fills out[65536*8] with doubled coordinates.  Returns the number of E8
 * points of squared norm <= 12 that were found (117361), or -1 on failure. */
int orc_codebook(int8_t* out) {
  /* Every E8 point with |x|^2 <= 12 has doubled coordinates either all even in
   * [-6,6] or all odd in [-5,5]; enumerate both boxes and keep the lattice
   * points (doubled coordinate sum divisible by 4) inside the ball. */
  const int n_even = 7, n_odd = 6;
  int64_t cap = 200000;
  orc_vec* pts = (orc_vec*)malloc(sizeof(orc_vec) * cap);
  if (!pts) return -1;
  int64_t np = 0;
  for (int coset = 0; coset < 2; ++coset) {
    int base = coset == 0 ? -6 : -5, nv = coset == 0 ? n_even : n_odd;
    int64_t total = 1;
    for (int i = 0; i < 8; ++i) total *= nv;
    for (int64_t c = 0; c < total; ++c) {
      int64_t r = c;
      orc_vec p;
      int sum = 0, n4 = 0;
      for (int i = 7; i >= 0; --i) {
        int d = (int)(r % nv); r /= nv;
        int x = base + 2 * d;
        p.v[i] = (int8_t)x;
        sum += x; n4 += x * x;
      }
      if (n4 > 48) continue;
      if (((sum % 4) + 4) % 4 != 0) continue;
      p.norm4 = n4;
      if (np >= cap) { free(pts); return -1; }
      pts[np++] = p;
    }
  }
  /* keep the origin and the positive representatives, sort by (shell, lex) */
  int64_t nrep = 0;
  orc_vec* reps = (orc_vec*)malloc(sizeof(orc_vec) * np);
  if (!reps) { free(pts); return -1; }
  for (int64_t i = 0; i < np; ++i)
    if (pts[i].norm4 == 0 || orc_first_nonzero_positive(pts[i].v)) reps[nrep++] = pts[i];
  qsort(reps, (size_t)nrep, sizeof(orc_vec), orc_lex_cmp);
  /* emit: origin, then p, -p for every positive representative, cut at 65536 */
  int64_t k = 0;
  for (int64_t i = 0; i < nrep && k < ORC_CB_SIZE; ++i) {
    if (reps[i].norm4 == 0) {
      memset(out + 8 * k, 0, 8); ++k;
      continue;
    }
    memcpy(out + 8 * k, reps[i].v, 8); ++k;
    if (k < ORC_CB_SIZE) {
      for (int j = 0; j < 8; ++j) out[8 * k + j] = (int8_t)(-reps[i].v[j]);
      ++k;
    }
  }
  free(reps); free(pts);
  if (k != ORC_CB_SIZE) return -1;
  return (int)np;
}

/* ------------------------------------------------------------------------- */
/* Randomized Hadamard transform pieces.                                      */
/* ------------------------------------------------------------------------- */

/* Largest power of two dividing K (the Hadamard block).  0 if K is not a
 * positive multiple of 8 or the block would exceed ORC_MAX_NH. */
int64_t orc_hadamard_block(int64_t K) {
  if (K <= 0 || (K % 8) != 0) return 0;
  int64_t n = 1;
  while ((K % (n * 2)) == 0) n *= 2;
  if (n > ORC_MAX_NH) return 0;
  return n;
}

/* SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): state advances by the golden
 * gamma, output is the state passed through the variant-13 mixer. */
static uint64_t orc_splitmix64(uint64_t* state) {
  uint64_t z = (*state += 0x9E3779B97F4A7C15ULL);
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Column sign vector: output word j of the stream seeded with rht_seed gives
 * the signs of columns 64j..64j+63, bit b set meaning column 64j+b is negated. */
void orc_signs(uint64_t rht_seed, int64_t K, int8_t* d) {
  uint64_t st = rht_seed, word = 0;
  for (int64_t k = 0; k < K; ++k) {
    if ((k & 63) == 0) word = orc_splitmix64(&st);
    d[k] = ((word >> (k & 63)) & 1ULL) ? (int8_t)-1 : (int8_t)1;
  }
}

/* In-place fp32 Walsh-Hadamard transform of length n, stages h = 1,2,4,...,
 * butterfly (a, b) -> (a + b, a - b), a at the lower index. */
static void orc_fwht_f32(float* y, int64_t n) {
  for (int64_t h = 1; h < n; h *= 2)
    for (int64_t i = 0; i < n; i += 2 * h)
      for (int64_t j = i; j < i + h; ++j) {
        float a = y[j], b = y[j + h];
        y[j] = a + b;
        y[j + h] = a - b;
      }
}

/* Same transform on integers (exact, so its order does not matter). */
static void orc_fwht_i64(int64_t* y, int64_t n) {
  for (int64_t h = 1; h < n; h *= 2)
    for (int64_t i = 0; i < n; i += 2 * h)
      for (int64_t j = i; j < i + h; ++j) {
        int64_t a = y[j], b = y[j + h];
        y[j] = a + b;
        y[j + h] = a - b;
      }
}

/* gamma = fl32(1 / (s * sqrt(n_h))), computed in binary64 then rounded. */
float orc_gamma(float scale, int64_t nh) {
  return (float)(1.0 / ((double)scale * sqrt((double)nh)));
}

/* alpha = fl32(s / (m * sqrt(n_h))), m = 2, 4, 8 for 2, 3, 4 bits per weight. */
float orc_alpha(float scale, int64_t nh, int bpw) {
  int m = bpw == 2 ? 2 : (bpw == 3 ? 4 : 8);
  return (float)((double)scale / ((double)m * sqrt((double)nh)));
}

/* The block size is left open by the pages (glq page, "How it works", item 2:
 * a randomized Hadamard transform on the input dimension).  The default block
 * is orc_hadamard_block(K); the *_nh entry points take any power of two n_h,
 * 8 <= n_h <= ORC_MAX_NH, that divides K (the small-block storage variant uses
 * n_h = 128 or 256).  Everything else -- signs, normalisation, rounding -- is
 * the same for every block size. */
int orc_valid_block(int64_t K, int64_t nh) {
  if (K <= 0 || (K % 8) != 0 || nh < 8 || nh > ORC_MAX_NH || (nh & (nh - 1)) != 0) return 0;
  return (K % nh) == 0;
}

/* Forward transform of every row: u = fl32(FWHT(D w) * gamma), per block of nh. */
int orc_rht_forward_nh(const float* W, int64_t N, int64_t K, int64_t nh, uint64_t rht_seed,
                       float scale, float* U, int nthreads) {
  if (!orc_valid_block(K, nh)) return -1;
  int8_t* d = (int8_t*)malloc((size_t)K);
  if (!d) return -1;
  orc_signs(rht_seed, K, d);
  float g = orc_gamma(scale, nh);
#ifdef _OPENMP
#pragma omp parallel for num_threads(nthreads) schedule(static)
#endif
  for (int64_t r = 0; r < N; ++r) {
    float* y = U + r * K;
    const float* w = W + r * K;
    for (int64_t k = 0; k < K; ++k) y[k] = d[k] < 0 ? -w[k] : w[k];
    for (int64_t b = 0; b < K; b += nh) orc_fwht_f32(y + b, nh);
    for (int64_t k = 0; k < K; ++k) y[k] = y[k] * g;
  }
  (void)nthreads;
  free(d);
  return 0;
}

int orc_rht_forward(const float* W, int64_t N, int64_t K, uint64_t rht_seed,
                    float scale, float* U, int nthreads) {
  int64_t nh = orc_hadamard_block(K);
  if (nh == 0) return -1;
  return orc_rht_forward_nh(W, N, K, nh, rht_seed, scale, U, nthreads);
}

/* ------------------------------------------------------------------------- */
/* Exact distance comparison.                                                 */
/*                                                                            */
/* Candidate points are Z/den with Z an integer 8-vector.  For two candidates */
/*   |u - Za/den|^2 - |u - Zb/den|^2                                          */
/*     = ( 2 den <u, Zb - Za> + |Za|^2 - |Zb|^2 ) / den^2.                    */
/* Each product 2*den*u_i*(Zb-Za)_i is exact in binary64 (24-bit significand  */
/* times an integer below 2^11); the sum is taken exactly in a long           */
/* fixed-point accumulator whose unit is 2^-160 (every fp32 value is a        */
/* multiple of 2^-149) and whose top lies above 2^160.                        */
/* ------------------------------------------------------------------------- */

#define ORC_ACC_LIMBS 6      /* 384 bits, two's complement, little endian */
#define ORC_ACC_LSB (-160)   /* exponent of bit 0 */

typedef struct { uint64_t w[ORC_ACC_LIMBS]; } orc_acc;

static void orc_acc_add_shifted(orc_acc* a, uint64_t mag, int shift, int neg) {
  /* adds (neg ? -1 : 1) * mag * 2^shift, shift >= 0 */
  uint64_t t[ORC_ACC_LIMBS];
  memset(t, 0, sizeof t);
  int limb = shift / 64, off = shift % 64;
  if (limb < ORC_ACC_LIMBS) t[limb] = mag << off;
  if (off != 0 && limb + 1 < ORC_ACC_LIMBS) t[limb + 1] = mag >> (64 - off);
  if (neg) { /* two's complement negate t */
    int carry = 1;
    for (int i = 0; i < ORC_ACC_LIMBS; ++i) {
      uint64_t x = ~t[i];
      uint64_t s = x + (uint64_t)carry;
      carry = (carry && s == 0) ? 1 : 0;
      t[i] = s;
    }
  }
  unsigned __int128 c = 0;
  for (int i = 0; i < ORC_ACC_LIMBS; ++i) {
    c += (unsigned __int128)a->w[i] + t[i];
    a->w[i] = (uint64_t)c;
    c >>= 64;
  }
}

static void orc_acc_add_double(orc_acc* a, double x) {
  if (x == 0.0) return;
  int e;
  double f = frexp(fabs(x), &e);           /* |x| = f 2^e, f in [0.5, 1) */
  uint64_t mag = (uint64_t)ldexp(f, 53);   /* exact 53-bit integer */
  int shift = e - 53 - ORC_ACC_LSB;        /* bit position of mag's LSB */
  /* inputs here are multiples of 2^-149 below 2^150, so 0 <= shift and the
   * value fits; strip trailing zero bits if shift would be negative */
  while (shift < 0) { mag >>= 1; ++shift; }
  orc_acc_add_shifted(a, mag, shift, x < 0);
}

static int orc_acc_sign(const orc_acc* a) {
  if ((int64_t)a->w[ORC_ACC_LIMBS - 1] < 0) return -1;
  for (int i = 0; i < ORC_ACC_LIMBS; ++i) if (a->w[i]) return 1;
  return 0;
}

/* Sign of |u - Za/den|^2 - |u - Zb/den|^2: +1 if b is strictly closer,
 * -1 if a is strictly closer, 0 on an exact tie. */
int orc_cmp_dist(const float* u, const int32_t* Za, const int32_t* Zb, int den) {
  orc_acc a;
  memset(&a, 0, sizeof a);
  int64_t na = 0, nb = 0;
  for (int i = 0; i < 8; ++i) {
    int64_t k = (int64_t)Zb[i] - Za[i];
    orc_acc_add_double(&a, (double)u[i] * (double)(2 * den * k));
    na += (int64_t)Za[i] * Za[i];
    nb += (int64_t)Zb[i] * Zb[i];
  }
  orc_acc_add_double(&a, (double)(na - nb));
  return orc_acc_sign(&a);
}

/* ------------------------------------------------------------------------- */
/* Nearest codebook point by brute force (the definition).                    */
/* ------------------------------------------------------------------------- */

static double orc_approx_dist(const float* u, const int32_t* Z, int den) {
  double s = 0.0;
  for (int i = 0; i < 8; ++i) {
    double x = (double)u[i] - (double)Z[i] / (double)den;
    s += x * x;
  }
  return s;
}

static int orc_all_finite(const float* u) {
  for (int i = 0; i < 8; ++i) if (!isfinite(u[i])) return 0;
  return 1;
}

/* argmin over candidates c in [0, ncand) of |u - (Zbase + q * v_c)/den|^2,
 * exact, smallest index on ties.  dist[] is caller scratch of ncand doubles. */
static int orc_argmin(const float* u, const int8_t* cb, int ncand,
                      const int32_t* Zbase, int q, int den, double* dist) {
  int32_t Z[8];
  double dmin = INFINITY;
  for (int c = 0; c < ncand; ++c) {
    for (int i = 0; i < 8; ++i) Z[i] = Zbase[i] + q * cb[8 * c + i];
    dist[c] = orc_approx_dist(u, Z, den);
    if (dist[c] < dmin) dmin = dist[c];
  }
  /* binary64 distances carry a relative error below 2^-48; any exact
   * minimiser lies within this window of the computed minimum */
  double lim = dmin * (1.0 + 0x1p-40);
  int best = -1;
  int32_t Zb[8], Zw[8];
  for (int c = 0; c < ncand; ++c) {
    if (!(dist[c] <= lim)) continue;
    for (int i = 0; i < 8; ++i) Zb[i] = Zbase[i] + q * cb[8 * c + i];
    if (best < 0 || orc_cmp_dist(u, Zw, Zb, den) > 0) {
      best = c;
      memcpy(Zw, Zb, sizeof Zw);
    }
  }
  return best;
}

/* Quantise groups of already-transformed weights u[G][8].
 * Stage 1: idx1 = argmin_{c in C} |u - c|^2.
 * Stage 2 (bpw 3, 4): idx2 = argmin_{c2 in C2} |u - c1 - beta c2|^2 with
 *   C2 = first 256 entries, beta = 1/2 (bpw 3) or C2 = C, beta = 1/4 (bpw 4).
 * Groups with a non-finite coordinate get index 0 at every stage. */
int orc_nearest_groups(const float* u, int64_t G, int bpw, const int8_t* cb,
                       uint16_t* idx1, void* idx2, int nthreads) {
  if (bpw < 2 || bpw > 4) return -1;
  int fail = 0;
#ifdef _OPENMP
#pragma omp parallel num_threads(nthreads)
#endif
  {
    double* dist = (double*)malloc(sizeof(double) * ORC_CB_SIZE);
    if (!dist) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
      fail = 1;
    }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 16)
#endif
    for (int64_t g = 0; g < G; ++g) {
      if (!dist) continue;
      const float* ug = u + 8 * g;
      const int32_t zero[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      int i1 = 0, i2 = 0;
      if (orc_all_finite(ug)) {
        i1 = orc_argmin(ug, cb, ORC_CB_SIZE, zero, 1, 2, dist);
        if (bpw > 2) {
          int m = bpw == 3 ? 4 : 8;
          int32_t Zb[8];
          for (int i = 0; i < 8; ++i) Zb[i] = (m / 2) * cb[8 * i1 + i];
          /* point = c1 + beta c2 = (m/2 v1 + (m beta / 2) v2) / m, m beta / 2 = 1 */
          i2 = orc_argmin(ug, cb, bpw == 3 ? 256 : ORC_CB_SIZE, Zb, 1, m, dist);
        }
      }
      idx1[g] = (uint16_t)i1;
      if (bpw == 3) ((uint8_t*)idx2)[g] = (uint8_t)i2;
      if (bpw == 4) ((uint16_t*)idx2)[g] = (uint16_t)i2;
    }
    free(dist);
  }
  (void)nthreads;
  return fail ? -1 : 0;
}

/* Full encoder: forward RHT of W [N][K] (blocks of nh) then nearest-point
 * quantisation. */
int orc_encode_nh(const float* W, int64_t N, int64_t K, int64_t nh, int bpw, uint64_t rht_seed,
                  float scale, const int8_t* cb, uint16_t* idx1, void* idx2, int nthreads) {
  if (!orc_valid_block(K, nh)) return -1;
  float* U = (float*)malloc(sizeof(float) * (size_t)(N * K));
  if (!U) return -1;
  int rc = orc_rht_forward_nh(W, N, K, nh, rht_seed, scale, U, nthreads);
  if (rc == 0) rc = orc_nearest_groups(U, N * K / 8, bpw, cb, idx1, idx2, nthreads);
  free(U);
  return rc;
}

int orc_encode(const float* W, int64_t N, int64_t K, int bpw, uint64_t rht_seed,
               float scale, const int8_t* cb, uint16_t* idx1, void* idx2, int nthreads) {
  int64_t nh = orc_hadamard_block(K);
  if (nh == 0) return -1;
  return orc_encode_nh(W, N, K, nh, bpw, rht_seed, scale, cb, idx1, idx2, nthreads);
}

/* ------------------------------------------------------------------------- */
/* Decoder: indices -> bf16 weights.                                          */
/* ------------------------------------------------------------------------- */

static uint16_t orc_bf16_rne(float f) {
  uint32_t x;
  memcpy(&x, &f, 4);
  if ((x & 0x7F800000u) == 0x7F800000u && (x & 0x007FFFFFu)) return (uint16_t)((x >> 16) | 0x40);
  uint32_t lsb = (x >> 16) & 1u;
  x += 0x7FFFu + lsb;
  return (uint16_t)(x >> 16);
}

/* Integer group vector z = m * (c1 + beta c2):  bpw 2: z = v1;  bpw 3:
 * z = 2 v1 + v2;  bpw 4: z = 4 v1 + v2 (v = doubled coordinates). */
static void orc_group_z(const int8_t* cb, int bpw, int i1, int i2, int64_t* z) {
  for (int j = 0; j < 8; ++j) {
    int64_t v1 = cb[8 * i1 + j];
    if (bpw == 2) z[j] = v1;
    else if (bpw == 3) z[j] = 2 * v1 + cb[8 * i2 + j];
    else z[j] = 4 * v1 + cb[8 * i2 + j];
  }
}

/* W_dec[n][k] = bf16_rne(d_k * fl32(t_k * alpha)), t = FWHT(z) per block of nh. */
int orc_decode_nh(const uint16_t* idx1, const void* idx2, int64_t N, int64_t K, int64_t nh,
                  int bpw, uint64_t rht_seed, float scale, const int8_t* cb, uint16_t* Wdec,
                  int nthreads) {
  if (!orc_valid_block(K, nh) || bpw < 2 || bpw > 4) return -1;
  int8_t* d = (int8_t*)malloc((size_t)K);
  if (!d) return -1;
  orc_signs(rht_seed, K, d);
  float alpha = orc_alpha(scale, nh, bpw);
  int fail = 0;
#ifdef _OPENMP
#pragma omp parallel num_threads(nthreads)
#endif
  {
    int64_t* t = (int64_t*)malloc(sizeof(int64_t) * (size_t)K);
    if (!t) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
      fail = 1;
    }
#ifdef _OPENMP
#pragma omp for schedule(static)
#endif
    for (int64_t r = 0; r < N; ++r) {
      if (!t) continue;
      for (int64_t g = 0; g < K / 8; ++g) {
        int64_t gi = r * (K / 8) + g;
        int i2 = 0;
        if (bpw == 3) i2 = ((const uint8_t*)idx2)[gi];
        if (bpw == 4) i2 = ((const uint16_t*)idx2)[gi];
        orc_group_z(cb, bpw, idx1[gi], i2, t + 8 * g);
      }
      for (int64_t b = 0; b < K; b += nh) orc_fwht_i64(t + b, nh);
      for (int64_t k = 0; k < K; ++k) {
        float p = (float)t[k] * alpha;    /* |t| < 2^24: exact conversion */
        if (d[k] < 0) p = -p;
        Wdec[r * K + k] = orc_bf16_rne(p);
      }
    }
    free(t);
  }
  (void)nthreads;
  free(d);
  return fail ? -1 : 0;
}

int orc_decode(const uint16_t* idx1, const void* idx2, int64_t N, int64_t K, int bpw,
               uint64_t rht_seed, float scale, const int8_t* cb, uint16_t* Wdec,
               int nthreads) {
  int64_t nh = orc_hadamard_block(K);
  if (nh == 0) return -1;
  return orc_decode_nh(idx1, idx2, N, K, nh, bpw, rht_seed, scale, cb, Wdec, nthreads);
}

/* ------------------------------------------------------------------------- */
/* GEMM: Y[m][n] = sum_k X[m][k] W[n][k], bf16 inputs, binary64 result.       */
/* ------------------------------------------------------------------------- */

static double orc_bf16_to_double(uint16_t h) {
  uint32_t x = (uint32_t)h << 16;
  float f;
  memcpy(&f, &x, 4);
  return (double)f;
}

int orc_gemm(const uint16_t* X, int64_t M, const uint16_t* W, int64_t N, int64_t K,
             double* Y, int nthreads) {
  double* xr = (double*)malloc(sizeof(double) * (size_t)(M * K));
  if (!xr) return -1;
  for (int64_t i = 0; i < M * K; ++i) xr[i] = orc_bf16_to_double(X[i]);
#ifdef _OPENMP
#pragma omp parallel for num_threads(nthreads) schedule(static)
#endif
  for (int64_t n = 0; n < N; ++n) {
    const uint16_t* w = W + n * K;
    for (int64_t m = 0; m < M; ++m) {
      const double* x = xr + m * K;
      double s = 0.0;
      for (int64_t k = 0; k < K; ++k) s += x[k] * orc_bf16_to_double(w[k]);
      Y[m * N + n] = s;
    }
  }
  (void)nthreads;
  free(xr);
  return 0;
}

int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
