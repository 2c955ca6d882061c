// Device-resident codebook tables shared by the encode, decode and GEMM kernels.
//
// Codebook (page "glq 0.1.1", "How it works", item 1): 65536 E8 lattice
// vectors from the shells of squared norm 0, 2, ..., 12, in canonical order --
// origin first, then shells by increasing norm, inside a shell the vectors
// whose first nonzero coordinate is positive sorted lexicographically on
// doubled coordinates, each emitted as p then -p, cut at 65536 entries.
//
// Representations (coordinates are always doubled, v = 2x, |v| <= 6):
//   vecs  [65536][8] int8        index -> vector, used by the exact slow path
//   table [32769] uint32         packed vector of pair slot j; index i maps to
//                                slot (i + 1) >> 1 and is negated when i is even
//                                and nonzero.  Nibble layout: bits 8j..8j+3 hold
//                                v_j + 8, bits 8j+4..8j+7 hold v_{j+4} + 8 (j < 4),
//                                so (e & 0x0F0F0F0F) are coordinates 0..3 and
//                                ((e >> 4) & 0x0F0F0F0F) coordinates 4..7, biased.
//   h8table [32769] uint32       the same pair slots holding H8 v / 4 instead of v,
//                                where H8 is the 8-point Walsh-Hadamard matrix in
//                                natural order.  For every codebook vector the
//                                entries of H8 v are multiples of 4 in [-16, 16]
//                                (checked when the table is built), so the
//                                transformed table keeps the nibble layout; the
//                                bf16 decoder starts from it and skips the three
//                                Hadamard stages inside a group.
//   hash  open addressing over kHashSlots slots: key = packed positive
//         representative, value = its pair slot q - 1 (0-based), used to
//         rank a vector (index 2q+1 for p, 2q+2 for -p).
#pragma once

#include <cstdint>

namespace e8 {

constexpr int kCbSize = 65536;
constexpr int kPairSlots = 32769;      // slot 0 = origin, slots 1..32768 = pairs
constexpr int kNumPosReps = 32768;     // positive representatives kept
constexpr int kHashSlots = 65536;
constexpr uint32_t kHashEmpty = 0u;    // packed keys are never 0 (every nibble >= 2)

__host__ __device__ __forceinline__ uint32_t pack_vec(const int* v) {
  uint32_t e = 0;
  for (int j = 0; j < 4; ++j) {
    e |= (uint32_t)(v[j] + 8) << (8 * j);
    e |= (uint32_t)(v[j + 4] + 8) << (8 * j + 4);
  }
  return e;
}

__host__ __device__ __forceinline__ uint32_t hash_slot(uint32_t key) {
  return (key * 2654435761u) >> 16;
}

// Packed decode of one group into 8 unsigned bytes z + 128 (two words, the
// coordinates 0..3 and 4..7).  ea / eb: pair-table entries of the stage-1 and
// stage-2 indices (8 nibbles v + 8); the sign of a stage is set when its index
// is even (index 0 is the zero vector, whose sign does not matter).  With
// B = v + 8 in [2, 14], the negated value's biased byte is B ^ 31 = 23 - v,
// so one XOR per word applies a stage's sign and a per-group constant fixes
// the bias:  byte = mul (B1 or B1 ^ 31) + (B2 or B2 ^ 31) + c(s1, s2) = z + 128.
template <int BPW>
__device__ __forceinline__ void decode_group_q8(uint32_t i1, uint32_t i2, uint32_t ea, uint32_t eb,
                                                uint32_t& lo, uint32_t& hi) {
  const uint32_t s1 = (~i1) & 1u;
  const uint32_t m1 = s1 * 0x1F1F1F1Fu;
  const uint32_t lo1 = (ea & 0x0F0F0F0Fu) ^ m1;
  const uint32_t hi1 = ((ea >> 4) & 0x0F0F0F0Fu) ^ m1;
  if (BPW == 2) {
    // v + 128: B + 120, or (23 - v) + 105 = -v + 128
    const uint32_t c = 0x78787878u - s1 * 0x0F0F0F0Fu;
    lo = lo1 + c;
    hi = hi1 + c;
  } else {
    const uint32_t s2 = (~i2) & 1u;
    const uint32_t m2 = s2 * 0x1F1F1F1Fu;
    const uint32_t lo2 = (eb & 0x0F0F0F0Fu) ^ m2;
    const uint32_t hi2 = ((eb >> 4) & 0x0F0F0F0Fu) ^ m2;
    if (BPW == 4) {
      // 4 (+-v1) + (+-v2) + 128
      const uint32_t c = 0x58585858u - s1 * 0x3C3C3C3Cu - s2 * 0x0F0F0F0Fu;
      lo = lo1 * 4u + lo2 + c;
      hi = hi1 * 4u + hi2 + c;
    } else {
      // 2 (+-v1) + (+-v2) + 128
      const uint32_t c = 0x68686868u - s1 * 0x1E1E1E1Eu - s2 * 0x0F0F0F0Fu;
      lo = lo1 * 2u + lo2 + c;
      hi = hi1 * 2u + hi2 + c;
    }
  }
}

struct DeviceCodebook {
  const int8_t* vecs;        // [65536][8]
  const uint32_t* table;     // [32769]
  const uint32_t* h8table;   // [32769]
  const uint32_t* hkeys;     // [kHashSlots]
  const uint32_t* hvals;     // [kHashSlots]
  const int32_t* clist;      // indices of the kept norm-12 points with x1 = 0, |x2| = 2
  int clist_len;
  uint32_t* status;          // device status word
};

// Codebook index of the lattice vector v (doubled coordinates), or -1 if v is
// not one of the 65536 entries; hkeys / hvals: the hash of the positive
// representatives.
__device__ __forceinline__ int rank_vector(const uint32_t* hkeys, const uint32_t* hvals,
                                           const int* v) {
  int first = 0;
  for (int j = 0; j < 8; ++j) {
    if (v[j] != 0) { first = v[j]; break; }
  }
  if (first == 0) return 0;
  int w[8];
  for (int j = 0; j < 8; ++j) {
    if (v[j] < -6 || v[j] > 6) return -1;
    w[j] = first > 0 ? v[j] : -v[j];
  }
  uint32_t key = pack_vec(w);
  uint32_t s = hash_slot(key);
  for (int probe = 0; probe < kHashSlots; ++probe) {
    uint32_t k = __ldg(hkeys + s);
    if (k == key) {
      int q = (int)__ldg(hvals + s);
      int idx = first > 0 ? 2 * q + 1 : 2 * q + 2;
      return idx < kCbSize ? idx : -1;
    }
    if (k == kHashEmpty) return -1;
    s = (s + 1) & (kHashSlots - 1);
  }
  return -1;
}

__device__ __forceinline__ int rank_vector(const DeviceCodebook& cb, const int* v) {
  return rank_vector(cb.hkeys, cb.hvals, v);
}

}  // namespace e8
