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

struct DeviceCodebook {
  const int8_t* vecs;        // [65536][8]
  const uint32_t* table;     // [32769]
  const uint32_t* hkeys;     // [kHashSlots]
  const uint32_t* hvals;     // [kHashSlots]
  uint32_t* status;          // device status word
};

// Codebook index of the lattice vector v (doubled coordinates), or -1 if v is
// not one of the 65536 entries.
__device__ __forceinline__ int rank_vector(const DeviceCodebook& cb, const int* v) {
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
    uint32_t k = __ldg(cb.hkeys + s);
    if (k == key) {
      int q = (int)__ldg(cb.hvals + s);
      int idx = first > 0 ? 2 * q + 1 : 2 * q + 2;
      return idx < kCbSize ? idx : -1;
    }
    if (k == kHashEmpty) return -1;
    s = (s + 1) & (kHashSlots - 1);
  }
  return -1;
}

}  // namespace e8
