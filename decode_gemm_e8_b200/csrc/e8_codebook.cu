// Device construction of the canonical E8 codebook tables.
//
// The canonical list is origin, then for each shell of squared norm 2..12 the
// positive representatives (first nonzero coordinate > 0) in lexicographic
// order of doubled coordinates, each followed by its negation, cut at 65536
// ("glq 0.1.1", "How it works", item 1: 65536 vectors from the first 7 shells).
//
// The work is split into "cells" = (shell, v0, v1).  Lexicographic order of
// whole vectors is the order of cells followed by the order inside a cell, so
// one thread per cell counts its representatives (pass 1), a scan gives every
// cell its first global representative number, and the same threads write
// their vectors in order (pass 2).  Inside a cell the six remaining doubled
// coordinates are enumerated by ascending nested loops, which is lexicographic.
#include "e8_common.cuh"
#include "e8_codebook.cuh"
#include "e8_internal.h"

namespace e8 {

constexpr int kShells = 6;                 // norms 2, 4, ..., 12
constexpr int kCells = kShells * 13 * 13;  // (shell, v0 + 6, v1 + 6)

struct CellSpec {
  int norm4, v0, v1, valid;
};

__device__ __forceinline__ CellSpec cell_spec(int cell) {
  CellSpec c;
  int s = cell / 169, r = cell % 169;
  c.norm4 = 8 * (s + 1);
  c.v0 = r / 13 - 6;
  c.v1 = r % 13 - 6;
  int p0 = c.v0 & 1, p1 = c.v1 & 1;
  c.valid = (p0 == p1) && (c.v0 >= 0) && !(c.v0 == 0 && c.v1 < 0) &&
            (c.v0 * c.v0 + c.v1 * c.v1 <= c.norm4);
  return c;
}

// Visits, in lexicographic order, every E8 vector of the cell's shell whose
// first two doubled coordinates are (v0, v1) and whose first nonzero
// coordinate is positive.  f(v) is called with the 8 doubled coordinates.
template <class F>
__device__ void visit_cell(const CellSpec& c, F&& f) {
  const bool odd = (c.v0 & 1) != 0;
  const int lo = odd ? -5 : -6, hi = -lo;
  const int rem0 = c.norm4 - c.v0 * c.v0 - c.v1 * c.v1;
  const int need_pos_suffix = (c.v0 == 0 && c.v1 == 0);
  int v[8];
  v[0] = c.v0;
  v[1] = c.v1;
  for (v[2] = lo; v[2] <= hi; v[2] += 2) {
    int r2 = rem0 - v[2] * v[2];
    if (r2 < 0) continue;
    for (v[3] = lo; v[3] <= hi; v[3] += 2) {
      int r3 = r2 - v[3] * v[3];
      if (r3 < 0) continue;
      for (v[4] = lo; v[4] <= hi; v[4] += 2) {
        int r4 = r3 - v[4] * v[4];
        if (r4 < 0) continue;
        for (v[5] = lo; v[5] <= hi; v[5] += 2) {
          int r5 = r4 - v[5] * v[5];
          if (r5 < 0) continue;
          for (v[6] = lo; v[6] <= hi; v[6] += 2) {
            int r6 = r5 - v[6] * v[6];
            if (r6 < 0) continue;
            for (v[7] = lo; v[7] <= hi; v[7] += 2) {
              if (r6 - v[7] * v[7] != 0) continue;
              int sum = 0;
              for (int j = 0; j < 8; ++j) sum += v[j];
              if ((sum & 3) != 0) continue;
              if (need_pos_suffix) {
                int first = 0;
                for (int j = 2; j < 8; ++j)
                  if (v[j] != 0) { first = v[j]; break; }
                if (first <= 0) continue;
              }
              f(v);
            }
          }
        }
      }
    }
  }
}

__global__ void k_cb_count(int* counts) {
  int cell = blockIdx.x * blockDim.x + threadIdx.x;
  if (cell >= kCells) return;
  CellSpec c = cell_spec(cell);
  int n = 0;
  if (c.valid) visit_cell(c, [&](const int*) { ++n; });
  counts[cell] = n;
}

__global__ void k_cb_scan(const int* counts, int* offsets, int* total) {
  if (blockIdx.x != 0 || threadIdx.x != 0) return;
  int acc = 0;
  for (int i = 0; i < kCells; ++i) {
    offsets[i] = acc;
    acc += counts[i];
  }
  *total = acc;
}

__global__ void k_cb_emit(const int* offsets, int8_t* vecs, uint32_t* table) {
  int cell = blockIdx.x * blockDim.x + threadIdx.x;
  if (cell == 0) {
    for (int j = 0; j < 8; ++j) vecs[j] = 0;
    int z[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    table[0] = pack_vec(z);
  }
  if (cell >= kCells) return;
  CellSpec c = cell_spec(cell);
  if (!c.valid) return;
  int q = offsets[cell];
  visit_cell(c, [&](const int* v) {
    if (q < kNumPosReps) {
      int64_t ip = 1 + 2 * (int64_t)q, in = ip + 1;
      for (int j = 0; j < 8; ++j) vecs[ip * 8 + j] = (int8_t)v[j];
      if (in < kCbSize)
        for (int j = 0; j < 8; ++j) vecs[in * 8 + j] = (int8_t)(-v[j]);
      table[q + 1] = pack_vec(v);
    }
    ++q;
  });
}

__global__ void k_cb_hash(const uint32_t* table, uint32_t* hkeys, uint32_t* hvals,
                          int* max_probe) {
  int q = blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= kNumPosReps) return;
  uint32_t key = table[q + 1];
  uint32_t s = hash_slot(key);
  for (int probe = 0; probe < kHashSlots; ++probe) {
    uint32_t prev = atomicCAS(hkeys + s, kHashEmpty, key);
    if (prev == kHashEmpty || prev == key) {
      hvals[s] = (uint32_t)q;
      atomicMax(max_probe, probe);
      return;
    }
    s = (s + 1) & (kHashSlots - 1);
  }
}

// Transformed pair table: slot q holds H8 v / 4 (v the slot's vector, H8 the
// natural-order 8-point Walsh-Hadamard matrix).  A slot whose transform is not
// a multiple of 4 in [-16, 16] is counted in *bad (none is expected).
__global__ void k_cb_h8(const uint32_t* table, uint32_t* h8, int* bad) {
  int q = blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= kPairSlots) return;
  const uint32_t e = table[q];
  int v[8];
  for (int j = 0; j < 4; ++j) {
    v[j] = (int)((e >> (8 * j)) & 0xFu) - 8;
    v[j + 4] = (int)((e >> (8 * j + 4)) & 0xFu) - 8;
  }
  for (int h = 1; h < 8; h <<= 1)
    for (int i = 0; i < 8; ++i)
      if ((i & h) == 0) {
        const int a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
  bool ok = true;
  for (int j = 0; j < 8; ++j) {
    ok = ok && (v[j] % 4 == 0) && v[j] >= -16 && v[j] <= 16;
    v[j] /= 4;
  }
  if (!ok) atomicAdd(bad, 1);
  h8[q] = pack_vec(v);
}

__global__ void k_cb_clist(const int8_t* vecs, int32_t* clist, int* count) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= kCbSize) return;
  const int8_t* v = vecs + 8 * i;
  int n = 0;
  for (int j = 0; j < 8; ++j) n += v[j] * v[j];
  if (n != 48 || v[0] != 0 || (v[1] != 4 && v[1] != -4)) return;
  const int slot = atomicAdd(count, 1);
  if (slot < kCListCap) clist[slot] = i;
}

int build_codebook_clist(const int8_t* d_vecs, int32_t* d_clist, cudaStream_t st) {
  int* d_count = nullptr;
  if (cudaMalloc(&d_count, sizeof(int)) != cudaSuccess) return -1;
  cudaMemsetAsync(d_count, 0, sizeof(int), st);
  k_cb_clist<<<kCbSize / 256, 256, 0, st>>>(d_vecs, d_clist, d_count);
  int h = -1;
  cudaMemcpyAsync(&h, d_count, sizeof(int), cudaMemcpyDeviceToHost, st);
  cudaError_t e = cudaStreamSynchronize(st);
  cudaFree(d_count);
  if (e != cudaSuccess || cudaGetLastError() != cudaSuccess || h > kCListCap) return -1;
  return h;
}

// Builds vecs, table, the transformed table and the hash on the current
// device (synchronous).
// Returns the number of positive representatives found over all shells
// (58680 for the E8 shells of norm 2..12), or -1 on a CUDA error.
int build_codebook_tables(int8_t* d_vecs, uint32_t* d_table, uint32_t* d_h8table,
                          uint32_t* d_hkeys, uint32_t* d_hvals, int* h_max_probe, cudaStream_t st) {
  int *d_counts = nullptr, *d_offsets = nullptr, *d_scalars = nullptr;
  if (cudaMalloc(&d_counts, kCells * sizeof(int)) != cudaSuccess) return -1;
  if (cudaMalloc(&d_offsets, kCells * sizeof(int)) != cudaSuccess) return -1;
  if (cudaMalloc(&d_scalars, 3 * sizeof(int)) != cudaSuccess) return -1;
  cudaMemsetAsync(d_scalars, 0, 3 * sizeof(int), st);
  cudaMemsetAsync(d_hkeys, 0, kHashSlots * sizeof(uint32_t), st);
  cudaMemsetAsync(d_hvals, 0, kHashSlots * sizeof(uint32_t), st);
  const int tpb = 128, nb = (kCells + tpb - 1) / tpb;
  k_cb_count<<<nb, tpb, 0, st>>>(d_counts);
  k_cb_scan<<<1, 1, 0, st>>>(d_counts, d_offsets, d_scalars);
  k_cb_emit<<<nb, tpb, 0, st>>>(d_offsets, d_vecs, d_table);
  k_cb_hash<<<(kNumPosReps + 255) / 256, 256, 0, st>>>(d_table, d_hkeys, d_hvals,
                                                       d_scalars + 1);
  k_cb_h8<<<(kPairSlots + 255) / 256, 256, 0, st>>>(d_table, d_h8table, d_scalars + 2);
  int h[3] = {0, 0, 0};
  cudaMemcpyAsync(h, d_scalars, sizeof(h), cudaMemcpyDeviceToHost, st);
  cudaError_t e = cudaStreamSynchronize(st);
  cudaFree(d_counts);
  cudaFree(d_offsets);
  cudaFree(d_scalars);
  if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) return -1;
  if (h[2] != 0) return -1;
  if (h_max_probe) *h_max_probe = h[1];
  return h[0];
}

}  // namespace e8
