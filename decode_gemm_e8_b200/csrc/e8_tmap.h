// Host helper: 2-D TMA tensor maps (cuTensorMapEncodeTiled).
//
// The driver entry point is fetched through the runtime at first use, so the
// library itself does not link against libcuda and loads on machines without
// a GPU driver.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace e8 {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// Row-major [rows][cols] tensor of `elem_bytes`-byte elements; box = [box_rows][box_cols].
// Returns false if the driver rejects the description.
// A map depends only on these arguments, so the last few encodings of each
// host thread are kept and reused (the steady state of a layer loop encodes
// nothing).
inline bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                         int elem_bytes, uint64_t rows, uint64_t cols, uint32_t box_rows,
                         uint32_t box_cols, CUtensorMapSwizzle swizzle) {
  struct Entry {
    const void* base;
    uint64_t rows, cols;
    uint32_t box_rows, box_cols;
    int dtype, elem_bytes, swizzle;
    CUtensorMap map;
  };
  constexpr int kEntries = 64;
  thread_local Entry cache[kEntries];
  thread_local int used = 0, next = 0;
  for (int i = 0; i < used; ++i) {
    const Entry& c = cache[i];
    if (c.base == base && c.rows == rows && c.cols == cols && c.box_rows == box_rows &&
        c.box_cols == box_cols && c.dtype == (int)dtype && c.elem_bytes == elem_bytes &&
        c.swizzle == (int)swizzle) {
      *map = c.map;
      return true;
    }
  }
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(cols * (uint64_t)elem_bytes)};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  Entry& e = cache[next];
  e.base = base;
  e.rows = rows;
  e.cols = cols;
  e.box_rows = box_rows;
  e.box_cols = box_cols;
  e.dtype = (int)dtype;
  e.elem_bytes = elem_bytes;
  e.swizzle = (int)swizzle;
  e.map = *map;
  next = (next + 1) % kEntries;
  if (used < kEntries) ++used;
  return true;
}

}  // namespace e8
