// C ABI of libe8 (declared in include/e8.h): argument checks, workspace
// carving, scale constants, kernel launches.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "e8.h"
#include "e8_common.cuh"
#include "e8_codebook.cuh"
#include "e8_internal.h"


namespace e8 {

cudaError_t ensure_smem_limit_ptr(const void* kernel, int bytes, bool carveout_max) {
  // fixed table, no heap use on any launch path
  constexpr int kSlots = 256;
  static std::mutex mu;
  static const void* kern[kSlots];
  static int devs[kSlots];
  static int used = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (kern[i] == kernel && devs[i] == dev) return cudaSuccess;
  // the limit may not exceed the opt-in maximum minus the kernel's static shared memory
  int optin = 0;
  cudaFuncAttributes fa;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess &&
      cudaFuncGetAttributes(&fa, kernel) == cudaSuccess) {
    const int cap = optin - (int)fa.sharedSizeBytes;
    if (bytes > cap) bytes = cap;
  }
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && carveout_max)
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && used < kSlots) {
    kern[used] = kernel;
    devs[used] = dev;
    ++used;
  }
  return e;
}

size_t act_scratch_bytes(int64_t M, int64_t K, int smem_variant, int64_t nh) {
  const int64_t rows = (2 * M + 15) / 16 * 16;
  if (!smem_variant && q8_eligible(M, K, nh)) return q8_layout(M, K, rows).total;
  return (((size_t)rows * (size_t)K * 2) + 255) & ~size_t(255);
}

cudaError_t run_act_gemm(const e8_codebook* cb, const uint16_t* X, int64_t M,
                         const uint16_t* idx1, const void* idx2, int64_t N, int64_t K, int bpw,
                         uint64_t seed, float alpha, float* Y, int smem_variant, void* scratch,
                         cudaStream_t st, int64_t nh) {
  DeviceCodebook d;
  d.vecs = cb->vecs;
  d.table = cb->table;
  d.h8table = cb->h8table;
  d.hkeys = cb->hkeys;
  d.hvals = cb->hvals;
  d.clist = cb->clist;
  d.clist_len = cb->clist_len;
  d.status = cb->status;
  const int rows = (int)((2 * M + 15) / 16 * 16);
  if (!smem_variant && q8_eligible(M, K, nh)) {
    const Q8Layout l = q8_layout(M, K, rows);
    uint8_t* buf = static_cast<uint8_t*>(scratch);
    ActQ8Args a;
    a.Xq = reinterpret_cast<int8_t*>(buf);
    a.scales = reinterpret_cast<float*>(buf + l.scales_off);
    a.M = M;
    a.N = N;
    a.K = K;
    a.rows_b = rows;
    a.idx1 = idx1;
    a.idx2 = idx2;
    a.bpw = bpw;
    a.alpha = alpha;
    a.Y = Y;
    a.pdl = 1;          // the fused kernel's prologue overlaps the transform
    a.early_codes = 1;  // which writes only the activation buffer
    cudaError_t e = launch_act_q8(X, M, K, seed, reinterpret_cast<int8_t*>(buf),
                                  reinterpret_cast<float*>(buf + l.scales_off), rows, st, 1, Y,
                                  M * N, nh);
    if (e != cudaSuccess) return e;
    return launch_act_gemm_q8(d, a, cb->sm_count, st);
  }
  uint16_t* Xt = static_cast<uint16_t*>(scratch);
  cudaError_t e = launch_act_rht(X, M, K, seed, Xt, rows, st, 0, nh);
  if (e != cudaSuccess) return e;
  ActGemmArgs a;
  a.Xt = Xt;
  a.M = M;
  a.N = N;
  a.K = K;
  a.rows_b = rows;
  a.idx1 = idx1;
  a.idx2 = idx2;
  a.bpw = bpw;
  a.alpha = alpha;
  a.Y = Y;
  a.variant = smem_variant ? 0 : 1;
  a.pdl = 0;
  a.early_codes = 0;
  return launch_act_gemm(d, a, cb->sm_count, st);
}

}  // namespace e8

namespace {

using e8::aligned16;
using e8::alpha_of;
using e8::valid_bpw;
using e8::valid_k;
constexpr size_t kTableAlloc = 131088;  // 32769 u32 padded to a multiple of 16 bytes

int check_device(const e8_codebook* cb) {
  if (!cb) return E8_EINVAL;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return E8_ECUDA;
  return dev == cb->device ? E8_OK : E8_EDEVICE;
}

float gamma_of(float scale, int64_t nh) {
  return (float)(1.0 / ((double)scale * std::sqrt((double)nh)));
}

e8::DeviceCodebook dev_view(const e8_codebook* cb) {
  e8::DeviceCodebook d;
  d.vecs = cb->vecs;
  d.table = cb->table;
  d.h8table = cb->h8table;
  d.hkeys = cb->hkeys;
  d.hvals = cb->hvals;
  d.clist = cb->clist;
  d.clist_len = cb->clist_len;
  d.status = cb->status;
  return d;
}

int rows_b_for(int64_t M) {
  int64_t r = 2 * M;
  r = (r + 15) / 16 * 16;
  return (int)r;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? E8_OK : E8_ECUDA; }

}  // namespace

extern "C" {

int e8_version(void) { return 100; }

const char* e8_status_str(int s) {
  switch (s) {
    case E8_OK: return "ok";
    case E8_EINVAL: return "invalid argument";
    case E8_EWORKSPACE: return "workspace too small";
    case E8_EDEVICE: return "unsupported or wrong device";
    case E8_ECUDA: return "CUDA error";
    case E8_ETIMEOUT: return "device wait timed out";
    case E8_ENOMEM: return "out of device memory";
    case E8_EDATA: return "malformed compressed stream";
    default: return "unknown status";
  }
}

int e8_codebook_build(e8_codebook** out, int device) {
  (void)cudaGetLastError();  // a failed earlier launch must not be reported here
  if (!out) return E8_EINVAL;
  *out = nullptr;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) return E8_EDEVICE;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) return E8_ECUDA;
  if (prop.major != 10) return E8_EDEVICE;
  int prev = -1;
  cudaGetDevice(&prev);
  if (cudaSetDevice(device) != cudaSuccess) return E8_ECUDA;
  e8_codebook* cb = new e8_codebook();
  cb->device = device;
  cb->sm_count = prop.multiProcessorCount;
  int rc = E8_OK;
  auto fail = [&](int code) {
    cudaFree(cb->vecs);
    cudaFree(cb->table);
    cudaFree(cb->h8table);
    cudaFree(cb->hkeys);
    cudaFree(cb->hvals);
    cudaFree(cb->clist);
    cudaFree(cb->status);
    delete cb;
    if (prev >= 0) cudaSetDevice(prev);
    return code;
  };
  if (cudaMalloc(&cb->vecs, (size_t)e8::kCbSize * 8) != cudaSuccess) return fail(E8_ENOMEM);
  if (cudaMalloc(&cb->table, kTableAlloc) != cudaSuccess) return fail(E8_ENOMEM);
  if (cudaMalloc(&cb->h8table, kTableAlloc) != cudaSuccess) return fail(E8_ENOMEM);
  if (cudaMalloc(&cb->hkeys, e8::kHashSlots * sizeof(uint32_t)) != cudaSuccess)
    return fail(E8_ENOMEM);
  if (cudaMalloc(&cb->hvals, e8::kHashSlots * sizeof(uint32_t)) != cudaSuccess)
    return fail(E8_ENOMEM);
  if (cudaMalloc(&cb->clist, e8::kCListCap * sizeof(int32_t)) != cudaSuccess)
    return fail(E8_ENOMEM);
  if (cudaMalloc(&cb->status, 16) != cudaSuccess) return fail(E8_ENOMEM);
  cudaStream_t st;
  if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess) return fail(E8_ECUDA);
  cudaMemsetAsync(cb->status, 0, 16, st);
  cudaMemsetAsync(cb->table, 0, kTableAlloc, st);
  cudaMemsetAsync(cb->h8table, 0, kTableAlloc, st);
  int reps = e8::build_codebook_tables(cb->vecs, cb->table, cb->h8table, cb->hkeys, cb->hvals,
                                       &cb->max_probe, st);
  // the kept norm-12 points with x1 = 0 and |x2| = 2: 888 positive
  // representatives and the negations of all but the last
  cb->clist_len = reps == 58680 ? e8::build_codebook_clist(cb->vecs, cb->clist, st) : -1;
  if (cb->clist_len != 1775) reps = -1;
  cudaStreamDestroy(st);
  // the E8 shells of squared norm 2..12 hold 117360 vectors, half of them
  // positive representatives
  if (reps != 58680) rc = E8_ECUDA;
  if (rc != E8_OK) return fail(rc);
  if (prev >= 0) cudaSetDevice(prev);
  *out = cb;
  return E8_OK;
}

void e8_codebook_free(e8_codebook* cb) {
  if (!cb) return;
  int prev = -1;
  cudaGetDevice(&prev);
  cudaSetDevice(cb->device);
  cudaFree(cb->vecs);
  cudaFree(cb->table);
  cudaFree(cb->h8table);
  cudaFree(cb->hkeys);
  cudaFree(cb->hvals);
  cudaFree(cb->clist);
  cudaFree(cb->status);
  if (prev >= 0) cudaSetDevice(prev);
  delete cb;
}

int e8_codebook_export(const e8_codebook* cb, int8_t* host_vecs) {
  if (!cb || !host_vecs) return E8_EINVAL;
  int prev = -1;
  cudaGetDevice(&prev);
  cudaSetDevice(cb->device);
  cudaError_t e = cudaMemcpy(host_vecs, cb->vecs, (size_t)e8::kCbSize * 8, cudaMemcpyDeviceToHost);
  if (prev >= 0) cudaSetDevice(prev);
  return cuda_status(e);
}

int e8_rht_forward_nh(const e8_codebook* cb, const float* W, int64_t N, int64_t K, int64_t nh,
                      uint64_t rht_seed, float scale, float* U, void* stream) {
  (void)cudaGetLastError();  // a failed earlier launch must not be reported here
  int rc = check_device(cb);
  if (rc != E8_OK) return rc;
  if (N < 0 || !valid_k(K) || !e8::valid_nh(K, nh) || !e8::valid_scale(scale)) return E8_EINVAL;
  if (N == 0) return E8_OK;
  if (!W || !U || !aligned16(W) || !aligned16(U) || W == U) return E8_EINVAL;
  const int64_t nb = e8::resolve_nh(K, nh);
  cudaError_t e = e8::launch_encode(dev_view(cb), W, N, K, 2, rht_seed, gamma_of(scale, nb),
                                    nullptr, nullptr, nullptr, nullptr, 0, U, 0, cb->sm_count,
                                    (cudaStream_t)stream, nb);
  return cuda_status(e);
}

int e8_rht_forward(const e8_codebook* cb, const float* W, int64_t N, int64_t K,
                   uint64_t rht_seed, float scale, float* U, void* stream) {
  return e8_rht_forward_nh(cb, W, N, K, 0, rht_seed, scale, U, stream);
}

size_t e8_workspace_bytes_nh(int op, int64_t M, int64_t N, int64_t K, int64_t nh, int bpw) {
  if (!valid_bpw(bpw) || N < 0 || M < 0 || !valid_k(K) || !e8::valid_nh(K, nh)) return 0;
  const size_t G = (size_t)N * (size_t)(K / 8);
  switch (op) {
    case E8_OP_ENCODE:
      return 256 + 2 * G * sizeof(e8::WorkItem);
    case E8_GEMM_AUTO:
      return e8_workspace_bytes_nh(e8_gemm_auto_mode(M, N, K, bpw), M, N, K, nh, bpw);
    case E8_GEMM_ACT_RHT:
      return e8::act_scratch_bytes(M, K, 0, nh);
    case E8_GEMM_ACT_RHT_SMEM:
      return e8::act_scratch_bytes(M, K, 1, nh);
    case E8_GEMM_DECODED_W:
    case E8_GEMM_SIMT:
      return round256((size_t)N * (size_t)K * 2);
    default:
      return 0;
  }
}

size_t e8_workspace_bytes(int op, int64_t M, int64_t N, int64_t K, int bpw) {
  return e8_workspace_bytes_nh(op, M, N, K, 0, bpw);
}

int e8_gemm_auto_mode(int64_t M, int64_t N, int64_t K, int bpw) {
  (void)N;
  (void)bpw;
  if (M <= 64 && (K % 128) == 0) return E8_GEMM_ACT_RHT;
  return E8_GEMM_DECODED_W;
}

int e8_encode_nh(const e8_codebook* cb, const float* W, int64_t N, int64_t K, int64_t nh,
                 int bpw, uint64_t rht_seed, float scale, uint16_t* idx1, void* idx2,
                 void* workspace, size_t ws_bytes, void* stream) {
  (void)cudaGetLastError();  // a failed earlier launch must not be reported here
  int rc = check_device(cb);
  if (rc != E8_OK) return rc;
  if (N < 0 || !valid_k(K) || !e8::valid_nh(K, nh) || !valid_bpw(bpw) ||
      !e8::valid_scale(scale))
    return E8_EINVAL;
  if ((bpw == 2) != (idx2 == nullptr)) return E8_EINVAL;
  if (N == 0) return E8_OK;
  if (!W || !idx1 || !aligned16(W) || !aligned16(idx1) || (idx2 && !aligned16(idx2)))
    return E8_EINVAL;
  const size_t need = e8_workspace_bytes(E8_OP_ENCODE, 0, N, K, bpw);
  if (!workspace || !aligned16(workspace) || ws_bytes < need) return E8_EWORKSPACE;
  const int64_t nb = e8::resolve_nh(K, nh);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* count = reinterpret_cast<uint32_t*>(ws);
  e8::WorkItem* items = reinterpret_cast<e8::WorkItem*>(ws + 256);
  const uint64_t cap = (uint64_t)N * (uint64_t)(K / 8);
  cudaError_t e = e8::launch_encode(dev_view(cb), W, N, K, bpw, rht_seed, gamma_of(scale, nb),
                                    idx1, idx2, items, count, cap, nullptr, 1, cb->sm_count,
                                    (cudaStream_t)stream, nb);
  return cuda_status(e);
}

int e8_encode(const e8_codebook* cb, const float* W, int64_t N, int64_t K, int bpw,
              uint64_t rht_seed, float scale, uint16_t* idx1, void* idx2, void* workspace,
              size_t ws_bytes, void* stream) {
  return e8_encode_nh(cb, W, N, K, 0, bpw, rht_seed, scale, idx1, idx2, workspace, ws_bytes,
                      stream);
}

int e8_decode_to_bf16_nh(const e8_codebook* cb, const uint16_t* idx1, const void* idx2,
                         int64_t N, int64_t K, int64_t nh, int bpw, uint64_t rht_seed,
                         float scale, uint16_t* W_dec, void* stream) {
  (void)cudaGetLastError();  // a failed earlier launch must not be reported here
  int rc = check_device(cb);
  if (rc != E8_OK) return rc;
  if (N < 0 || !valid_k(K) || !e8::valid_nh(K, nh) || !valid_bpw(bpw) ||
      !e8::valid_scale(scale))
    return E8_EINVAL;
  if ((bpw == 2) != (idx2 == nullptr)) return E8_EINVAL;
  if (N == 0) return E8_OK;
  if (!idx1 || !W_dec || !aligned16(idx1) || !aligned16(W_dec) || (idx2 && !aligned16(idx2)))
    return E8_EINVAL;
  const int64_t nb = e8::resolve_nh(K, nh);
  cudaError_t e = e8::launch_decode(dev_view(cb), idx1, idx2, N, K, bpw, rht_seed,
                                    alpha_of(scale, nb, bpw), W_dec, cb->sm_count,
                                    (cudaStream_t)stream, nb);
  return cuda_status(e);
}

int e8_decode_to_bf16(const e8_codebook* cb, const uint16_t* idx1, const void* idx2, int64_t N,
                      int64_t K, int bpw, uint64_t rht_seed, float scale, uint16_t* W_dec,
                      void* stream) {
  return e8_decode_to_bf16_nh(cb, idx1, idx2, N, K, 0, bpw, rht_seed, scale, W_dec, stream);
}

int e8_act_rht(const uint16_t* X, int64_t M, int64_t K, uint64_t rht_seed, uint16_t* Xt,
               int64_t rows, void* stream) {
  (void)cudaGetLastError();  // a failed earlier launch must not be reported here
  if (M < 0 || !valid_k(K) || rows < 2 * M) return E8_EINVAL;
  if (M == 0) return E8_OK;
  if (!X || !Xt || !aligned16(X) || !aligned16(Xt)) return E8_EINVAL;
  return cuda_status(e8::launch_act_rht(X, M, K, rht_seed, Xt, rows, (cudaStream_t)stream));
}

int e8_gemm_nh(const e8_codebook* cb, const uint16_t* X, int64_t M, const uint16_t* idx1,
               const void* idx2, int64_t N, int64_t K, int64_t nh, int bpw, uint64_t rht_seed,
               float scale, float* Y, int mode, void* workspace, size_t ws_bytes, void* stream) {
  (void)cudaGetLastError();  // a failed earlier launch must not be reported here
  int rc = check_device(cb);
  if (rc != E8_OK) return rc;
  if (M < 0 || N < 0 || !valid_k(K) || !e8::valid_nh(K, nh) || !valid_bpw(bpw) ||
      !e8::valid_scale(scale))
    return E8_EINVAL;
  if ((bpw == 2) != (idx2 == nullptr)) return E8_EINVAL;
  if (mode == E8_GEMM_AUTO) mode = e8_gemm_auto_mode(M, N, K, bpw);
  if (mode < E8_GEMM_ACT_RHT || mode > E8_GEMM_SIMT) return E8_EINVAL;
  const bool act = mode == E8_GEMM_ACT_RHT || mode == E8_GEMM_ACT_RHT_SMEM;
  if (act && !e8::act_shape_ok(M, K)) return E8_EINVAL;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return E8_EINVAL;
  if (M == 0 || N == 0) return E8_OK;
  if (!X || !idx1 || !Y || !aligned16(X) || !aligned16(idx1) || !aligned16(Y) ||
      (idx2 && !aligned16(idx2)))
    return E8_EINVAL;
  const size_t need = e8_workspace_bytes_nh(mode, M, N, K, nh, bpw);
  if (!workspace || !aligned16(workspace) || ws_bytes < need) return E8_EWORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  const int64_t nb = e8::resolve_nh(K, nh);
  const float alpha = alpha_of(scale, nb, bpw);
  const e8::DeviceCodebook d = dev_view(cb);
  cudaError_t e;
  if (act) {
    e = e8::run_act_gemm(cb, X, M, idx1, idx2, N, K, bpw, rht_seed, alpha, Y,
                         mode == E8_GEMM_ACT_RHT_SMEM ? 1 : 0, workspace, st, nb);
    return cuda_status(e);
  }
  uint16_t* Wd = static_cast<uint16_t*>(workspace);
  e = e8::launch_decode(d, idx1, idx2, N, K, bpw, rht_seed, alpha, Wd, cb->sm_count, st, nb);
  if (e != cudaSuccess) return E8_ECUDA;
  if (mode == E8_GEMM_SIMT)
    e = e8::launch_simt_gemm(X, M, Wd, N, K, Y, st);
  else
    e = e8::launch_dense_gemm(X, M, Wd, N, K, Y, cb->status, cb->sm_count, st);
  return cuda_status(e);
}

int e8_gemm(const e8_codebook* cb, const uint16_t* X, int64_t M, const uint16_t* idx1,
            const void* idx2, int64_t N, int64_t K, int bpw, uint64_t rht_seed, float scale,
            float* Y, int mode, void* workspace, size_t ws_bytes, void* stream) {
  return e8_gemm_nh(cb, X, M, idx1, idx2, N, K, 0, bpw, rht_seed, scale, Y, mode, workspace,
                    ws_bytes, stream);
}

size_t e8_gemm_host_workspace_bytes(int mode, int64_t M, int64_t N, int64_t K, int bpw) {
  if (M < 1 || N < 1 || !valid_bpw(bpw) || !valid_k(K)) return 0;
  if (mode == E8_GEMM_AUTO) mode = e8_gemm_auto_mode(M, N, K, bpw);
  if (mode < E8_GEMM_ACT_RHT || mode > E8_GEMM_SIMT) return 0;
  return round256((size_t)M * (size_t)K * 2) + round256((size_t)M * (size_t)N * 4) +
         e8_workspace_bytes(mode, M, N, K, bpw);
}

int e8_gemm_host(const e8_codebook* cb, const uint16_t* X_host, int64_t M, const uint16_t* idx1,
                 const void* idx2, int64_t N, int64_t K, int bpw, uint64_t rht_seed,
                 float scale, float* Y_host, int mode, void* workspace, size_t ws_bytes,
                 void* stream) {
  // every argument is checked before anything is queued (no CUDA call before
  // the device check)
  if (!cb || M < 0 || N < 0 || !valid_k(K) || !valid_bpw(bpw) || !(scale > 0.0f) ||
      !std::isfinite(scale))
    return E8_EINVAL;
  if ((bpw == 2) != (idx2 == nullptr)) return E8_EINVAL;
  if (M == 0 || N == 0) return E8_OK;
  const int m = mode == E8_GEMM_AUTO ? e8_gemm_auto_mode(M, N, K, bpw) : mode;
  if (m < E8_GEMM_ACT_RHT || m > E8_GEMM_SIMT) return E8_EINVAL;
  if ((m == E8_GEMM_ACT_RHT || m == E8_GEMM_ACT_RHT_SMEM) && (M > 64 || (K % 128) != 0))
    return E8_EINVAL;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return E8_EINVAL;
  if (!X_host || !Y_host || !idx1 || !aligned16(X_host) || !aligned16(Y_host) ||
      !aligned16(idx1) || (idx2 && !aligned16(idx2)))
    return E8_EINVAL;
  const size_t xb = (size_t)M * (size_t)K * 2, yb = (size_t)M * (size_t)N * 4;
  {
    const uintptr_t x0 = reinterpret_cast<uintptr_t>(X_host), y0 = reinterpret_cast<uintptr_t>(Y_host);
    if (x0 < y0 + yb && y0 < x0 + xb) return E8_EINVAL;
  }
  const size_t need = e8_gemm_host_workspace_bytes(m, M, N, K, bpw);
  if (need == 0) return E8_EINVAL;
  if (!workspace || !aligned16(workspace) || ws_bytes < need) return E8_EWORKSPACE;
  (void)cudaGetLastError();  // a failed earlier launch must not be reported here
  const int dc = check_device(cb);
  if (dc != E8_OK) return dc;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  uint16_t* Xd = reinterpret_cast<uint16_t*>(w);
  float* Yd = reinterpret_cast<float*>(w + round256(xb));
  uint8_t* inner = w + round256(xb) + round256(yb);
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemcpyAsync(Xd, X_host, xb, cudaMemcpyHostToDevice, st) != cudaSuccess) return E8_ECUDA;
  const int rc = e8_gemm(cb, Xd, M, idx1, idx2, N, K, bpw, rht_seed, scale, Yd, m, inner,
                         ws_bytes - round256(xb) - round256(yb), stream);
  if (rc != E8_OK) return rc;
  if (cudaMemcpyAsync(Y_host, Yd, yb, cudaMemcpyDeviceToHost, st) != cudaSuccess) return E8_ECUDA;
  return E8_OK;
}

int e8_act_rht_q8(const uint16_t* X, int64_t M, int64_t K, uint64_t rht_seed, void* buf,
                  void* stream) {
  (void)cudaGetLastError();  // a failed earlier launch must not be reported here
  if (M < 0 || !valid_k(K)) return E8_EINVAL;
  if (M == 0) return E8_OK;
  if (!e8::q8_eligible(M, K)) return E8_EINVAL;
  if (!X || !buf || !aligned16(X) || !aligned16(buf)) return E8_EINVAL;
  const int64_t rows = rows_b_for(M);
  const e8::Q8Layout l = e8::q8_layout(M, K, rows);
  uint8_t* b = static_cast<uint8_t*>(buf);
  return cuda_status(e8::launch_act_q8(X, M, K, rht_seed, reinterpret_cast<int8_t*>(b),
                                       reinterpret_cast<float*>(b + l.scales_off), rows,
                                       (cudaStream_t)stream, 0));
}

size_t e8_act_q8_bytes(int64_t M, int64_t K) {
  if (M < 1 || !valid_k(K) || !e8::q8_eligible(M, K)) return 0;
  return e8::q8_layout(M, K, rows_b_for(M)).total;
}

int e8_gemm_xt(const e8_codebook* cb, const void* xq, int64_t M, const uint16_t* idx1,
               const void* idx2, int64_t N, int64_t K, int bpw, float scale, float* Y,
               void* stream) {
  (void)cudaGetLastError();  // a failed earlier launch must not be reported here
  int rc = check_device(cb);
  if (rc != E8_OK) return rc;
  if (M < 0 || N < 0 || !valid_k(K) || !valid_bpw(bpw) || !(scale > 0.0f) ||
      !std::isfinite(scale))
    return E8_EINVAL;
  if ((bpw == 2) != (idx2 == nullptr)) return E8_EINVAL;
  if (N > INT32_MAX) return E8_EINVAL;
  if (M == 0 || N == 0) return E8_OK;
  if (!e8::q8_eligible(M, K)) return E8_EINVAL;
  if (!xq || !idx1 || !Y || !aligned16(xq) || !aligned16(idx1) || !aligned16(Y) ||
      (idx2 && !aligned16(idx2)))
    return E8_EINVAL;
  const int64_t rows = rows_b_for(M);
  const e8::Q8Layout l = e8::q8_layout(M, K, rows);
  const uint8_t* b = static_cast<const uint8_t*>(xq);
  e8::ActQ8Args a;
  a.Xq = reinterpret_cast<const int8_t*>(b);
  a.scales = reinterpret_cast<const float*>(b + l.scales_off);
  a.M = M;
  a.N = N;
  a.K = K;
  a.rows_b = (int)rows;
  a.idx1 = idx1;
  a.idx2 = idx2;
  a.bpw = bpw;
  a.alpha = alpha_of(scale, e8::hadamard_block(K), bpw);
  a.Y = Y;
  a.pdl = 1;          // table and codes are read before the previous kernel ends
  a.early_codes = 1;
  return cuda_status(e8::launch_act_gemm_q8(dev_view(cb), a, cb->sm_count, (cudaStream_t)stream));
}

int e8_gemm_xt_rows(int64_t M) { return M < 0 ? 0 : rows_b_for(M); }

size_t e8_gemm_grouped_workspace_bytes(int64_t M, int64_t K, int bpw, int count) {
  if (M < 1 || !valid_k(K) || !valid_bpw(bpw) || count < 1 || count > E8_GROUP_MAX ||
      !e8::q8_eligible(M, K))
    return 0;
  return (size_t)count * e8::q8_layout(M, K, rows_b_for(M)).total;
}

int e8_gemm_grouped(const e8_codebook* cb, const uint16_t* X, int64_t M, int64_t K, int bpw,
                    const e8_gemm_item* items, int count, void* workspace, size_t ws_bytes,
                    void* stream) {
  // every argument and the workspace are checked before the first CUDA call
  if (!cb || !items || count < 1 || count > E8_GROUP_MAX || M < 0 || !valid_k(K) ||
      !valid_bpw(bpw))
    return E8_EINVAL;
  for (int g = 0; g < count; ++g) {
    const e8_gemm_item& it = items[g];
    if (it.N < 0 || it.N > INT32_MAX || !e8::valid_scale(it.scale) ||
        (it.N > 0 && (bpw == 2) != (it.idx2 == nullptr)))
      return E8_EINVAL;
    if (it.N > 0 && M > 0 &&
        (!it.idx1 || !it.Y || !aligned16(it.idx1) || !aligned16(it.Y) ||
         (it.idx2 && !aligned16(it.idx2))))
      return E8_EINVAL;
  }
  if (M == 0) return E8_OK;
  if (!e8::q8_eligible(M, K) || !X || !aligned16(X)) return E8_EINVAL;
  const size_t need = e8_gemm_grouped_workspace_bytes(M, K, bpw, count);
  if (!workspace || !aligned16(workspace) || ws_bytes < need) return E8_EWORKSPACE;
  int nonempty = 0;
  for (int g = 0; g < count; ++g) nonempty += items[g].N > 0 ? 1 : 0;
  if (nonempty == 0) return E8_OK;
  (void)cudaGetLastError();  // a failed earlier launch must not be reported here
  int rc = check_device(cb);
  if (rc != E8_OK) return rc;
  const int64_t rows = rows_b_for(M);
  const e8::Q8Layout l = e8::q8_layout(M, K, rows);
  const int64_t nh = e8::hadamard_block(K);
  e8::ActQ8Out outs[e8::kMaxGroup];
  e8::Q8Item its[e8::kMaxGroup];
  int n = 0;
  for (int g = 0; g < count; ++g) {
    const e8_gemm_item& it = items[g];
    if (it.N == 0) continue;   // nothing to compute for an empty matrix
    uint8_t* buf = static_cast<uint8_t*>(workspace) + (size_t)g * l.total;
    outs[n].seed = it.rht_seed;
    outs[n].Xq = reinterpret_cast<int8_t*>(buf);
    outs[n].scales = reinterpret_cast<float*>(buf + l.scales_off);
    outs[n].Yz = it.Y;   // zeroed by the transform, accumulated into by the GEMM
    outs[n].yz_elems = M * it.N;
    its[n].idx1 = it.idx1;
    its[n].idx2 = it.idx2;
    its[n].N = it.N;
    its[n].alpha = alpha_of(it.scale, nh, bpw);
    its[n].Xq = outs[n].Xq;
    its[n].scales = outs[n].scales;
    its[n].Y = it.Y;
    ++n;
  }
  cudaStream_t st = (cudaStream_t)stream;
  // programmatic launches, as the single-matrix int8 path: the GEMM's prologue
  // and index loads overlap the transform, which writes only the workspace and Y
  cudaError_t e = e8::launch_act_q8_group(X, M, K, outs, n, rows, st, 1);
  if (e != cudaSuccess) return E8_ECUDA;
  e = e8::launch_gemm_q8_group(dev_view(cb), its, n, M, K, (int)rows, bpw, 1, 1, cb->sm_count,
                               st);
  return cuda_status(e);
}

int e8_sync_status(const e8_codebook* cb, void* stream) {
  int rc = check_device(cb);
  if (rc != E8_OK) return rc;
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return E8_ECUDA;
  uint32_t s = 0;
  if (cudaMemcpy(&s, cb->status, sizeof(s), cudaMemcpyDeviceToHost) != cudaSuccess) return E8_ECUDA;
  if (s != 0 && cudaMemset(cb->status, 0, sizeof(s)) != cudaSuccess) return E8_ECUDA;
  if (s & (e8::kDevTimeoutFull | e8::kDevTimeoutEmpty | e8::kDevTimeoutMma | e8::kDevTimeoutCluster))
    return E8_ETIMEOUT;
  if (s & e8::kDevWorklistOverflow) return E8_EWORKSPACE;
  if (s & e8::kDevBadStream) return E8_EDATA;
  if (s & e8::kDevBadInput) return E8_EINVAL;
  return E8_OK;
}

int e8_debug_wait_timeout(const e8_codebook* cb, int wait_ms, void* stream) {
  (void)cudaGetLastError();  // a failed earlier launch must not be reported here
  int rc = check_device(cb);
  if (rc != E8_OK) return rc;
  if (wait_ms < 1 || wait_ms > 5000) return E8_EINVAL;
  return cuda_status(e8::launch_wait_never_signalled(cb->status, (uint64_t)wait_ms * 1000000ull,
                                                     (cudaStream_t)stream));
}

}  // extern "C"
