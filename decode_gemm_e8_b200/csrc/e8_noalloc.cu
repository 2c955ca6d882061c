// e8_gemm_act_noalloc: the small-batch fused GEMM (E8_GEMM_ACT_RHT) for callers
// that cannot hand the library a workspace.
//
// Some callers may not allocate device memory at the point where they run a
// layer: plugins whose host framework owns every byte of device memory and
// hands them none when they are enqueued, services that run under a fixed
// device-memory budget decided at start-up, and latency-critical loops where
// an allocation could synchronise the device or fail half-way through a
// request.  This entry point keeps its only scratch buffer -- the transformed
// activations -- in a fixed-size array that lives in the library's own device
// image, so it needs neither a workspace argument nor any allocation.
//
// Limits and rules (also stated in include/e8.h):
//   - the scratch is 2 MiB: requests for which e8_workspace_bytes(
//     E8_GEMM_ACT_RHT, M, N, K, bpw) exceeds 2 MiB return E8_EWORKSPACE
//     without launching anything;
//   - every GPU that loads the library keeps this 2 MiB until the process exits;
//   - all calls share the one array and it keeps the last call's contents; the
//     padding rows that must be zero are cleared by every call, but two calls
//     whose kernels overlap on the GPU (different streams without ordering)
//     race on the array and give wrong results;
//   - the first call on each device looks up the array's device address there
//     (cudaGetSymbolAddress, with that device current); make that first call
//     before any stream capture begins.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "e8.h"
#include "e8_common.cuh"
#include "e8_codebook.cuh"
#include "e8_internal.h"

namespace {

constexpr int64_t kNoallocXtElems = 1 << 20;   // 1 Mi bf16 = 2 MiB
constexpr int64_t kNoallocBytes = kNoallocXtElems * 2;
constexpr int kMaxDevices = 64;

// Device-resident scratch: transformed activations of the last call.
static __device__ __align__(256) uint16_t g_noalloc_xt[kNoallocXtElems];

std::mutex g_mu;
void* g_xt_addr[kMaxDevices];   // device address of g_noalloc_xt, per device

// Device address of the scratch array on the current device (looked up once).
int scratch_address(int dev, uint16_t** out) {
  if (dev < 0 || dev >= kMaxDevices) return E8_EDEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_xt_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_xt) != cudaSuccess || !p) return E8_ECUDA;
    g_xt_addr[dev] = p;
  }
  *out = static_cast<uint16_t*>(g_xt_addr[dev]);
  return E8_OK;
}

}  // namespace

extern "C" int e8_gemm_act_noalloc(const e8_codebook* cb, const uint16_t* X, int64_t M,
                                   const uint16_t* idx1, const void* idx2, int64_t N, int64_t K,
                                   int bpw, uint64_t rht_seed, float scale, float* Y,
                                   void* stream) {
  if (!cb) return E8_EINVAL;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return E8_ECUDA;
  if (dev != cb->device) return E8_EDEVICE;
  (void)cudaGetLastError();  // an earlier failed launch must not be reported here
  // the argument rules of e8_gemm in mode E8_GEMM_ACT_RHT (shared helpers)
  if (M < 0 || N < 0 || !e8::valid_k(K) || !e8::valid_bpw(bpw) || !e8::valid_scale(scale))
    return E8_EINVAL;
  if ((bpw == 2) != (idx2 == nullptr)) return E8_EINVAL;
  if (!e8::act_shape_ok(M, K) || N > INT32_MAX || K > INT32_MAX) return E8_EINVAL;
  if (M == 0 || N == 0) return E8_OK;
  const size_t need = e8::act_scratch_bytes(M, K, 0);
  if (need > (size_t)kNoallocBytes) return E8_EWORKSPACE;
  if (!X || !idx1 || !Y || !e8::aligned16(X) || !e8::aligned16(idx1) || !e8::aligned16(Y) ||
      (idx2 && !e8::aligned16(idx2)))
    return E8_EINVAL;
  uint16_t* xt = nullptr;
  int rc = scratch_address(dev, &xt);
  if (rc != E8_OK) return rc;
  const float alpha = e8::alpha_of(scale, e8::hadamard_block(K), bpw);
  const cudaError_t e = e8::run_act_gemm(cb, X, M, idx1, idx2, N, K, bpw, rht_seed, alpha, Y, 0,
                                         xt, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? E8_OK : E8_ECUDA;
}
