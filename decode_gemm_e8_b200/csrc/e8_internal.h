// Declarations shared between the kernel translation units and the C ABI layer.
#pragma once

#include <cmath>
#include <cstdint>
#include <cuda_runtime.h>

#include "e8_codebook.cuh"
#include "e8_common.cuh"

// The opaque handle of include/e8.h: device tables of one codebook.
struct e8_codebook {
  int device;
  int sm_count;
  int8_t* vecs;
  uint32_t* table;
  uint32_t* h8table;
  uint32_t* hkeys;
  uint32_t* hvals;
  int32_t* clist;     // indices of the kept norm-12 points with x1 = 0, |x2| = 2
  uint32_t* status;
  int max_probe;
  int clist_len;
};

namespace e8 {

// Argument rules shared by every C entry point (one definition, so that the
// entry points that must agree -- e8_gemm in E8_GEMM_ACT_RHT and
// e8_gemm_act_noalloc, for instance -- cannot drift apart).
constexpr int64_t kMaxNh = 32768;
// K: positive multiple of 8 whose Hadamard block is at most 32768.
inline bool valid_k(int64_t K) { return K >= 8 && (K % 8) == 0 && hadamard_block(K) <= kMaxNh; }
inline bool valid_bpw(int bpw) { return bpw >= 2 && bpw <= 4; }
inline bool valid_scale(float s) { return s > 0.0f && std::isfinite(s); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// Shapes of the activation-side GEMM (E8_GEMM_ACT_RHT and _SMEM).
inline bool act_shape_ok(int64_t M, int64_t K) { return M <= 64 && (K % 128) == 0; }
// Hadamard block: 0 selects the default (the largest power of two dividing K);
// an explicit block is a power of two in [8, 32768] that divides K.
inline bool valid_nh(int64_t K, int64_t nh) {
  return nh == 0 || (nh >= 8 && nh <= kMaxNh && (nh & (nh - 1)) == 0 && (K % nh) == 0);
}
inline int64_t resolve_nh(int64_t K, int64_t nh) { return nh ? nh : hadamard_block(K); }
// Integer multiplier of the group vectors: z = m (c1 + beta c2).
inline int m_of(int bpw) { return bpw == 2 ? 2 : (bpw == 3 ? 4 : 8); }
// Decode constant alpha = fl32(scale / (m sqrt(n_h))), computed in binary64.
inline float alpha_of(float scale, int64_t nh, int bpw) {
  return (float)((double)scale / ((double)m_of(bpw) * std::sqrt((double)nh)));
}

// One group that the encoder's fast path could not decide exactly.
struct WorkItem {
  float u[8];      // transformed, scaled weights of the group
  int64_t group;   // global group index (row * K/8 + column / 8)
  uint32_t mask;   // kWork* bits
  uint32_t cand;   // with kWorkStage*List: best index outside the listed set
};
static_assert(sizeof(WorkItem) == 48, "WorkItem layout");
enum : uint32_t {
  kWorkStage1 = 1u,       // stage 1 undecided
  kWorkStage2 = 2u,       // stage 2 undecided (or pending behind stage 1)
  kWorkStage1List = 4u,   // stage 1: only the listed set and `cand` compete
  kWorkStage2List = 8u,   // stage 2: likewise
};

int build_codebook_tables(int8_t* d_vecs, uint32_t* d_table, uint32_t* d_h8table,
                          uint32_t* d_hkeys, uint32_t* d_hvals, int* h_max_probe, cudaStream_t st);
// Fills clist with the codebook indices of the norm-12 entries with x1 = 0 and
// |x2| = 2 (doubled: 0 and 4); returns their number or -1.
int build_codebook_clist(const int8_t* d_vecs, int32_t* d_clist, cudaStream_t st);
constexpr int kCListCap = 2048;

int encode_elems_per_cta(int nh);
// Encoder workspace: four item counters (256 bytes), then two item regions of
// `work_cap` items each.
cudaError_t launch_encode(const DeviceCodebook& cb, const float* W, int64_t N, int64_t K, int bpw,
                          uint64_t seed, float gamma, uint16_t* idx1, void* idx2,
                          WorkItem* work, uint32_t* work_count, uint64_t work_cap, float* U,
                          int do_quantise, int sm_count, cudaStream_t st, int64_t nh = 0);
cudaError_t launch_encode_leader(const DeviceCodebook& cb, const WorkItem* in,
                                 const uint32_t* in_count, uint64_t cap, WorkItem* out,
                                 uint32_t* out_count, int bpw, uint16_t* idx1, void* idx2,
                                 int sm_count, cudaStream_t st);

cudaError_t launch_decode(const DeviceCodebook& cb, const uint16_t* idx1, const void* idx2,
                          int64_t N, int64_t K, int bpw, uint64_t seed, float alpha,
                          uint16_t* Wdec, int sm_count, cudaStream_t st, int64_t nh = 0);
// Tensor-core decoder (n_h = 1024, 2048, 4096; N K a multiple of 8192;
// 16-byte aligned buffers); same contract and bit-identical result as
// launch_decode.  Returns cudaErrorNotSupported, launching nothing, for other
// shapes.
bool decode_tc_eligible(int64_t N, int64_t K, const void* idx1, const void* idx2,
                        const void* out, int64_t nh = 0);
cudaError_t launch_decode_tc(const DeviceCodebook& cb, const uint16_t* idx1, const void* idx2,
                             int64_t N, int64_t K, int bpw, uint64_t seed, float alpha,
                             uint16_t* Wdec, int sm_count, cudaStream_t st, int64_t nh = 0);

// X [M][K] bf16 -> Xt [rows][K] bf16: rows [0, M) hi parts, [M, 2M) lo parts of
// FWHT(D x), rows [2M, rows) zero.
cudaError_t launch_act_rht(const uint16_t* X, int64_t M, int64_t K, uint64_t seed, uint16_t* Xt,
                           int64_t rows, cudaStream_t st, int pdl = 0, int64_t nh = 0);

// Fused decode + GEMM with the transform moved onto the activations:
// Y[m][n] = alpha * sum_k Xt[m][k] Z[n][k] (hi + lo rows), Z decoded on chip.
struct ActGemmArgs {
  const uint16_t* Xt;   // [rows_b][K], rows_b = padded 2M
  int64_t M, N, K;
  int rows_b;           // MMA N dimension (16..256, multiple of 16)
  const uint16_t* idx1;
  const void* idx2;
  int bpw;
  float alpha;
  float* Y;             // [M][N] fp32
  int variant;          // 0: decoded operand in shared memory, 1: in tensor memory
  int pdl;              // 1: launch with programmatic stream serialization
  int early_codes;      // 1: codes may be fetched before the predecessor kernel ends
};
cudaError_t launch_act_gemm(const DeviceCodebook& cb, const ActGemmArgs& a, int sm_count,
                            cudaStream_t st);

// int8 path for up to 32 tokens: Xq int8 [rows_b][K] (token m: rows 2m, 2m + 1),
// per-token steps and per-row column sums from launch_act_q8.  The kernel adds
// its partial tiles into Y, which must hold zeros when it starts (the
// transform kernel zeroes it when given Y).
struct ActQ8Args {
  const int8_t* Xq;
  const float* scales;   // [M]
  int64_t M, N, K;
  int rows_b;
  const uint16_t* idx1;
  const void* idx2;
  int bpw;
  float alpha;
  float* Y;
  int pdl;
  int early_codes;
};
cudaError_t launch_act_gemm_q8(const DeviceCodebook& cb, const ActQ8Args& a, int sm_count,
                               cudaStream_t st);

// Grouped int8 path: up to kMaxGroup weight matrices that share K, bpw and the
// token count, each with its own transformed activations (its own RHT seed),
// alpha and output, in one launch whose stream-K units run over the
// concatenated 128-row tiles of all of them.
constexpr int kMaxGroup = 4;
struct Q8Item {
  const uint16_t* idx1;
  const void* idx2;
  int64_t N;
  float alpha;
  const int8_t* Xq;       // [rows_b][K], token m: rows 2m, 2m + 1
  const float* scales;    // [M]
  float* Y;               // [M][N], zero when the kernel starts
};
cudaError_t launch_gemm_q8_group(const DeviceCodebook& cb, const Q8Item* items, int count,
                                 int64_t M, int64_t K, int rows_b, int bpw, int pdl,
                                 int early_codes, int sm_count, cudaStream_t st);
// When Yz is not null the kernel also zeroes Yz[0, yz_elems) (the fp32 output
// that launch_act_gemm_q8 accumulates into), after the preceding kernel ends.
cudaError_t launch_act_q8(const uint16_t* X, int64_t M, int64_t K, uint64_t seed, int8_t* Xq,
                          float* scales, int64_t rows, cudaStream_t st, int pdl,
                          float* Yz = nullptr, int64_t yz_elems = 0, int64_t nh = 0);
// One output set of the grouped transform: X transformed with `seed` into
// Xq / scales, and Yz[0, yz_elems) zeroed (Yz may be null).
struct ActQ8Out {
  uint64_t seed;
  int8_t* Xq;
  float* scales;
  float* Yz;
  int64_t yz_elems;
};
// The same transform for up to kMaxGroup seeds in one launch.
cudaError_t launch_act_q8_group(const uint16_t* X, int64_t M, int64_t K, const ActQ8Out* outs,
                                int count, int64_t rows, cudaStream_t st, int pdl,
                                int64_t nh = 0);

// Layout of the int8 activation buffer: Xq [rows][K] int8, then the per-token
// steps (fp32 [M]), each part starting on a 256-byte boundary.
struct Q8Layout {
  size_t scales_off, total;
};
inline Q8Layout q8_layout(int64_t M, int64_t K, int64_t rows) {
  auto r256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  Q8Layout l;
  l.scales_off = r256((size_t)rows * (size_t)K);
  l.total = l.scales_off + r256((size_t)M * 4);
  return l;
}
// Shapes served by the int8 path: up to 32 tokens, K a multiple of 256 whose
// Hadamard block lies in 256..4096, K <= 32768.
inline bool q8_eligible(int64_t M, int64_t K, int64_t nh = 0) {
  if (nh == 0) nh = K & (-K);
  return M >= 1 && M <= 32 && (K % 256) == 0 && (K % nh) == 0 && nh >= 256 && nh <= 4096 &&
         K <= 32768;
}

// Activation-side GEMM (E8_GEMM_ACT_RHT / _SMEM) on caller-provided scratch of
// act_scratch_bytes() bytes: the transform and the fused kernel.
size_t act_scratch_bytes(int64_t M, int64_t K, int smem_variant, int64_t nh = 0);
cudaError_t run_act_gemm(const e8_codebook* cb, const uint16_t* X, int64_t M,
                         const uint16_t* idx1, const void* idx2, int64_t N, int64_t K, int bpw,
                         uint64_t seed, float alpha, float* Y, int smem_variant, void* scratch,
                         cudaStream_t st, int64_t nh = 0);

// Entropy-coded E8 variant (e8_ep.cu).
constexpr int kEpBlockGroups = 64;    // groups of 8 weights per independently decodable block
constexpr int kEpTableWords = 770;    // frequency tables: c, m|0, m|1, q|0, q|1
int64_t ep_num_blocks(int64_t N, int64_t K);
int64_t ep_max_words(int64_t N, int64_t K);
size_t ep_encode_workspace_bytes(int64_t N, int64_t K);
// 0 ok, 1 CUDA error, 2 frequency normalisation impossible, 3 stream longer
// than max_words.  Synchronises the stream.
int ep_encode(const float* W, int64_t N, int64_t K, float delta, uint16_t* words,
              int64_t max_words, uint32_t* offsets, float* t, uint16_t* tables, void* ws,
              uint32_t* status, int sm_count, cudaStream_t st, int64_t* total_words);
int ep_estimate_bpp(const float* W, int64_t N, int64_t K, float delta, void* ws,
                    uint32_t* status, int sm_count, cudaStream_t st, double* bpp);
cudaError_t launch_ep_decode(const uint16_t* words, int64_t n_words, const uint32_t* offsets,
                             const float* t, const uint16_t* tables, int64_t N, int64_t K,
                             uint16_t* out, uint32_t* status, int sm_count, cudaStream_t st);

// Dense Y[M][N] fp32 = X[M][K] bf16 * W[N][K]^T bf16 on tcgen05.
cudaError_t launch_dense_gemm(const uint16_t* X, int64_t M, const uint16_t* W, int64_t N,
                              int64_t K, float* Y, uint32_t* status, int sm_count,
                              cudaStream_t st);

// Reference-quality CUDA-core GEMM used by the simt mode (diagnostics).
cudaError_t launch_simt_gemm(const uint16_t* X, int64_t M, const uint16_t* W, int64_t N,
                             int64_t K, float* Y, cudaStream_t st);

// Failure-detection check: a bounded wait on a barrier nobody signals.
cudaError_t launch_wait_never_signalled(uint32_t* status, uint64_t limit_ns, cudaStream_t st);

}  // namespace e8
