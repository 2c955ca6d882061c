/*
 * libe8 -- E8 lattice-codebook weights decoded on a B200 (sm_100a) GPU and
 * fed into a bf16 tensor-core GEMM, plus the data-parallel encoder.
 *
 * The method is the one described on the PyPI page of "glq 0.1.1"
 * (section "How it works" and the "Bit widths" table):
 *   - a codebook of 65536 vectors of the E8 lattice taken from its first seven
 *     shells (squared norms 0, 2, ..., 12); each group of 8 consecutive weights
 *     of a row is replaced by a 16-bit codebook index (2 bits per weight);
 *   - for 3 and 4 bits per weight a second-stage residual codebook adds an
 *     8-bit or a 16-bit index per group;
 *   - before quantisation every weight row is passed through a randomized
 *     Hadamard transform (random sign flips, then a fast Walsh-Hadamard
 *     transform), and each group is mapped to its Euclidean nearest codebook
 *     vector;
 *   - one global scale per layer, no per-group scales, so the storage is
 *     exactly bpw * N * K / 8 bytes plus the scale (and the transform seed).
 *
 * Conventions fixed by this library where the page is silent:
 *   - weights W are [N][K] row-major (output rows, input columns); groups and
 *     the transform run along K; the Hadamard block n_h is the largest power
 *     of two dividing K (block-diagonal transform when K is not a power of
 *     two); n_h must not exceed 32768;
 *   - codebook order: origin first, then shells by increasing norm; inside a
 *     shell the vectors whose first nonzero coordinate is positive, sorted
 *     lexicographically on their coordinates, each followed by its negation;
 *     cut at 65536 entries;
 *   - residual codebook: the first 256 entries at scale 1/2 (3 bpw) or the
 *     whole codebook at scale 1/4 (4 bpw), chosen greedily after stage 1;
 *   - nearest means exact Euclidean distance on the fp32 transformed weights,
 *     ties resolved to the smallest index;
 *   - sign vector: SplitMix64 stream seeded with rht_seed, output word j gives
 *     the signs of columns 64j..64j+63 (bit set = negate);
 *   - forward transform: u = fl32(FWHT(D w) * gamma) in fp32, stages
 *     h = 1, 2, 4, ..., butterfly (a, b) -> (a + b, a - b),
 *     gamma = fl32(1 / (scale * sqrt(n_h)));
 *   - decoded weight: w = bf16_rne(d * fl32(t * alpha)), t = FWHT(z) computed
 *     exactly on the integer group vectors z = m (c1 + beta c2), m = 2, 4, 8
 *     for 2, 3, 4 bpw, alpha = fl32(scale / (m * sqrt(n_h))).
 *
 * General rules for every call below:
 *   - all pointers are device pointers unless a parameter says "host";
 *     device pointers must be 16-byte aligned;
 *   - the caller owns every buffer; only e8_codebook_build allocates (device
 *     tables, freed by e8_codebook_free);
 *   - calls are asynchronous on `stream` (a cudaStream_t, NULL = legacy
 *     default stream) and never synchronise, except e8_codebook_build,
 *     e8_codebook_export and e8_sync_status, which are synchronous;
 *   - the current CUDA device must be the device the codebook was built on;
 *   - N == 0 or M == 0 is a valid empty call that launches nothing;
 *   - argument errors are reported before anything is launched.
 */
#ifndef E8_H
#define E8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define E8_OK 0          /* success */
#define E8_EINVAL 1      /* bad argument: null/misaligned pointer, shape, bpw, scale, mode */
#define E8_EWORKSPACE 2  /* workspace missing or smaller than e8_workspace_bytes() */
#define E8_EDEVICE 3     /* no sm_100 device, or the current device is not the codebook's */
#define E8_ECUDA 4       /* a CUDA runtime or driver call failed */
#define E8_ETIMEOUT 5    /* a kernel gave up on a bounded wait (reported by e8_sync_status) */
#define E8_ENOMEM 6      /* device allocation failed (e8_codebook_build only) */
#define E8_EDATA 7       /* an entropy-coded stream did not decode exactly (e8_sync_status) */

/* GEMM modes (e8_gemm `mode`, and `op` of e8_workspace_bytes). */
#define E8_GEMM_AUTO 0          /* ACT_RHT for M <= 64 and K % 128 == 0, else DECODED_W */
#define E8_GEMM_ACT_RHT 1       /* transform on the activations, codes decoded on chip into
                                   tensor memory, fused tcgen05 GEMM (M <= 64, K % 128 == 0);
                                   int8 MMA for the shapes of e8_act_rht_q8, bf16 otherwise */
#define E8_GEMM_DECODED_W 2     /* decode to a bf16 workspace, then a dense tcgen05 GEMM */
#define E8_GEMM_ACT_RHT_SMEM 3  /* as ACT_RHT, decoded operand staged in shared memory */
#define E8_GEMM_SIMT 4          /* decode to bf16, CUDA-core fp32 GEMM (diagnostic) */
#define E8_OP_ENCODE 100        /* e8_workspace_bytes: workspace of e8_encode */

typedef struct e8_codebook e8_codebook;

/* Builds the canonical codebook tables on CUDA device `device` ("How it
 * works", item 1) and stores an opaque handle in *out.  Synchronous.
 * Allocates about 1.2 MB of device memory.  Errors: E8_EINVAL (out NULL),
 * E8_EDEVICE (device missing or not compute capability 10.x), E8_ENOMEM,
 * E8_ECUDA. */
int e8_codebook_build(e8_codebook** out, int device);

/* Releases the tables of a codebook built by e8_codebook_build (NULL is a no-op). */
void e8_codebook_free(e8_codebook* cb);

/* Copies the 65536 codebook vectors, doubled coordinates (2x, all in [-6, 6]),
 * as int8 [65536][8] into the HOST buffer host_vecs.  Synchronous. */
int e8_codebook_export(const e8_codebook* cb, int8_t* host_vecs);

/* Forward randomized Hadamard transform of every row ("How it works", item 2):
 * U = fl32(FWHT_{n_h}(D W) * gamma), W and U fp32 [N][K] (may not alias).
 * Bit-exact to the sequential definition given at the top of this file. */
int e8_rht_forward(const e8_codebook* cb, const float* W, int64_t N, int64_t K,
                   uint64_t rht_seed, float scale, float* U, void* stream);

/* Encoder ("How it works", items 1-2; "Bit widths" table): W fp32 [N][K] ->
 * idx1 uint16 [N][K/8] and, for bpw 3, idx2 uint8 [N][K/8], for bpw 4 idx2
 * uint16 [N][K/8] (idx2 must be NULL for bpw 2).  scale > 0 is the layer's
 * global scale.  Every index equals the exact nearest codebook point of the
 * transformed, scaled group (smallest index on ties); groups with a
 * non-finite coordinate get index 0.  workspace: at least
 * e8_workspace_bytes(E8_OP_ENCODE, 0, N, K, bpw) bytes, contents ignored.
 * When the call has completed on the stream, the first four uint32 words of
 * the workspace hold diagnostic counts of groups: [0] left open by the
 * Conway-Sloane fast path (one class search per open stage follows), [1]
 * left for the exact brute force after it, [2] stage-2 searches of groups
 * whose stage 1 the brute force settled, [3] of those, left for a second
 * brute force. */
int e8_encode(const e8_codebook* cb, const float* W, int64_t N, int64_t K, int bpw,
              uint64_t rht_seed, float scale, uint16_t* idx1, void* idx2, void* workspace,
              size_t ws_bytes, void* stream);

/* Decoder ("How it works", items 1-2; "Bit widths" table): indices -> bf16
 * weights W_dec [N][K] (raw bf16 bits).  Each group's vector is rebuilt from
 * the codebook (z = m (c1 + beta c2)), the sign flips and the Walsh-Hadamard
 * transform are undone exactly, then the two roundings given at the top of
 * this file are applied; bit-exact.  idx1 / idx2 as e8_encode writes them
 * (idx2 NULL for bpw 2).  Needs no workspace. */
int e8_decode_to_bf16(const e8_codebook* cb, const uint16_t* idx1, const void* idx2, int64_t N,
                      int64_t K, int bpw, uint64_t rht_seed, float scale, uint16_t* W_dec,
                      void* stream);

/* Activation-side transform used by E8_GEMM_ACT_RHT: X bf16 [M][K] ->
 * Xt bf16 [rows][K] with rows >= 2M; row 2m holds hi = bf16(FWHT(D x_m)) and
 * row 2m + 1 holds lo = bf16(FWHT(D x_m) - hi); rows 2M..rows-1 are zeroed.
 * No normalisation is applied (the GEMM multiplies by alpha). */
int e8_act_rht(const uint16_t* X, int64_t M, int64_t K, uint64_t rht_seed, uint16_t* Xt,
               int64_t rows, void* stream);

/* GEMM with compressed weights ("How it works", items 1-2: the weights are
 * rebuilt from their codebook indices and the inverse transform at run time):
 * Y fp32 [M][N] = X bf16 [M][K] * W_dec^T, where
 * W_dec is what e8_decode_to_bf16 returns for (idx1, idx2, scale, rht_seed).
 * In the DECODED_W and SIMT modes the product uses W_dec itself; in the
 * ACT_RHT modes it uses the unrounded decoded weights (relative Frobenius
 * difference to the W_dec product about 1.7e-3, from the bf16 rounding of
 * W_dec).  In E8_GEMM_ACT_RHT with up to 32 tokens (the int8 path, see
 * e8_gemm_xt) the K range of an output is split over several CTAs whose
 * partial sums are added in arrival order (TMA reduce-add, or fp32 atomics
 * when N is not a multiple of 4): the last bits of Y can differ between runs.
 * workspace: at least e8_workspace_bytes(mode, M, N, K, bpw) bytes.
 * Ordering: the int8 path launches its kernels with programmatic dependent
 * launch; its kernels may read X, idx1, idx2 and the codebook
 * before the kernel that precedes the call on the stream has finished, if
 * that kernel releases its dependents early (griddepcontrol.launch_dependents).
 * Kernels that do not release early (every kernel of this library that writes
 * X-sized inputs or indices included) are waited for in full.  Y, the
 * workspace and everything else are written only after the preceding kernel
 * has finished. */
int e8_gemm(const e8_codebook* cb, const uint16_t* X, int64_t M, const uint16_t* idx1,
            const void* idx2, int64_t N, int64_t K, int bpw, uint64_t rht_seed, float scale,
            float* Y, int mode, void* workspace, size_t ws_bytes, void* stream);

/* int8 activation transform, first half of E8_GEMM_ACT_RHT for up to 32
 * tokens: X bf16 [M][K] -> one buffer of e8_act_q8_bytes(M, K) bytes holding
 *   Xq int8 [rows][K], rows = e8_gemm_xt_rows(M): row 2m = q0 and row 2m + 1 =
 *     q1 of token m, where xt = FWHT(D x_m) per Hadamard block,
 *     s_m = max|xt| / 127, q0 = rint(xt / s_m), q1 = rint((xt - q0 s_m) 128 / s_m),
 *     so xt = s_m (q0 + q1 / 128) within s_m / 256; padding rows are zero;
 *   then s_m (fp32 [M]), starting on a 256-byte boundary after Xq.
 * Shapes: 1 <= M <= 32, K a multiple of 256 whose Hadamard block is 256..4096,
 * K <= 32768 (else E8_EINVAL). */
int e8_act_rht_q8(const uint16_t* X, int64_t M, int64_t K, uint64_t rht_seed, void* buf,
                  void* stream);

/* Explicit Hadamard block ("How it works", item 2: the transform is a
 * randomized Hadamard transform of the input dimension; the page does not fix
 * its block size).  The calls without a suffix use the default block, the
 * largest power of two dividing K.  These take the block n_h explicitly: a
 * power of two with 8 <= n_h <= 32768 that divides K (n_h = 0 selects the
 * default), for instance n_h = 128 or 256 for every K, so that every K tile of
 * 128 or 256 columns is transformed on its own.  Everything else -- signs,
 * gamma = fl32(1 / (scale sqrt(n_h))), alpha = fl32(scale / (m sqrt(n_h))),
 * the roundings, the codebooks -- is as above with n_h in place of the
 * default block; codes written with one block must be decoded and multiplied
 * with the same block.  Arguments, results and errors as the calls without the
 * suffix (E8_EINVAL also for an invalid n_h). */
int e8_rht_forward_nh(const e8_codebook* cb, const float* W, int64_t N, int64_t K, int64_t n_h,
                      uint64_t rht_seed, float scale, float* U, void* stream);
int e8_encode_nh(const e8_codebook* cb, const float* W, int64_t N, int64_t K, int64_t n_h,
                 int bpw, uint64_t rht_seed, float scale, uint16_t* idx1, void* idx2,
                 void* workspace, size_t ws_bytes, void* stream);
int e8_decode_to_bf16_nh(const e8_codebook* cb, const uint16_t* idx1, const void* idx2,
                         int64_t N, int64_t K, int64_t n_h, int bpw, uint64_t rht_seed,
                         float scale, uint16_t* W_dec, void* stream);
/* E8_GEMM_ACT_RHT with n_h < 256 takes the bf16 activation path (the int8 one
 * needs 256 <= n_h <= 4096); the workspace is e8_workspace_bytes_nh's. */
int e8_gemm_nh(const e8_codebook* cb, const uint16_t* X, int64_t M, const uint16_t* idx1,
               const void* idx2, int64_t N, int64_t K, int64_t n_h, int bpw, uint64_t rht_seed,
               float scale, float* Y, int mode, void* workspace, size_t ws_bytes, void* stream);
size_t e8_workspace_bytes_nh(int op, int64_t M, int64_t N, int64_t K, int64_t n_h, int bpw);

/* Size in bytes of the e8_act_rht_q8 buffer (0 if the shape is not served). */
size_t e8_act_q8_bytes(int64_t M, int64_t K);

/* Second half of E8_GEMM_ACT_RHT: the fused decode + int8 tensor-core GEMM on
 * a buffer written by e8_act_rht_q8 for the same M, K and rht_seed:
 * Y fp32 [M][N] += alpha * s_m * ((q0 + q1 / 128) . z) over each weight row, z
 * the integer codebook vectors decoded on chip.  The product is ADDED into Y
 * (zero Y first for a plain product); the partial sums of one output, from
 * the CTAs that split its K range, are added with fp32 atomics, so the last
 * bits of Y can differ from run to run (relative differences of order 1e-7).
 * One transform can serve every weight matrix that shares K and rht_seed (for
 * instance q, k and v).  Same shape limits as e8_act_rht_q8.  No workspace. */
int e8_gemm_xt(const e8_codebook* cb, const void* xq, int64_t M, const uint16_t* idx1,
               const void* idx2, int64_t N, int64_t K, int bpw, float scale, float* Y,
               void* stream);

/* Row count of the transformed-activation buffers for M tokens: 2M rounded up to
 * a multiple of 16. */
int e8_gemm_xt_rows(int64_t M);

/* One weight matrix of e8_gemm_grouped: its codes (as e8_encode writes them;
 * idx2 NULL for bpw 2), row count N, transform seed, global scale and output
 * Y fp32 [M][N] (device). */
typedef struct e8_gemm_item {
  const uint16_t* idx1;
  const void* idx2;
  int64_t N;
  uint64_t rht_seed;
  float scale;
  float* Y;
} e8_gemm_item;

#define E8_GROUP_MAX 4

/* Small-batch GEMM of several weight matrices that read the same activations
 * ("How it works", items 1-2: weights rebuilt from their indices and the
 * inverse transform at run time), for instance the q, k and v or the gate and
 * up projections of a decoder layer: for every item,
 *   Y_i = X * W_dec_i^T,
 * as e8_gemm in mode E8_GEMM_ACT_RHT computes it on the int8 path (same
 * accuracy, same arrival-order partial sums), in two launches for the whole
 * group: one activation transform per item seed and one fused decode + GEMM
 * whose work runs over the concatenated row tiles of all items, so the
 * per-launch costs (codebook table load, grid boundaries, tail) are paid once.
 * X bf16 [M][K]; 1 <= M <= 32; K as for e8_act_rht_q8; all items share K and
 * bpw; 1 <= count <= E8_GROUP_MAX; an item with N == 0 is skipped; the Y
 * buffers may not overlap one another, X or the workspace.  workspace: at least
 * e8_gemm_grouped_workspace_bytes(M, K, bpw, count) bytes (the int8
 * activations of every item).  Ordering as e8_gemm's int8 path.  Errors:
 * E8_EINVAL (arguments, shapes, alignment), E8_EWORKSPACE, E8_EDEVICE,
 * E8_ECUDA; all are reported before anything is launched except E8_ECUDA. */
int e8_gemm_grouped(const e8_codebook* cb, const uint16_t* X, int64_t M, int64_t K, int bpw,
                    const e8_gemm_item* items, int count, void* workspace, size_t ws_bytes,
                    void* stream);

/* Workspace bytes for e8_gemm_grouped; 0 if the arguments are invalid. */
size_t e8_gemm_grouped_workspace_bytes(int64_t M, int64_t K, int bpw, int count);

/* E8_GEMM_ACT_RHT without a workspace, for callers that may not allocate device
 * memory where they run the layer: plugins whose host framework owns all
 * device memory and hands them none when they are enqueued, services held to
 * a device-memory budget fixed at start-up, and latency-critical loops that
 * cannot risk an allocation synchronising the device or failing mid-request.
 * The paper has no counterpart; this is a deployment convenience of this
 * library.
 * Same arguments and result as e8_gemm with mode E8_GEMM_ACT_RHT, minus the
 * workspace.  The transformed activations go to a fixed 2 MiB array compiled
 * into the library (every GPU that loads the library holds it until the process
 * exits): requests for which e8_workspace_bytes(E8_GEMM_ACT_RHT, ...) exceeds
 * 2 MiB return E8_EWORKSPACE and launch nothing.  Nothing is allocated.  All calls share that array and it
 * keeps the last call's contents (each call clears what must start at zero);
 * calls whose kernels overlap on the GPU race on it, so order them on one
 * stream.  The first call on a device looks up the array's address on that
 * device; make it before any stream capture begins. */
int e8_gemm_act_noalloc(const e8_codebook* cb, const uint16_t* X, int64_t M,
                        const uint16_t* idx1, const void* idx2, int64_t N, int64_t K, int bpw,
                        uint64_t rht_seed, float scale, float* Y, void* stream);

/* e8_gemm with X and Y in host memory: one call queues, on `stream`, the copy
 * of X (bf16 [M][K], host) into the workspace, the product of e8_gemm in mode
 * `mode` into a device copy of Y, and the copy of that Y (fp32 [M][N]) back
 * to Y_host.  Nothing is waited for: Y_host holds the product once the stream
 * has passed this call.  Page-locked host buffers (cudaHostAlloc /
 * cudaHostRegister) make both copies asynchronous; with pageable memory the
 * CUDA runtime stages them and the call may block until they are done.
 * Arguments are those of e8_gemm; X_host and Y_host must be 16-byte aligned
 * and may not overlap.  workspace: at least
 * e8_gemm_host_workspace_bytes(mode, M, N, K, bpw) bytes of device memory,
 * laid out as [X copy][Y copy][the workspace of e8_gemm], each part on a
 * 256-byte boundary; it must not be used by other work until the stream
 * passes this call.  Errors as e8_gemm (E8_ECUDA also for a failed copy);
 * argument and workspace errors are returned before anything is queued. */
int e8_gemm_host(const e8_codebook* cb, const uint16_t* X_host, int64_t M, const uint16_t* idx1,
                 const void* idx2, int64_t N, int64_t K, int bpw, uint64_t rht_seed,
                 float scale, float* Y_host, int mode, void* workspace, size_t ws_bytes,
                 void* stream);

/* Workspace bytes for e8_gemm_host; 0 if the arguments are invalid. */
size_t e8_gemm_host_workspace_bytes(int mode, int64_t M, int64_t N, int64_t K, int bpw);

/* Mode that E8_GEMM_AUTO selects for these sizes. */
int e8_gemm_auto_mode(int64_t M, int64_t N, int64_t K, int bpw);

/* Workspace bytes for e8_encode (op = E8_OP_ENCODE) or for e8_gemm in mode
 * `op`; 0 if the arguments are invalid or nothing is needed. */
size_t e8_workspace_bytes(int op, int64_t M, int64_t N, int64_t K, int bpw);

/* Synchronises `stream`, then reads and clears the codebook's device status
 * word.  Returns E8_ETIMEOUT if a kernel gave up on a bounded wait since the
 * last call, E8_EWORKSPACE on an encoder work-list overflow, E8_EDATA if an
 * entropy-coded stream did not decode exactly, E8_EINVAL if an entropy-coded
 * encode met a weight outside the quantiser's range (non-finite), E8_ECUDA if
 * the stream reported an error, else E8_OK. */
int e8_sync_status(const e8_codebook* cb, void* stream);

/* ---------------------------------------------------------------------------
 * Entropy-coded E8 variant (page "Transformers Proposes EntroPack Integration
 * for Configurable Non-Integer-Bit-Rate Weight Compression", second paragraph:
 * per-row normalised E8 lattice quantisation, a conditional probability model,
 * entropy coding into independently decodable blocks, fused symbol decoding and
 * weight reconstruction on the GPU; third paragraph: the actual rate counts
 * the metadata).  The page fixes no detail; this library's format:
 *   - row scale t_n = fl32(max_k |w_nk| * delta) (0 when below FLT_MIN), for a
 *     global step delta >= 1/120; u = fl32(w * fl32(1 / t_n)) per group of 8;
 *   - V = the E8 point of u in doubled coordinates chosen by Conway & Sloane's
 *     algorithm in fp32 with fixed tie rules (whole lattice, no codebook);
 *   - decoded weight w' = bf16_rne(fl32(V * fl32(t_n / 2)));
 *   - per group 9 symbols: coset c, seven m_i = (V_i - c) / 2, q = floor(m_7 / 2),
 *     coded by rANS (32-bit state, 16-bit words, 12-bit frequencies) with the
 *     models P(c), P(m | c), P(q | c) counted over the matrix;
 *   - the groups of the row-major matrix in blocks of E8_EP_BLOCK_GROUPS, each
 *     block its own stream of 16-bit words from offsets[b] to offsets[b + 1];
 *   - tables: E8_EP_TABLE_WORDS uint16 frequencies (c[2], m|0[256], m|1[256],
 *     q|0[128], q|1[128]), each model summing to 4096;
 *   - actual bits per weight = (16 words + 32 (blocks + 1) + 32 N
 *     + 16 E8_EP_TABLE_WORDS + 32) / (N K).
 * Shapes: K >= 8, K % 8 == 0, N K / 8 <= 2^31.  The codebook handle only
 * selects the device and carries the status word. */
#define E8_EP_BLOCK_GROUPS 64
#define E8_EP_TABLE_WORDS 770

/* Blocks of an N x K matrix (ceil(N K / 8 / 64)) and the most stream words an
 * encode can produce (9 per group + 2 per block); -1 for an invalid shape. */
int64_t e8_ep_num_blocks(int64_t N, int64_t K);
int64_t e8_ep_max_words(int64_t N, int64_t K);

/* Actual bits per weight of an encoded matrix, metadata included (formula
 * above); -1 for an invalid shape or N = 0. */
double e8_ep_actual_bpp(int64_t N, int64_t K, int64_t total_words);

/* Workspace bytes of e8_ep_encode / e8_ep_estimate_bpp / e8_ep_choose_delta
 * (symbols, block sizes, row scales, histogram), and of e8_ep_gemm (the
 * decoded bf16 weights); 0 for an invalid shape. */
size_t e8_ep_encode_workspace_bytes(int64_t N, int64_t K);
size_t e8_ep_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* Encoder: W fp32 [N][K] (finite) at step delta -> words uint16
 * [max_words >= the stream], offsets uint32 [blocks + 1], t fp32 [N], tables
 * uint16 [E8_EP_TABLE_WORDS]; *total_words (host) = offsets[blocks].
 * Synchronous (it reads the histogram and the block sizes back to the host).
 * E8_EWORKSPACE if max_words is too small or the workspace is. */
int e8_ep_encode(const e8_codebook* cb, const float* W, int64_t N, int64_t K, float delta,
                 uint16_t* words, int64_t max_words, uint32_t* offsets, float* t,
                 uint16_t* tables, int64_t* total_words, void* workspace, size_t ws_bytes,
                 void* stream);

/* Estimated bits per weight at step delta, metadata included (the model's
 * ideal code lengths plus 32 bits of final state per block); synchronous.
 * e8_ep_choose_delta: the smallest step in [1/120, 16] (bisection on log
 * delta) whose estimate is at most target_bpp; synchronous. */
int e8_ep_estimate_bpp(const e8_codebook* cb, const float* W, int64_t N, int64_t K, float delta,
                       double* bpp, void* workspace, size_t ws_bytes, void* stream);
int e8_ep_choose_delta(const e8_codebook* cb, const float* W, int64_t N, int64_t K,
                       double target_bpp, float* delta, void* workspace, size_t ws_bytes,
                       void* stream);

/* Decoder: the compressed form -> bf16 weights out [N][K] (16-byte aligned),
 * one thread per block.  n_words: length of `words` (no read goes past it).
 * A block whose offsets leave [0, n_words], whose stream runs past its end or
 * does not return to the initial state sets E8_EDATA (read by
 * e8_sync_status); its weights are then unspecified. */
int e8_ep_decode_to_bf16(const e8_codebook* cb, const uint16_t* words, int64_t n_words,
                         const uint32_t* offsets, const float* t, const uint16_t* tables,
                         int64_t N, int64_t K, uint16_t* out, void* stream);

/* Y fp32 [M][N] = X bf16 [M][K] * W'^T: the decoder into the workspace
 * (e8_ep_gemm_workspace_bytes), then the dense tcgen05 GEMM of E8_GEMM_DECODED_W. */
int e8_ep_gemm(const e8_codebook* cb, const uint16_t* X, int64_t M, const uint16_t* words,
               int64_t n_words, const uint32_t* offsets, const float* t, const uint16_t* tables,
               int64_t N, int64_t K, float* Y, void* workspace, size_t ws_bytes, void* stream);

/* Failure-detection check (diagnostic): launches one thread that waits on a
 * barrier nothing ever signals, gives up after wait_ms (1..5000) milliseconds
 * and sets the timeout bit of the codebook's status word, the same way every
 * pipeline kernel reports a wait that ran out.  The next e8_sync_status then
 * returns E8_ETIMEOUT; the CUDA context stays usable.  The paper has no
 * counterpart; this exists to test the library's error reporting. */
int e8_debug_wait_timeout(const e8_codebook* cb, int wait_ms, void* stream);

/* Human-readable name of a status code (static string). */
const char* e8_status_str(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int e8_version(void);

#ifdef __cplusplus
}
#endif

#endif /* E8_H */
