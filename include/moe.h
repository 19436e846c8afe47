/*
 * moe.h -- C ABI of libmoe: one FP8 x FP4 Mixture-of-Experts layer forward
 * on a single NVIDIA B200 (sm_100a).
 *
 * What the layer computes.  The MoE forward named in
 *   "DeepSeek DeepGEMM 2026年4月重磅更新：Mega MoE融合算子、FP4精度与极致性能优化"
 *   (chenxutan.com), section 3.1 and 3.2 (dispatch -> linear1 (FP8xFP4) ->
 *   SwiGLU -> linear2 (FP8xFP4) -> combine, fused), section 3.3 (the call's
 *   inputs: x (FP8), x_sf, topk_idx, topk_weights, weights l1 / l2 in FP4 with
 *   UE8M0 scale factors, a caller-allocated BF16 y) and section 4.2 (UE8M0
 *   scale factors packed four per 32-bit int, FP32 accumulation);
 *   "DeepGEMM: DeepSeek 把大模型核心算子打包成一座 CUDA 训练场"
 *   (zevenfang.github.io), section 4 (SM100 consumes packed UE8M0 scales)
 *   and section 5 (the five fused steps).
 * On one GPU, dispatch is an on-device permutation of token rows into
 * expert-contiguous order and combine is an on-device weighted reduction.
 *
 * For every token t and slot s with e = topk_idx[t][s] != -1:
 *   g   = W1[e] . x[t]                       (2I outputs; rows [0,I) gate, [I,2I) up)
 *   a   = silu(g[0:I]) * g[I:2I]             (FP32; silu(z) = z / (1 + exp(-z)))
 *   a'  = E4M3 requantisation of a, one UE8M0 scale per 32 consecutive values,
 *         scale exponent = smallest e with 448 * 2^e >= amax (0 for amax 0)
 *   o_s = W2[e] . a'                         (H outputs)
 *   y[t] = BF16_RNE( sum over s in slot order of topk_w[t][s] * o_s )
 * (This implementation rounds each weighted slot output to BF16 and sums
 * those in FP32 in slot order; against the definition, the error stays
 * within normwise 5e-3 and 2e-2 * (|y| + rms(y)) per element.)
 * All products are block-scaled: every 1x32 block along K of x, W1, W2 and a'
 * carries one UE8M0 scale (value 2^(b-127)).
 *
 * Canonical layouts (row-major, little-endian):
 *   x        uint8  [T, H]        E4M3 codes (OCP e4m3fn: bias 7, max 448, no Inf)
 *   x_sf     int32  [T, H/128]    byte j of word i = UE8M0 scale of K-block 4i+j
 *   topk_idx int32  [T, k]        expert ids; -1 = unused slot
 *   topk_w   fp32   [T, k]
 *   w1       uint8  [E, 2I, H/2]  E2M1 codes, two per byte, low nibble = even k
 *   w1_sf    uint8  [E, 2I, H/32] UE8M0 per 1x32 block
 *   w2       uint8  [E, H, I/2],  w2_sf uint8 [E, H, I/32]
 *   y        uint16 [T, H]        BF16 bits
 *
 * Conventions shared by every entry point:
 *   - Pointers are DEVICE pointers owned by the caller unless the parameter
 *     says "host".  The library never allocates device memory and never
 *     frees anything it did not allocate.
 *   - Arguments are validated on the host before anything is launched; an
 *     invalid call returns an error status and launches nothing.
 *   - moe_plan and moe_forward enqueue work on `stream` and return without
 *     synchronising; data-dependent problems (an expert id outside
 *     [-1, E), a device wait that timed out) are recorded in a status word
 *     inside the workspace and read back by moe_get_device_status.
 *   - A workspace is used by one call sequence at a time; calls that share a
 *     workspace must be ordered on one stream.
 *   - Supported shapes: H % 128 == 0, I % 128 == 0, 1 <= k <= 32,
 *     1 <= E <= 1024, 0 <= T, T * k <= 2^24.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,      /* null pointer, misaligned pointer, negative size */
  MOE_ERR_UNSUPPORTED_SHAPE = 2,/* shape outside the supported set above */
  MOE_ERR_WORKSPACE = 3,        /* workspace too small */
  MOE_ERR_CUDA = 4,             /* a CUDA runtime / driver call failed */
  MOE_ERR_TIMEOUT = 5,          /* device status: a bounded device wait expired */
  MOE_ERR_BAD_EXPERT_ID = 6     /* device status: an id outside [-1, E) was skipped */
} moe_status;

typedef struct {
  int T;    /* tokens */
  int H;    /* hidden size (K of linear1, N of linear2) */
  int I;    /* intermediate size after SwiGLU (linear1 has 2I outputs) */
  int E;    /* experts */
  int topk; /* experts per token */
} moe_shape;

/* Human-readable name of a status code (static storage). */
const char* moe_status_string(moe_status s);

/* Row granularity of the padded expert-contiguous layout (rows of one
 * expert start at a multiple of this).  Returns 128. */
int moe_block_m(void);

/* Cap on the number of SMs used by the persistent kernels (0 = all SMs).
 * "DeepSeek DeepGEMM 2026年4月重磅更新" section 9.2 (set_num_sms).
 * Process-wide; takes effect for calls enqueued afterwards. */
void moe_set_num_sms(int num_sms);

/* Enable (1) or disable (0) programmatic dependent launch between the
 * kernels of one forward.  "DeepSeek DeepGEMM 2026年4月重磅更新" section 6
 * (PDL moves kernel-to-kernel dependencies onto the GPU).  Default 1. */
void moe_set_pdl(int enable);

/* Tiling of the two grouped GEMMs: 0 (default) = one SM per 128 x 256
 * output tile; 1 = SM pairs (thread-block clusters of 2, tcgen05
 * cta_group::2) per 256 x 256 tile, used where the weight row count is a
 * multiple of 256.  Both give identical results.  Process-wide. */
void moe_set_gemm_variant(int variant);

/* Experts with at most `rows` routed rows (0..64; default 0 = off) run with
 * swapped operand roles: the weights take the MMA's M side and the expert's
 * rows the N side (N = rows rounded up to 16), so a decode-sized expert no
 * longer pays for a 128-row tile ("DeepSeek DeepGEMM 2026年4月重磅更新" section
 * 8.1, Dynamic Swap A/B).  moe_plan takes the value current when it is
 * called; changing it between moe_plan and moe_forward is safe (moe_forward
 * runs every expert the plan listed).  0 disables.  Results are the same
 * either way.  Process-wide. */
void moe_set_swap_max(int rows);

/* Narrow tiles for experts with 1..32 routed rows: their A operand stages
 * only 32 rows per 128-K step, which leaves room for a fifth pipeline stage
 * and so a deeper stream of the expert's weights (decode-sized batches are
 * bound by that stream).  -1 (default): on when the layer has at most 128
 * routed rows per expert on average; 0: off; 1: on.  Never with SM-pair
 * tiles.  moe_plan takes the value current when it is called; changing it
 * between moe_plan and moe_forward is safe.  Results are the same either
 * way.  Process-wide. */
void moe_set_narrow_tiles(int mode);

/* ---------------------------------------------------------------- weights */
/* Bytes of one transformed weight: which = 1 for W1, 2 for W2.  Returns the
 * FP4 byte count and writes the scale-factor byte count to *sf_bytes (may
 * be NULL).  Returns 0 for an unsupported shape. */
size_t moe_transformed_bytes(const moe_shape* shape, int which, size_t* sf_bytes);

/* One-time weight transform into the layout the GEMM kernels stream
 * ("DeepSeek DeepGEMM 2026年4月重磅更新" section 3.3,
 * transform_weights_for_mega_moe, FP4 + UE8M0 SF):
 *   - W1 rows are interleaved in 128-row granules (gate rows 128g..128g+127
 *     then up rows I+128g..I+128g+127) so that one 256-row tile holds the
 *     gate and up rows of the same 128 SwiGLU outputs;
 *   - FP4 codes are regrouped K-block-major: [E][K/128][rows][64 bytes], so
 *     that each tile of one K-block is one contiguous run of memory (the
 *     128-byte shared-memory swizzle is applied by the tensor-memory
 *     accelerator on load);
 *   - UE8M0 scales are regrouped into 512-byte chunks [E][K/128][rows/128]
 *     of 128 rows x 4 K-blocks; byte (r%32)*16 + (r/32)*4 + j of a chunk is
 *     row r, K-block j (four UE8M0 per 32-bit word).
 * Inputs are the canonical w1 / w1_sf / w2 / w2_sf (device).  Outputs need
 * moe_transformed_bytes() bytes each, 256-byte aligned, and must not alias
 * the inputs.  Enqueued on `stream`. */
moe_status moe_transform_weights(const moe_shape* shape, const uint8_t* w1, const uint8_t* w1_sf,
                                 const uint8_t* w2, const uint8_t* w2_sf, void* w1_t,
                                 void* w1_sf_t, void* w2_t, void* w2_sf_t, moe_stream_t stream);

/* -------------------------------------------------------------- workspace */
/* Bytes of workspace one forward needs for this shape: the plan, the
 * permuted activations and their scales, the requantised intermediate and
 * its scales, and the BF16 weighted partial outputs.  It is an upper bound
 * over every possible routing (rows padded per expert to moe_block_m()). */
size_t moe_workspace_bytes(const moe_shape* shape);

/* ------------------------------------------------------------------- plan */
/* Routing plan (the dispatch bookkeeping of "DeepSeek DeepGEMM 2026年4月重磅
 * 更新" section 3.1): per-expert histogram of topk_idx, exclusive prefix sum,
 * padded offsets (multiples of moe_block_m()), the row of every assignment
 * (rows of one expert ordered by ascending t*k+s) and the tile schedule.
 * topk_idx: device int32 [T, k].  workspace: device, 256-byte aligned,
 * at least moe_workspace_bytes(shape) bytes.  Resets the device status word.
 * Enqueued on `stream`; nothing is synchronised. */
moe_status moe_plan(const moe_shape* shape, const int32_t* topk_idx, void* workspace,
                    size_t ws_bytes, moe_stream_t stream);

/* ---------------------------------------------------------------- forward */
/* The layer forward, using the plan already in `workspace` (moe_plan must be
 * enqueued before it on the same stream with the same topk_idx):
 * permute -> grouped GEMM1 + SwiGLU + E4M3 requant -> grouped GEMM2 x topk_w
 * -> per-token combine into BF16.  x, x_sf, topk_w in canonical layout;
 * w1_t / w1_sf_t / w2_t / w2_sf_t from moe_transform_weights; y: device
 * uint16 [T, H] written completely.  All device pointers 16-byte aligned
 * (transformed weights and workspace 256-byte aligned).  Enqueued on
 * `stream`; nothing is synchronised. */
moe_status moe_forward(const moe_shape* shape, const uint8_t* x, const int32_t* x_sf,
                       const int32_t* topk_idx, const float* topk_w, const void* w1_t,
                       const void* w1_sf_t, const void* w2_t, const void* w2_sf_t, uint16_t* y,
                       void* workspace, size_t ws_bytes, moe_stream_t stream);

/* Host-buffer variant for callers whose activations live in host memory:
 * copies x / x_sf / topk_idx / topk_w (HOST, preferably pinned) to the
 * device staging area at the end of `workspace`, runs moe_plan and
 * moe_forward, copies y back to `y_host` (HOST) and synchronises `stream`.
 * Needs moe_workspace_bytes_host(shape) bytes of workspace. */
size_t moe_workspace_bytes_host(const moe_shape* shape);
moe_status moe_forward_host(const moe_shape* shape, const uint8_t* x_host,
                            const int32_t* x_sf_host, const int32_t* topk_idx_host,
                            const float* topk_w_host, const void* w1_t, const void* w1_sf_t,
                            const void* w2_t, const void* w2_sf_t, uint16_t* y_host,
                            void* workspace, size_t ws_bytes, moe_stream_t stream);

/* A sequence of n_batches independent host-buffer forwards of one shape, for
 * a caller that feeds successive micro-batches from host memory.  Batch i
 * reads x_host[i], x_sf_host[i], topk_idx_host[i], topk_w_host[i] and writes
 * y_host[i] (HOST arrays of HOST pointers, layouts as for moe_forward_host;
 * batches may share input buffers; a y buffer that several batches share
 * ends up holding the last of them).  The copies run on two streams of
 * the call's own: batch i + 1's inputs go up and batch i - 1's y comes down
 * while batch i's kernels run on `stream`, through two staging slots at the
 * end of `workspace`, which needs moe_workspace_bytes_host_pipelined(shape)
 * bytes.  The copies only overlap when the host buffers are pinned; pageable
 * buffers give the same results at the speed of moe_forward_host.  The call
 * creates two streams and seven events and destroys them before it returns;
 * it returns after every copy-out has landed (also when it fails part-way,
 * with the first error).  n_batches < 0 or a NULL pointer: INVALID_ARG
 * before anything is enqueued; T == 0 or n_batches == 0: MOE_OK, nothing done. */
size_t moe_workspace_bytes_host_pipelined(const moe_shape* shape);
moe_status moe_forward_host_pipelined(const moe_shape* shape, int n_batches,
                                      const uint8_t* const* x_host,
                                      const int32_t* const* x_sf_host,
                                      const int32_t* const* topk_idx_host,
                                      const float* const* topk_w_host, const void* w1_t,
                                      const void* w1_sf_t, const void* w2_t,
                                      const void* w2_sf_t, uint16_t* const* y_host,
                                      void* workspace, size_t ws_bytes, moe_stream_t stream);

/* ---------------------------------------------------- allocation-free call */
/* The pages describe no counterpart of this entry point.  It is for callers
 * that cannot call cudaMalloc themselves: a serving runtime whose memory
 * manager reserves the free device memory at start-up for its own pool (a
 * further cudaMalloc would fail, or would take memory the pool counts on),
 * or a plug-in / custom operator inside another framework that is handed
 * only its input and output buffers and has no way to reach that
 * framework's allocator for scratch space.  It performs moe_plan + moe_forward with the
 * workspace taken from a fixed 32 MiB array inside the library (a
 * file-scope __device__ array: every GPU that loads the library holds those
 * 32 MiB until the process exits).  The caller passes the inputs and y
 * exactly as for moe_forward (device pointers, canonical layouts,
 * transformed weights).
 *   - Shapes whose moe_workspace_bytes() exceeds 32 MiB are rejected with
 *     MOE_ERR_WORKSPACE before anything is launched (for example T = 256,
 *     H = 2048, I = 1024, E = 8, top-2 fits; the large workloads do not).
 *   - The first call on a device looks up the array's device address, with
 *     that device current.
 *   - Nothing is allocated: no cudaMalloc, no cudaFree, no allocating
 *     library routine.  The header part of the array is cleared by every
 *     call; the rest keeps the last call's contents and is rewritten before
 *     it is read.
 *   - All calls share the one array: calls whose GPU work overlaps (two
 *     streams, two host threads) race and corrupt each other.  Order them
 *     on one stream.
 * Data-dependent problems (bad expert ids, device timeouts) are recorded in
 * the array's status word as for moe_forward. */
moe_status moe_forward_noalloc(const moe_shape* shape, const uint8_t* x, const int32_t* x_sf,
                               const int32_t* topk_idx, const float* topk_w, const void* w1_t,
                               const void* w1_sf_t, const void* w2_t, const void* w2_sf_t,
                               uint16_t* y, moe_stream_t stream);

/* ------------------------------------------------------------- diagnostics */
/* Synchronises `stream` and returns the device status word of the last
 * plan / forward that used `workspace` (MOE_OK, MOE_ERR_BAD_EXPERT_ID or
 * MOE_ERR_TIMEOUT), or MOE_ERR_CUDA if the stream itself failed. */
moe_status moe_get_device_status(const void* workspace, moe_stream_t stream);

/* Synchronises `stream` and returns where the first bounded device wait of
 * the last forward on `workspace` expired: 0 none; 10 + j the TMA producer,
 * 20 + j the MMA issuer, 30 + j the epilogue warps of the one-SM grouped
 * GEMM, with j = 1 for linear1, 2 for linear2, 3 for the standalone GEMM;
 * 40 + j, 50 + j, 60 + j the same roles in the SM-pair kernel; 70 + j,
 * 80 + j, 90 + j in the swapped-role kernel; in the FP4 indexer 110-114 the
 * producer (key stage, weight slot, query slot, end, query-slot release),
 * 120 / 121 the first / second MMA thread, 130 the epilogue warps (the same
 * workspace word, read after moe_fp8_fp4_mqa_logits).  -1 if the stream
 * failed.
 * Every wait on another role of the kernel is bounded (2 s for a stage's
 * data, 4 s for the waits that can only end after such a stage); when one
 * expires the kernel records MOE_ERR_TIMEOUT and this site, the other roles
 * of the CTA stop waiting, copies and MMAs already in flight are waited for,
 * tensor memory is freed and the kernel returns. */
int moe_get_timeout_site(const void* workspace, moe_stream_t stream);

/* Test hook for the failure path above (the pages' change list fixes a
 * kernel hang; this checks that a wait which never ends is reported instead):
 * in every following moe_forward, the producer of each CTA of the linear1
 * kernel (one-SM tiles, normal m-tiles) skips the loads of its pipeline
 * iteration `skip_iteration` (-1: off), and the waits of that kernel use
 * `wait_limit_ns` for a stage's data and twice that otherwise (0: the
 * defaults above).  In every following moe_fp8_fp4_mqa_logits the producer
 * of each CTA leaves the first key stage of its active tile number
 * `skip_iteration` unfilled, with the same wait limits.  Process-wide; both
 * off by default. */
void moe_debug_set_fault(int skip_iteration, unsigned long long wait_limit_ns);

/* Copies the plan out of `workspace` for bit-exact checking (synchronises
 * `stream`).  All outputs are HOST buffers: counts [E], offs [E+1],
 * padded_offs [E+1], row_of [T*k] (-1 for skipped slots), src_of [P] where
 * P = padded_offs[E] (-1 for padding rows); *P_out receives P.  src_of may be
 * NULL; otherwise it must hold moe_plan_max_rows(shape) entries. */
int moe_plan_max_rows(const moe_shape* shape);
moe_status moe_plan_export(const moe_shape* shape, const void* workspace, int32_t* counts,
                           int32_t* offs, int32_t* padded_offs, int32_t* row_of, int32_t* src_of,
                           int32_t* P_out, moe_stream_t stream);

/* Kernel timing: when `events` is not NULL and n >= 5, every following
 * moe_forward records events[0..4] (cudaEvent_t handles owned by the
 * caller) on its stream: before the permute kernel, after it, after the
 * linear1 kernels, after the linear2 kernels (normal, narrow and swapped-role
 * tiles each) and after the combine kernel.
 * NULL stops it.  Process-wide; the handles must outlive their use. */
void moe_set_timing_events(void* const* events, int n);

/* Test hook: runs the GEMM1 epilogue's requantiser on `a` (device fp32
 * [rows, cols], cols % 32 == 0) and writes E4M3 codes (device uint8
 * [rows, cols]) and UE8M0 bytes (device uint8 [rows, cols/32]).  Same
 * device code as the fused epilogue. */
moe_status moe_debug_requant(const float* a, int rows, int cols, uint8_t* codes, uint8_t* sbytes,
                             moe_stream_t stream);

/* ------------------------------------------------- standalone FP8 x FP4 GEMM */
/* D = A . B^T with A FP8 E4M3 [M, K] (one UE8M0 scale per 1x32 block, four
 * per int32 as x_sf), B FP4 E2M1 [N, K/2] (low nibble = even k, one UE8M0
 * byte per 1x32 block) and D BF16 [M, N], FP32 accumulation, one BF16
 * rounding ("DeepSeek DeepGEMM 2026年4月重磅更新" section 4.3, the
 * fp8_fp4_gemm call).  The masked grouped form computes G such products
 * with A [G, M_max, K], B [G, N, K/2], D [G, M_max, N], where only rows
 * m < masked_m[g] of group g are computed and written; masked_m lives on
 * the device, so a captured CUDA graph follows the counts of each replay
 * (the masked layout for CUDA-graph decode: "DeepGEMM: DeepSeek
 * 把大模型核心算子打包成一座 CUDA 训练场" section 2).  Same tensor-core
 * kernel as the MoE layer's linears.
 *
 * Shapes: N and K multiples of 128 (N, K <= 65536), G >= 1, G * M_max <=
 * 2^24; the masked form needs M_max % 128 == 0; the dense form takes any
 * M >= 0.  Errors: MOE_ERR_UNSUPPORTED_SHAPE, MOE_ERR_INVALID_ARG (NULL or
 * misaligned pointer: A, A scales and D 16-byte aligned; transformed B and
 * the workspace 256-byte aligned), MOE_ERR_WORKSPACE; a masked_m value
 * outside [0, M_max] is clamped on the device and reported as
 * MOE_ERR_INVALID_ARG by moe_get_device_status(workspace).  All pointers
 * are caller-owned device memory; calls are enqueued on `stream`. */

/* Bytes of B after moe_gemm_transform_b (codes; *sf_bytes: scales), 0 for
 * an unsupported shape. */
size_t moe_gemm_b_bytes(int G, int N, int K, size_t* sf_bytes);

/* One-time repack of B (G groups, canonical layout above) into the
 * K-block-major layout and 512-byte scale chunks the kernel streams (the
 * layout moe_transform_weights gives W2). */
moe_status moe_gemm_transform_b(int G, int N, int K, const uint8_t* b, const uint8_t* b_sf,
                                void* b_t, void* b_sf_t, moe_stream_t stream);

/* Workspace bytes of one call (tile lists and A's scale chunks), 0 for an
 * unsupported shape.  For the dense form pass G = 1, M_max = M. */
size_t moe_gemm_workspace_bytes(int G, int M_max, int N, int K);

moe_status moe_gemm_fp8_fp4(int M, int N, int K, const uint8_t* a, const int32_t* a_sf,
                            const void* b_t, const void* b_sf_t, uint16_t* d, void* workspace,
                            size_t ws_bytes, moe_stream_t stream);

/* masked_m: device int32 [G]. */
moe_status moe_gemm_fp8_fp4_masked(int G, int M_max, int N, int K, const uint8_t* a,
                                   const int32_t* a_sf, const int32_t* masked_m, const void* b_t,
                                   const void* b_sf_t, uint16_t* d, void* workspace,
                                   size_t ws_bytes, moe_stream_t stream);

/* ------------------------------------------------------ FP4 indexer (MQA) */
/* MQA logits of the lightning indexer with FP8 queries and FP4 keys
 * ("DeepSeek DeepGEMM 2026年4月重磅更新" section 5.1, the fp8_fp4_mqa_logits
 * call: q, kv, per-head weights, per-query key ranges cu_seq_len_k_start /
 * cu_seq_len_k_end, clean_logits; section 5.2, the logit of query i and
 * key j).  The page's formula is garbled (a ReLU of a softmax); this library
 * computes, for every query token i and key j with ks[i] <= j < ke[i]:
 *   logits[i][j] = sum_h weights[i][h] * max(0, sum_d q[i][h][d] * k[j][d])
 * with FP32 accumulation; entries outside the range are -inf when `clean`
 * is non-zero and are not written otherwise.
 *   q       uint8 [S, Hh, D]  E4M3 codes (the query heads of each token)
 *   q_sf    int32 [S, Hh, D/128]  UE8M0 scales per 1x32 block along D, four
 *                             per word as x_sf
 *   kv      uint8 [N, D/2]    E2M1 codes, two per byte, low nibble = even d
 *   kv_sf   uint8 [N, D/32]   UE8M0 per 1x32 block
 *   weights fp32  [S, Hh]
 *   ks, ke  int32 [S]         key range of each query (clamped to [0, N];
 *                             an empty range gives a row of -inf)
 *   logits  fp32  [S, N]      row-major
 * Shapes: Hh in {16, 32, 64, 128}, D a multiple of 128 up to 1024, S, N >= 0,
 * S * Hh <= 2^24, N <= 2^24.  Pointers are caller-owned device memory: q, kv
 * and weights 16-byte aligned, the rest 4-byte aligned, the workspace
 * 256-byte aligned with moe_mqa_logits_workspace_bytes() bytes (the keys in
 * the tile layout and the scale chunks, rebuilt by every call from the
 * canonical inputs).  Errors: MOE_ERR_UNSUPPORTED_SHAPE, MOE_ERR_INVALID_ARG,
 * MOE_ERR_WORKSPACE, MOE_ERR_CUDA; a device wait that expires is reported by
 * moe_get_device_status(workspace).  Enqueued on `stream`; nothing is
 * synchronised. */
size_t moe_mqa_logits_workspace_bytes(int S, int Hh, int D, int N);
moe_status moe_fp8_fp4_mqa_logits(int S, int Hh, int D, int N, const uint8_t* q,
                                  const int32_t* q_sf, const uint8_t* kv, const uint8_t* kv_sf,
                                  const float* weights, const int32_t* ks, const int32_t* ke,
                                  int clean, float* logits, void* workspace, size_t ws_bytes,
                                  moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
