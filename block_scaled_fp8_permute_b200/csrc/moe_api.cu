// moe_api.cu -- the extern "C" entry points of libmoe (declared in
// include/moe.h): argument validation, workspace carving, tensor-map
// encoding and the launch sequence of one MoE layer forward.
#include <atomic>
#include <cstring>
#include <mutex>

#include "moe_internal.cuh"

namespace moe {
cudaError_t launch_gemm(int epi, bool narrow, const CUtensorMap& tmA, const CUtensorMap& tmAn,
                        const CUtensorMap& tmB, const CUtensorMap& tmOut, const GemmArgs& args,
                        int grid, bool pdl, cudaStream_t stream);
cudaError_t launch_gemm_pair(int epi, const CUtensorMap& tmA, const CUtensorMap& tmB,
                             const CUtensorMap& tmSFA, const CUtensorMap& tmSFB,
                             const CUtensorMap& tmOut, const GemmArgs& args, int num_pairs_grid,
                             bool pdl, cudaStream_t stream);
cudaError_t launch_requant_debug(const float* a, int rows, int cols, uint8_t* codes,
                                 uint8_t* sbytes, cudaStream_t stream);
cudaError_t launch_plan(const int32_t* idx, int R, int E, int NCH, int P_max, int swap_max,
                        int narrow_max,
                        int* chunk, int* counts, int* offs, int* poffs, int* tile_expert,
                        int* mpair, int* norm_mtiles, int* swap_experts, int* narrow_mtiles,
                        int* row_of, int* src_of, int* hdr, bool pdl, cudaStream_t stream);
cudaError_t launch_gemm_swap(int epi, const CUtensorMap& tmW, const CUtensorMap& tmX,
                             const GemmArgs& args, int grid, bool pdl, cudaStream_t stream);
cudaError_t launch_permute(const uint8_t* x, const int32_t* x_sf, const int* src_of,
                           const int* hdr, int H, int topk, uint8_t* xp, uint8_t* xp_sf, int grid,
                           bool pdl, cudaStream_t stream);
cudaError_t launch_combine(const uint16_t* yp, const int* row_of, int T, int H, int topk,
                           uint16_t* y, int grid, bool pdl, cudaStream_t stream);
cudaError_t launch_transform(const uint8_t* w, const uint8_t* w_sf, int E, int N, int K,
                             int interleave, uint8_t* wt, uint8_t* wt_sf, cudaStream_t stream);
cudaError_t launch_gemm_prep(const int* masked_m, int G, int m_max, int mt_per_g, int* tile_expert,
                             int* norm_mtiles, int* hdr, const int32_t* a_sf, long long rows, int KG,
                             uint8_t* sf_chunks, cudaStream_t stream);

cudaError_t launch_sf_chunks(const int32_t* a_sf, long long rows, int KG, uint8_t* sf_chunks,
                             cudaStream_t stream);
int mqa_tokens_per_tile(int Hh);
size_t mqa_qsf_bytes_per_group(int D);
cudaError_t launch_mqa_logits(const CUtensorMap& tmK, const CUtensorMap& tmQ, const uint8_t* kv,
                              const uint8_t* kv_sf, uint8_t* codes, uint8_t* sfa, int Np,
                              const int32_t* q_sf, uint8_t* sfb, const float* w, const int* ks,
                              const int* ke, float* out, int* hdr, uint8_t* act, int S, int Hh,
                              int N, int KB, int clean, int grid, bool pdl,
                              unsigned long long wait_limit_ns, int fault_skip_tile,
                              cudaStream_t stream);

namespace {

std::atomic<int> g_num_sms_cap{0};
std::atomic<int> g_pdl{1};
std::atomic<int> g_gemm_variant{0};
std::atomic<int> g_swap_max{0};
std::atomic<int> g_narrow_mode{-1};
// Every value the two plan-time knobs have held in this process.  moe_plan
// takes the knobs' values at plan time and moves the experts it gives to
// narrow or swapped-role tiles out of the normal tile list; moe_forward
// launches those kernels whenever any value seen so far could have listed
// such experts, so changing a knob between moe_plan and moe_forward (or from
// another thread) never drops rows.  The launched kernels read the plan's
// own counts on the device and exit at once when their list is empty.
std::atomic<int> g_narrow_modes_seen{1};  // bit 0: auto (-1), bit 1: off (0), bit 2: on (1)
std::atomic<int> g_swap_max_seen{0};      // largest swapped-role threshold ever set
std::atomic<int> g_fault_skip_it{0};               // test hook, 0 = off
std::atomic<unsigned long long> g_fault_wait_ns{0}; // test hook, 0 = default limits
std::mutex g_ev_mu;
cudaEvent_t g_events[5];
bool g_events_on = false;

void record_event(int i, cudaStream_t s) {
  std::lock_guard<std::mutex> lk(g_ev_mu);
  if (g_events_on) cudaEventRecord(g_events[i], s);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (EncodeTiledFn) nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  int cap = g_num_sms_cap.load();
  return (cap > 0 && cap < n) ? cap : n;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

moe_status check_shape(const moe_shape* s) {
  if (!s) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->H <= 0 || s->I <= 0 || s->E <= 0 || s->topk <= 0)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s->H % 128 || s->I % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s->E > kMaxE || s->topk > kMaxTopk || s->topk > s->E) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((long long)s->T * s->topk > (1LL << 24)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((long long)s->H * s->I > (1LL << 31) || s->H > 65536 || s->I > 65536)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

// activations [rows, K] uint8 E4M3: box 128 x box_rows, 128-byte swizzle
bool encode_act(CUtensorMap* m, const void* base, int rows, int K, int box_rows = 128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K};
  cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// transformed weights [E*KB][n_rows][128 E2M1 = 64 bytes]: box 128 x box_rows x 1;
// the TMA unpacks every 16 codes (8 bytes) into a 16-byte shared-memory slot.
bool encode_wgt(CUtensorMap* m, const void* base, int E, int KB, int n_rows, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)n_rows, (cuuint64_t)E * KB};
  cuuint64_t strides[2] = {64, (cuuint64_t)n_rows * 64};
  cuuint32_t box[3] = {128, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, const_cast<void*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// BF16 partial rows [rows, N]: TMA store box 32 columns x 32 rows, 64-byte swizzle
bool encode_out_bf16(CUtensorMap* m, const void* base, int rows, int N) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)N * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// scale chunks [nchunks][512 bytes] as uint32 [nchunks][128]: box of
// `chunks` consecutive chunks
bool encode_sf(CUtensorMap* m, const void* base, long long nchunks, int chunks) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {128, (cuuint64_t)nchunks};
  cuuint64_t strides[1] = {512};
  cuuint32_t box[2] = {128, (cuuint32_t)chunks};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Ws {
  WsLayout L;
  uint8_t* base;
  int* hdr() const { return reinterpret_cast<int*>(base + L.hdr); }
  int* counts() const { return reinterpret_cast<int*>(base + L.counts); }
  int* offs() const { return reinterpret_cast<int*>(base + L.offs); }
  int* poffs() const { return reinterpret_cast<int*>(base + L.poffs); }
  int* chunk() const { return reinterpret_cast<int*>(base + L.chunk); }
  int* row_of() const { return reinterpret_cast<int*>(base + L.row_of); }
  int* src_of() const { return reinterpret_cast<int*>(base + L.src_of); }
  int* tile_expert() const { return reinterpret_cast<int*>(base + L.tile_expert); }
  int* mpair() const { return reinterpret_cast<int*>(base + L.mpair); }
  int* norm_mt() const { return reinterpret_cast<int*>(base + L.norm_mt); }
  int* swap_e() const { return reinterpret_cast<int*>(base + L.swap_e); }
  int* narrow_mt() const { return reinterpret_cast<int*>(base + L.narrow_mt); }
  uint8_t* xp() const { return base + L.xp; }
  uint8_t* xp_sf() const { return base + L.xp_sf; }
  uint8_t* a2() const { return base + L.a2; }
  uint8_t* a2_sf() const { return base + L.a2_sf; }
  uint16_t* yp() const { return reinterpret_cast<uint16_t*>(base + L.yp); }
};

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// Narrow-tile threshold of a shape, the same in moe_plan and moe_forward: on
// (experts with 1..kNarrowRows rows) with one-SM tiles when the layer has at
// most 128 rows per expert on average (decode-sized and fine-grained layers),
// or always / never when set so; off with SM-pair tiles.
bool narrow_auto_on(const moe_shape& s) {
  return (long long)s.T * s.topk <= (long long)kBlockM * s.E;
}
bool narrow_enabled(const moe_shape& s) {
  const int mode = g_narrow_mode.load();
  if (mode == 0) return false;
  return mode > 0 || narrow_auto_on(s);
}
int narrow_max_for(const moe_shape& s) {
  return (g_gemm_variant.load() != 1 && narrow_enabled(s)) ? kNarrowRows : 0;
}
// Could a plan of this shape made at any time in this process have listed
// narrow-tiled experts?  (A superset of the plan's actual choice.)
bool narrow_possible(const moe_shape& s) {
  const int seen = g_narrow_modes_seen.load();
  return (seen & 4) != 0 || ((seen & 1) != 0 && narrow_auto_on(s));
}

// standalone GEMM: shape rules and workspace (header, tile lists, A's scale chunks)
moe_status check_gemm(int G, int M_max, int N, int K) {
  if (G < 1 || M_max < 0 || N <= 0 || K <= 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (N % 128 || K % 128 || N > 65536 || K > 65536) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((long long)G * M_max > (1LL << 24) || (long long)G * N * (K / 128) > (1LL << 31))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

struct GemmWs {
  size_t hdr, tile_expert, norm_mt, sf, total;
  int mt_per_g, MT;
};
GemmWs gemm_ws(int G, int M_max, int K) {
  GemmWs w{};
  w.mt_per_g = (M_max + kBlockM - 1) / kBlockM;
  w.MT = G * w.mt_per_g;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 1024);
    return o;
  };
  w.hdr = take(kHdrWords * 4);
  w.tile_expert = take((size_t)w.MT * 4 + 4);
  w.norm_mt = take((size_t)w.MT * 4 + 4);
  w.sf = take((size_t)w.MT * (K / 128) * kSfChunk);
  w.total = off;
  return w;
}

moe_status gemm_run(int G, int M_max, int N, int K, const uint8_t* a, const int32_t* a_sf,
                    const int32_t* masked_m, const void* b_t, const void* b_sf_t, uint16_t* d,
                    void* workspace, size_t ws_bytes, cudaStream_t s) {
  const GemmWs L = gemm_ws(G, M_max, K);
  if (!workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  const long long rows = (long long)G * M_max;
  if (rows == 0) return MOE_OK;
  const void* p16[] = {a, a_sf, d};
  for (const void* p : p16)
    if (!p || !aligned(p, 16)) return MOE_ERR_INVALID_ARG;
  if (!b_t || !b_sf_t || !aligned(b_t, 256) || !aligned(b_sf_t, 256)) return MOE_ERR_INVALID_ARG;
  if (masked_m && !aligned(masked_m, 4)) return MOE_ERR_INVALID_ARG;
  const int sms = device_sms();
  if (sms <= 0) return MOE_ERR_CUDA;
  uint8_t* base = static_cast<uint8_t*>(workspace);
  int* hdr = reinterpret_cast<int*>(base + L.hdr);
  int* tile_expert = reinterpret_cast<int*>(base + L.tile_expert);
  int* norm_mt = reinterpret_cast<int*>(base + L.norm_mt);
  uint8_t* sf = base + L.sf;
  const int KB = K / 128, NT = (N + kBlockN - 1) / kBlockN;
  CUtensorMap tmA, tmB, tmD;
  if (!encode_act(&tmA, a, (int)rows, K) || !encode_wgt(&tmB, b_t, G, KB, N, 256) ||
      !encode_out_bf16(&tmD, d, (int)rows, N))
    return MOE_ERR_CUDA;
  cudaError_t e = cudaMemsetAsync(hdr, 0, kHdrWords * 4, s);
  if (e == cudaSuccess)
    e = launch_gemm_prep(masked_m, G, M_max, L.mt_per_g, tile_expert, norm_mt, hdr, a_sf, rows,
                         KB, sf, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  GemmArgs g{};
  g.sfa = sf;
  g.sfb = static_cast<const uint8_t*>(b_sf_t);
  g.hdr = hdr;
  g.tile_expert = tile_expert;
  g.norm_mtiles = norm_mt;
  g.tiles_word = kHdrNormMTiles;
  g.KB = KB;
  g.n_rows = N;
  g.NT = NT;
  g.d = d;
  g.masked_m = masked_m;
  g.m_max = M_max;
  const long long tiles = (long long)L.MT * NT;
  const int grid = (int)(tiles < sms ? tiles : sms);
  return cuda_status(
      launch_gemm(3, false, tmA, tmA, tmB, tmD, g, grid < 1 ? 1 : grid, g_pdl.load() != 0, s));
}

// FP4 indexer (MQA logits): shape rules and workspace (status header, keys in
// the tile layout, key and query scale chunks)
moe_status check_mqa(int S, int Hh, int D, int N) {
  if (S < 0 || N < 0 || D <= 0 || Hh <= 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (Hh != 16 && Hh != 32 && Hh != 64 && Hh != 128) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (D % 128 || D > 1024) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((long long)S * Hh > (1LL << 24) || N > (1 << 24) || (long long)S * N > (1LL << 34))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

struct MqaWs {
  size_t hdr, codes, kchunks, qchunks, act, total;
  int Np, n_groups;
};
MqaWs mqa_ws(int S, int Hh, int D, int N) {
  MqaWs w{};
  w.Np = (N + 127) / 128 * 128;
  w.n_groups = (S + mqa_tokens_per_tile(Hh) - 1) / mqa_tokens_per_tile(Hh);
  const int KB = D / 128;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 1024);
    return o;
  };
  w.hdr = take(kHdrWords * 4);
  w.codes = take((size_t)KB * w.Np * 64);
  w.kchunks = take((size_t)KB * (w.Np / 128) * kSfChunk);
  w.qchunks = take((size_t)w.n_groups * mqa_qsf_bytes_per_group(D));
  w.act = take((size_t)w.n_groups * (w.Np / 128));
  w.total = off;
  return w;
}

// staging area of moe_forward_host, after the regular workspace
struct HostStage {
  size_t x, x_sf, idx, w, y, total;
};
HostStage host_stage(const moe_shape& s, size_t base) {
  HostStage h{};
  size_t off = base;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 1024);
    return o;
  };
  h.x = take((size_t)s.T * s.H);
  h.x_sf = take((size_t)s.T * (s.H / 128) * 4);
  h.idx = take((size_t)s.T * s.topk * 4);
  h.w = take((size_t)s.T * s.topk * 4);
  h.y = take((size_t)s.T * s.H * 2);
  h.total = off;
  return h;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "MOE_ERR_UNSUPPORTED_SHAPE";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_BAD_EXPERT_ID: return "MOE_ERR_BAD_EXPERT_ID";
  }
  return "MOE_ERR_UNKNOWN";
}

int moe_block_m(void) { return kBlockM; }

void moe_set_num_sms(int num_sms) { g_num_sms_cap.store(num_sms > 0 ? num_sms : 0); }

void moe_set_pdl(int enable) { g_pdl.store(enable ? 1 : 0); }

void moe_set_gemm_variant(int variant) { g_gemm_variant.store(variant == 1 ? 1 : 0); }

void moe_set_narrow_tiles(int mode) {
  const int m = mode < 0 ? -1 : (mode ? 1 : 0);
  g_narrow_modes_seen.fetch_or(m < 0 ? 1 : (m == 0 ? 2 : 4));  // before any plan can use it
  g_narrow_mode.store(m);
}

void moe_set_swap_max(int rows) {
  const int r = rows < 0 ? 0 : (rows > kMaxSwapRows ? kMaxSwapRows : rows);
  int seen = g_swap_max_seen.load();
  while (r > seen && !g_swap_max_seen.compare_exchange_weak(seen, r)) {
  }
  g_swap_max.store(r);
}

void moe_set_timing_events(void* const* events, int n) {
  std::lock_guard<std::mutex> lk(g_ev_mu);
  g_events_on = (events != nullptr && n >= 5);
  if (g_events_on)
    for (int i = 0; i < 5; ++i) g_events[i] = static_cast<cudaEvent_t>(events[i]);
}

size_t moe_transformed_bytes(const moe_shape* shape, int which, size_t* sf_bytes) {
  if (check_shape(shape) != MOE_OK || (which != 1 && which != 2)) {
    if (sf_bytes) *sf_bytes = 0;
    return 0;
  }
  const size_t E = shape->E, H = shape->H, I = shape->I;
  const size_t elems = (which == 1) ? E * 2 * I * H : E * H * I;
  if (sf_bytes) *sf_bytes = elems / 32;
  return elems / 2;
}

moe_status moe_transform_weights(const moe_shape* shape, const uint8_t* w1, const uint8_t* w1_sf,
                                 const uint8_t* w2, const uint8_t* w2_sf, void* w1_t,
                                 void* w1_sf_t, void* w2_t, void* w2_sf_t, moe_stream_t stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  const void* ptrs[] = {w1, w1_sf, w2, w2_sf, w1_t, w1_sf_t, w2_t, w2_sf_t};
  for (const void* p : ptrs)
    if (!p || !aligned(p, 16)) return MOE_ERR_INVALID_ARG;
  for (const void* p : {(const void*)w1_t, (const void*)w1_sf_t, (const void*)w2_t,
                        (const void*)w2_sf_t})
    if (!aligned(p, 256)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_transform(w1, w1_sf, shape->E, 2 * shape->I, shape->H, 1,
                                   static_cast<uint8_t*>(w1_t), static_cast<uint8_t*>(w1_sf_t), s);
  if (e == cudaSuccess)
    e = launch_transform(w2, w2_sf, shape->E, shape->H, shape->I, 0, static_cast<uint8_t*>(w2_t),
                         static_cast<uint8_t*>(w2_sf_t), s);
  return cuda_status(e);
}

size_t moe_workspace_bytes(const moe_shape* shape) {
  if (check_shape(shape) != MOE_OK) return 0;
  return ws_layout(*shape).total;
}

int moe_plan_max_rows(const moe_shape* shape) {
  if (check_shape(shape) != MOE_OK) return 0;
  return ws_layout(*shape).P_max;
}

moe_status moe_plan(const moe_shape* shape, const int32_t* topk_idx, void* workspace,
                    size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (!workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!topk_idx || !aligned(topk_idx, 4))) return MOE_ERR_INVALID_ARG;
  Ws ws{ws_layout(*shape), static_cast<uint8_t*>(workspace)};
  if (ws_bytes < ws.L.total) return MOE_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(ws.hdr(), 0, kHdrWords * 4, s);
  if (e == cudaSuccess)
    e = launch_plan(topk_idx, ws.L.R, shape->E, ws.L.NCH, ws.L.P_max, g_swap_max.load(),
                    narrow_max_for(*shape), ws.chunk(), ws.counts(), ws.offs(), ws.poffs(),
                    ws.tile_expert(), ws.mpair(), ws.norm_mt(), ws.swap_e(), ws.narrow_mt(),
                    ws.row_of(), ws.src_of(), ws.hdr(), g_pdl.load() != 0, s);
  return cuda_status(e);
}

moe_status moe_forward(const moe_shape* shape, const uint8_t* x, const int32_t* x_sf,
                       const int32_t* topk_idx, const float* topk_w, const void* w1_t,
                       const void* w1_sf_t, const void* w2_t, const void* w2_sf_t, uint16_t* y,
                       void* workspace, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  const moe_shape sh = *shape;
  if (!workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
  Ws ws{ws_layout(sh), static_cast<uint8_t*>(workspace)};
  if (ws_bytes < ws.L.total) return MOE_ERR_WORKSPACE;
  if (sh.T == 0) return MOE_OK;
  const void* p16[] = {x, x_sf, topk_w, y};
  for (const void* p : p16)
    if (!p || !aligned(p, 16)) return MOE_ERR_INVALID_ARG;
  const void* p256[] = {w1_t, w1_sf_t, w2_t, w2_sf_t};
  for (const void* p : p256)
    if (!p || !aligned(p, 256)) return MOE_ERR_INVALID_ARG;
  if (!topk_idx || !aligned(topk_idx, 4)) return MOE_ERR_INVALID_ARG;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int sms = device_sms();
  if (sms <= 0) return MOE_ERR_CUDA;
  const bool pdl = g_pdl.load() != 0;
  const int KB1 = sh.H / 128, KB2 = sh.I / 128;
  const int NT1 = (2 * sh.I + kBlockN - 1) / kBlockN, NT2 = (sh.H + kBlockN - 1) / kBlockN;

  // SM-pair tiles (variant 1) for linear1 (2I is a multiple of 256) and for
  // linear2 when H is; one-SM tiles otherwise (and for 128-column tail tiles)
  const bool pair1 = g_gemm_variant.load() == 1;
  const bool pair2 = pair1 && (sh.H % 256) == 0;
  CUtensorMap tmX, tmW1, tmA2, tmW2, tmYp, tmXsf, tmW1sf, tmA2sf, tmW2sf;
  // swapped-role kernel: 16-row token boxes; tmW1s / tmW2s (256-row weight boxes)
  // also serve the narrow tiles
  CUtensorMap tmX16, tmA216, tmW1s, tmW2s;
  CUtensorMap tmXn, tmA2n;                   // narrow tiles: kNarrowRows-row A boxes
  if (!encode_act(&tmXn, ws.xp(), ws.L.P_max, sh.H, kNarrowRows) ||
      !encode_act(&tmA2n, ws.a2(), ws.L.P_max, sh.I, kNarrowRows))
    return MOE_ERR_CUDA;
  if (!encode_act(&tmX16, ws.xp(), ws.L.P_max, sh.H, 16) ||
      !encode_act(&tmA216, ws.a2(), ws.L.P_max, sh.I, 16) ||
      !encode_wgt(&tmW1s, w1_t, sh.E, KB1, 2 * sh.I, 256) ||
      !encode_wgt(&tmW2s, w2_t, sh.E, KB2, sh.H, 256))
    return MOE_ERR_CUDA;
  if (!encode_act(&tmX, ws.xp(), ws.L.P_max, sh.H) ||
      !encode_wgt(&tmW1, w1_t, sh.E, KB1, 2 * sh.I, pair1 ? 128 : 256) ||
      !encode_act(&tmA2, ws.a2(), ws.L.P_max, sh.I) ||
      !encode_wgt(&tmW2, w2_t, sh.E, KB2, sh.H, pair2 ? 128 : 256) ||
      !encode_out_bf16(&tmYp, ws.yp(), ws.L.P_max, sh.H) ||
      !encode_sf(&tmXsf, ws.xp_sf(), (long long)ws.L.MT_max * KB1, 1) ||
      !encode_sf(&tmW1sf, w1_sf_t, (long long)sh.E * KB1 * (2 * sh.I / 128), 2) ||
      !encode_sf(&tmA2sf, ws.a2_sf(), (long long)ws.L.MT_max * KB2, 1) ||
      (pair2 && !encode_sf(&tmW2sf, w2_sf_t, (long long)sh.E * KB2 * (sh.H / 128), 2)))
    return MOE_ERR_CUDA;

  // dispatch: permute rows into expert-contiguous order
  record_event(0, s);
  int pgrid = (ws.L.P_max + 7) / 8;
  if (pgrid > sms * 16) pgrid = sms * 16;
  if (pgrid < 1) pgrid = 1;
  cudaError_t e = launch_permute(x, x_sf, ws.src_of(), ws.hdr(), sh.H, sh.topk, ws.xp(),
                                 ws.xp_sf(), pgrid, pdl, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  record_event(1, s);

  const int max_pairs_grid = sms / 2 > 0 ? sms / 2 : 1;
  GemmArgs g1{};
  g1.sfa = ws.xp_sf();
  g1.sfb = static_cast<const uint8_t*>(w1_sf_t);
  g1.hdr = ws.hdr();
  g1.tile_expert = ws.tile_expert();
  g1.src_of = ws.src_of();
  g1.mpair = ws.mpair();
  g1.norm_mtiles = ws.norm_mt();
  g1.tiles_word = kHdrNormMTiles;
  g1.swap_experts = ws.swap_e();
  g1.poffs = ws.poffs();
  g1.counts = ws.counts();
  g1.KB = KB1;
  g1.n_rows = 2 * sh.I;
  g1.NT = NT1;
  g1.a2 = ws.a2();
  g1.a2_sf = ws.a2_sf();
  g1.I = sh.I;
  g1.H = sh.H;
  g1.narrow_mtiles = ws.narrow_mt();
  // experts with at most kNarrowRows rows: narrow tiles (a deeper weight stream).
  // Launched whenever the plan may have listed such experts, whatever the knobs
  // say now (an empty list costs one short launch).  With one-SM normal tiles
  // the launches are mixed: the normal-tile kernel also runs the narrow m-tiles
  // when the plan has normal m-tiles too, so their weight streams overlap the
  // compute-bound tiles; otherwise the narrow-tile kernel runs them.
  const bool narrow = narrow_possible(sh);
  g1.mixed = (narrow && !pair1) ? 1 : 0;
  GemmArgs g1f = g1;  // the normal one-SM linear1 launch carries the test hook
  g1f.fault_skip_it = g_fault_skip_it.load();
  g1f.wait_limit_ns = g_fault_wait_ns.load();
  if (pair1) {
    long long work = (long long)ws.L.MP_max * NT1;
    int pairs = (int)(work < max_pairs_grid ? work : max_pairs_grid);
    e = launch_gemm_pair(1, tmX, tmW1, tmXsf, tmW1sf, tmYp, g1, pairs < 1 ? 1 : pairs, pdl, s);
  } else {
    long long tiles1 = (long long)ws.L.MT_max * NT1;
    int grid1 = (int)(tiles1 < sms ? tiles1 : sms);
    e = launch_gemm(1, false, tmX, tmXn, tmW1, tmYp, g1f, grid1 < 1 ? 1 : grid1, pdl, s);
  }
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  const int narrow_grid1 = (int)((long long)sh.E * NT1 < sms ? (long long)sh.E * NT1 : sms);
  if (narrow) {
    GemmArgs g1n = g1;
    g1n.norm_mtiles = ws.narrow_mt();
    g1n.tiles_word = kHdrNarrowMTiles;
    // 256-row weight boxes, whatever box the SM-pair tiles use
    e = launch_gemm(1, true, tmXn, tmXn, tmW1s, tmYp, g1n, narrow_grid1, pdl, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
  }
  // swapped-role tiles exist only when the plan was made with a threshold > 0
  const bool use_swap = g_swap_max_seen.load() > 0;
  if (use_swap) {
    const int swap_grid1 = (int)((long long)sh.E * NT1 < sms ? (long long)sh.E * NT1 : sms);
    e = launch_gemm_swap(1, tmW1s, tmX16, g1, swap_grid1, pdl, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
  }
  record_event(2, s);

  GemmArgs g2 = g1;
  g2.sfa = ws.a2_sf();
  g2.sfb = static_cast<const uint8_t*>(w2_sf_t);
  g2.KB = KB2;
  g2.n_rows = sh.H;
  g2.NT = NT2;
  g2.yp = ws.yp();
  g2.topk_w = topk_w;
  g2.mixed = (narrow && !pair2) ? 1 : 0;
  if (pair2) {
    long long work = (long long)ws.L.MP_max * NT2;
    int pairs = (int)(work < max_pairs_grid ? work : max_pairs_grid);
    e = launch_gemm_pair(2, tmA2, tmW2, tmA2sf, tmW2sf, tmYp, g2, pairs < 1 ? 1 : pairs, pdl, s);
  } else {
    long long tiles2 = (long long)ws.L.MT_max * NT2;
    int grid2 = (int)(tiles2 < sms ? tiles2 : sms);
    e = launch_gemm(2, false, tmA2, tmA2n, tmW2, tmYp, g2, grid2 < 1 ? 1 : grid2, pdl, s);
  }
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (narrow) {
    GemmArgs g2n = g2;
    g2n.norm_mtiles = ws.narrow_mt();
    g2n.tiles_word = kHdrNarrowMTiles;
    const int narrow_grid2 = (int)((long long)sh.E * NT2 < sms ? (long long)sh.E * NT2 : sms);
    e = launch_gemm(2, true, tmA2n, tmA2n, tmW2s, tmYp, g2n, narrow_grid2, pdl, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (use_swap) {
    const int swap_grid2 = (int)((long long)sh.E * NT2 < sms ? (long long)sh.E * NT2 : sms);
    e = launch_gemm_swap(2, tmW2s, tmA216, g2, swap_grid2, pdl, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
  }
  record_event(3, s);

  int cgrid = sh.T < 65535 ? sh.T : 65535;
  e = launch_combine(ws.yp(), ws.row_of(), sh.T, sh.H, sh.topk, y, cgrid, pdl, s);
  record_event(4, s);
  return cuda_status(e);
}

size_t moe_workspace_bytes_host(const moe_shape* shape) {
  if (check_shape(shape) != MOE_OK) return 0;
  WsLayout L = ws_layout(*shape);
  return host_stage(*shape, L.total).total;
}

moe_status moe_forward_host(const moe_shape* shape, const uint8_t* x_host,
                            const int32_t* x_sf_host, const int32_t* topk_idx_host,
                            const float* topk_w_host, const void* w1_t, const void* w1_sf_t,
                            const void* w2_t, const void* w2_sf_t, uint16_t* y_host,
                            void* workspace, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  const moe_shape sh = *shape;
  if (!workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
  WsLayout L = ws_layout(sh);
  HostStage hs = host_stage(sh, L.total);
  if (ws_bytes < hs.total) return MOE_ERR_WORKSPACE;
  if (sh.T == 0) return MOE_OK;
  if (!x_host || !x_sf_host || !topk_idx_host || !topk_w_host || !y_host)
    return MOE_ERR_INVALID_ARG;
  uint8_t* base = static_cast<uint8_t*>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t nx = (size_t)sh.T * sh.H, nsf = (size_t)sh.T * (sh.H / 128) * 4,
               nk = (size_t)sh.T * sh.topk * 4, ny = (size_t)sh.T * sh.H * 2;
  cudaError_t e = cudaMemcpyAsync(base + hs.x, x_host, nx, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(base + hs.x_sf, x_sf_host, nsf, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(base + hs.idx, topk_idx_host, nk, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(base + hs.w, topk_w_host, nk, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  const int32_t* idx_d = reinterpret_cast<const int32_t*>(base + hs.idx);
  st = moe_plan(shape, idx_d, workspace, L.total, stream);
  if (st != MOE_OK) return st;
  st = moe_forward(shape, base + hs.x, reinterpret_cast<const int32_t*>(base + hs.x_sf), idx_d,
                   reinterpret_cast<const float*>(base + hs.w), w1_t, w1_sf_t, w2_t, w2_sf_t,
                   reinterpret_cast<uint16_t*>(base + hs.y), workspace, L.total, stream);
  if (st != MOE_OK) return st;
  e = cudaMemcpyAsync(y_host, base + hs.y, ny, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return cuda_status(e);
}

size_t moe_workspace_bytes_host_pipelined(const moe_shape* shape) {
  if (check_shape(shape) != MOE_OK) return 0;
  WsLayout L = ws_layout(*shape);
  return host_stage(*shape, host_stage(*shape, L.total).total).total;
}

moe_status moe_forward_host_pipelined(const moe_shape* shape, int n_batches,
                                      const uint8_t* const* x_host,
                                      const int32_t* const* x_sf_host,
                                      const int32_t* const* topk_idx_host,
                                      const float* const* topk_w_host, const void* w1_t,
                                      const void* w1_sf_t, const void* w2_t,
                                      const void* w2_sf_t, uint16_t* const* y_host,
                                      void* workspace, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (n_batches < 0) return MOE_ERR_INVALID_ARG;
  const moe_shape sh = *shape;
  if (!workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(sh);
  const HostStage slot[2] = {host_stage(sh, L.total), host_stage(sh, host_stage(sh, L.total).total)};
  if (ws_bytes < slot[1].total) return MOE_ERR_WORKSPACE;
  if (sh.T == 0 || n_batches == 0) return MOE_OK;
  if (!x_host || !x_sf_host || !topk_idx_host || !topk_w_host || !y_host)
    return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n_batches; ++i)
    if (!x_host[i] || !x_sf_host[i] || !topk_idx_host[i] || !topk_w_host[i] || !y_host[i])
      return MOE_ERR_INVALID_ARG;
  uint8_t* base = static_cast<uint8_t*>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t nx = (size_t)sh.T * sh.H, nsf = (size_t)sh.T * (sh.H / 128) * 4,
               nk = (size_t)sh.T * sh.topk * 4, ny = (size_t)sh.T * sh.H * 2;

  // Copy-in and copy-out run on streams of their own, so batch i + 1's inputs
  // go up and batch i - 1's y comes down while batch i's kernels run on
  // `stream`.  Staging slot i % 2 holds batch i; the events order its reuse.
  cudaStream_t cin = nullptr, cout = nullptr;
  cudaEvent_t ev_start = nullptr, ev_in[2] = {}, ev_comp[2] = {}, ev_out[2] = {};
  cudaError_t e = cudaStreamCreateWithFlags(&cin, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&cout, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_start, cudaEventDisableTiming);
  for (int b = 0; b < 2 && e == cudaSuccess; ++b) {
    e = cudaEventCreateWithFlags(&ev_in[b], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_comp[b], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_out[b], cudaEventDisableTiming);
  }
  // both copy streams start after whatever the caller enqueued on `stream`
  if (e == cudaSuccess) e = cudaEventRecord(ev_start, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cin, ev_start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cout, ev_start, 0);
  st = cuda_status(e);
  for (int i = 0; i < n_batches && st == MOE_OK; ++i) {
    const int b = i & 1;
    const HostStage& h = slot[b];
    // slot b's inputs are overwritten once batch i - 2's kernels have read them
    if (i >= 2) e = cudaStreamWaitEvent(cin, ev_comp[b], 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(base + h.x, x_host[i], nx, cudaMemcpyHostToDevice, cin);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(base + h.x_sf, x_sf_host[i], nsf, cudaMemcpyHostToDevice, cin);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(base + h.idx, topk_idx_host[i], nk, cudaMemcpyHostToDevice, cin);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(base + h.w, topk_w_host[i], nk, cudaMemcpyHostToDevice, cin);
    if (e == cudaSuccess) e = cudaEventRecord(ev_in[b], cin);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev_in[b], 0);
    // slot b's y is overwritten once batch i - 2's copy-out has read it
    if (e == cudaSuccess && i >= 2) e = cudaStreamWaitEvent(s, ev_out[b], 0);
    st = cuda_status(e);
    if (st != MOE_OK) break;
    const int32_t* idx_d = reinterpret_cast<const int32_t*>(base + h.idx);
    st = moe_plan(shape, idx_d, workspace, L.total, stream);
    if (st == MOE_OK)
      st = moe_forward(shape, base + h.x, reinterpret_cast<const int32_t*>(base + h.x_sf), idx_d,
                       reinterpret_cast<const float*>(base + h.w), w1_t, w1_sf_t, w2_t, w2_sf_t,
                       reinterpret_cast<uint16_t*>(base + h.y), workspace, L.total, stream);
    if (st != MOE_OK) break;
    e = cudaEventRecord(ev_comp[b], s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cout, ev_comp[b], 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(y_host[i], base + h.y, ny, cudaMemcpyDeviceToHost, cout);
    if (e == cudaSuccess) e = cudaEventRecord(ev_out[b], cout);
    st = cuda_status(e);
  }
  // `stream` is ordered after the last copy-out; then drain all three streams
  // (also after a failure: nothing may still be reading the caller's host
  // buffers when this returns)
  if (st == MOE_OK) st = cuda_status(cudaStreamWaitEvent(s, ev_out[(n_batches - 1) & 1], 0));
  cudaError_t e1 = cin ? cudaStreamSynchronize(cin) : cudaSuccess;
  cudaError_t e2 = cout ? cudaStreamSynchronize(cout) : cudaSuccess;
  cudaError_t e3 = cudaStreamSynchronize(s);
  for (int b = 0; b < 2; ++b) {
    if (ev_in[b]) cudaEventDestroy(ev_in[b]);
    if (ev_comp[b]) cudaEventDestroy(ev_comp[b]);
    if (ev_out[b]) cudaEventDestroy(ev_out[b]);
  }
  if (ev_start) cudaEventDestroy(ev_start);
  if (cin) cudaStreamDestroy(cin);
  if (cout) cudaStreamDestroy(cout);
  if (st != MOE_OK) return st;
  if (e1 != cudaSuccess || e2 != cudaSuccess || e3 != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

void moe_debug_set_fault(int skip_iteration, unsigned long long wait_limit_ns) {
  g_fault_skip_it.store(skip_iteration >= 0 ? skip_iteration + 1 : 0);
  g_fault_wait_ns.store(wait_limit_ns);
}

int moe_get_timeout_site(const void* workspace, moe_stream_t stream) {
  if (!workspace) return -1;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return -1;
  int hdr[kHdrWords];
  if (cudaMemcpy(hdr, workspace, sizeof(hdr), cudaMemcpyDeviceToHost) != cudaSuccess) return -1;
  return hdr[kHdrTimeoutSite];
}

moe_status moe_get_device_status(const void* workspace, moe_stream_t stream) {
  if (!workspace) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  int hdr[kHdrWords];
  if (cudaMemcpy(hdr, workspace, sizeof(hdr), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOE_ERR_CUDA;
  return static_cast<moe_status>(hdr[kHdrStatus]);
}

moe_status moe_plan_export(const moe_shape* shape, const void* workspace, int32_t* counts,
                           int32_t* offs, int32_t* padded_offs, int32_t* row_of, int32_t* src_of,
                           int32_t* P_out, moe_stream_t stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (!workspace || !counts || !offs || !padded_offs || !row_of || !P_out)
    return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  Ws ws{ws_layout(*shape), static_cast<uint8_t*>(const_cast<void*>(workspace))};
  const int E = shape->E;
  int hdr[kHdrWords];
  cudaError_t e = cudaMemcpy(hdr, ws.hdr(), sizeof(hdr), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(counts, ws.counts(), E * 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(offs, ws.offs(), (E + 1) * 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(padded_offs, ws.poffs(), (E + 1) * 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && ws.L.R > 0)
    e = cudaMemcpy(row_of, ws.row_of(), (size_t)ws.L.R * 4, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  *P_out = hdr[kHdrP];
  if (src_of && hdr[kHdrP] > 0) {
    if (hdr[kHdrP] > ws.L.P_max) return MOE_ERR_CUDA;
    if (cudaMemcpy(src_of, ws.src_of(), (size_t)hdr[kHdrP] * 4, cudaMemcpyDeviceToHost) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

size_t moe_gemm_b_bytes(int G, int N, int K, size_t* sf_bytes) {
  if (check_gemm(G, 0, N, K) != MOE_OK) {
    if (sf_bytes) *sf_bytes = 0;
    return 0;
  }
  const size_t elems = (size_t)G * N * K;
  if (sf_bytes) *sf_bytes = elems / 32;
  return elems / 2;
}

moe_status moe_gemm_transform_b(int G, int N, int K, const uint8_t* b, const uint8_t* b_sf,
                                void* b_t, void* b_sf_t, moe_stream_t stream) {
  moe_status st = check_gemm(G, 0, N, K);
  if (st != MOE_OK) return st;
  if (!b || !b_sf || !aligned(b, 16) || !aligned(b_sf, 16)) return MOE_ERR_INVALID_ARG;
  if (!b_t || !b_sf_t || !aligned(b_t, 256) || !aligned(b_sf_t, 256)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_transform(b, b_sf, G, N, K, 0, static_cast<uint8_t*>(b_t),
                                      static_cast<uint8_t*>(b_sf_t),
                                      reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_gemm_workspace_bytes(int G, int M_max, int N, int K) {
  if (check_gemm(G, M_max, N, K) != MOE_OK) return 0;
  return gemm_ws(G, M_max, K).total;
}

moe_status moe_gemm_fp8_fp4(int M, int N, int K, const uint8_t* a, const int32_t* a_sf,
                            const void* b_t, const void* b_sf_t, uint16_t* d, void* workspace,
                            size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_gemm(1, M, N, K);
  if (st != MOE_OK) return st;
  return gemm_run(1, M, N, K, a, a_sf, nullptr, b_t, b_sf_t, d, workspace, ws_bytes,
                  reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_gemm_fp8_fp4_masked(int G, int M_max, int N, int K, const uint8_t* a,
                                   const int32_t* a_sf, const int32_t* masked_m, const void* b_t,
                                   const void* b_sf_t, uint16_t* d, void* workspace,
                                   size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_gemm(G, M_max, N, K);
  if (st != MOE_OK) return st;
  if (M_max % kBlockM) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!masked_m) return MOE_ERR_INVALID_ARG;
  return gemm_run(G, M_max, N, K, a, a_sf, masked_m, b_t, b_sf_t, d, workspace, ws_bytes,
                  reinterpret_cast<cudaStream_t>(stream));
}

size_t moe_mqa_logits_workspace_bytes(int S, int Hh, int D, int N) {
  if (check_mqa(S, Hh, D, N) != MOE_OK) return 0;
  return mqa_ws(S, Hh, D, N).total;
}

moe_status moe_fp8_fp4_mqa_logits(int S, int Hh, int D, int N, const uint8_t* q,
                                  const int32_t* q_sf, const uint8_t* kv, const uint8_t* kv_sf,
                                  const float* weights, const int32_t* ks, const int32_t* ke,
                                  int clean, float* logits, void* workspace, size_t ws_bytes,
                                  moe_stream_t stream) {
  moe_status st = check_mqa(S, Hh, D, N);
  if (st != MOE_OK) return st;
  const MqaWs L = mqa_ws(S, Hh, D, N);
  if (!workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (S == 0 || N == 0) return MOE_OK;
  const void* p16[] = {q, kv, weights};
  for (const void* p : p16)
    if (!p || !aligned(p, 16)) return MOE_ERR_INVALID_ARG;
  const void* p4[] = {q_sf, kv_sf, ks, ke, logits};
  for (const void* p : p4)
    if (!p || !aligned(p, 4)) return MOE_ERR_INVALID_ARG;
  const int sms = device_sms();
  if (sms <= 0) return MOE_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  int* hdr = reinterpret_cast<int*>(base + L.hdr);
  uint8_t* codes = base + L.codes;
  uint8_t* kchunks = base + L.kchunks;
  uint8_t* qchunks = base + L.qchunks;
  const int KB = D / 128;
  CUtensorMap tmK, tmQ;
  if (!encode_wgt(&tmK, codes, 1, KB, L.Np, 128) ||
      !encode_act(&tmQ, q, S * Hh, D, mqa_tokens_per_tile(Hh) * Hh))
    return MOE_ERR_CUDA;
  // two launches: the prep kernel (status words, key layout, query scale
  // chunks, tile activity) and the logits kernel
  const long long tiles = (long long)(L.Np / 128) * L.n_groups;
  const int grid = (int)(tiles < sms ? tiles : sms);
  return cuda_status(launch_mqa_logits(tmK, tmQ, kv, kv_sf, codes, kchunks, L.Np, q_sf, qchunks,
                                       weights, ks, ke, logits, hdr, base + L.act, S, Hh, N, KB,
                                       clean ? 1 : 0, grid, g_pdl.load() != 0,
                                       g_fault_wait_ns.load(), g_fault_skip_it.load(), s));
}

moe_status moe_debug_requant(const float* a, int rows, int cols, uint8_t* codes, uint8_t* sbytes,
                             moe_stream_t stream) {
  if (rows < 0 || cols <= 0 || cols % 32) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return MOE_OK;
  if (!a || !codes || !sbytes || !aligned(a, 16) || !aligned(codes, 16))
    return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_requant_debug(a, rows, cols, codes, sbytes,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
