// moe_internal.cuh -- shared definitions of the libmoe CUDA sources:
// workspace layout, device status word, tile constants.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// ---------------------------------------------------------------- constants
constexpr int kBlockM = 128;        // rows per M tile (padding granule of the expert layout)
constexpr int kBlockN = 256;        // weight rows per N tile
constexpr int kBlockK = 128;        // K elements per pipeline stage (4 MMAs of K=32)
constexpr int kSfChunk = 512;       // bytes of one 128-row x 4-K-block scale chunk
constexpr int kPlanChunk = 1024;    // assignments per plan block
constexpr int kMaxE = 1024;
constexpr int kMaxTopk = 32;

// header words at the start of the workspace
enum HdrWord : int {
  kHdrStatus = 0,     // moe_status of the last plan/forward (device side)
  kHdrP = 1,          // padded rows P
  kHdrMTiles = 2,     // P / kBlockM
  kHdrBadIds = 3,     // number of skipped invalid expert ids
  kHdrTimeoutSite = 4,
  kHdrMPairs = 5,     // number of m-tile pairs of normal-tiled experts (SM-pair work rows)
  kHdrNormMTiles = 6, // m-tiles of experts run with normal tiles
  kHdrSwapExperts = 7,// experts run with swapped operand roles (n <= swap threshold)
  kHdrSwapMax = 8,    // the threshold the plan used
  kHdrPlanDone = 9,   // blocks of the plan's counting kernel that have finished
  kHdrNarrowMTiles = 10,  // m-tiles of experts run with narrow tiles (1..narrow_max rows)
  kHdrNarrowMax = 11,     // the narrow threshold the plan used
  kHdrWords = 64
};

// byte offsets of every region of the workspace (all 1024-byte aligned)
struct WsLayout {
  size_t hdr, counts, offs, poffs, chunk, row_of, src_of, tile_expert, mpair, norm_mt, swap_e;
  size_t narrow_mt;
  size_t xp, xp_sf, a2, a2_sf, yp;
  size_t total;
  int R, P_max, MT_max, MP_max, NCH;
};

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Upper bound on padded rows over every routing: each non-empty expert adds
// at most kBlockM-1 rows of padding, and at most min(E, R) experts are
// non-empty.
__host__ __device__ inline int max_padded_rows(int R, int E) {
  long long nonempty = R < E ? R : E;
  long long p = (long long)R + nonempty * (kBlockM - 1);
  return (int)align_up((size_t)p, kBlockM);
}

inline WsLayout ws_layout(const moe_shape& s) {
  WsLayout L{};
  L.R = s.T * s.topk;
  L.P_max = max_padded_rows(L.R, s.E);
  L.MT_max = L.P_max / kBlockM;
  // pairs of m-tiles of one expert: at most one odd m-tile per non-empty expert
  L.MP_max = L.MT_max / 2 + (L.R < s.E ? L.R : s.E) + 1;
  L.NCH = (L.R + kPlanChunk - 1) / kPlanChunk;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 1024);
    return o;
  };
  L.hdr = take(kHdrWords * 4);
  L.counts = take((size_t)s.E * 4);
  L.offs = take((size_t)(s.E + 1) * 4);
  L.poffs = take((size_t)(s.E + 1) * 4);
  L.chunk = take((size_t)L.NCH * s.E * 4);
  L.row_of = take((size_t)L.R * 4);
  L.src_of = take((size_t)L.P_max * 4);
  L.tile_expert = take((size_t)L.MT_max * 4);
  L.mpair = take((size_t)L.MP_max * 4);
  L.norm_mt = take((size_t)L.MT_max * 4);
  L.swap_e = take((size_t)s.E * 4);
  L.narrow_mt = take((size_t)s.E * 4);
  L.xp = take((size_t)L.P_max * s.H);
  L.xp_sf = take((size_t)L.MT_max * (s.H / 128) * kSfChunk);
  L.a2 = take((size_t)L.P_max * s.I);
  L.a2_sf = take((size_t)L.MT_max * (s.I / 128) * kSfChunk);
  L.yp = take((size_t)L.P_max * s.H * 2);
  L.total = off;
  return L;
}

// arguments of the grouped GEMM kernel (both linears)
struct GemmArgs {
  const uint8_t* sfa;      // activation scale chunks [MT][KB][512]
  const uint8_t* sfb;      // weight scale chunks [E][KB][n_rows/128][512]
  int* hdr;                // workspace header
  const int* tile_expert;  // expert of every m-tile
  const int* src_of;       // assignment of every padded row (-1 = padding)
  int KB;                  // K / 128
  int n_rows;              // weight rows per expert
  int NT;                  // ceil(n_rows / 256)
  uint8_t* a2;             // linear1 out: E4M3 [P, I]
  uint8_t* a2_sf;          // linear1 out: scale chunks [MT][I/128][512]
  int I;
  uint16_t* yp;            // linear2 out: BF16 [P, H], rows times their top-k weight
  const float* topk_w;     // [T*k]
  int H;
  const int* mpair;        // m-tile pairs: first m-tile | (1 << 31) when the pair has one m-tile
  const int* norm_mtiles;  // m-tiles this launch runs (normal or narrow list)
  int tiles_word;          // header word holding their count
  const int* swap_experts; // experts with swapped operand roles
  const int* poffs;        // padded first row of every expert
  const int* counts;       // rows of every expert
  // standalone GEMM (epilogue 3): D rows [G * m_max, n_rows] BF16; group g of an
  // m-tile = tile_expert[mt]; rows at and past masked_m[g] (m_max when NULL) are not written
  uint16_t* d;
  const int* masked_m;
  int m_max;
  // mixed launches (one-SM tiles, layers with both large and narrow-tiled
  // experts): the normal-tile kernel also runs the narrow m-tiles, spread
  // evenly among its own, when the plan listed normal m-tiles, and the
  // narrow-tile kernel then has nothing to do; without normal m-tiles the
  // narrow-tile kernel runs them (its deeper ring suits a pure weight stream)
  int mixed;
  const int* narrow_mtiles;
  // test hooks (moe_debug_set_fault), both off when 0: the wait limit of the
  // MMA issuer's wait for a stage's data (the other waits of the kernel get
  // twice this), and 1 + a pipeline iteration whose loads the producer of
  // every CTA skips, so that the wait for that stage expires
  unsigned long long wait_limit_ns;
  int fault_skip_it;
};

// experts with at most this many routed rows use swapped operand roles
constexpr int kMaxSwapRows = 64;
// narrow tiles: the A operand of a stage holds this many rows (the MMA still
// spans 128; the rows past them are padding and never stored)
constexpr int kNarrowRows = 32;

// record the first error of a call in the status word
__device__ inline void set_status(int* hdr, int code) { atomicCAS(&hdr[kHdrStatus], 0, code); }

// a bounded wait expired: MOE_ERR_TIMEOUT and the site of the first expiry
// (10 + epilogue: producer, 20 + epilogue: MMA issuer, 30 + epilogue:
// epilogue warps of the one-SM kernel; 40/50/60 + epilogue the same roles of
// the SM-pair kernel, 70/80/90 + epilogue of the swapped-role kernel)
__device__ inline void record_timeout(int* hdr, int site) {
  set_status(hdr, MOE_ERR_TIMEOUT);
  atomicCAS(&hdr[kHdrTimeoutSite], 0, site);
}

}  // namespace moe
