// moe_indexer.cu -- the FP4 indexer: MQA logits of FP8 queries against FP4
// keys ("DeepSeek DeepGEMM 2026年4月重磅更新：Mega MoE融合算子、FP4精度与极致性能优化",
// sections 5.1-5.2, the fp8_fp4_mqa_logits call):
//
//   logits[i][j] = sum_h w[i][h] * max(0, q[i][h] . k[j])   for ks[i] <= j < ke[i]
//                = -inf                                      elsewhere (when cleaning)
//
// q: FP8 E4M3 [S, Hh, D], k: FP4 E2M1 [N, D], both with one UE8M0 scale per
// 1x32 block along D; FP32 accumulation and output.
//
// Tiling.  The keys sit on the MMA's M side (128 keys per tile) and a group
// of query tokens' (token, head) rows on its N side (kTok tokens, kN =
// kTok * Hh <= 192 rows), so every epilogue thread owns one key and holds all
// heads of its tokens in its accumulator columns: the head-weighted ReLU sum
// is a per-thread loop, no cross-lane reduction.  That sum costs about as
// much as the tile's MMAs, so the accumulator is double-buffered in TMEM
// (two 192-column buffers) and the MMAs of one tile run while the epilogue
// reduces the previous one.
//
// Work order.  A unit is a run of up to C consecutive key tiles of one query
// group; units are numbered chunk-major (unit = chunk * n_groups + group), and
// CTA c takes units c, c + grid, ...  A CTA therefore meets the same query
// group for up to C tiles in a row, and the group's query block (kN rows x D,
// with its scales) is loaded once into a query slot and read by all of them;
// only the 8 KB key tile streams per tile (the 24 KB query block would
// otherwise be most of a tile's bytes).  One CTA per SM, persistent, 480
// threads:
//   warp 0     TMA producer: query blocks into 1-2 query slots (one per group
//              change), key tiles 128 x 128 (E2M1, unpacked by the TMA) with
//              their scale chunk into a ring of up to 8 stages, and the
//              group's head weights into a 4-deep weight ring
//   warps 1,14 TMEM allocator (warp 1) and two MMA-issuing threads
//              (tcgen05.mma kind::mxf8f6f4, A = keys E2M1, B = queries E4M3,
//              M=128, N=kN, K=32) taking alternate tiles, each with its own
//              half of the key ring and its own accumulator buffer
//   warps 2-13 epilogue: three warps per 32-lane TMEM subpartition, the
//              group's tokens split between them
// Tiles whose keys lie outside every token's [ks, ke) skip the loads and the
// MMAs; the epilogue only writes their -inf entries.
#include "moe_device.cuh"
#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int kIdxMaxStages = 8;
constexpr int kIdxSmemA = 128 * 128;   // keys, one byte per E2M1 element
constexpr int kIdxQBlock = 192 * 128;  // one K-block of a query block (up to 192 rows), E4M3
constexpr int kIdxSfbBlock = 2 * kSfChunk;  // the query scales of one K-block
constexpr int kIdxTxA = 128 * 128 / 2; // bytes the TMA moves for the packed keys
constexpr int kIdxEpiWarps = 12;  // three per 32-lane TMEM subpartition
constexpr int kIdxMma2Warp = 2 + kIdxEpiWarps;  // the second MMA thread's warp (14)
constexpr int kIdxThreads = 32 * (kIdxMma2Warp + 1);
constexpr uint32_t kIdxTmemCols = 512;
constexpr uint32_t kIdxAccStride = 256;  // accumulator buffer b at column 256 b
constexpr uint32_t kIdxSfCol = 448;      // scale buffers: SFA at +16x (4 cols), SFB at +16x+4 (8)
constexpr int kIdxWSlot = 1024;          // the group's kN weights, up to 768 bytes
constexpr int kIdxWSlots = 4;
constexpr int kIdxSmemMax = 232448;      // shared memory per CTA
constexpr int kIdxBarBytes = 512;
// Stage info word (producer -> MMA thread): bits 0-1 kind, then for a key
// stage: bit 2 the tile's first K-block, bit 3 its last, bit 4 the parity of
// the query slot's load, bit 5 the query slot, bits 8-15 kb, bits 16-31 the
// query epoch (group change count) mod 2^16; for a release: bit 5 the slot.
constexpr int kStKey = 0;     // a key stage of a tile
constexpr int kStRelQ = 1;    // release a query slot (a stage without loads)
constexpr int kStEnd = 2;     // no more work (a stage without loads)
constexpr int kStFirst = 4, kStLast = 8, kStQPar = 16, kStQSlot = 32;
static_assert(kIdxSmemA % 1024 == 0 && kIdxQBlock % 1024 == 0, "swizzled block alignment");

// tokens per tile for Hh heads: kN = kTok * Hh query rows on the MMA's N side
__host__ __device__ constexpr int idx_tokens(int Hh) { return Hh >= 128 ? 1 : 192 / Hh; }

// Shared-memory plan for KB K-blocks: key stages (16 KB of unpacked codes +
// one 512-byte scale chunk each) and query slots (KB blocks of 24 KB + KB
// scale pairs of 1 KB).  Two query slots when they leave room for two key
// stages, else one; then as many key stages as fit, at most 8.
struct IdxSmem {
  int stages, qslots;
  int a_off, q_off, sfa_off, sfb_off, w_off, bar_off, total;
};
__host__ __device__ inline IdxSmem idx_smem(int KB) {
  IdxSmem p{};
  const int stage = kIdxSmemA + kSfChunk;
  const int qslot = KB * (kIdxQBlock + kIdxSfbBlock);
  const int avail = kIdxSmemMax - kIdxWSlots * kIdxWSlot - kIdxBarBytes;
  p.qslots = (2 * qslot + 2 * stage <= avail) ? 2 : 1;
  p.stages = (avail - p.qslots * qslot) / stage;
  if (p.stages > kIdxMaxStages) p.stages = kIdxMaxStages;
  p.a_off = 0;
  p.q_off = p.a_off + p.stages * kIdxSmemA;
  p.sfa_off = p.q_off + p.qslots * KB * kIdxQBlock;
  p.sfb_off = p.sfa_off + p.stages * kSfChunk;
  p.w_off = p.sfb_off + p.qslots * KB * kIdxSfbBlock;
  p.bar_off = p.w_off + kIdxWSlots * kIdxWSlot;
  p.total = p.bar_off + kIdxBarBytes;
  return p;
}

struct IdxArgs {
  const uint8_t* sfa;    // key scale chunks [KB][ceil(N/128)][512]
  const uint8_t* sfb;    // query scale chunks [group][KB][2][512]
  const float* w;        // [S, Hh]
  const int* ks;         // [S]
  const int* ke;         // [S]
  float* out;            // [S, N]
  int* hdr;              // status header
  const uint8_t* act;    // [n_groups * n_tiles_k]: 1 when some token of the group sees a key of the tile
  int S, Hh, N, KB, clean;
  int n_tiles_k;         // ceil(N / 128)
  int n_groups;          // ceil(S / tokens per tile)
  int chunk_log2;        // C = 2^chunk_log2 key tiles per unit (1..16)
  int n_chunks;          // ceil(n_tiles_k / C)
  int n_units;           // n_groups * n_chunks (< 2^28 for the supported shapes)
  unsigned long long wait_limit_ns;  // 0: the default limits (a test hook shortens them)
  int fault_skip_tile;   // test hook: 1 + the active tile whose key stage is never filled (0 = off)
};

// Does any token of query group g see a key of key tile kt?  (Decided the
// same way by every role of the CTA.)
template <int kTok>
__device__ __forceinline__ bool tile_active(const IdxArgs& a, int kt, int g) {
  const int j0 = kt * 128, j1 = min(j0 + 128, a.N);
#pragma unroll 1
  for (int t = 0; t < kTok; ++t) {
    const int i = g * kTok + t;
    if (i >= a.S) break;
    const int lo = max(__ldg(a.ks + i), 0), hi = min(__ldg(a.ke + i), a.N);
    if (lo < j1 && hi > j0 && lo < hi) return true;
  }
  return false;
}

// Columns [c0, c0 + kHh) of this warp's 32 TMEM lanes -> registers.
template <int kHh>
__device__ __forceinline__ void load_head_cols(uint32_t taddr, uint32_t (&v)[kHh]) {
  using namespace ptx;
  if constexpr (kHh == 16) {
    tmem_ld_32x32b_x16(taddr, v);
  } else {
#pragma unroll
    for (int c = 0; c < kHh / 32; ++c)
      tmem_ld_32x32b_x32(taddr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
  }
}

// Unit m of this CTA (u = blockIdx.x + m * gridDim.x): its group g = u %
// n_groups and first key tile kt0 = (u / n_groups) * C.  False past the last
// unit.  (32-bit: u < n_units + gridDim.x.)
__device__ __forceinline__ bool cta_unit(const IdxArgs& a, int m, int& g, int& kt0) {
  const int u = (int)blockIdx.x + m * (int)gridDim.x;
  if (u >= a.n_units) return false;
  const int c = u / a.n_groups;
  g = u - c * a.n_groups;
  kt0 = c << a.chunk_log2;
  return true;
}
// The k-th tile of this CTA: tile k % C of unit k / C.  False when it lies
// past the last unit or past the last key tile.
__device__ __forceinline__ bool cta_tile(const IdxArgs& a, long long k, int& g, int& kt) {
  int kt0;
  if (!cta_unit(a, (int)(k >> a.chunk_log2), g, kt0)) return false;
  kt = kt0 + (int)(k & ((1 << a.chunk_log2) - 1));
  return kt < a.n_tiles_k;
}

template <int kHh>  // heads per query token (16, 32, 64 or 128)
__global__ void __launch_bounds__(kIdxThreads, 1)
    mqa_logits_kernel(const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmQ, const IdxArgs args) {
  using namespace ptx;
  constexpr int kTok = idx_tokens(kHh);
  constexpr int kN = kTok * kHh;
  static_assert(kN % 16 == 0 && kN <= 192, "MMA N");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {  // the swizzled layout needs it; no work done yet
    pdl_wait();  // the status word is cleared by the previous kernel
    if (threadIdx.x == 0) set_status(args.hdr, MOE_ERR_CUDA);
    return;
  }
  const int KB = args.KB;
  const IdxSmem L = idx_smem(KB);
  const unsigned long long lim = args.wait_limit_ns ? args.wait_limit_ns : kWaitLimitNs;
  const int NS = L.stages, NQ = L.qslots;
  uint8_t* sA = smem_raw + L.a_off;      // [NS][128 x 128]
  uint8_t* sQ = smem_raw + L.q_off;      // [NQ][KB][kN x 128]
  uint8_t* sSFA = smem_raw + L.sfa_off;  // [NS][512]
  uint8_t* sSFB = smem_raw + L.sfb_off;  // [NQ][KB][1 KB]
  float* wslot = reinterpret_cast<float*>(smem_raw + L.w_off);  // [kIdxWSlots][kIdxWSlot / 4]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw + L.bar_off);  // [kIdxMaxStages]
  uint64_t* empty = full + kIdxMaxStages;     // [kIdxMaxStages]
  uint64_t* q_full = empty + kIdxMaxStages;   // [2] query slot loaded
  uint64_t* q_empty = q_full + 2;             // [2] query slot no longer read by MMAs
  uint64_t* acc_full = q_empty + 2;           // [2]
  uint64_t* acc_empty = acc_full + 2;         // [2]
  uint64_t* w_full = acc_empty + 2;           // [kIdxWSlots] weight slot loaded
  uint64_t* w_empty = w_full + kIdxWSlots;    // [kIdxWSlots] weight slot read by every epilogue warp
  uint64_t* drain = w_empty + kIdxWSlots;   // [2] one per MMA thread
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  // what the MMA thread does with stage s (written by the producer before
  // the stage's loads are issued; read after the stage's full barrier)
  int* sinfo = const_cast<int*>(abort_flag) + 1;  // [kIdxMaxStages]
  // Two MMA threads (warp 1 and warp 14, on different SMSPs) take alternate
  // active tiles, each with its own half of the key ring and its own
  // accumulator buffer, so one thread's bookkeeping overlaps the other's
  // MMAs.  With a single key stage (8 K-blocks) there is one ring and one
  // MMA thread.
  const int n_rings = NS >= 2 ? 2 : 1;
  const int ring_a = n_rings == 2 ? (NS + 1) / 2 : NS;  // ring 0: stages [0, ring_a), ring 1: the rest

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&q_full[b], 1);
      mbar_init(&q_empty[b], n_rings);
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kIdxEpiWarps);
    }
    for (int b = 0; b < kIdxWSlots; ++b) {
      mbar_init(&w_full[b], 1);
      mbar_init(&w_empty[b], kIdxEpiWarps);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmQ);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kIdxTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  pdl_wait();  // the key layout, query scale chunks and tile activity come from the prep kernel
  uint32_t issued_mask = 0, last_phase = 0;  // key stages loaded (producer lane), for the failure path
  uint32_t w_issued = 0, w_phase = 0;        // weight slots loaded
  uint32_t q_issued = 0, q_phase = 0;        // query slots loaded

  // This CTA's tiles k = 0 .. n_mine - 1 (cta_tile).  Every role walks them
  // in batches of 32: each lane reads the activity flag of one tile of the
  // next batch while the current batch is worked through, and a ballot turns
  // the 32 flags into a mask, so no tile waits on a global load.
  const long long n_mine =
      args.n_units > (int)blockIdx.x
          ? (long long)((args.n_units - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x)
                << args.chunk_log2
          : 0;
  auto act_flag = [&](long long k) -> uint32_t {
    int g, kt;
    if (k >= n_mine || !cta_tile(args, k, g, kt)) return 0u;
    return (uint32_t)args.act[(size_t)g * args.n_tiles_k + kt];
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Ring positions advance by increments (no division on the per-tile
    // path); the unit is looked up once per unit.  Active tile number tp
    // goes to key ring tp % n_rings.
    struct Ring {
      int s, lo, hi;
      uint32_t ph;
    };
    Ring rg0{0, 0, ring_a, 0}, rg1{ring_a, ring_a, NS, 0};
    int wb = 0, qs = 0, tp = 0;
    uint32_t w_ph = 0, q_ph = 0;
    int qe = -1, cur_g = -1, cur_m = -1, g = 0, kt0 = 0;
    bool ok = true;
    const uint32_t tx = kIdxTxA + kSfChunk;
    const uint32_t qtx = (uint32_t)KB * (kN * 128 + kIdxSfbBlock);
    // the next stage of ring R: wait for it to be free
    auto take = [&](Ring& R, int site) -> bool {
      if (!mbar_wait_or_abort(&empty[R.s], R.ph ^ 1u, 2 * lim, abort_flag)) {
        if (!*abort_flag) record_timeout(args.hdr, site);
        *abort_flag = 1;
        return false;
      }
      return true;
    };
    auto advance = [&](Ring& R) {
      if (++R.s == R.hi) {
        R.s = R.lo;
        R.ph ^= 1u;
      }
    };
    // a stage without loads: only its info word
    auto send_info = [&](Ring& R, int code, int site) -> bool {
      if (!take(R, site)) return false;
      sinfo[R.s] = code;
      mbar_arrive(&full[R.s]);
      advance(R);
      return true;
    };
    // the key stages of one tile
    auto send_tile = [&](Ring& R, int kt, int qinfo) -> bool {
      for (int kb = 0; kb < KB; ++kb) {
        if (kb == 0 && tp + 1 == args.fault_skip_tile) {  // test hook: this stage never fills
          advance(R);
          continue;
        }
        if (!take(R, 110)) return false;
        const int st = R.s;
        sinfo[st] = kStKey | (kb == 0 ? kStFirst : 0) | (kb == KB - 1 ? kStLast : 0) | qinfo |
                    (kb << 8);
        mbar_arrive_expect_tx(&full[st], tx);
        tma_load_3d(sA + (size_t)st * kIdxSmemA, &tmK, &full[st], 0, kt * 128, kb);
        bulk_load(sSFA + st * kSfChunk, args.sfa + ((size_t)kb * args.n_tiles_k + kt) * kSfChunk,
                  kSfChunk, &full[st]);
        issued_mask |= 1u << st;
        last_phase = (last_phase & ~(1u << st)) | (R.ph << st);
        advance(R);
      }
      return true;
    };
    uint32_t fnext = act_flag(lane);
    for (long long k0 = 0; k0 < n_mine && ok; k0 += 32) {
      uint32_t mask = __ballot_sync(0xffffffffu, fnext != 0);
      fnext = act_flag(k0 + 32 + lane);
      while (mask != 0 && ok) {
        const long long k = k0 + __ffs(mask) - 1;
        mask &= mask - 1;
        if (lane == 0) {
          const int m = (int)(k >> args.chunk_log2);
          if (m != cur_m) {
            cur_m = m;
            (void)cta_unit(args, m, g, kt0);  // an active tile: its unit exists
          }
          const int kt = kt0 + (int)(k & ((1 << args.chunk_log2) - 1));
          if (g != cur_g) {
            if (qe >= 0) {
              // Info-only stages tell both MMA threads that the current query
              // slot is read by no later MMA: each releases it once its MMAs
              // issued so far complete.  (With one slot the wait below needs
              // exactly that release.)
              const int code = kStRelQ | (qs ? kStQSlot : 0);
              ok = send_info(rg0, code, 114) && (n_rings == 1 || send_info(rg1, code, 114));
              if (++qs == NQ) {
                qs = 0;
                q_ph ^= 1u;
              }
            }
            if (ok) {
              // a new query group: its query block and scales into the next slot
              ++qe;
              cur_g = g;
              if (!mbar_wait_or_abort(&q_empty[qs], q_ph ^ 1u, 2 * lim, abort_flag)) {
                if (!*abort_flag) record_timeout(args.hdr, 112);
                *abort_flag = 1;
                ok = false;
              } else {
                mbar_arrive_expect_tx(&q_full[qs], qtx);
                for (int kb = 0; kb < KB; ++kb)
                  tma_load_2d(sQ + (size_t)(qs * KB + kb) * kIdxQBlock, &tmQ, &q_full[qs],
                              kb * 128, g * kN);
                bulk_load(sSFB + (size_t)qs * KB * kIdxSfbBlock,
                          args.sfb + (size_t)g * KB * kIdxSfbBlock, (uint32_t)KB * kIdxSfbBlock,
                          &q_full[qs]);
                q_issued |= 1u << qs;
                q_phase = (q_phase & ~(1u << qs)) | (q_ph << qs);
              }
            }
          }
          if (ok) {
            const int qinfo = (q_ph ? kStQPar : 0) | (qs ? kStQSlot : 0) | ((qe & 0xffff) << 16);
            ok = (n_rings == 2 && (tp & 1)) ? send_tile(rg1, kt, qinfo) : send_tile(rg0, kt, qinfo);
          }
          if (ok) {
            // the group's weights into the next slot of the weight ring (rows
            // of tokens past S are not read: the slot keeps stale values there)
            if (!mbar_wait_or_abort(&w_empty[wb], w_ph ^ 1u, 2 * lim, abort_flag)) {
              if (!*abort_flag) record_timeout(args.hdr, 111);
              *abort_flag = 1;
              ok = false;
            } else {
              const int ntok = min(kTok, args.S - g * kTok);
              const uint32_t wbytes = (uint32_t)(ntok * kHh * 4);
              mbar_arrive_expect_tx(&w_full[wb], wbytes);
              bulk_load(wslot + wb * (kIdxWSlot / 4), args.w + (size_t)g * kN, wbytes, &w_full[wb]);
              w_issued |= 1u << wb;
              w_phase = (w_phase & ~(1u << wb)) | (w_ph << wb);
              if (++wb == kIdxWSlots) {
                wb = 0;
                w_ph ^= 1u;
              }
              ++tp;
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
    }
    // one more stage per ring, without loads, tells the MMA threads that the work ends
    if (lane == 0 && ok) {
      if (send_info(rg0, kStEnd, 113) && n_rings == 2) (void)send_info(rg1, kStEnd, 113);
    }
  } else if ((warp == 1 || (warp == kIdxMma2Warp && n_rings == 2)) && lane == 0) {
    // ----------------------------------------------------------------- MMA
    // Each MMA thread shares its SMSP with three epilogue warps and each of
    // its instructions takes tens of cycles while the tensor pipe waits for
    // it; so it walks no tile list: it takes its ring's stages in order and
    // reads from each stage's info word what to do around its MMAs.
    const int r = warp == 1 ? 0 : 1;  // ring, and (with two rings) accumulator buffer
    const int lo = r == 0 ? 0 : ring_a, hi = r == 0 ? ring_a : NS;
    int s = lo, b = r, cur_q = -1;
    uint32_t ph = 0, acc_ph = 0, x = 0;  // x: which of this thread's two TMEM scale buffers
    int sfb_tag0 = -1, sfb_tag1 = -1;  // (epoch << 8 | kb) + 1 whose query scales each scale buffer holds
    bool issued_any = false, ok = true;
    const uint32_t idesc0 = idesc_mxf8f6f4(/*A E2M1*/ 5, /*B E4M3*/ 0, 128, kN);
    uint32_t id[4];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) id[kk] = idesc_with_sf_id(idesc0, kk, kk);
    const uint64_t a_desc0 = sdesc_sw128(smem_u32(sA)), q_desc0 = sdesc_sw128(smem_u32(sQ));
    const uint64_t sfa_desc0 = sdesc_sf(smem_u32(sSFA)), sfb_desc0 = sdesc_sf(smem_u32(sSFB));
    for (;;) {
      if (!mbar_wait_or_abort(&full[s], ph, lim, abort_flag)) {
        ok = false;
        break;
      }
      const int info = sinfo[s];
      const int kind = info & 3;
      if (kind == kStEnd) break;
      const int qs = (info & kStQSlot) ? 1 : 0;
      if (kind == kStRelQ) {
        // the query slot is free once this thread's MMAs issued so far complete
        tc_commit(&q_empty[qs]);
        mbar_arrive(&empty[s]);  // the stage carried no data
      } else {
        const int qtag = info >> 16;  // query epoch mod 2^16
        if (qtag != cur_q) {
          cur_q = qtag;
          if (!mbar_wait_or_abort(&q_full[qs], (info & kStQPar) ? 1u : 0u, 2 * lim,
                                  abort_flag)) {
            ok = false;
            break;
          }
        }
        if ((info & kStFirst) &&
            !mbar_wait_or_abort(&acc_empty[b], acc_ph ^ 1u, 2 * lim, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int kb = (info >> 8) & 0xff;
        const uint32_t acc = tmem + kIdxAccStride * (uint32_t)b;
        const uint32_t sfa_t = tmem + kIdxSfCol + 16u * (2u * (uint32_t)r + x);
        const uint32_t sfb_t = sfa_t + 4u;
        tc_cp_32x128b_warpx4(sfa_t, sfa_desc0 + (uint64_t)(((uint32_t)s * kSfChunk) >> 4));
        const int tag = ((qtag << 8) | kb) + 1;
        if ((x ? sfb_tag1 : sfb_tag0) != tag) {  // else the buffer still holds these query scales
          const uint32_t sfb_off = (uint32_t)(qs * KB + kb) * kIdxSfbBlock;
          tc_cp_32x128b_warpx4(sfb_t, sfb_desc0 + (uint64_t)(sfb_off >> 4));
          if (kN > 128)
            tc_cp_32x128b_warpx4(sfb_t + 4u, sfb_desc0 + (uint64_t)((sfb_off + kSfChunk) >> 4));
          if (x)
            sfb_tag1 = tag;
          else
            sfb_tag0 = tag;
        }
        const uint64_t adesc = a_desc0 + (uint64_t)(((uint32_t)s * kIdxSmemA) >> 4);
        const uint64_t bdesc = q_desc0 + (uint64_t)(((uint32_t)(qs * KB + kb) * kIdxQBlock) >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_mxf8f6f4(acc, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), id[kk],
                       (kb | kk) != 0 ? 1u : 0u, sfa_t | ((uint32_t)kk << 30),
                       sfb_t | ((uint32_t)kk << 30));
        issued_any = true;
        tc_commit(&empty[s]);
        if (info & kStLast) {
          tc_commit(&acc_full[b]);
          if (n_rings == 1) {
            b ^= 1;
            if (b == 0) acc_ph ^= 1u;
          } else {
            acc_ph ^= 1u;
          }
        }
        x ^= 1u;
      }
      if (++s == hi) {
        s = lo;
        ph ^= 1u;
      }
    }
    if (!ok) {
      if (!*abort_flag) record_timeout(args.hdr, 120 + r);
      *abort_flag = 1;
      if (issued_any) {  // wait for the MMAs in flight before TMEM is released
        tc_commit(&drain[r]);
        (void)mbar_wait(&drain[r], 0);
      }
    }
  } else if (warp >= 2 && warp < kIdxMma2Warp) {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;          // 0..11
    const int q = warp & 3;           // TMEM lane subpartition this warp can read
    const int h = ew >> 2;            // which of the group's tokens: t = h, h + 3, ...
    const int r = q * 32 + lane;      // key within the tile
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    constexpr int kMine = (kTok + 2) / 3;
    int ta = 0;
    bool dead = false;
    int unit_m = -1, g = 0, kt0 = 0;  // the current unit, looked up once per unit
    uint32_t fnext = act_flag(lane);
    for (long long k0 = 0; k0 < n_mine && !dead; k0 += 32) {
      const uint32_t mask = __ballot_sync(0xffffffffu, fnext != 0);
      fnext = act_flag(k0 + 32 + lane);
      const int nb = (int)(n_mine - k0 < 32 ? n_mine - k0 : 32);
      for (int bit = 0; bit < nb; ++bit) {
        const long long k = k0 + bit;
        const int m = (int)(k >> args.chunk_log2);
        if (m != unit_m) {
          unit_m = m;
          (void)cta_unit(args, m, g, kt0);  // k < n_mine: the unit exists
        }
        const int kt = kt0 + (int)(k & ((1 << args.chunk_log2) - 1));
        if (kt >= args.n_tiles_k) continue;  // past the last key tile: no entries
        const int j = kt * 128 + r;
        const bool active = (mask >> bit) & 1u;
        // key ranges of this warp's tokens (loaded before the waits)
        int lo[kMine], hi[kMine];
#pragma unroll
        for (int m = 0; m < kMine; ++m) {
          const int i = g * kTok + h + 3 * m;
          const bool tok = active && h + 3 * m < kTok && i < args.S;
          lo[m] = tok ? max(__ldg(args.ks + i), 0) : 0;
          hi[m] = tok ? min(__ldg(args.ke + i), args.N) : 0;
        }
        const int b = ta & 1;            // accumulator buffer
        const int wb = ta % kIdxWSlots;  // weight slot
        bool use = false;  // this tile's accumulator (and weight slot) is read
        if (active) {
          const uint32_t par = (ta >> 1) & 1, wpar = (uint32_t)(ta / kIdxWSlots) & 1u;
          const bool ready =
              __all_sync(0xffffffffu,
                         mbar_wait_or_abort(&acc_full[b], par, 2 * lim, abort_flag) &&
                             mbar_wait_or_abort(&w_full[wb], wpar, 2 * lim, abort_flag));
          if (!ready) {
            if (lane == 0) {
              if (!*abort_flag) record_timeout(args.hdr, 130);
              *abort_flag = 1;
            }
            dead = true;
            break;
          }
          tc_fence_after();
          use = true;
        }
        const float* w_s = wslot + wb * (kIdxWSlot / 4);
        // this warp's tokens t = h + 3m, in column chunks of at most 64: every
        // TMEM load of a chunk first, one wait, then the weighted ReLU sums on
        // eight independent accumulator chains (head c goes to chain c % 8),
        // two chains per packed FP32x2 instruction
        constexpr int kC = kHh > 64 ? 64 : kHh;  // columns per chunk
        uint64_t acc[kMine][4];
#pragma unroll
        for (int m = 0; m < kMine; ++m)
#pragma unroll
          for (int u = 0; u < 4; ++u) acc[m][u] = 0ull;
#pragma unroll
        for (int c0 = 0; c0 < kHh; c0 += kC) {
          uint32_t v[kMine][kC];
          if (use) {  // warp-uniform: the TMEM loads are collective
#pragma unroll
            for (int m = 0; m < kMine; ++m)
              if (h + 3 * m < kTok)
                load_head_cols<kC>(trow + kIdxAccStride * (uint32_t)b +
                                       (uint32_t)((h + 3 * m) * kHh + c0), v[m]);
            tc_wait_ld();
            if (c0 + kC >= kHh) {
              // the last chunk is in registers: the accumulator buffer is free
              // for the next tile's MMAs while the sums below run
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&acc_empty[b]);
            }
#pragma unroll
            for (int m = 0; m < kMine; ++m) {
              const int t = h + 3 * m;
              if (t < kTok) {
                const ulonglong2* wt = reinterpret_cast<const ulonglong2*>(w_s + t * kHh + c0);
#pragma unroll
                for (int h4 = 0; h4 < kC / 4; ++h4) {
                  const ulonglong2 w4 = wt[h4];  // heads c0 + 4 h4 .. + 3, two per word
                  const uint64_t x01 = relu_pack_f32x2(v[m][4 * h4], v[m][4 * h4 + 1]);
                  const uint64_t x23 = relu_pack_f32x2(v[m][4 * h4 + 2], v[m][4 * h4 + 3]);
                  acc[m][(2 * h4) & 3] = fma_f32x2(w4.x, x01, acc[m][(2 * h4) & 3]);
                  acc[m][(2 * h4 + 1) & 3] = fma_f32x2(w4.y, x23, acc[m][(2 * h4 + 1) & 3]);
                }
              }
            }
          }
        }
        if (use) {  // the weights are read: release their slot
          __syncwarp();
          if (lane == 0) mbar_arrive(&w_empty[wb]);
        }
#pragma unroll
        for (int m = 0; m < kMine; ++m) {
          const int t = h + 3 * m;
          const int i = g * kTok + t;
          const bool here = t < kTok && i < args.S && j < args.N;  // an entry of the output
          const bool scored = use && here && j >= lo[m] && j < hi[m];
          float a8[8];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            a8[2 * u] = __uint_as_float((uint32_t)acc[m][u]);
            a8[2 * u + 1] = __uint_as_float((uint32_t)(acc[m][u] >> 32));
          }
          const float logit = scored ? ((a8[0] + a8[1]) + (a8[2] + a8[3])) +
                                           ((a8[4] + a8[5]) + (a8[6] + a8[7]))
                                     : -INFINITY;
          if (scored || (here && args.clean)) args.out[(size_t)i * args.N + j] = logit;
        }
        if (active) ++ta;
      }
    }
  }

  pdl_launch();
  tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0 && *abort_flag) {
    // copies issued that nobody consumed land before the CTA's memory goes away
    for (int s = 0; s < NS; ++s)
      if (issued_mask & (1u << s)) (void)mbar_wait(&full[s], (last_phase >> s) & 1);
    for (int b = 0; b < kIdxWSlots; ++b)
      if (w_issued & (1u << b)) (void)mbar_wait(&w_full[b], (w_phase >> b) & 1);
    for (int b = 0; b < 2; ++b)
      if (q_issued & (1u << b)) (void)mbar_wait(&q_full[b], (q_phase >> b) & 1);
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kIdxTmemCols);
  }
}

// Keys into the layout the key tiles stream, for any N: codes [KB][Np][64 B]
// (Np = N rounded up to 128; padding rows zero) and UE8M0 chunks
// [KB][Np/128][512 B] (byte (r%32)*16 + (r/32)*4 + j of a chunk = row r,
// K-block j of the 128-element slice; padding rows zero).  Item x = one
// (K-block, row).
struct KvPrep {
  const uint8_t* kv;
  const uint8_t* kv_sf;
  int N, Np, D;
  uint8_t* codes;
  uint8_t* chunks;
};
__device__ __forceinline__ void kv_prep_item(const KvPrep& p, long long x) {
  const int n = (int)(x % p.Np), kb = (int)(x / p.Np);
  uint4* d4 = reinterpret_cast<uint4*>(p.codes + ((size_t)kb * p.Np + n) * 64);
  uint32_t sfw = 0;
  if (n < p.N) {
    const uint4* s4 = reinterpret_cast<const uint4*>(p.kv + (size_t)n * (p.D / 2) + (size_t)kb * 64);
#pragma unroll
    for (int c = 0; c < 4; ++c) d4[c] = s4[c];
    sfw = *reinterpret_cast<const uint32_t*>(p.kv_sf + (size_t)n * (p.D / 32) + (size_t)kb * 4);
  } else {
#pragma unroll
    for (int c = 0; c < 4; ++c) d4[c] = make_uint4(0, 0, 0, 0);
  }
  const size_t chunk = (size_t)kb * (p.Np / 128) + (n >> 7);
  *reinterpret_cast<uint32_t*>(p.chunks + chunk * kSfChunk + (n & 31) * 16 + ((n >> 5) & 3) * 4) = sfw;
}

// Query scales into per-group chunk pairs [group][KB][2][512 B]: query row r
// (token * Hh + head) belongs to group r / kN, row rr = r % kN of it; chunk
// rr / 128 of the pair, byte (rr%32)*16 + ((rr%128)/32)*4 + j.  Rows of the
// pair past kN (or past the last token) stay whatever they were: their MMA
// columns are never read.  Item x = one (row, K-block).
struct QPrep {
  const int32_t* q_sf;
  int KB, kN;
  uint8_t* out;
};
__device__ __forceinline__ void q_prep_item(const QPrep& p, long long x) {
  const long long r = x / p.KB;
  const int kb = (int)(x - r * p.KB);
  const long long g = r / p.kN;
  const int rr = (int)(r - g * p.kN);
  uint8_t* dst = p.out + ((size_t)g * p.KB + kb) * kIdxSfbBlock + (rr >> 7) * kSfChunk;
  const int r7 = rr & 127;
  *reinterpret_cast<int32_t*>(dst + (r7 & 31) * 16 + (r7 >> 5) * 4) = p.q_sf[x];
}

// Everything the logits kernel reads that the call derives from its inputs,
// in one launch: the status words cleared, the key layout, the query scale
// chunks, and act[g * n_tiles_k + kt] = 1 when some token of query group g
// sees a key of key tile kt.  The three jobs are independent; one grid-stride
// loop walks their items back to back.
template <int kTok>
__global__ void mqa_prep_kernel(KvPrep kvp, long long n_kv, QPrep qp, long long n_q, IdxArgs a,
                                uint8_t* __restrict__ act, long long n_act) {
  if (blockIdx.x == 0 && threadIdx.x < kHdrWords) a.hdr[threadIdx.x] = 0;
  const long long total = n_kv + n_q + n_act;
  for (long long x = blockIdx.x * (long long)blockDim.x + threadIdx.x; x < total;
       x += (long long)gridDim.x * blockDim.x) {
    if (x < n_kv) {
      kv_prep_item(kvp, x);
    } else if (x < n_kv + n_q) {
      q_prep_item(qp, x - n_kv);
    } else {
      const long long y = x - n_kv - n_q;
      const int g = (int)(y / a.n_tiles_k), kt = (int)(y - (long long)g * a.n_tiles_k);
      act[y] = tile_active<kTok>(a, kt, g) ? 1 : 0;
    }
  }
}

}  // namespace

int mqa_tokens_per_tile(int Hh) { return idx_tokens(Hh); }
size_t mqa_qsf_bytes_per_group(int D) { return (size_t)(D / 128) * kIdxSfbBlock; }

cudaError_t launch_mqa_logits(const CUtensorMap& tmK, const CUtensorMap& tmQ, const uint8_t* kv,
                              const uint8_t* kv_sf, uint8_t* codes, uint8_t* sfa, int Np,
                              const int32_t* q_sf, uint8_t* sfb, const float* w, const int* ks,
                              const int* ke, float* out, int* hdr, uint8_t* act, int S, int Hh,
                              int N, int KB, int clean, int grid, bool pdl,
                              unsigned long long wait_limit_ns, int fault_skip_tile,
                              cudaStream_t stream) {
  typedef void (*Fn)(CUtensorMap, CUtensorMap, IdxArgs);
  typedef void (*ActFn)(KvPrep, long long, QPrep, long long, IdxArgs, uint8_t*, long long);
  Fn fn;
  ActFn afn;
  int slot;
  switch (Hh) {
    case 16: fn = mqa_logits_kernel<16>; afn = mqa_prep_kernel<idx_tokens(16)>; slot = 0; break;
    case 32: fn = mqa_logits_kernel<32>; afn = mqa_prep_kernel<idx_tokens(32)>; slot = 1; break;
    case 64: fn = mqa_logits_kernel<64>; afn = mqa_prep_kernel<idx_tokens(64)>; slot = 2; break;
    case 128: fn = mqa_logits_kernel<128>; afn = mqa_prep_kernel<idx_tokens(128)>; slot = 3; break;
    default: return cudaErrorInvalidValue;
  }
  static bool attr_set[4] = {};
  if (!attr_set[slot]) {
    cudaError_t err = cudaFuncSetAttribute((const void*)fn,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kIdxSmemMax);
    if (err != cudaSuccess) return err;
    attr_set[slot] = true;
  }
  IdxArgs a{};
  a.sfa = sfa;
  a.sfb = sfb;
  a.w = w;
  a.ks = ks;
  a.ke = ke;
  a.out = out;
  a.hdr = hdr;
  a.S = S;
  a.Hh = Hh;
  a.N = N;
  a.KB = KB;
  a.clean = clean;
  a.n_tiles_k = (N + 127) / 128;
  a.n_groups = (S + idx_tokens(Hh) - 1) / idx_tokens(Hh);
  a.act = act;
  // key tiles per unit: 16, halved while the units would number fewer than
  // four per CTA, and no more than the key tiles round up to
  int lg = 4;
  while (lg > 0 && ((long long)a.n_groups * ((a.n_tiles_k + (1 << lg) - 1) >> lg) < 4LL * grid ||
                    (1 << (lg - 1)) >= a.n_tiles_k))
    --lg;
  a.chunk_log2 = lg;
  a.n_chunks = (a.n_tiles_k + (1 << lg) - 1) >> lg;
  a.n_units = a.n_groups * a.n_chunks;
  a.wait_limit_ns = wait_limit_ns;
  a.fault_skip_tile = fault_skip_tile;
  const IdxSmem L = idx_smem(KB);
  if (L.stages < 1 || L.total > kIdxSmemMax) return cudaErrorInvalidValue;
  {
    const KvPrep kvp{kv, kv_sf, N, Np, KB * 128, codes, sfa};
    const QPrep qp{q_sf, KB, idx_tokens(Hh) * Hh, sfb};
    const long long n_kv = (long long)KB * Np, n_q = (long long)S * Hh * KB;
    const long long n_act = (long long)a.n_tiles_k * a.n_groups;
    long long pgrid = (n_kv + n_q + n_act + 255) / 256;
    if (pgrid > 148LL * 16) pgrid = 148LL * 16;
    if (pgrid < 1) pgrid = 1;
    afn<<<(unsigned)pgrid, 256, 0, stream>>>(kvp, n_kv, qp, n_q, a, act, n_act);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kIdxThreads);
  cfg.dynamicSmemBytes = (size_t)L.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, fn, tmK, tmQ, a);
}

}  // namespace moe
