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
// reduces the previous one.  One CTA per SM, persistent, 320 threads:
//   warp 0     TMA producer: key tile 128 x 128 (E2M1, unpacked by the TMA),
//              query tile kN x 128 (E4M3), their scale chunks; 4-stage ring
//   warp 1     TMEM allocator and MMA issuer (tcgen05.mma kind::mxf8f6f4,
//              A = keys E2M1, B = queries E4M3, M=128, N=kN, K=32)
//   warps 2-13 epilogue: three warps per 32-lane TMEM subpartition, the
//              group's tokens split between them
// Tiles whose keys lie outside every token's [ks, ke) skip the loads and the
// MMAs; the epilogue only writes their -inf entries.
#include "moe_device.cuh"
#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int kIdxStages = 4;
constexpr int kIdxSmemA = 128 * 128;   // keys, one byte per E2M1 element
constexpr int kIdxSmemB = 192 * 128;   // queries (up to 192 rows), E4M3
constexpr int kIdxSmemSFB = 2 * kSfChunk;
constexpr int kIdxTxA = 128 * 128 / 2; // bytes the TMA moves for the packed keys
constexpr int kIdxEpiWarps = 12;  // three per 32-lane TMEM subpartition
constexpr int kIdxThreads = 64 + 32 * kIdxEpiWarps;
constexpr uint32_t kIdxTmemCols = 512;
constexpr uint32_t kIdxAccStride = 256;  // accumulator buffer b at column 256 b
constexpr uint32_t kIdxSfCol = 448;      // scale buffers: SFA at +16b (4 cols), SFB at +16b+4 (8)
// stage ring, then a ring of weight slots (the group's kN weights, up to 768
// bytes each; four deep, so a slot's bulk load is issued while the epilogue
// is still three tiles behind it), then barriers
constexpr size_t kIdxSmemStage = (size_t)kIdxStages * (kIdxSmemA + kIdxSmemB + kSfChunk + kIdxSmemSFB);
constexpr int kIdxWSlot = 1024;
constexpr int kIdxWSlots = 4;
constexpr size_t kIdxSmemBytes = kIdxSmemStage + kIdxWSlots * kIdxWSlot + 256;
static_assert(kIdxSmemBytes <= 232448, "shared memory per CTA");
static_assert(kIdxSmemA % 1024 == 0 && kIdxSmemB % 1024 == 0, "swizzled stage alignment");

// tokens per tile for Hh heads: kN = kTok * Hh query rows on the MMA's N side
__host__ __device__ constexpr int idx_tokens(int Hh) { return Hh >= 128 ? 1 : 192 / Hh; }

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
    if (threadIdx.x == 0) set_status(args.hdr, MOE_ERR_CUDA);
    return;
  }
  uint8_t* sA = smem_raw;
  uint8_t* sB = sA + kIdxStages * kIdxSmemA;
  uint8_t* sSFA = sB + kIdxStages * kIdxSmemB;
  uint8_t* sSFB = sSFA + kIdxStages * kSfChunk;
  float* wslot = reinterpret_cast<float*>(smem_raw + kIdxSmemStage);  // [kIdxWSlots][kIdxWSlot / 4]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw + kIdxSmemStage + kIdxWSlots * kIdxWSlot);
  uint64_t* empty = full + kIdxStages;
  uint64_t* acc_full = empty + kIdxStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint64_t* w_full = acc_empty + 2;         // [kIdxWSlots] weight slot loaded
  uint64_t* w_empty = w_full + kIdxWSlots;  // [kIdxWSlots] weight slot read by every epilogue warp
  uint64_t* drain = w_empty + kIdxWSlots;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kIdxStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kIdxEpiWarps);
    }
    for (int b = 0; b < kIdxWSlots; ++b) {
      mbar_init(&w_full[b], 1);
      mbar_init(&w_empty[b], kIdxEpiWarps);
    }
    mbar_init(drain, 1);
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

  pdl_wait();  // the transformed keys and the query scale chunks come from the previous kernels
  const int KB = args.KB;
  const int num_tiles = args.n_tiles_k * args.n_groups;
  uint32_t issued_mask = 0, last_phase = 0;
  uint32_t w_issued = 0, w_phase = 0;  // weight slots loaded (producer lane), for the failure path

  // This CTA's tiles are blockIdx.x + k * gridDim.x, k = 0 .. n_mine - 1.
  // Every role walks them in batches of 32: each lane reads the activity flag
  // of one tile of the next batch while the current batch is worked through,
  // and a ballot turns the 32 flags into a mask, so no tile waits on a global
  // load.
  const long long n_mine =
      num_tiles > (int)blockIdx.x ? (num_tiles - (long long)blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  auto act_flag = [&](long long k) -> uint32_t {
    const long long t = blockIdx.x + k * gridDim.x;
    return (k < n_mine && t < num_tiles) ? (uint32_t)args.act[t] : 0u;
  };
  auto tile_of = [&](long long k) -> int { return (int)(blockIdx.x + k * gridDim.x); };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint32_t it = 0;
    int tp = 0;  // active tiles so far
    bool ok = true;
    const uint32_t tx = kIdxTxA + kN * 128 + kSfChunk + kIdxSmemSFB;
    uint32_t fnext = act_flag(lane);
    for (long long k0 = 0; k0 < n_mine && ok; k0 += 32) {
      uint32_t mask = __ballot_sync(0xffffffffu, fnext != 0);
      fnext = act_flag(k0 + 32 + lane);
      while (mask != 0 && ok) {
        const int tile = tile_of(k0 + __ffs(mask) - 1);
        mask &= mask - 1;
        if (lane == 0) {
          const int g = tile / args.n_tiles_k, kt = tile - g * args.n_tiles_k;
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = it % kIdxStages;
            const uint32_t ph = (it / kIdxStages) & 1;
            if (!mbar_wait_or_abort(&empty[s], ph ^ 1, 2 * kWaitLimitNs, abort_flag)) {
              if (!*abort_flag) record_timeout(args.hdr, 110);
              *abort_flag = 1;
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[s], tx);
            tma_load_3d(sA + s * kIdxSmemA, &tmK, &full[s], 0, kt * 128, kb);
            tma_load_2d(sB + s * kIdxSmemB, &tmQ, &full[s], kb * 128, g * kN);
            bulk_load(sSFA + s * kSfChunk,
                      args.sfa + ((size_t)kb * args.n_tiles_k + kt) * kSfChunk, kSfChunk, &full[s]);
            bulk_load(sSFB + s * kIdxSmemSFB, args.sfb + ((size_t)g * KB + kb) * kIdxSmemSFB,
                      kIdxSmemSFB, &full[s]);
            issued_mask |= 1u << s;
            last_phase = (last_phase & ~(1u << s)) | (ph << s);
          }
          if (ok) {
            // the group's weights into the next slot of the weight ring (rows
            // of tokens past S are not read: the slot keeps stale values there)
            const int b = tp % kIdxWSlots;
            const uint32_t wpar = (uint32_t)(tp / kIdxWSlots) & 1u;
            if (!mbar_wait_or_abort(&w_empty[b], wpar ^ 1, 2 * kWaitLimitNs, abort_flag)) {
              if (!*abort_flag) record_timeout(args.hdr, 111);
              *abort_flag = 1;
              ok = false;
            } else {
              const int ntok = min(kTok, args.S - g * kTok);
              const uint32_t wbytes = (uint32_t)(ntok * kHh * 4);
              mbar_arrive_expect_tx(&w_full[b], wbytes);
              bulk_load(wslot + b * (kIdxWSlot / 4), args.w + (size_t)g * kN, wbytes, &w_full[b]);
              w_issued |= 1u << b;
              w_phase = (w_phase & ~(1u << b)) | (wpar << b);
              ++tp;
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    uint32_t it = 0;
    int ta = 0;  // active tiles so far
    bool issued_any = false, ok = true;
    const uint32_t idesc0 = idesc_mxf8f6f4(/*A E2M1*/ 5, /*B E4M3*/ 0, 128, kN);
    const uint64_t a_desc0 = sdesc_sw128(smem_u32(sA)), b_desc0 = sdesc_sw128(smem_u32(sB));
    const uint64_t sfa_desc0 = sdesc_sf(smem_u32(sSFA)), sfb_desc0 = sdesc_sf(smem_u32(sSFB));
    uint32_t fnext = act_flag(lane);
    for (long long k0 = 0; k0 < n_mine && ok; k0 += 32) {
      uint32_t mask = __ballot_sync(0xffffffffu, fnext != 0);
      fnext = act_flag(k0 + 32 + lane);
      // only the count of active tiles matters here: the stages arrive in order
      for (int n = __popc(mask); n > 0 && ok; --n) {
        if (lane == 0) {
          const int b = ta & 1;
          if (!mbar_wait_or_abort(&acc_empty[b], ((ta >> 1) & 1) ^ 1, 2 * kWaitLimitNs,
                                  abort_flag)) {
            ok = false;
          } else {
            tc_fence_after();
            const uint32_t acc = tmem + kIdxAccStride * (uint32_t)b;
            for (int kb = 0; kb < KB; ++kb, ++it) {
              const int s = it % kIdxStages;
              const uint32_t ph = (it / kIdxStages) & 1;
              if (!mbar_wait_or_abort(&full[s], ph, kWaitLimitNs, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t sfa_t = tmem + kIdxSfCol + 16u * (it & 1u);
              const uint32_t sfb_t = sfa_t + 4u;
              tc_cp_32x128b_warpx4(sfa_t, sfa_desc0 + (uint64_t)((s * kSfChunk) >> 4));
              tc_cp_32x128b_warpx4(sfb_t, sfb_desc0 + (uint64_t)((s * kIdxSmemSFB) >> 4));
              if (kN > 128)
                tc_cp_32x128b_warpx4(sfb_t + 4u,
                                     sfb_desc0 + (uint64_t)((s * kIdxSmemSFB + kSfChunk) >> 4));
              const uint64_t adesc = a_desc0 + (uint64_t)((s * kIdxSmemA) >> 4);
              const uint64_t bdesc = b_desc0 + (uint64_t)((s * kIdxSmemB) >> 4);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint32_t id = idesc_with_sf_id(idesc0, kk, kk);
                mma_mxf8f6f4(acc, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), id,
                             (kb | kk) != 0 ? 1u : 0u, sfa_t | ((uint32_t)kk << 30),
                             sfb_t | ((uint32_t)kk << 30));
              }
              issued_any = true;
              tc_commit(&empty[s]);
            }
            if (ok) {
              tc_commit(&acc_full[b]);
              ++ta;
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
    }
    if (lane == 0 && !ok) {
      if (!*abort_flag) record_timeout(args.hdr, 120);
      *abort_flag = 1;
      if (issued_any) {  // wait for the MMAs in flight before TMEM is released
        tc_commit(drain);
        (void)mbar_wait(drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;          // 0..11
    const int q = warp & 3;           // TMEM lane subpartition this warp can read
    const int h = ew >> 2;            // which of the group's tokens: t = h, h + 3, ...
    const int r = q * 32 + lane;      // key within the tile
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    constexpr int kMine = (kTok + 2) / 3;
    int ta = 0;
    bool dead = false;
    uint32_t fnext = act_flag(lane);
    for (long long k0 = 0; k0 < n_mine && !dead; k0 += 32) {
      const uint32_t mask = __ballot_sync(0xffffffffu, fnext != 0);
      fnext = act_flag(k0 + 32 + lane);
      const int nb = (int)(n_mine - k0 < 32 ? n_mine - k0 : 32);
      for (int bit = 0; bit < nb; ++bit) {
        const int tile = tile_of(k0 + bit);
        const int g = tile / args.n_tiles_k, kt = tile - g * args.n_tiles_k;
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
                         mbar_wait_or_abort(&acc_full[b], par, 2 * kWaitLimitNs, abort_flag) &&
                             mbar_wait_or_abort(&w_full[wb], wpar, 2 * kWaitLimitNs, abort_flag));
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
        if (use) {  // accumulator and weights are in registers: release both
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&acc_empty[b]);
            mbar_arrive(&w_empty[wb]);
          }
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
    for (int s = 0; s < kIdxStages; ++s)
      if (issued_mask & (1u << s)) (void)mbar_wait(&full[s], (last_phase >> s) & 1);
    for (int b = 0; b < kIdxWSlots; ++b)
      if (w_issued & (1u << b)) (void)mbar_wait(&w_full[b], (w_phase >> b) & 1);
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kIdxTmemCols);
  }
}

// act[g * n_tiles_k + kt] = 1 when some token of query group g sees a key
// of key tile kt.  One thread per tile.
template <int kTok>
__global__ void tile_activity_kernel(IdxArgs a, uint8_t* __restrict__ act) {
  const long long total = (long long)a.n_groups * a.n_tiles_k;
  for (long long x = blockIdx.x * (long long)blockDim.x + threadIdx.x; x < total;
       x += (long long)gridDim.x * blockDim.x) {
    const int g = (int)(x / a.n_tiles_k), kt = (int)(x - (long long)g * a.n_tiles_k);
    act[x] = tile_active<kTok>(a, kt, g) ? 1 : 0;
  }
}

// Keys into the layout the key tiles stream, for any N: codes [KB][Np][64 B]
// (Np = N rounded up to 128; padding rows zero) and UE8M0 chunks
// [KB][Np/128][512 B] (byte (r%32)*16 + (r/32)*4 + j of a chunk = row r,
// K-block j of the 128-element slice; padding rows zero).  One thread per
// (K-block, row).
__global__ void kv_prep_kernel(const uint8_t* __restrict__ kv, const uint8_t* __restrict__ kv_sf,
                               int N, int Np, int D, uint8_t* __restrict__ codes,
                               uint8_t* __restrict__ chunks) {
  const int KB = D / 128;
  const long long total = (long long)KB * Np;
  for (long long x = blockIdx.x * (long long)blockDim.x + threadIdx.x; x < total;
       x += (long long)gridDim.x * blockDim.x) {
    const int n = (int)(x % Np), kb = (int)(x / Np);
    uint4* d4 = reinterpret_cast<uint4*>(codes + ((size_t)kb * Np + n) * 64);
    uint32_t sfw = 0;
    if (n < N) {
      const uint4* s4 = reinterpret_cast<const uint4*>(kv + (size_t)n * (D / 2) + (size_t)kb * 64);
#pragma unroll
      for (int c = 0; c < 4; ++c) d4[c] = s4[c];
      sfw = *reinterpret_cast<const uint32_t*>(kv_sf + (size_t)n * (D / 32) + (size_t)kb * 4);
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) d4[c] = make_uint4(0, 0, 0, 0);
    }
    const size_t chunk = (size_t)kb * (Np / 128) + (n >> 7);
    *reinterpret_cast<uint32_t*>(chunks + chunk * kSfChunk + (n & 31) * 16 + ((n >> 5) & 3) * 4) = sfw;
  }
}

// Query scales into per-group chunk pairs [group][KB][2][512 B]: query row r
// (token * Hh + head) belongs to group r / kN, row rr = r % kN of it; chunk
// rr / 128 of the pair, byte (rr%32)*16 + ((rr%128)/32)*4 + j.  Rows of the
// pair past kN (or past the last token) stay whatever they were: their MMA
// columns are never read.  One thread per (row, K-block).
__global__ void q_sf_prep_kernel(const int32_t* __restrict__ q_sf, long long rows, int KB, int kN,
                                 uint8_t* __restrict__ out) {
  const long long total = rows * KB;
  for (long long x = blockIdx.x * (long long)blockDim.x + threadIdx.x; x < total;
       x += (long long)gridDim.x * blockDim.x) {
    const long long r = x / KB;
    const int kb = (int)(x - r * KB);
    const long long g = r / kN;
    const int rr = (int)(r - g * kN);
    uint8_t* dst = out + ((size_t)g * KB + kb) * kIdxSmemSFB + (rr >> 7) * kSfChunk;
    const int r7 = rr & 127;
    *reinterpret_cast<int32_t*>(dst + (r7 & 31) * 16 + (r7 >> 5) * 4) = q_sf[x];
  }
}

}  // namespace

int mqa_tokens_per_tile(int Hh) { return idx_tokens(Hh); }
size_t mqa_qsf_bytes_per_group(int D) { return (size_t)(D / 128) * kIdxSmemSFB; }

cudaError_t launch_kv_prep(const uint8_t* kv, const uint8_t* kv_sf, int N, int Np, int D,
                           uint8_t* codes, uint8_t* chunks, cudaStream_t stream) {
  const long long total = (long long)(D / 128) * Np;
  if (total == 0) return cudaSuccess;
  long long grid = (total + 255) / 256;
  if (grid > 148LL * 32) grid = 148LL * 32;
  kv_prep_kernel<<<(unsigned)grid, 256, 0, stream>>>(kv, kv_sf, N, Np, D, codes, chunks);
  return cudaGetLastError();
}

cudaError_t launch_q_sf_prep(const int32_t* q_sf, long long rows, int D, int Hh, uint8_t* out,
                             cudaStream_t stream) {
  const int KB = D / 128;
  const long long total = rows * KB;
  if (total == 0) return cudaSuccess;
  long long grid = (total + 255) / 256;
  if (grid > 148LL * 16) grid = 148LL * 16;
  q_sf_prep_kernel<<<(unsigned)grid, 256, 0, stream>>>(q_sf, rows, KB,
                                                       idx_tokens(Hh) * Hh, out);
  return cudaGetLastError();
}

cudaError_t launch_mqa_logits(const CUtensorMap& tmK, const CUtensorMap& tmQ, const uint8_t* sfa,
                              const uint8_t* sfb, const float* w, const int* ks, const int* ke,
                              float* out, int* hdr, uint8_t* act, int S, int Hh, int N, int KB,
                              int clean, int grid, bool pdl, cudaStream_t stream) {
  typedef void (*Fn)(CUtensorMap, CUtensorMap, IdxArgs);
  typedef void (*ActFn)(IdxArgs, uint8_t*);
  Fn fn;
  ActFn afn;
  int slot;
  switch (Hh) {
    case 16: fn = mqa_logits_kernel<16>; afn = tile_activity_kernel<idx_tokens(16)>; slot = 0; break;
    case 32: fn = mqa_logits_kernel<32>; afn = tile_activity_kernel<idx_tokens(32)>; slot = 1; break;
    case 64: fn = mqa_logits_kernel<64>; afn = tile_activity_kernel<idx_tokens(64)>; slot = 2; break;
    case 128: fn = mqa_logits_kernel<128>; afn = tile_activity_kernel<idx_tokens(128)>; slot = 3; break;
    default: return cudaErrorInvalidValue;
  }
  static bool attr_set[4] = {};
  if (!attr_set[slot]) {
    cudaError_t err = cudaFuncSetAttribute((const void*)fn,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)kIdxSmemBytes);
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
  {
    const long long tiles = (long long)a.n_tiles_k * a.n_groups;
    long long agrid = (tiles + 255) / 256;
    if (agrid > 148LL * 8) agrid = 148LL * 8;
    if (agrid < 1) agrid = 1;
    afn<<<(unsigned)agrid, 256, 0, stream>>>(a, act);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kIdxThreads);
  cfg.dynamicSmemBytes = kIdxSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, fn, tmK, tmQ, a);
}

}  // namespace moe
