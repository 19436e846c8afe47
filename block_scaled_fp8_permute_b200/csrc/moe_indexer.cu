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
// Tiling.  The keys sit on the MMA's M side (128 keys per tile) and the
// queries' (token, head) rows on its N side (256 rows = 256/Hh tokens), so
// every epilogue thread owns one key and holds all heads of its tokens in
// its accumulator columns: the head-weighted ReLU sum is a per-thread loop,
// no cross-lane reduction.  One CTA per SM, persistent, 320 threads:
//   warp 0     TMA producer: key tile 128 x 128 (E2M1, unpacked by the TMA),
//              query tile 256 x 128 (E4M3), their scale chunks; 4-stage ring
//   warp 1     TMEM allocator and MMA issuer (tcgen05.mma kind::mxf8f6f4,
//              A = keys E2M1, B = queries E4M3, M=128, N=256, K=32)
//   warps 2-9  epilogue: two warps per 32-lane TMEM subpartition, one column
//              half (128 columns = 128/Hh tokens) each
// Tiles whose keys lie outside every token's [ks, ke) skip the loads and the
// MMAs; the epilogue only writes their -inf entries.
#include "moe_device.cuh"
#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int kIdxStages = 4;
constexpr int kIdxSmemA = 128 * 128;                 // keys, one byte per E2M1 element
constexpr int kIdxSmemB = 256 * 128;                 // queries, E4M3
constexpr int kIdxTxA = 128 * 128 / 2;               // bytes the TMA moves for the packed keys
constexpr int kIdxEpiWarps = 8;
constexpr int kIdxThreads = 64 + 32 * kIdxEpiWarps;
constexpr uint32_t kIdxTmemCols = 512;
constexpr uint32_t kIdxSfCol = 256;
constexpr size_t kIdxSmemBytes =
    (size_t)kIdxStages * (kIdxSmemA + kIdxSmemB + kSfChunk + 2 * kSfChunk) + 256;
static_assert(kIdxSmemBytes <= 232448, "shared memory per CTA");

struct IdxArgs {
  const uint8_t* sfa;    // key scale chunks [KB][ceil(N/128)][512]
  const uint8_t* sfb;    // query scale chunks [ceil(S*Hh/128)][KB][512]
  const float* w;        // [S, Hh]
  const int* ks;         // [S]
  const int* ke;         // [S]
  float* out;            // [S, N]
  int* hdr;              // status header
  int S, Hh, N, KB, clean;
  int n_tiles_k;         // ceil(N / 128)
  int n_groups;          // ceil(S / (256 / Hh))
};

// Does any token of query group g see a key of key tile kt?  (Decided the
// same way by every role of the CTA.)
__device__ __forceinline__ bool tile_active(const IdxArgs& a, int kt, int g) {
  const int tpg = 256 / a.Hh;
  const int j0 = kt * 128, j1 = min(j0 + 128, a.N);
  for (int t = 0; t < tpg; ++t) {
    const int i = g * tpg + t;
    if (i >= a.S) break;
    const int lo = max(a.ks[i], 0), hi = min(a.ke[i], a.N);
    if (lo < j1 && hi > j0 && lo < hi) return true;
  }
  return false;
}

template <int kHh>  // heads per query token (divides 128)
__global__ void __launch_bounds__(kIdxThreads, 1)
    mqa_logits_kernel(const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmQ, const IdxArgs args) {
  using namespace ptx;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {  // the swizzled layout needs it; no work done yet
    if (threadIdx.x == 0) set_status(args.hdr, MOE_ERR_CUDA);
    return;
  }
  uint8_t* sA = smem_raw;
  uint8_t* sB = sA + kIdxStages * kIdxSmemA;
  uint8_t* sSFA = sB + kIdxStages * kIdxSmemB;
  uint8_t* sSFB = sSFA + kIdxStages * kSfChunk;
  uint64_t* full = reinterpret_cast<uint64_t*>(sSFB + kIdxStages * 2 * kSfChunk);
  uint64_t* empty = full + kIdxStages;
  uint64_t* acc_full = empty + kIdxStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kIdxStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kIdxEpiWarps);
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int g = tile / args.n_tiles_k, kt = tile - g * args.n_tiles_k;
        if (!tile_active(args, kt, g)) continue;
        const uint32_t tx = kIdxTxA + kIdxSmemB + 3 * kSfChunk;
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
          tma_load_2d(sB + s * kIdxSmemB, &tmQ, &full[s], kb * 128, g * 256);
          bulk_load(sSFA + s * kSfChunk,
                    args.sfa + ((size_t)kb * args.n_tiles_k + kt) * kSfChunk, kSfChunk, &full[s]);
          // the group's 256 query rows are two 128-row chunks: [chunk][KB][512]
          bulk_load(sSFB + s * 2 * kSfChunk,
                    args.sfb + ((size_t)(2 * g) * KB + kb) * kSfChunk, kSfChunk, &full[s]);
          bulk_load(sSFB + s * 2 * kSfChunk + kSfChunk,
                    args.sfb + ((size_t)(2 * g + 1) * KB + kb) * kSfChunk, kSfChunk, &full[s]);
          issued_mask |= 1u << s;
          last_phase = (last_phase & ~(1u << s)) | (ph << s);
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      uint32_t it = 0;
      int ta = 0;  // active tiles so far
      bool issued_any = false, ok = true;
      const uint32_t idesc0 = idesc_mxf8f6f4(/*A E2M1*/ 5, /*B E4M3*/ 0, 128, 256);
      const uint64_t a_desc0 = sdesc_sw128(smem_u32(sA)), b_desc0 = sdesc_sw128(smem_u32(sB));
      const uint64_t sfa_desc0 = sdesc_sf(smem_u32(sSFA)), sfb_desc0 = sdesc_sf(smem_u32(sSFB));
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int g = tile / args.n_tiles_k, kt = tile - g * args.n_tiles_k;
        if (!tile_active(args, kt, g)) continue;
        if (!mbar_wait_or_abort(acc_empty, (ta & 1) ^ 1, 2 * kWaitLimitNs, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
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
          tc_cp_32x128b_warpx4(sfb_t, sfb_desc0 + (uint64_t)((s * 2 * kSfChunk) >> 4));
          tc_cp_32x128b_warpx4(sfb_t + 4u, sfb_desc0 + (uint64_t)((s * 2 * kSfChunk + kSfChunk) >> 4));
          const uint64_t adesc = a_desc0 + (uint64_t)((s * kIdxSmemA) >> 4);
          const uint64_t bdesc = b_desc0 + (uint64_t)((s * kIdxSmemB) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t id = idesc_with_sf_id(idesc0, kk, kk);
            mma_mxf8f6f4(tmem, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), id,
                         (kb | kk) != 0 ? 1u : 0u, sfa_t | ((uint32_t)kk << 30),
                         sfb_t | ((uint32_t)kk << 30));
          }
          issued_any = true;
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(acc_full);
        ++ta;
      }
      if (!ok) {
        if (!*abort_flag) record_timeout(args.hdr, 120);
        *abort_flag = 1;
        if (issued_any) {  // wait for the MMAs in flight before TMEM is released
          tc_commit(drain);
          (void)mbar_wait(drain, 0);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;        // 0..7
    const int q = warp & 3;         // TMEM lane subpartition this warp can read
    const int h = ew >> 2;          // column half: columns [128h, 128h + 128)
    const int r = q * 32 + lane;    // key within the tile
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    constexpr int tpg = 256 / kHh, tph = 128 / kHh;  // tokens per group / per column half
    int ta = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int g = tile / args.n_tiles_k, kt = tile - g * args.n_tiles_k;
      const int j = kt * 128 + r;
      const bool active = tile_active(args, kt, g);
      uint32_t v[4][32];
      if (active) {
        const bool ready =
            __all_sync(0xffffffffu, mbar_wait_or_abort(acc_full, ta & 1, 2 * kWaitLimitNs, abort_flag));
        if (!ready) {
          if (lane == 0) {
            if (!*abort_flag) record_timeout(args.hdr, 130);
            *abort_flag = 1;
          }
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(trow + 128 * h + 32 * c, v[c]);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
        ++ta;
      }
      // this thread's tokens: tph of them, kHh accumulator columns each
#pragma unroll
      for (int t = 0; t < tph; ++t) {
        const int i = g * tpg + h * tph + t;
        if (i < args.S && j < args.N) {
          const int lo = max(args.ks[i], 0), hi = min(args.ke[i], args.N);
          float* dst = args.out + (size_t)i * args.N + j;
          if (!active || j < lo || j >= hi) {
            if (args.clean) *dst = -INFINITY;
          } else {
            const float4* wi = reinterpret_cast<const float4*>(args.w + (size_t)i * kHh);
            float acc = 0.0f;
#pragma unroll
            for (int h4 = 0; h4 < kHh / 4; ++h4) {
              const float4 w4 = __ldg(wi + h4);
              const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int col = t * kHh + 4 * h4 + u;  // 0..127 inside the half
                acc = fmaf(wv[u], fmaxf(__uint_as_float(v[col >> 5][col & 31]), 0.0f), acc);
              }
            }
            *dst = acc;
          }
        }
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

}  // namespace

cudaError_t launch_kv_prep(const uint8_t* kv, const uint8_t* kv_sf, int N, int Np, int D,
                           uint8_t* codes, uint8_t* chunks, cudaStream_t stream) {
  const long long total = (long long)(D / 128) * Np;
  if (total == 0) return cudaSuccess;
  long long grid = (total + 255) / 256;
  if (grid > 148LL * 32) grid = 148LL * 32;
  kv_prep_kernel<<<(unsigned)grid, 256, 0, stream>>>(kv, kv_sf, N, Np, D, codes, chunks);
  return cudaGetLastError();
}

cudaError_t launch_mqa_logits(const CUtensorMap& tmK, const CUtensorMap& tmQ, const uint8_t* sfa,
                              const uint8_t* sfb, const float* w, const int* ks, const int* ke,
                              float* out, int* hdr, int S, int Hh, int N, int KB, int clean,
                              int grid, bool pdl, cudaStream_t stream) {
  typedef void (*Fn)(CUtensorMap, CUtensorMap, IdxArgs);
  Fn fn;
  int slot;
  switch (Hh) {
    case 16: fn = mqa_logits_kernel<16>; slot = 0; break;
    case 32: fn = mqa_logits_kernel<32>; slot = 1; break;
    case 64: fn = mqa_logits_kernel<64>; slot = 2; break;
    case 128: fn = mqa_logits_kernel<128>; slot = 3; break;
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
  a.n_groups = (S * Hh + 255) / 256;
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
