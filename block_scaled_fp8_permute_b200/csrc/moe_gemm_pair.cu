// moe_gemm_pair.cu -- the grouped block-scaled GEMM of both linears on SM
// pairs (thread-block clusters of 2, tcgen05 cta_group::2).
//
// One work item is a 256 x 256 output tile: two 128-row m-tiles of one
// expert (CTA r of the pair owns m-tile mt0 + r) times 256 weight rows.  The
// even CTA issues tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 32,
// kind::mxf8f6f4 with UE8M0 block scales); each CTA keeps its own 128 A rows
// and its own 128 of the 256 B rows in shared memory, so per SM the
// shared-memory traffic of a K step is A 4 KB + B 4 KB written by the TMA
// and read by the tensor core, instead of 4 KB + 8 KB for a one-SM
// 128 x 256 tile (the FP4 weights occupy one byte per element in shared
// memory for this MMA kind).  That halves the shared-memory bandwidth per
// MMA and leaves room for a 6-stage pipeline.
// ("DeepSeek DeepGEMM 2026年4月重磅更新：Mega MoE融合算子、FP4精度与极致性能优化",
//  section 3.2: fused linear1 / SwiGLU / linear2; section 11.3: multi-stage
//  TMA pipelines.)
//
// Roles per CTA (320 threads):
//   warp 0     TMA producer (both CTAs): its A rows, its half of B, its A
//              scale chunk and all 256 rows of B scales, signalling the even
//              CTA's full barrier (cp.async.bulk.tensor .cta_group::2).
//   warp 1     TMEM allocation (both CTAs, cta_group::2); in the even CTA it
//              also copies the stage's scales to TMEM in both CTAs and issues
//              the MMAs; completions are committed to the barriers of both
//              CTAs at once.
//   warps 2-9  epilogue (both CTAs): drain the CTA's own 128 accumulator rows,
//              release them to the even CTA, compute and store.
// A pair whose expert has an odd number of m-tiles ends with a one-m-tile
// item: the odd CTA then mirrors the even CTA's rows and stores nothing.
#include "moe_epilogue.cuh"

namespace moe {
namespace pairk {

constexpr int kStages = 6;
constexpr int kSmemA = kBlockM * kBlockK;        // 16384: this CTA's 128 rows
constexpr int kSmemB = 128 * kBlockK;            // 16384: this CTA's 128 weight rows, unpacked
constexpr int kSmemSFA = kSfChunk;               // 512
constexpr int kSmemSFB = 2 * kSfChunk;           // 1024: all 256 weight rows
constexpr uint32_t kTxPair = 2u * (kSmemA + kSmemB / 2 + kSmemSFA + kSmemSFB);
constexpr int kNumEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kNumEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;
constexpr uint32_t kSfCol = 256;
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * (kSmemA + kSmemB + kSmemSFA + kSmemSFB) +
                              (size_t)kNumEpiWarps * kEpiOutStage + 256;

}  // namespace pairk

template <int kEpi>
__global__ void __launch_bounds__(pairk::kThreads, 1)
    moe_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmSFA,
                         const __grid_constant__ CUtensorMap tmSFB,
                         const __grid_constant__ CUtensorMap tmOut, const GemmArgs args) {
  using namespace ptx;
  using namespace pairk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<size_t>(smem_raw), 1024));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kStages * kSmemA;
  uint8_t* sSFA = sB + kStages * kSmemB;
  uint8_t* sSFB = sSFA + kStages * kSmemSFA;
  uint8_t* sOut = sSFB + kStages * kSmemSFB;
  uint64_t* full = reinterpret_cast<uint64_t*>(sOut + kNumEpiWarps * kEpiOutStage);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the CTA that issues the MMAs
  const int cid = (int)cluster_id_x(), ncl = (int)num_clusters_x();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kNumEpiWarps);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmSFA);
    prefetch_tmap(&tmSFB);
    if (kEpi == 2) prefetch_tmap(&tmOut);
  }
  cluster_sync();  // both CTAs' barriers exist before either CTA signals the other
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  pdl_wait();  // inputs come from the previous kernel of the forward
  const int NT = args.NT, KB = args.KB, n_rows = args.n_rows;
  const int num_work = args.hdr[kHdrMPairs] * NT;
  const uint32_t full0_leader = mapa_shared(smem_u32(&full[0]), 0);
  const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true, issued = false;
      for (int w = cid; w < num_work && ok; w += ncl) {
        const int p = w / NT, nt = w - (w / NT) * NT;
        const int ent = args.mpair[p];
        const int mt0 = ent & 0x7FFFFFFF;
        const bool single = ent < 0;
        const int my_mt = (single && rank == 1) ? mt0 : mt0 + (int)rank;
        const int e = args.tile_expert[mt0];
        const int n0 = nt * kBlockN;
        const int sfb_chunk0 = e * KB * (n_rows / 128) + n0 / 128;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!mbar_wait_cluster(&empty[s], ph ^ 1) || *abort_flag) {
            record_timeout(args.hdr, 40 + kEpi);
            *abort_flag = 1;
            ok = false;
            break;
          }
          const uint32_t bar = full0_leader + 8u * (uint32_t)s;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], kTxPair);
          tma_load_2d_pair(sA + s * kSmemA, &tmA, bar, kb * kBlockK, my_mt * kBlockM);
          tma_load_3d_pair(sB + s * kSmemB, &tmB, bar, 0, n0 + 128 * (int)rank, e * KB + kb);
          tma_load_2d_pair(sSFA + s * kSmemSFA, &tmSFA, bar, 0, my_mt * KB + kb);
          tma_load_2d_pair(sSFB + s * kSmemSFB, &tmSFB, bar, 0,
                           sfb_chunk0 + kb * (n_rows / 128));
          issued = true;
        }
      }
      if (!ok && issued) {  // let copies in flight land before the CTA's memory goes away
        const unsigned long long t0 = globaltimer();
        while (globaltimer() - t0 < 100000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA (even CTA)
    if (rank == 0 && lane == 0) {
      const uint32_t idesc0 = idesc_mxf8f6f4(/*A E4M3*/ 0, /*B E2M1*/ 5, 2 * kBlockM, kBlockN);
      uint32_t it = 0;
      int ti = 0;
      bool ok = true, issued_any = false;
      for (int w = cid; w < num_work && ok; w += ncl, ++ti) {
        if (!mbar_wait_cluster(acc_empty, (ti & 1) ^ 1) || *abort_flag) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!mbar_wait(&full[s], ph) || *abort_flag) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_t = tmem + kSfCol + 16u * (it & 1u);
          const uint32_t sfb_t = sfa_t + 4u;
          tc_cp_pair_32x128b_warpx4(sfa_t, sdesc_sf(smem_u32(sSFA + s * kSmemSFA)));
          tc_cp_pair_32x128b_warpx4(sfb_t, sdesc_sf(smem_u32(sSFB + s * kSmemSFB)));
          tc_cp_pair_32x128b_warpx4(sfb_t + 4u,
                                    sdesc_sf(smem_u32(sSFB + s * kSmemSFB + kSfChunk)));
          const uint64_t adesc = sdesc_sw128(smem_u32(sA + s * kSmemA));
          const uint64_t bdesc = sdesc_sw128(smem_u32(sB + s * kSmemB));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            mma_mxf8f6f4_pair(tmem + kAccCol, adesc + (uint64_t)(kk * 2),
                              bdesc + (uint64_t)(kk * 2), idesc_with_sf_id(idesc0, kk, kk),
                              (kb | kk) != 0 ? 1u : 0u, sfa_t | ((uint32_t)kk << 30),
                              sfb_t | ((uint32_t)kk << 30));
          }
          issued_any = true;
          tc_commit_pair(&empty[s], 0x3);
        }
        if (!ok) break;
        tc_commit_pair(acc_full, 0x3);
      }
      if (!ok) {
        record_timeout(args.hdr, 50 + kEpi);
        *abort_flag = 1;
        if (issued_any) {  // wait for the MMAs in flight before TMEM is released
          tc_commit_pair(drain, 0x1);
          (void)mbar_wait(drain, 0);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;      // 0..7
    const int q = warp & 3;       // TMEM lane subpartition this warp can read
    const int h = ew >> 2;        // column half
    const int r = q * 32 + lane;  // row within the CTA's m-tile
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16) + kAccCol;
    int ti = 0;
    for (int w = cid; w < num_work; w += ncl, ++ti) {
      const int p = w / NT, nt = w - (w / NT) * NT;
      const int ent = args.mpair[p];
      const int mt0 = ent & 0x7FFFFFFF;
      const bool mirror = ent < 0 && rank == 1;  // one-m-tile item: nothing to store here
      const bool ready = __all_sync(0xffffffffu, mbar_wait(acc_full, ti & 1) && !*abort_flag);
      if (!ready) {
        if (lane == 0) {
          record_timeout(args.hdr, 60 + kEpi);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      uint32_t v[4][32];
      if (!mirror) {
        epilogue_load<kEpi>(v, trow, h);
        tc_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader);
      if (!mirror)
        epilogue_store<kEpi>(v, args, &tmOut, sOut + ew * kEpiOutStage, mt0 + (int)rank, nt, r,
                             h, q, lane);
    }
    if (kEpi == 2 && lane == 0) bulk_wait_group0();  // stores complete before the CTA exits
  }

  pdl_launch();
  tc_fence_before();
  __syncwarp();
  __syncthreads();
  cluster_sync();  // the pair is done with each other's barriers, shared memory and TMEM
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------ host launcher
cudaError_t launch_gemm_pair(int epi, const CUtensorMap& tmA, const CUtensorMap& tmB,
                             const CUtensorMap& tmSFA, const CUtensorMap& tmSFB,
                             const CUtensorMap& tmOut, const GemmArgs& args, int num_pairs_grid,
                             bool pdl, cudaStream_t stream) {
  static bool attr_set[3] = {false, false, false};
  void (*fn)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, GemmArgs) =
      (epi == 1) ? moe_gemm_pair_kernel<1> : moe_gemm_pair_kernel<2>;
  if (!attr_set[epi]) {
    cudaError_t err = cudaFuncSetAttribute((const void*)fn,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)pairk::kSmemBytes);
    if (err != cudaSuccess) return err;
    attr_set[epi] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * num_pairs_grid);
  cfg.blockDim = dim3(pairk::kThreads);
  cfg.dynamicSmemBytes = pairk::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, fn, tmA, tmB, tmSFA, tmSFB, tmOut, args);
}

}  // namespace moe
