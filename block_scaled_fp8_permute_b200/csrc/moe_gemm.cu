// moe_gemm.cu -- persistent grouped GEMM on 5th-generation tensor cores for
// the two linear layers of the MoE layer.
//
//   linear1: G = Xp_e . W1_e^T  (FP8 E4M3 activations x FP4 E2M1 weights,
//            UE8M0 scale per 1x32 block on both sides, FP32 accumulation) with
//            the SwiGLU + E4M3 requantisation epilogue fused in;
//   linear2: O = A2_e . W2_e^T with the top-k weight applied in the epilogue,
//            BF16 partial rows written in expert-contiguous row order;
//   the standalone FP8 x FP4 GEMM (dense or masked grouped): D = A_g . B_g^T,
//            BF16 rows.
// ("DeepSeek DeepGEMM 2026年4月重磅更新：Mega MoE融合算子、FP4精度与极致性能优化",
//  section 3.2 (fusing linear1 / SwiGLU / linear2), section 4.2 (UE8M0 scale
//  factors, FP32 accumulation), section 11.3 (TMA multi-stage loads).)
//
// One CTA per SM, 320 threads:
//   warp 0     TMA producer: A tile 128x128 (E4M3), B tile 256x128 (E2M1,
//              unpacked by the TMA to one byte per element as the block-scaled
//              MMA requires), and the two 512/1024-byte scale chunks, into a
//              shared-memory ring (4 stages; 5 for narrow tiles, TileCfg).
//   warp 1     TMEM allocator and MMA issuer: copies the stage's scales into
//              TMEM (tcgen05.cp) and issues 4 x tcgen05.mma kind::mxf8f6f4
//              (M=128, N=256, K=32) per stage into one FP32 TMEM accumulator.
//   warps 2-9  epilogue: drain the accumulator from TMEM (two warps per
//              32-lane subpartition, one column half each), release it to
//              the MMA warp, then compute and store.
// Tiles: (m-tile of 128 padded rows, n-tile of 256 weight rows); each m-tile
// belongs to one expert (rows are padded per expert to 128).
#include <cuda_fp8.h>

#include "moe_epilogue.cuh"

namespace moe {

constexpr int kSmemB = kBlockN * kBlockK;  // 32768 bytes (one byte per E2M1 element in smem)
constexpr int kTxB = kBlockN * kBlockK / 2;  // bytes the TMA moves for B (packed)
// Scale factors of one stage: the 512-byte chunk of A's 128 rows and the two
// chunks of B's 256 rows, copied into TMEM by tcgen05.cp .32x128b.warpx4
// (the layout the block-scaled MMA reads: every 32-lane subpartition holds
// all rows).  (Copies without replication from four replicas per chunk are
// cheaper in the tensor pipe, but the extra loads per stage cost more.)
constexpr int kSmemSFA = kSfChunk;
constexpr int kSmemSFB = 2 * kSfChunk;
constexpr int kNumEpiWarps = 8;
constexpr int kGemmThreads = 64 + 32 * kNumEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;    // FP32 accumulator, 256 columns
constexpr uint32_t kSfCol = 256;   // scale buffers: buf b -> SFA at +16b (4 cols), SFB at +16b+4 (8)

constexpr int kOutStage = kEpiOutStage;

// Stage geometry.  Normal tiles stage 128 A rows (16 KB) per 128-K step in a
// 4-deep ring.  Narrow tiles (experts with at most kNarrowRows rows: decode-
// sized batches) stage only kNarrowRows A rows, and the 12 KB saved per stage
// buy a fifth stage, i.e. 25 % more weight bytes in flight per SM.  The MMA
// still spans 128 rows: rows past kNarrowRows read whatever the shared memory
// after the stage's A rows holds, and those accumulator rows (padding) are
// never stored.
template <int kEpi, bool kNarrow>
struct TileCfg {
  static constexpr int kARows = kNarrow ? kNarrowRows : kBlockM;
  static constexpr int kStages = kNarrow ? 5 : 4;
  static constexpr int kSmemA = kARows * kBlockK;
  static constexpr int kStageBytes = kSmemA + kSmemB + kSmemSFA + kSmemSFB;
  static constexpr int kOutBytes = kEpi == 1 ? 0 : kNumEpiWarps * kOutStage;
  // the dynamic shared memory base is 1024-byte aligned (checked at kernel start)
  static constexpr size_t kSmemBytes = (size_t)kStages * kStageBytes + kOutBytes + 256;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  // A and B stage buffers keep the 1024-byte alignment of the 128-byte
  // swizzle; the epilogue staging after all stage arrays the 512 bytes of the
  // 64-byte swizzle
  static_assert(kSmemA % 1024 == 0 && kSmemB % 1024 == 0, "swizzled stage alignment");
  static_assert(((size_t)kStages * kStageBytes) % 512 == 0, "staging alignment");
};

__global__ void requant_debug_kernel(const float* __restrict__ a, int rows, int cols,
                                     uint8_t* __restrict__ codes, uint8_t* __restrict__ sbytes) {
  const int nblk = cols / 32;
  for (long long b = blockIdx.x * (long long)blockDim.x + threadIdx.x; b < (long long)rows * nblk;
       b += (long long)gridDim.x * blockDim.x) {
    float v[32];
    const float* src = a + b * 32;
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = src[i];
    uint32_t packed[8], sb;
    requant32(v, packed, sb);
    uint4* dst = reinterpret_cast<uint4*>(codes + b * 32);
    dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    sbytes[b] = (uint8_t)sb;
  }
}

// Order of the tiles of one list (n_mt m-tiles x NT n-tiles): the m-tiles
// go in chunks of kMChunk, and within a chunk the m-tile index runs fastest.
// The CTAs working at one time then cover a few n-tiles of many m-tiles of
// the same expert: each weight slice is read from DRAM about once per chunk
// and reused from L2 by the chunk's m-tiles, while the chunk's activation rows
// (kMChunk x 128 rows) stay in L2 across its n-tiles.  idx -> (m-tile list
// position, n-tile).
constexpr int kMChunk = 16;
__device__ __forceinline__ void chunked_tile(int idx, int n_mt, int NT, int& mpos, int& nt) {
  const int per_chunk = kMChunk * NT;
  const int c = idx / per_chunk, rem = idx - c * per_chunk;
  const int in_chunk = min(kMChunk, n_mt - c * kMChunk);  // the last chunk may be short
  nt = rem / in_chunk;
  mpos = c * kMChunk + (rem - nt * in_chunk);
}

// Tile v of a launch with `total` tiles of which `n_mix` are mixed-in narrow
// tiles: narrow tiles sit at the positions where floor(v * n_mix / total)
// steps up, so they are spread evenly over the launch and every CTA (which
// takes every gridDim-th tile) gets its share.  Returns true for a narrow
// tile; mt / nt: its m-tile and n-tile.
// The narrow-tile kernel (kChunked false) keeps the plain order: its m-tiles
// are single small experts that share no weights, and walking one expert's
// n-tiles on neighbouring CTAs streams its weights in address order.
template <bool kChunked>
__device__ __forceinline__ bool decode_tile(int v, int total, int n_mix, int NT,
                                            const GemmArgs& args, int& mt, int& nt) {
  int mpos;
  if (n_mix == 0) {
    if (kChunked) {
      chunked_tile(v, total / NT, NT, mpos, nt);
    } else {
      mpos = v / NT;
      nt = v - mpos * NT;
    }
    mt = args.norm_mtiles[mpos];
    return false;
  }
  const long long before = (long long)v * n_mix / total;          // narrow tiles before v
  const long long upto = ((long long)v + 1) * n_mix / total;      // ... up to and with v
  const bool nar = upto > before;
  const int idx = nar ? (int)before : v - (int)before;
  if (nar) {
    mt = args.narrow_mtiles[idx / NT];
    nt = idx - (idx / NT) * NT;
  } else {
    chunked_tile(idx, (total - n_mix) / NT, NT, mpos, nt);
    mt = args.norm_mtiles[mpos];
  }
  return nar;
}

// -------------------------------------------------------------------- kernel
template <int kEpi,    // 1: SwiGLU + requant (linear1), 2: x topk_w, BF16 rows (linear2),
                       // 3: BF16 rows of the standalone GEMM
          bool kNarrow>  // stage only kNarrowRows A rows (TileCfg)
__global__ void __launch_bounds__(kGemmThreads, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmAn,  // kNarrowRows-row A boxes
                    const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmOut, const GemmArgs args) {
  using namespace ptx;
  using Cfg = TileCfg<kEpi, kNarrow>;
  constexpr int kStages = Cfg::kStages;
  constexpr int kSmemA = Cfg::kSmemA;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {  // the layout below needs it; no work done yet
    if (threadIdx.x == 0) set_status(args.hdr, MOE_ERR_CUDA);
    return;
  }
  uint8_t* smem = smem_raw;
  uint8_t* sA = smem;
  uint8_t* sB = sA + kStages * kSmemA;
  uint8_t* sSFA = sB + kStages * kSmemB;
  uint8_t* sSFB = sSFA + kStages * kSmemSFA;
  uint8_t* sOut = sSFB + kStages * kSmemSFB;  // epilogue staging, 1024-aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(sOut + Cfg::kOutBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kNumEpiWarps);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if (kEpi != 1) prefetch_tmap(&tmOut);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  pdl_wait();  // inputs come from the previous kernel of the forward
  const int NT = args.NT, KB = args.KB, n_rows = args.n_rows;
  // wait limits: a stage's data (MMA issuer) gets L, the waits that can only
  // end after such a stage (free slots, the accumulator) get 2L, so that the
  // wait nearest the cause expires first
  const unsigned long long lim = args.wait_limit_ns ? args.wait_limit_ns : kWaitLimitNs;
  // tiles of this launch: its own list, plus (mixed normal-tile launch) the
  // narrow m-tiles spread evenly among them; a mixed narrow-tile launch has
  // nothing to do when the normal-tile launch took its tiles
  const int n_norm_mt = args.hdr[kHdrNormMTiles];
  int n_own = args.hdr[args.tiles_word] * NT, n_mix = 0;
  if (args.mixed) {
    if (kNarrow && n_norm_mt > 0) n_own = 0;
    if (!kNarrow && n_norm_mt > 0) n_mix = args.hdr[kHdrNarrowMTiles] * NT;
  }
  const int num_tiles = n_own + n_mix;

  // stages the producer has issued loads into, and the phase of the last one
  // (producer lane only): after a failure they are waited for before exit
  uint32_t issued_mask = 0, last_phase = 0;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int mt, nt;
        const bool nar = decode_tile<!kNarrow>(tile, num_tiles, n_mix, NT, args, mt, nt);
        const int e = args.tile_expert[mt];
        const int n0 = nt * kBlockN;
        const bool two_chunks = n_rows - n0 > 128;  // 256 weight rows (else the 128-row tail)
        const uint32_t a_bytes = nar ? kNarrowRows * kBlockK : kSmemA;
        const uint32_t tx = a_bytes + kTxB + kSfChunk + (two_chunks ? 2 : 1) * kSfChunk;
        const uint8_t* sfa_src = args.sfa + (size_t)mt * KB * kSfChunk;
        const uint8_t* sfb_src = args.sfb + ((size_t)e * KB * (n_rows / 128) + n0 / 128) * kSfChunk;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!mbar_wait_or_abort(&empty[s], ph ^ 1, 2 * lim, abort_flag)) {
            if (!*abort_flag) record_timeout(args.hdr, 10 + kEpi);
            *abort_flag = 1;
            ok = false;
            break;
          }
          if ((int)it + 1 == args.fault_skip_it) continue;  // test hook: this stage never fills
          mbar_arrive_expect_tx(&full[s], tx);
          tma_load_2d(sA + s * kSmemA, nar ? &tmAn : &tmA, &full[s], kb * kBlockK, mt * kBlockM);
          tma_load_3d(sB + s * kSmemB, &tmB, &full[s], 0, n0, e * KB + kb);
          bulk_load(sSFA + s * kSmemSFA, sfa_src + (size_t)kb * kSfChunk, kSfChunk, &full[s]);
          bulk_load(sSFB + s * kSmemSFB, sfb_src + (size_t)kb * (n_rows / 128) * kSfChunk,
                    (two_chunks ? 2 : 1) * kSfChunk, &full[s]);
          issued_mask |= 1u << s;
          last_phase = (last_phase & ~(1u << s)) | (ph << s);
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      uint32_t it = 0;
      int ti = 0;
      bool issued_any = false, ok = true;
      // descriptors of stage 0; stage s adds its byte offset >> 4 to the start field
      const uint64_t a_desc0 = sdesc_sw128(smem_u32(sA)), b_desc0 = sdesc_sw128(smem_u32(sB));
      const uint64_t sfa_desc0 = sdesc_sf(smem_u32(sSFA)), sfb_desc0 = sdesc_sf(smem_u32(sSFB));
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++ti) {
        int mt, nt;
        (void)decode_tile<!kNarrow>(tile, num_tiles, n_mix, NT, args, mt, nt);
        const int n_tile = min(kBlockN, n_rows - nt * kBlockN);
        const uint32_t idesc0 = idesc_mxf8f6f4(/*A E4M3*/ 0, /*B E2M1*/ 5, kBlockM, n_tile);
        if (!mbar_wait_or_abort(acc_empty, (ti & 1) ^ 1, 2 * lim, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!mbar_wait_or_abort(&full[s], ph, lim, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_t = tmem + kSfCol + 16u * (it & 1u);
          const uint32_t sfb_t = sfa_t + 4u;
          tc_cp_32x128b_warpx4(sfa_t, sfa_desc0 + (uint64_t)((s * kSmemSFA) >> 4));
          tc_cp_32x128b_warpx4(sfb_t, sfb_desc0 + (uint64_t)((s * kSmemSFB) >> 4));
          if (n_tile > 128)
            tc_cp_32x128b_warpx4(sfb_t + 4u, sfb_desc0 + (uint64_t)((s * kSmemSFB + kSfChunk) >> 4));
          const uint64_t adesc = a_desc0 + (uint64_t)((s * kSmemA) >> 4);
          const uint64_t bdesc = b_desc0 + (uint64_t)((s * kSmemB) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t id = idesc_with_sf_id(idesc0, kk, kk);
            mma_mxf8f6f4(tmem + kAccCol, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), id,
                         (kb | kk) != 0 ? 1u : 0u, sfa_t | ((uint32_t)kk << 30),
                         sfb_t | ((uint32_t)kk << 30));
          }
          issued_any = true;
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      if (!ok) {
        if (!*abort_flag) record_timeout(args.hdr, 20 + kEpi);
        *abort_flag = 1;
        if (issued_any) {  // wait for the MMAs in flight before TMEM is released
          tc_commit(drain);
          (void)mbar_wait(drain, 0);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;      // 0..7
    const int q = warp & 3;       // TMEM lane subpartition this warp can read
    const int h = ew >> 2;        // column half
    const int r = q * 32 + lane;  // row within the tile
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16) + kAccCol;
    int ti = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++ti) {
      int mt, nt;
      (void)decode_tile<!kNarrow>(tile, num_tiles, n_mix, NT, args, mt, nt);
      // warp-uniform decision: every lane leaves or every lane continues
      const bool ready =
          __all_sync(0xffffffffu, mbar_wait_or_abort(acc_full, ti & 1, 2 * lim, abort_flag));
      if (!ready) {
        if (lane == 0) {
          if (!*abort_flag) record_timeout(args.hdr, 30 + kEpi);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      uint32_t v[4][32];
      epilogue_load<kEpi>(v, trow, h);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      epilogue_store<kEpi>(v, args, &tmOut, sOut + ew * kOutStage, mt, nt, r, h, q, lane);
    }
    if (kEpi != 1 && lane == 0) bulk_wait_group0();  // stores complete before the CTA exits
  }

  pdl_launch();
  tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0 && *abort_flag) {
    // a role failed, possibly after the producer had finished: copies it
    // issued that nobody consumed land before the CTA's memory goes away
    for (int s = 0; s < kStages; ++s)
      if (issued_mask & (1u << s)) (void)mbar_wait(&full[s], (last_phase >> s) & 1);
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------ host launchers
cudaError_t launch_gemm(int epi, bool narrow, const CUtensorMap& tmA, const CUtensorMap& tmAn,
                        const CUtensorMap& tmB, const CUtensorMap& tmOut, const GemmArgs& args,
                        int grid, bool pdl, cudaStream_t stream) {
  typedef void (*Fn)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, GemmArgs);
  static bool attr_set[2][4] = {};
  Fn fn;
  size_t smem;
  if (narrow) {
    if (epi != 1 && epi != 2) return cudaErrorInvalidValue;
    fn = epi == 1 ? moe_gemm_kernel<1, true> : moe_gemm_kernel<2, true>;
    smem = epi == 1 ? TileCfg<1, true>::kSmemBytes : TileCfg<2, true>::kSmemBytes;
  } else {
    fn = epi == 1 ? moe_gemm_kernel<1, false>
                  : (epi == 2 ? moe_gemm_kernel<2, false> : moe_gemm_kernel<3, false>);
    smem = epi == 1 ? TileCfg<1, false>::kSmemBytes
                    : (epi == 2 ? TileCfg<2, false>::kSmemBytes : TileCfg<3, false>::kSmemBytes);
  }
  if (!attr_set[narrow][epi]) {
    cudaError_t err =
        cudaFuncSetAttribute((const void*)fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    attr_set[narrow][epi] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, fn, tmA, tmAn, tmB, tmOut, args);
}

cudaError_t launch_requant_debug(const float* a, int rows, int cols, uint8_t* codes,
                                 uint8_t* sbytes, cudaStream_t stream) {
  long long nblk = (long long)rows * (cols / 32);
  int grid = (int)((nblk + 255) / 256);
  if (grid < 1) grid = 1;
  if (grid > 4096) grid = 4096;
  requant_debug_kernel<<<grid, 256, 0, stream>>>(a, rows, cols, codes, sbytes);
  return cudaGetLastError();
}

}  // namespace moe
