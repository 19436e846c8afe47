// moe_gemm_swap.cu -- grouped block-scaled GEMM with swapped operand roles
// for experts that receive few tokens ("DeepSeek DeepGEMM 2026年4月重磅更新：
// Mega MoE融合算子、FP4精度与极致性能优化" section 8.1, Dynamic Swap A/B: the
// operand roles follow the per-expert shape).
//
// An expert with n <= 64 routed rows would waste most of a 128-row MMA
// tile; here the weights take the MMA's M side (two M = 128 MMAs per K step
// over one 256-row weight group) and the expert's n rows take the N side
// (N = n rounded up to 16).  The accumulators are transposed: TMEM lane =
// weight row, column = token.
//   linear1: the group holds the gate rows (MMA 0) and the up rows (MMA 1) of
//            the same 128 SwiGLU outputs, so one thread owns gate and up of
//            one output j for every token; the 32 outputs of a requant block
//            are the 32 lanes of a warp (amax by warp reduction).
//   linear2: MMA 0 / MMA 1 cover output columns h0..h0+127 / h0+128..h0+255;
//            one warp writes 32 consecutive BF16 outputs of a token row.
// Work item = (expert, 256-row weight group); each item streams that group's
// weights once, so the kernel is bound by HBM weight traffic.
//
// One CTA per SM, 320 threads: warp 0 TMA producer, warp 1 TMEM + MMA issue,
// warps 2-9 epilogue (warp w reads TMEM lanes 32*(w%4).., column half
// (w-2)/4).  Bounded waits as in the other GEMM kernels.
#include "moe_epilogue.cuh"

namespace moe {
namespace swapk {

constexpr int kStages = 5;
constexpr int kMaxN = kMaxSwapRows;              // tokens per item (N of the MMA)
constexpr int kSmemW = kBlockN * kBlockK;        // 32768: 256 weight rows, unpacked
constexpr int kSmemX = kMaxN * kBlockK;          // 8192: up to 64 token rows
constexpr int kSmemSFW = 2 * kSfChunk;           // 1024
constexpr int kSmemSFX = kSfChunk;               // 512
constexpr int kNumEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kNumEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;     // MMA 0 accumulator at [0,128), MMA 1 at [128,256)
constexpr uint32_t kSfCol = 256;    // buf b: weight scales +16b (8 cols), token scales +16b+8 (4)
constexpr size_t kSmemBytes =
    1024 + (size_t)kStages * (kSmemW + kSmemX + kSmemSFW + kSmemSFX) + 256;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
constexpr int kMaxChunks = kMaxN / 16;

}  // namespace swapk

template <int kEpi>
__global__ void __launch_bounds__(swapk::kThreads, 1)
    moe_gemm_swap_kernel(const __grid_constant__ CUtensorMap tmW,   // weights, box 128 x 256
                         const __grid_constant__ CUtensorMap tmX,   // activations, box 128 x 16
                         const GemmArgs args) {
  using namespace ptx;
  using namespace swapk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<size_t>(smem_raw), 1024));
  uint8_t* sW = smem;
  uint8_t* sX = sW + kStages * kSmemW;
  uint8_t* sSFW = sX + kStages * kSmemX;
  uint8_t* sSFX = sSFW + kStages * kSmemSFW;
  uint64_t* full = reinterpret_cast<uint64_t*>(sSFX + kStages * kSmemSFX);
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
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  pdl_wait();
  const int KB = args.KB, n_rows = args.n_rows;
  const int NG = (n_rows + kBlockN - 1) / kBlockN;  // 256-row weight groups
  const int num_items = args.hdr[kHdrSwapExperts] * NG;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      uint32_t issued_mask = 0, last_phase = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < num_items && ok; item += gridDim.x) {
        const int e = args.swap_experts[item / NG];
        const int wg = item - (item / NG) * NG;
        const int r0 = args.poffs[e];  // 128-aligned first row of the expert
        const int n = args.counts[e];
        const int n16 = (n + 15) >> 4;
        const int w0 = wg * kBlockN;
        const uint32_t sfw_bytes = (n_rows - w0 > 128) ? 2 * kSfChunk : kSfChunk;
        const uint32_t tx = kBlockN * kBlockK / 2 + n16 * 16 * kBlockK + sfw_bytes + kSfChunk;
        const uint8_t* sfw_src = args.sfb + ((size_t)e * KB * (n_rows / 128) + w0 / 128) * kSfChunk;
        const uint8_t* sfx_src = args.sfa + (size_t)(r0 / kBlockM) * KB * kSfChunk;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1) || *abort_flag) {
            record_timeout(args.hdr, 70 + kEpi);
            *abort_flag = 1;
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], tx);
          tma_load_3d(sW + s * kSmemW, &tmW, &full[s], 0, w0, e * KB + kb);
          for (int i = 0; i < n16; ++i)
            tma_load_2d(sX + s * kSmemX + i * 16 * kBlockK, &tmX, &full[s], kb * kBlockK,
                        r0 + 16 * i);
          bulk_load(sSFW + s * kSmemSFW, sfw_src + (size_t)kb * (n_rows / 128) * kSfChunk,
                    sfw_bytes, &full[s]);
          bulk_load(sSFX + s * kSmemSFX, sfx_src + (size_t)kb * kSfChunk, kSfChunk, &full[s]);
          issued_mask |= 1u << s;
          last_phase = (last_phase & ~(1u << s)) | (ph << s);
        }
      }
      if (!ok) {
        for (int s = 0; s < kStages; ++s)
          if (issued_mask & (1u << s)) (void)mbar_wait(&full[s], (last_phase >> s) & 1);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      uint32_t it = 0;
      int ti = 0;
      bool ok = true, issued_any = false;
      for (int item = blockIdx.x; item < num_items && ok; item += gridDim.x, ++ti) {
        const int e = args.swap_experts[item / NG];
        const int wg = item - (item / NG) * NG;
        const int n16 = (args.counts[e] + 15) >> 4;
        const bool two = n_rows - wg * kBlockN > 128;  // second 128-row half present
        const uint32_t idesc0 = idesc_mxf8f6f4(/*A E2M1*/ 5, /*B E4M3*/ 0, kBlockM, 16 * n16);
        if (!mbar_wait(acc_empty, (ti & 1) ^ 1) || *abort_flag) {
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
          const uint32_t sfw_t = tmem + kSfCol + 16u * (it & 1u);
          const uint32_t sfx_t = sfw_t + 8u;
          tc_cp_32x128b_warpx4(sfw_t, sdesc_sf(smem_u32(sSFW + s * kSmemSFW)));
          if (two)
            tc_cp_32x128b_warpx4(sfw_t + 4u, sdesc_sf(smem_u32(sSFW + s * kSmemSFW + kSfChunk)));
          tc_cp_32x128b_warpx4(sfx_t, sdesc_sf(smem_u32(sSFX + s * kSmemSFX)));
          const uint64_t wdesc = sdesc_sw128(smem_u32(sW + s * kSmemW));
          const uint64_t xdesc = sdesc_sw128(smem_u32(sX + s * kSmemX));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t id = idesc_with_sf_id(idesc0, kk, kk);
            const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
            mma_mxf8f6f4(tmem + kAccCol, wdesc + (uint64_t)(kk * 2), xdesc + (uint64_t)(kk * 2),
                         id, acc, sfw_t | ((uint32_t)kk << 30), sfx_t | ((uint32_t)kk << 30));
            if (two)  // rows 128..255 of the group: 128 rows x 128 bytes further on
              mma_mxf8f6f4(tmem + kAccCol + 128u, wdesc + (uint64_t)(1024 + kk * 2),
                           xdesc + (uint64_t)(kk * 2), id, acc,
                           (sfw_t + 4u) | ((uint32_t)kk << 30), sfx_t | ((uint32_t)kk << 30));
          }
          issued_any = true;
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      if (!ok) {
        record_timeout(args.hdr, 80 + kEpi);
        *abort_flag = 1;
        if (issued_any) {
          tc_commit(drain);
          (void)mbar_wait(drain, 0);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;   // 0..7
    const int q = warp & 3;    // TMEM lanes 32q..32q+31 = weight rows of this warp
    const int h = ew >> 2;     // token columns [8h, 8h+8) of every 16
    int ti = 0;
    for (int item = blockIdx.x; item < num_items; item += gridDim.x, ++ti) {
      const int e = args.swap_experts[item / NG];
      const int wg = item - (item / NG) * NG;
      const int r0 = args.poffs[e];
      const int n = args.counts[e];
      const int n16 = (n + 15) >> 4;
      const bool ready = __all_sync(0xffffffffu, mbar_wait(acc_full, ti & 1) && !*abort_flag);
      if (!ready) {
        if (lane == 0) {
          record_timeout(args.hdr, 90 + kEpi);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      // this warp's token columns: 8 of every 16, i.e. chunks c = 2*i + h
      uint32_t g[kMaxChunks][8], u[kMaxChunks][8];  // [chunk][column]: MMA-0 / MMA-1 accumulators
      const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16) + kAccCol;
#pragma unroll
      for (int i = 0; i < kMaxChunks; ++i) {
        if (i < n16) {
          tmem_ld_32x32b_x8(tl + 16 * i + 8 * h, g[i]);
          tmem_ld_32x32b_x8(tl + 128 + 16 * i + 8 * h, u[i]);
        }
      }
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);

      if (kEpi == 1) {
        // output j = 128*wg + 32q + lane; token t = 16 i + 8 h + c
        const int j = wg * 128 + q * 32 + lane;
#pragma unroll
        for (int i = 0; i < kMaxChunks; ++i) {
          if (i >= n16) break;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int t = 16 * i + 8 * h + c;
            const float gv = __uint_as_float(g[i][c]);
            const float uv = __uint_as_float(u[i][c]);
            const float a = gv * __frcp_rn(1.0f + __expf(-gv)) * uv;  // silu(gate) * up
            // block amax over the warp's 32 outputs (non-negative floats order as integers)
            const float amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(a))));
            const int ex = e4m3_block_exponent(amax);
            const float inv = __uint_as_float((uint32_t)(127 - ex) << 23);
            const uint8_t code = (uint8_t)(__nv_cvt_float2_to_fp8x2(make_float2(a * inv, 0.0f),
                                                                    __NV_SATFINITE, __NV_E4M3) &
                                           0xFF);
            if (t < n) {
              const int row = r0 + t;
              args.a2[(size_t)row * args.I + j] = code;
              if (lane == 0)
                args.a2_sf[((size_t)(row >> 7) * (args.I / 128) + wg) * kSfChunk +
                           (row & 31) * 16 + ((row >> 5) & 3) * 4 + q] = (uint8_t)(ex + 127);
            }
          }
        }
      } else {
        // output columns h0 = 256*wg + 32q + lane (MMA 0) and +128 (MMA 1)
        const int hc0 = wg * kBlockN + q * 32 + lane;
#pragma unroll
        for (int i = 0; i < kMaxChunks; ++i) {
          if (i >= n16) break;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int t = 16 * i + 8 * h + c;
            if (t < n) {
              const int row = r0 + t;
              const int src = args.src_of[row];
              const float w = args.topk_w[src];
              __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(args.yp) + (size_t)row * args.H;
              dst[hc0] = __float2bfloat16_rn(w * __uint_as_float(g[i][c]));
              if (hc0 + 128 < n_rows) dst[hc0 + 128] = __float2bfloat16_rn(w * __uint_as_float(u[i][c]));
            }
          }
        }
      }
    }
  }

  pdl_launch();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

cudaError_t launch_gemm_swap(int epi, const CUtensorMap& tmW, const CUtensorMap& tmX,
                             const GemmArgs& args, int grid, bool pdl, cudaStream_t stream) {
  static bool attr_set[3] = {false, false, false};
  void (*fn)(CUtensorMap, CUtensorMap, GemmArgs) =
      (epi == 1) ? moe_gemm_swap_kernel<1> : moe_gemm_swap_kernel<2>;
  if (!attr_set[epi]) {
    cudaError_t err = cudaFuncSetAttribute((const void*)fn,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)swapk::kSmemBytes);
    if (err != cudaSuccess) return err;
    attr_set[epi] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(swapk::kThreads);
  cfg.dynamicSmemBytes = swapk::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, fn, tmW, tmX, args);
}

}  // namespace moe
