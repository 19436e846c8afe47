// moe_epilogue.cuh -- the two fused GEMM epilogues, shared by the one-SM and
// the SM-pair grouped GEMM kernels.  One thread owns one accumulator row
// (TMEM lane) and one 128-column half of the 256-column tile.
//   linear1 (kEpi 1): columns [0,128) of the tile are gate outputs, [128,256)
//     the matching up outputs (the weight transform interleaves them);
//     a = silu(gate) * up in FP32, requantised per 32 values to E4M3 + UE8M0
//     ("DeepSeek DeepGEMM 2026年4月重磅更新" section 3.1: SwiGLU between
//     linear1 and linear2; section 4.2: UE8M0 scale factors, four per int32).
//   linear2 (kEpi 2): rows scaled by their top-k weight, rounded to BF16
//     (the GEMM's output type, section 4.3) and written through swizzled
//     shared-memory staging and TMA tensor stores.
//   standalone GEMM (kEpi 3): the same BF16 rows, unscaled, for the rows of
//     each group below its row count.
#pragma once

#include <cuda_bf16.h>

#include "moe_device.cuh"
#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {

constexpr int kEpiOutStage = 2048;  // bytes of staging per epilogue warp (32 rows x 32 BF16)

// TMEM -> registers: the columns this thread's half of the epilogue needs.
template <int kEpi>
__device__ __forceinline__ void epilogue_load(uint32_t (&v)[4][32], uint32_t trow, int h) {
  using namespace ptx;
  if (kEpi == 1) {
    tmem_ld_32x32b_x32(trow + 64 * h, v[0]);
    tmem_ld_32x32b_x32(trow + 64 * h + 32, v[1]);
    tmem_ld_32x32b_x32(trow + 128 + 64 * h, v[2]);
    tmem_ld_32x32b_x32(trow + 128 + 64 * h + 32, v[3]);
  } else {
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(trow + 128 * h + 32 * c, v[c]);
  }
}

// 32 rows x 128 FP32 columns of the accumulator (this warp's rows, one column
// half) times w, rounded to BF16 and written by TMA tensor stores: 4 chunks of
// 32 x 32 staged in 64-byte-swizzled shared memory.  row0: first of the 32
// rows in the output tensor map.  Warp-collective.
__device__ __forceinline__ void store_rows_bf16(const uint32_t (&v)[4][32], float w,
                                                const CUtensorMap* tmOut, uint8_t* stg, int col0,
                                                int row0, int lane) {
  using namespace ptx;
  const uint32_t stg_row = smem_u32(stg) + (uint32_t)lane * 64u;
  const uint32_t swz = ((uint32_t)lane >> 1) & 3u;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    if (lane == 0) bulk_wait_group_read0();  // staging free again
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t p[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(w * __uint_as_float(v[c][8 * j + 2 * i]),
                                                       w * __uint_as_float(v[c][8 * j + 2 * i + 1]));
        p[i] = *reinterpret_cast<const uint32_t*>(&b);
      }
      st_shared_v4(stg_row + 16u * ((uint32_t)j ^ swz), p[0], p[1], p[2], p[3]);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tmOut, stg, col0 + 32 * c, row0);
      bulk_commit_group();
    }
  }
}

// Compute and store one (row, half) of a finished tile.  mt: m-tile (128
// padded rows), nt: n-tile (256 weight rows), r: row in the tile, q: the
// warp's 32-row group, stg: the warp's staging buffer.  Warp-collective for
// kEpi 2 (all lanes must call it together).
template <int kEpi>
__device__ __forceinline__ void epilogue_store(const uint32_t (&v)[4][32], const GemmArgs& args,
                                               const CUtensorMap* tmOut, uint8_t* stg, int mt,
                                               int nt, int r, int h, int q, int lane) {
  using namespace ptx;
  const int row = mt * kBlockM + r;
  const int src = kEpi == 3 ? 0 : args.src_of[row];
  if (kEpi == 1) {
    if (src < 0) return;  // padding row
    uint32_t sbytes = 0;
    uint8_t* dst = args.a2 + (size_t)row * args.I + nt * 128 + 64 * h;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      float a[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float g = __uint_as_float(v[b][i]);
        const float u = __uint_as_float(v[2 + b][i]);
        a[i] = g * __frcp_rn(1.0f + __expf(-g)) * u;  // silu(g) * u
      }
      uint32_t packed[8], sb;
      requant32(a, packed, sb);
      uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * b);
      d4[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      d4[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
      sbytes |= sb << (8 * b);
    }
    uint8_t* sfdst = args.a2_sf + ((size_t)mt * (args.I / 128) + nt) * kSfChunk + (r & 31) * 16 +
                     (r >> 5) * 4 + 2 * h;
    *reinterpret_cast<uint16_t*>(sfdst) = (uint16_t)sbytes;
  } else if (kEpi == 2) {
    const int col0 = nt * kBlockN + 128 * h;
    if (col0 >= args.n_rows) return;  // half tile at the end of N (warp-uniform)
    // 32 padding rows (an expert's last m-tile, decode-sized batches): nothing to store
    if (__all_sync(0xffffffffu, src < 0)) return;
    const float w = src >= 0 ? args.topk_w[src] : 0.0f;
    store_rows_bf16(v, w, tmOut, stg, col0, mt * kBlockM + q * 32, lane);
  } else {
    // plain D rows of the standalone GEMM: whole 32-row boxes by TMA; in a box
    // that crosses the group's row count each lane writes its own row
    const int col0 = nt * kBlockN + 128 * h;
    if (col0 >= args.n_rows) return;
    const int g = args.tile_expert[mt];
    const int rin = row - g * args.m_max;  // row within its group
    int cnt = args.masked_m ? args.masked_m[g] : args.m_max;
    cnt = cnt < 0 ? 0 : (cnt > args.m_max ? args.m_max : cnt);
    const bool valid = rin < cnt;
    if (__all_sync(0xffffffffu, !valid)) return;
    if (__all_sync(0xffffffffu, valid)) {
      store_rows_bf16(v, 1.0f, tmOut, stg, col0, mt * kBlockM + q * 32, lane);
    } else if (valid) {
      uint4* dst = reinterpret_cast<uint4*>(args.d + (size_t)row * args.n_rows + col0);
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t p[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(v[c][8 * j + 2 * i]),
                                                           __uint_as_float(v[c][8 * j + 2 * i + 1]));
            p[i] = *reinterpret_cast<const uint32_t*>(&b);
          }
          dst[4 * c + j] = make_uint4(p[0], p[1], p[2], p[3]);
        }
    }
  }
}

}  // namespace moe
