// moe_kernels.cu -- the HBM-bound kernels of the MoE layer forward:
//   plan    (routing bookkeeping: histogram, prefix sums, stable scatter),
//   permute (dispatch: gather token rows and their scales into
//            expert-contiguous order),
//   combine (top-k reduction of the weighted BF16 partial rows into BF16),
//   transform (one-time weight repack).
// ("DeepSeek DeepGEMM 2026年4月重磅更新：Mega MoE融合算子、FP4精度与极致性能优化",
//  section 3.1: the dispatch and combine steps around the two expert linears;
//  section 3.3: transform_weights_for_mega_moe and the buffer fields.)
#include <cuda_bf16.h>

#include "moe_internal.cuh"

namespace moe {

__device__ __forceinline__ void pdl_wait_k() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_k() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// byte offset of (row, K-group) inside scale chunks laid out [row/128][G][512]
__device__ __forceinline__ size_t sf_chunk_offset(int row, int kg, int G) {
  return ((size_t)(row >> 7) * G + kg) * kSfChunk + (row & 31) * 16 + ((row >> 5) & 3) * 4;
}

// ------------------------------------------------------------------- plan
// K1 (count + scan, one launch): every block fills its share of src_of with
// -1 (padding) and histograms its chunk of kPlanChunk consecutive flattened
// slots into chunk_counts[b][e]; the last block to finish then turns the
// chunk histograms into per-chunk starting ranks (exclusive, in place),
// expert counts, offsets, padded offsets, the m-tile -> expert table, the
// m-tile pairs and m-tiles of normal-tiled experts, the list of swapped-role
// experts (1 <= count <= swap_max) and the m-tiles of narrow-tiled experts
// (1 <= count <= narrow_max).
__global__ void __launch_bounds__(1024) plan_count_scan_kernel(
    const int32_t* __restrict__ idx, int R, int E, int NCH, int P_max, int swap_max, int narrow_max,
    int* __restrict__ chunk_counts, int* __restrict__ counts, int* __restrict__ offs,
    int* __restrict__ poffs, int* __restrict__ tile_expert, int* __restrict__ mpair,
    int* __restrict__ norm_mtiles, int* __restrict__ swap_experts, int* __restrict__ narrow_mtiles,
    int* __restrict__ src_of,
    int* __restrict__ hdr) {
  __shared__ int hist[kMaxE];
  __shared__ int last_block;
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) hist[e] = 0;
  // every row starts as padding (-1); the scatter kernel that follows
  // overwrites the rows that hold assignments.  Filled by all blocks, so no
  // single block writes the padding of every expert.
  for (int r = blockIdx.x * blockDim.x + tid; r < P_max; r += gridDim.x * blockDim.x)
    src_of[r] = -1;
  __syncthreads();
  const int a = blockIdx.x * kPlanChunk + tid;
  if (a < R) {
    const int e = idx[a];
    if (e >= 0 && e < E) {
      atomicAdd(&hist[e], 1);
    } else if (e != -1) {
      atomicAdd(&hdr[kHdrBadIds], 1);
      set_status(hdr, MOE_ERR_BAD_EXPERT_ID);
    }
  }
  __syncthreads();
  if (R > 0)
    for (int e = tid; e < E; e += blockDim.x) chunk_counts[(size_t)blockIdx.x * E + e] = hist[e];
  __threadfence();
  __syncthreads();
  if (tid == 0) last_block = atomicAdd(&hdr[kHdrPlanDone], 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!last_block) return;
  __threadfence();
  if (tid == 0) hdr[kHdrPlanDone] = 0;

  // ---- scan (last block only): count, padded count, m-tile pairs and
  // m-tiles of the normal-tiled experts, swapped-role experts
  constexpr int NV = 6;
  __shared__ int warp_tot[NV][32];
  __shared__ int carry[NV];
  const int lane = tid & 31, wid = tid >> 5;
  if (tid < NV) carry[tid] = 0;
  __syncthreads();
  for (int e0 = 0; e0 < E; e0 += 1024) {
    const int e = e0 + tid;
    int c = 0;
    if (e < E && R > 0) {
      // chunk histograms of this expert: exclusive prefix in place, several loads in flight
      int b = 0;
      for (; b + 8 <= NCH; b += 8) {
        int v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = chunk_counts[(size_t)(b + j) * E + e];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          chunk_counts[(size_t)(b + j) * E + e] = c;
          c += v[j];
        }
      }
      for (; b < NCH; ++b) {
        const int v = chunk_counts[(size_t)b * E + e];
        chunk_counts[(size_t)b * E + e] = c;
        c += v;
      }
    }
    if (e < E) counts[e] = c;
    const int pc = (c + kBlockM - 1) / kBlockM * kBlockM;
    const bool swapped = c > 0 && c <= swap_max;
    const bool narrow = !swapped && c > 0 && c <= narrow_max;  // one m-tile, <= kNarrowRows rows
    const int nm = (swapped || narrow) ? 0 : pc / kBlockM;
    const int np = (nm + 1) / 2;
    const int ns = swapped ? 1 : 0;
    const int nn = narrow ? 1 : 0;
    const int val[NV] = {c, pc, np, nm, ns, nn};
    int incl[NV] = {c, pc, np, nm, ns, nn};
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        const int t = __shfl_up_sync(0xffffffffu, incl[j], d);
        if (lane >= d) incl[j] += t;
      }
    }
    if (lane == 31)
      for (int j = 0; j < NV; ++j) warp_tot[j][wid] = incl[j];
    __syncthreads();
    if (wid == 0) {
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        int w = warp_tot[j][lane];
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, w, d);
          if (lane >= d) w += t;
        }
        warp_tot[j][lane] = w;
      }
    }
    __syncthreads();
    int pre[NV];
#pragma unroll
    for (int j = 0; j < NV; ++j)
      pre[j] = carry[j] + (wid ? warp_tot[j][wid - 1] : 0) + incl[j] - val[j];
    if (e < E) {
      offs[e] = pre[0];
      poffs[e] = pre[1];
      const int mt_first = pre[1] / kBlockM, nmt = pc / kBlockM;
      for (int mt = mt_first; mt < mt_first + nmt; ++mt) tile_expert[mt] = e;
      for (int i = 0; i < np; ++i)
        mpair[pre[2] + i] = (mt_first + 2 * i) | ((2 * i + 1 == nm) ? (int)0x80000000 : 0);
      for (int i = 0; i < nm; ++i) norm_mtiles[pre[3] + i] = mt_first + i;
      if (swapped) swap_experts[pre[4]] = e;
      if (narrow) narrow_mtiles[pre[5]] = mt_first;
    }
    __syncthreads();
    if (tid < NV) carry[tid] += warp_tot[tid][31];
    __syncthreads();
  }
  if (tid == 0) {
    offs[E] = carry[0];
    poffs[E] = carry[1];
    hdr[kHdrP] = carry[1];
    hdr[kHdrMTiles] = carry[1] / kBlockM;
    hdr[kHdrMPairs] = carry[2];
    hdr[kHdrNormMTiles] = carry[3];
    hdr[kHdrSwapExperts] = carry[4];
    hdr[kHdrSwapMax] = swap_max;
    hdr[kHdrNarrowMTiles] = carry[5];
    hdr[kHdrNarrowMax] = narrow_max;
  }
}

// K2: stable scatter.  Thread i of block b owns assignment b*kPlanChunk+i;
// its row is padded_offs[e] + (assignments of e in earlier chunks) +
// (assignments of e in earlier warps of this chunk) + (earlier lanes of its
// warp with the same expert), which orders each expert's rows by ascending
// flattened index.
__global__ void __launch_bounds__(1024) plan_scatter_kernel(const int32_t* __restrict__ idx, int R,
                                                            int E,
                                                            const int* __restrict__ chunk_base,
                                                            const int* __restrict__ poffs,
                                                            int* __restrict__ row_of,
                                                            int* __restrict__ src_of) {
  extern __shared__ unsigned short wcnt[];  // [32 warps][E]
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  for (int i = tid; i < 32 * E; i += blockDim.x) wcnt[i] = 0;
  pdl_wait_k();  // chunk bases and padded offsets come from K1
  __syncthreads();
  const int a = blockIdx.x * kPlanChunk + tid;
  int e = -1;
  if (a < R) {
    e = idx[a];
    if (e < 0 || e >= E) e = -1;
  }
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int rank_w = __popc(peers & ((1u << lane) - 1u));
  if (e >= 0 && rank_w == 0) wcnt[wid * E + e] = (unsigned short)__popc(peers);
  __syncthreads();
  if (a < R) {
    if (e < 0) {
      row_of[a] = -1;
    } else {
      int rank = chunk_base[(size_t)blockIdx.x * E + e] + rank_w;
      for (int w = 0; w < wid; ++w) rank += wcnt[w * E + e];
      const int row = poffs[e] + rank;
      row_of[a] = row;
      src_of[row] = a;
    }
  }
}

// ---------------------------------------------------------------- permute
// One warp per padded row: copy x[t] (H bytes) into Xp[row] and its scale
// words into the chunked layout the GEMM streams.  Padding rows are skipped.
__global__ void permute_kernel(const uint8_t* __restrict__ x, const int32_t* __restrict__ x_sf,
                               const int* __restrict__ src_of, const int* __restrict__ hdr, int H,
                               int topk, uint8_t* __restrict__ xp, uint8_t* __restrict__ xp_sf) {
  pdl_wait_k();
  const int P = hdr[kHdrP];
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int G = H / 128;
  for (int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < P; row += warps) {
    const int src = src_of[row];
    if (src < 0) continue;
    const int t = src / topk;
    const uint4* s4 = reinterpret_cast<const uint4*>(x + (size_t)t * H);
    uint4* d4 = reinterpret_cast<uint4*>(xp + (size_t)row * H);
    for (int i = lane; i < H / 16; i += 32) d4[i] = __ldg(&s4[i]);
    for (int kg = lane; kg < G; kg += 32)
      *reinterpret_cast<int32_t*>(xp_sf + sf_chunk_offset(row, kg, G)) = x_sf[(size_t)t * G + kg];
  }
  pdl_launch_k();
}

// ---------------------------------------------------------------- combine
// y[t] = BF16_RNE( sum_s Yp[row_of[t][s]] ), slot order, FP32 sum of the
// BF16 partial rows (the top-k weight was applied by the linear2 epilogue).
// One block per token, 8 columns (16 bytes) per thread and slot.
__global__ void combine_kernel(const uint16_t* __restrict__ yp, const int* __restrict__ row_of,
                               int T, int H, int topk, __nv_bfloat16* __restrict__ y) {
  pdl_wait_k();
  __shared__ int rows[kMaxTopk];
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    __syncthreads();
    if (threadIdx.x < topk) rows[threadIdx.x] = row_of[(size_t)t * topk + threadIdx.x];
    __syncthreads();
    for (int c = threadIdx.x * 8; c < H; c += blockDim.x * 8) {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll 4
      for (int s = 0; s < topk; ++s) {
        const int r = rows[s];
        if (r < 0) continue;
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(yp + (size_t)r * H + c));
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] += __uint_as_float(w4[i] << 16);
          acc[2 * i + 1] += __uint_as_float(w4[i] & 0xFFFF0000u);
        }
      }
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        o[i] = *reinterpret_cast<const uint32_t*>(&b);
      }
      *reinterpret_cast<uint4*>(y + (size_t)t * H + c) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  pdl_launch_k();
}

// ------------------------------------------------------- standalone GEMM
// Tile lists of the FP8 x FP4 GEMM (dense or masked grouped): group g owns
// m-tiles g*mt_per_g .. g*mt_per_g + ceil(rows_g / 128) - 1 with rows_g =
// masked_m[g] (m_max when masked_m is NULL), read on the device so a
// captured graph follows the counts of each replay.  One block of 1024.
__global__ void __launch_bounds__(1024) gemm_plan_kernel(const int* __restrict__ masked_m, int G,
                                                         int m_max, int mt_per_g,
                                                         int* __restrict__ tile_expert,
                                                         int* __restrict__ norm_mtiles,
                                                         int* __restrict__ hdr) {
  __shared__ int wsum[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int g0 = 0; g0 < G; g0 += blockDim.x) {
    const int g = g0 + tid;
    int c = 0;
    if (g < G) {
      int rows = masked_m ? masked_m[g] : m_max;
      if (rows < 0 || rows > m_max) {
        set_status(hdr, MOE_ERR_INVALID_ARG);
        rows = rows < 0 ? 0 : m_max;
      }
      c = (rows + kBlockM - 1) / kBlockM;
      for (int i = 0; i < mt_per_g; ++i) tile_expert[(size_t)g * mt_per_g + i] = g;
    }
    int incl = c;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += t;
    }
    if (lane == 31) wsum[wid] = incl;
    __syncthreads();
    if (wid == 0) {
      int w = wsum[lane];
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, w, d);
        if (lane >= d) w += t;
      }
      wsum[lane] = w;
    }
    __syncthreads();
    const int pre = carry + (wid ? wsum[wid - 1] : 0) + incl - c;
    for (int i = 0; i < c; ++i) norm_mtiles[pre + i] = g * mt_per_g + i;
    __syncthreads();
    if (tid == 0) carry += wsum[31];
    __syncthreads();
  }
  if (tid == 0) hdr[kHdrNormMTiles] = carry;
}

// A's scale words [rows][KG] into the 512-byte chunks the GEMM streams.
__global__ void sf_chunks_kernel(const int32_t* __restrict__ a_sf, long long rows, int KG,
                                 uint8_t* __restrict__ out) {
  const long long n = rows * KG;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(i / KG), kg = (int)(i - (long long)r * KG);
    *reinterpret_cast<int32_t*>(out + sf_chunk_offset(r, kg, KG)) = a_sf[i];
  }
}

cudaError_t launch_sf_chunks(const int32_t* a_sf, long long rows, int KG, uint8_t* sf_chunks,
                             cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  long long grid = (rows * KG + 255) / 256;
  if (grid > 148LL * 16) grid = 148LL * 16;
  sf_chunks_kernel<<<(unsigned)grid, 256, 0, stream>>>(a_sf, rows, KG, sf_chunks);
  return cudaGetLastError();
}

cudaError_t launch_gemm_prep(const int* masked_m, int G, int m_max, int mt_per_g, int* tile_expert,
                             int* norm_mtiles, int* hdr, const int32_t* a_sf, long long rows, int KG,
                             uint8_t* sf_chunks, cudaStream_t stream) {
  gemm_plan_kernel<<<1, 1024, 0, stream>>>(masked_m, G, m_max, mt_per_g, tile_expert, norm_mtiles,
                                           hdr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || rows == 0) return e;
  long long grid = (rows * KG + 255) / 256;
  if (grid > 148LL * 16) grid = 148LL * 16;
  sf_chunks_kernel<<<(unsigned)grid, 256, 0, stream>>>(a_sf, rows, KG, sf_chunks);
  return cudaGetLastError();
}

// -------------------------------------------------------------- transform
// One thread per (expert, K-block, transformed row): 64 bytes of codes and
// one 32-bit word of scales.  interleave != 0 applies the W1 gate/up
// interleave: transformed row n' = 256g + j takes gate row 128g + j (j < 128)
// or up row half + 128g + (j - 128).
__global__ void transform_kernel(const uint8_t* __restrict__ w, const uint8_t* __restrict__ w_sf,
                                 int E, int N, int K, int interleave, uint8_t* __restrict__ wt,
                                 uint8_t* __restrict__ wt_sf) {
  const int KB = K / 128;
  const long long total = (long long)E * KB * N;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int n = (int)(i % N);
    const int kb = (int)((i / N) % KB);
    const int e = (int)(i / ((long long)N * KB));
    int src_row = n;
    if (interleave) {
      const int g = n >> 8, j = n & 255;
      src_row = (j < 128) ? (g * 128 + j) : (N / 2 + g * 128 + (j - 128));
    }
    const size_t srow = (size_t)e * N + src_row;
    const uint4* s4 = reinterpret_cast<const uint4*>(w + srow * (K / 2) + (size_t)kb * 64);
    uint4* d4 = reinterpret_cast<uint4*>(wt + (((size_t)e * KB + kb) * N + n) * 64);
#pragma unroll
    for (int v = 0; v < 4; ++v) d4[v] = s4[v];
    const uint32_t sfw = *reinterpret_cast<const uint32_t*>(w_sf + srow * (K / 32) + (size_t)kb * 4);
    const size_t chunk = ((size_t)e * KB + kb) * (N / 128) + (n >> 7);
    *reinterpret_cast<uint32_t*>(wt_sf + chunk * kSfChunk + (n & 31) * 16 + ((n >> 5) & 3) * 4) = sfw;
  }
}

// ---------------------------------------------------------------- launchers
static cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, size_t smem, bool pdl,
                              cudaStream_t stream, void** args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

cudaError_t launch_plan(const int32_t* idx, int R, int E, int NCH, int P_max, int swap_max,
                        int narrow_max,
                        int* chunk, int* counts, int* offs, int* poffs, int* tile_expert,
                        int* mpair, int* norm_mtiles, int* swap_experts, int* narrow_mtiles,
                        int* row_of, int* src_of, int* hdr, bool pdl, cudaStream_t stream) {
  static bool attr_set = false;
  const size_t scatter_smem = (size_t)32 * E * sizeof(unsigned short);
  if (!attr_set) {
    cudaError_t err = cudaFuncSetAttribute((const void*)plan_scatter_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           32 * kMaxE * (int)sizeof(unsigned short));
    if (err != cudaSuccess) return err;
    attr_set = true;
  }
  plan_count_scan_kernel<<<NCH > 0 ? NCH : 1, 1024, 0, stream>>>(
      idx, R, E, NCH, P_max, swap_max, narrow_max, chunk, counts, offs, poffs, tile_expert, mpair,
      norm_mtiles, swap_experts, narrow_mtiles, src_of, hdr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || R == 0) return e;
  const int32_t* cidx = idx;
  const int* cchunk = chunk;
  const int* cpoffs = poffs;
  void* args[] = {(void*)&cidx, (void*)&R, (void*)&E, (void*)&cchunk, (void*)&cpoffs,
                  (void*)&row_of, (void*)&src_of};
  return launch_pdl((const void*)plan_scatter_kernel, dim3(NCH), dim3(1024), scatter_smem, pdl,
                    stream, args);
}

cudaError_t launch_permute(const uint8_t* x, const int32_t* x_sf, const int* src_of,
                           const int* hdr, int H, int topk, uint8_t* xp, uint8_t* xp_sf, int grid,
                           bool pdl, cudaStream_t stream) {
  void* args[] = {(void*)&x, (void*)&x_sf, (void*)&src_of, (void*)&hdr, (void*)&H,
                  (void*)&topk, (void*)&xp, (void*)&xp_sf};
  return launch_pdl((const void*)permute_kernel, dim3(grid), dim3(256), 0, pdl, stream, args);
}

cudaError_t launch_combine(const uint16_t* yp, const int* row_of, int T, int H, int topk,
                           uint16_t* y, int grid, bool pdl, cudaStream_t stream) {
  __nv_bfloat16* yb = reinterpret_cast<__nv_bfloat16*>(y);
  void* args[] = {(void*)&yp, (void*)&row_of, (void*)&T, (void*)&H, (void*)&topk, (void*)&yb};
  int threads = H / 8 < 256 ? ((H / 8 + 31) / 32) * 32 : 256;
  return launch_pdl((const void*)combine_kernel, dim3(grid), dim3(threads), 0, pdl, stream, args);
}

cudaError_t launch_transform(const uint8_t* w, const uint8_t* w_sf, int E, int N, int K,
                             int interleave, uint8_t* wt, uint8_t* wt_sf, cudaStream_t stream) {
  const long long total = (long long)E * (K / 128) * N;
  long long grid = (total + 255) / 256;
  if (grid > 65535LL * 16) grid = 65535LL * 16;
  if (grid < 1) grid = 1;
  transform_kernel<<<(unsigned)grid, 256, 0, stream>>>(w, w_sf, E, N, K, interleave, wt, wt_sf);
  return cudaGetLastError();
}

}  // namespace moe
