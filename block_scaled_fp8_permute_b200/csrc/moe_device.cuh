// moe_device.cuh -- device helpers shared by the GEMM kernels: the E4M3
// block requantiser of the linear1 epilogue and programmatic-dependent-launch
// hooks.
#pragma once

#include <cuda_fp8.h>
#include <stdint.h>

namespace moe {

// ------------------------------------------------------------- requantiser
// Smallest e with 448 * 2^e >= amax, from the bits of amax (448 = 1.75 * 2^8):
// amax = m * 2^x with m in [1,2) needs e = x - 8 when m <= 1.75, else x - 7.
// amax == 0 gives 0; results are clamped to [-127, 127].
__device__ __forceinline__ int e4m3_block_exponent(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  const int biased = (int)((bits >> 23) & 0xFF);
  if (amax == 0.0f) return 0;
  if (biased == 0) return -127;
  const int x = biased - 127;
  int e = ((bits & 0x7FFFFFu) > 0x600000u) ? x - 7 : x - 8;
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// Requantise 32 floats: E4M3 codes (little-endian packed, 4 per word) and
// the UE8M0 byte of the block.
__device__ __forceinline__ void requant32(const float (&a)[32], uint32_t (&packed)[8],
                                          uint32_t& sbyte) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(a[i]));
  const int e = e4m3_block_exponent(amax);
  const float inv = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e, exact
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const __nv_fp8x2_storage_t lo =
        __nv_cvt_float2_to_fp8x2(make_float2(a[4 * i] * inv, a[4 * i + 1] * inv), __NV_SATFINITE,
                                 __NV_E4M3);
    const __nv_fp8x2_storage_t hi =
        __nv_cvt_float2_to_fp8x2(make_float2(a[4 * i + 2] * inv, a[4 * i + 3] * inv),
                                 __NV_SATFINITE, __NV_E4M3);
    packed[i] = (uint32_t)lo | ((uint32_t)hi << 16);
  }
  sbyte = (uint32_t)(e + 127);
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace moe
