// Shared device helpers for the SRNL scan kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace srnl {

constexpr int kD = 32;              // head dim built
constexpr int kGen = 2 * kD + 2;    // generating rows: M_k (d), M_v (d), m_eta, m_alpha
constexpr int kMemRows = kD + kGen; // all five memories stacked row-wise (98)
constexpr int kStateFloats = 3 * kD * kD + 2 * kD;

// Raster index p = i*W + j of the t-th token of route r.
//   r0: forward row-major, r1: reverse row-major,
//   r2: forward column-major (t = j*H + i), r3: reverse column-major.
// ("VisionHOPE Model Overview", section "Four-Directional Scanning and
//  Spatial Chunking".)
__host__ __device__ __forceinline__ int route_pos(int r, int t, int H, int W) {
  const int N = H * W;
  if (r & 1) t = N - 1 - t;
  if (r < 2) return t;
  const int j = t / H;
  const int i = t - j * H;
  return i * W + j;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float round_bf16(float v) {
  return __bfloat162float(__float2bfloat16_rn(v));
}

// Load 4 consecutive activations (fp32 or bf16) as fp32.
__device__ __forceinline__ float4 load4(const void* base, int64_t idx, bool bf16) {
  if (bf16) {
    const uint2 raw = *reinterpret_cast<const uint2*>(
        reinterpret_cast<const __nv_bfloat16*>(base) + idx);
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
    const float2 a = __bfloat1622float2(lo);
    const float2 b = __bfloat1622float2(hi);
    return make_float4(a.x, a.y, b.x, b.y);
  }
  return *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx);
}

}  // namespace srnl
