// SRNL four-direction chunked scan: projection, fusion and index kernels (sm_100a).
//
// Method sources (web pages on VisionHOPE; no page prints an equation):
//   "VisionHOPE: Visual Backbones as Self-Modifying Learning Systems" (summary
//   of arXiv 2609.33325) — write-rule, stability and 2D-maps paragraphs;
//   "VisionHOPE Model Overview: Architecture, Benchmarks, and Practical
//   Limits" — "Four-Directional Scanning and Spatial Chunking" and "Why the
//   Stability Controls Matter";
//   "VisionHOPE" README — "SRNL and VisionHOPE operator".
//
// The sequence kernel itself lives in srnl_scan.cu.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "srnl_common.cuh"
#include "srnl_launch.h"

namespace srnl {

// ---------------------------------------------------------------------------
// Query projection (SIMT, 64x64 output tiles, fp32 accumulate).
// q = x W_q^T is shared by all four routes ("Four-Directional Scanning ..."
// and the caveats paragraph of the paper summary: the query projection stays
// outside the recurrence).
// ---------------------------------------------------------------------------
constexpr int kQpBM = 64, kQpBO = 64, kQpBK = 32, kQpThreads = 256;

__global__ void __launch_bounds__(kQpThreads)
query_projection_kernel(const void* __restrict__ x, const float* __restrict__ Wq,
                        void* __restrict__ q, int64_t M, int C, bool act_bf16, bool q_bf16) {
  __shared__ float xs[kQpBK][kQpBM + 4];
  __shared__ float ws[kQpBK][kQpBO + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int64_t m0 = (int64_t)blockIdx.x * kQpBM;
  const int o0 = blockIdx.y * kQpBO;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < C; k0 += kQpBK) {
    // 64 rows x 32 k of x and of W: 512 float4 each, 2 per thread.
#pragma unroll
    for (int rep = 0; rep < 2; ++rep) {
      const int idx = tid + rep * kQpThreads;
      const int row = idx >> 3, kq = (idx & 7) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (m0 + row < M && k0 + kq < C) v = load4(x, (m0 + row) * C + k0 + kq, act_bf16);
      xs[kq + 0][row] = v.x; xs[kq + 1][row] = v.y; xs[kq + 2][row] = v.z; xs[kq + 3][row] = v.w;
      float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
      if (o0 + row < C && k0 + kq < C)
        w = *reinterpret_cast<const float4*>(Wq + (int64_t)(o0 + row) * C + k0 + kq);
      ws[kq + 0][row] = w.x; ws[kq + 1][row] = w.y; ws[kq + 2][row] = w.z; ws[kq + 3][row] = w.w;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kQpBK; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&xs[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&ws[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    const int o = o0 + tx * 4;
    if (m >= M || o >= C) continue;
    if (q_bf16) {
      __nv_bfloat162 lo = __floats2bfloat162_rn(acc[i][0], acc[i][1]);
      __nv_bfloat162 hi = __floats2bfloat162_rn(acc[i][2], acc[i][3]);
      uint2 raw;
      raw.x = *reinterpret_cast<uint32_t*>(&lo);
      raw.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(q) + m * C + o) = raw;
    } else {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(q) + m * C + o) =
          make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    }
  }
}

// ---------------------------------------------------------------------------
// Fusion epilogue: y = yr0 + yr1 + yr2 + yr3 (fixed order), 8 channels per
// thread, 16-byte loads and stores.
// ---------------------------------------------------------------------------
// [n][heads][d] <-> [n][heads][32] element copies (zeros in the padded lanes).
template <typename T>
__global__ void pad_heads_kernel(const T* __restrict__ src, T* __restrict__ dst, int64_t n, int heads, int d) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // over dst
  if (i >= n * heads * kD) return;
  const int j = (int)(i % kD);
  const int64_t th = i / kD;  // token * heads + head
  dst[i] = j < d ? src[th * d + j] : T(0);
}

template <typename T>
__global__ void unpad_heads_kernel(const T* __restrict__ src, T* __restrict__ dst, int64_t n, int heads, int d) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // over dst
  if (i >= n * heads * d) return;
  const int64_t th = i / d;
  dst[i] = src[th * kD + (int)(i - th * d)];
}

__global__ void unpad_states_kernel(const float* __restrict__ src, float* __restrict__ dst, int64_t S, int d) {
  const int per = 3 * d * d + 2 * d;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= S * per) return;
  const int64_t sq = i / per;
  const int e = (int)(i - sq * per);
  const float* s = src + sq * kStateFloats;
  int off;
  if (e < 3 * d * d) {  // M_mem, M_k, M_v: top-left d x d of each 32 x 32
    const int m = e / (d * d), rc = e - m * d * d;
    off = m * kD * kD + (rc / d) * kD + rc % d;
  } else {  // m_eta, m_alpha: first d of each 32
    const int v = (e - 3 * d * d) / d, c = (e - 3 * d * d) % d;
    off = 3 * kD * kD + v * kD + c;
  }
  dst[i] = s[off];
}

// Element-wise bf16 <-> fp32 conversion (fp32 -> bf16 rounds to nearest even).
__global__ void convert_kernel(const void* __restrict__ src, bool src_bf16, void* __restrict__ dst, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  if (src_bf16)
    reinterpret_cast<float*>(dst)[i] = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(src)[i]);
  else
    reinterpret_cast<__nv_bfloat16*>(dst)[i] = __float2bfloat16_rn(reinterpret_cast<const float*>(src)[i]);
}

__global__ void fuse_kernel(const float* __restrict__ yr, void* __restrict__ y, int64_t total,
                            int routes, bool act_bf16, bool part_bf16) {
  const int64_t i8 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (i8 >= total) return;
  float acc[8];
#pragma unroll
  for (int r = 0; r < 4; ++r) {   // fixed order r0 + r1 + r2 + r3
    if (r >= routes) break;
    float v[8];
    if (part_bf16) {
      const uint4 raw = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(yr) + r * total + i8);
      const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
        v[2 * e] = f.x;
        v[2 * e + 1] = f.y;
      }
    } else {
      const float4 a = *reinterpret_cast<const float4*>(yr + r * total + i8);
      const float4 b = *reinterpret_cast<const float4*>(yr + r * total + i8 + 4);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = r == 0 ? v[e] : acc[e] + v[e];
  }
  if (act_bf16) {
    uint4 raw;
    __nv_bfloat162 p0 = __floats2bfloat162_rn(acc[0], acc[1]);
    __nv_bfloat162 p1 = __floats2bfloat162_rn(acc[2], acc[3]);
    __nv_bfloat162 p2 = __floats2bfloat162_rn(acc[4], acc[5]);
    __nv_bfloat162 p3 = __floats2bfloat162_rn(acc[6], acc[7]);
    raw.x = *reinterpret_cast<uint32_t*>(&p0);
    raw.y = *reinterpret_cast<uint32_t*>(&p1);
    raw.z = *reinterpret_cast<uint32_t*>(&p2);
    raw.w = *reinterpret_cast<uint32_t*>(&p3);
    *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(y) + i8) = raw;
  } else {
    float* yo = reinterpret_cast<float*>(y) + i8;
    *reinterpret_cast<float4*>(yo) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    *reinterpret_cast<float4*>(yo + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

__global__ void route_index_kernel(int route, int H, int W, int32_t* out) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < H * W) out[t] = route_pos(route, t, H, W);
}

// xr[b][t][:] = x[b][route_pos(t)][:], 16-byte chunks.
__global__ void gather_kernel(const uint4* __restrict__ x, uint4* __restrict__ xr, int route, int H,
                              int W, int64_t vec_per_token, int64_t total_vec) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total_vec) return;
  const int64_t tok = i / vec_per_token, part = i - tok * vec_per_token;
  const int N = H * W;
  const int64_t b = tok / N;
  const int t = (int)(tok - b * N);
  xr[i] = x[(b * N + route_pos(route, t, H, W)) * vec_per_token + part];
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
cudaError_t prepare_kernels() {
  cudaError_t e = prepare_scan_kernels();
  if (e != cudaSuccess) return e;
  if ((e = prepare_backward_kernel()) != cudaSuccess) return e;
  if ((e = prepare_backward64_kernel()) != cudaSuccess) return e;
  if ((e = prepare_scan_d64_kernel()) != cudaSuccess) return e;
  return prepare_projection_kernel();
}

cudaError_t launch_query_projection(const ScanGeom& g, const ScanParamsDev& p, const void* x,
                                    void* q, int* err, cudaStream_t s) {
  if (p.Wqb != nullptr && query_projection_tc_supported(g)) return launch_query_projection_tc(g, p, x, q, err, s);
  const int64_t M = (int64_t)g.B * g.H * g.W;
  dim3 grid((unsigned)((M + kQpBM - 1) / kQpBM), (unsigned)((g.C + kQpBO - 1) / kQpBO));
  query_projection_kernel<<<grid, kQpThreads, 0, s>>>(x, p.Wq, q, M, g.C, g.act_bf16, g.gen_bf16);
  return cudaGetLastError();
}

cudaError_t launch_fuse(const ScanGeom& g, const float* yr, void* y, cudaStream_t s) {
  const int64_t total = (int64_t)g.B * g.H * g.W * g.C;
  const int64_t threads = total / 8;
  const int bs = 256;
  fuse_kernel<<<(unsigned)((threads + bs - 1) / bs), bs, 0, s>>>(yr, y, total, g.routes, g.act_bf16,
                                                                partials_bf16(g));
  return cudaGetLastError();
}

cudaError_t launch_pad_heads(const void* src, void* dst, int64_t n, int heads, int d, int elt, cudaStream_t s) {
  const int64_t total = n * heads * kD;
  const unsigned grid = (unsigned)((total + 255) / 256);
  if (elt == 2)
    pad_heads_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(src), static_cast<__nv_bfloat16*>(dst),
                                          n, heads, d);
  else
    pad_heads_kernel<<<grid, 256, 0, s>>>(static_cast<const float*>(src), static_cast<float*>(dst), n, heads, d);
  return cudaGetLastError();
}

cudaError_t launch_unpad_heads(const void* src, void* dst, int64_t n, int heads, int d, int elt, cudaStream_t s) {
  const int64_t total = n * heads * d;
  const unsigned grid = (unsigned)((total + 255) / 256);
  if (elt == 2)
    unpad_heads_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(src),
                                            static_cast<__nv_bfloat16*>(dst), n, heads, d);
  else
    unpad_heads_kernel<<<grid, 256, 0, s>>>(static_cast<const float*>(src), static_cast<float*>(dst), n, heads, d);
  return cudaGetLastError();
}

cudaError_t launch_unpad_states(const float* src, float* dst, int64_t S, int d, cudaStream_t s) {
  const int64_t total = S * (3 * d * d + 2 * d);
  unpad_states_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(src, dst, S, d);
  return cudaGetLastError();
}

cudaError_t launch_convert(const void* src, bool src_bf16, void* dst, int64_t n, cudaStream_t s) {
  const int bs = 256;
  convert_kernel<<<(unsigned)((n + bs - 1) / bs), bs, 0, s>>>(src, src_bf16, dst, n);
  return cudaGetLastError();
}

cudaError_t launch_route_index(int route, int H, int W, int32_t* out, cudaStream_t s) {
  const int N = H * W, bs = 256;
  route_index_kernel<<<(N + bs - 1) / bs, bs, 0, s>>>(route, H, W, out);
  return cudaGetLastError();
}

cudaError_t launch_gather(const ScanGeom& g, int route, const void* x, void* xr, cudaStream_t s) {
  const int64_t bytes_per_token = (int64_t)g.C * (g.act_bf16 ? 2 : 4);
  const int64_t vpt = bytes_per_token / 16;
  const int64_t total = vpt * g.B * g.H * g.W;
  const int bs = 256;
  gather_kernel<<<(unsigned)((total + bs - 1) / bs), bs, 0, s>>>(
      reinterpret_cast<const uint4*>(x), reinterpret_cast<uint4*>(xr), route, g.H, g.W, vpt, total);
  return cudaGetLastError();
}

}  // namespace srnl
