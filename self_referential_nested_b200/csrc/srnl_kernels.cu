// SRNL four-direction chunked scan: device kernels for sm_100a.
//
// Method sources (web pages on VisionHOPE; no page prints an equation):
//   "VisionHOPE: Visual Backbones as Self-Modifying Learning Systems" (summary
//   of arXiv 2609.33325) — write-rule, stability and 2D-maps paragraphs;
//   "VisionHOPE Model Overview: Architecture, Benchmarks, and Practical
//   Limits" — "Four-Directional Scanning and Spatial Chunking" and "Why the
//   Stability Controls Matter";
//   "VisionHOPE" README — "SRNL and VisionHOPE operator".
//
// Single-product form.  Every write right-multiplies each of the five memories
// by the same matrix T_t = alpha_t I - eta_t u_t k_t^T, u_t = (1 + alpha_t) k_t - v_t,
// because the retained transition alpha_t (I - eta k k^T) and the L2 signal
// (X k - X v) k^T are both X times a factor that does not depend on X.  So
// every memory is its initial state times one d x d product Q_t = T_1 ... T_t,
// and the kernels carry Q instead of five memories:
//   generation   [k~ v a beta] = (G Q_b) x_t,   G = [M_k0; M_v0; m_eta0; m_alpha0]
//   readout      y_t = M_mem0 (Q_t q_t)
// Rows of Q evolve independently: row_t = alpha_t row - eta_t (row . u_t) k_t.
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
// Scan: one CTA per (route, batch, head) sequence, 128 threads.
// ---------------------------------------------------------------------------
constexpr int kScanThreads = 128;
constexpr int kSub = 64;  // tokens staged in shared memory at a time

struct ScanSmem {
  // 16-byte aligned rows first: they are read and written as float4.
  alignas(16) float x[kSub][kD];  // head slice of x, route order
  alignas(16) float q[kSub][kD];  // head slice of q
  alignas(16) float k[kSub][kD];  // normalised keys
  alignas(16) float u[kSub][kD];  // u = (1 + alpha_t) k - v
  alignas(16) float z[kSub][kD];  // Q_t q_t
  alignas(16) float G[kGen][kD];  // generating initials of this (route, head)
  alignas(16) float Qb[kD][kD + 1];    // boundary product Q_b
  alignas(16) float Hb[kGen][kD + 1];  // boundary generating states G Q_b
  alignas(16) float2 ae[kSub];         // (alpha_t, eta_t)
  alignas(16) int pos[kSub];           // raster index of each staged token
};
static_assert(offsetof(ScanSmem, x) % 16 == 0 && offsetof(ScanSmem, q) % 16 == 0 &&
              offsetof(ScanSmem, k) % 16 == 0 && offsetof(ScanSmem, u) % 16 == 0 &&
              offsetof(ScanSmem, z) % 16 == 0, "float4 rows must be 16-byte aligned");
static_assert(sizeof(ScanSmem) <= 227 * 1024, "shared memory budget");

struct ScanKernelArgs {
  const void* x;
  const void* q;
  float* yr;
  float* finals;
  const float* G;
  const float* Mm;
  const float* scales;
  int B, H, W, C, heads, Lrow, Lcol;
  float alpha, eps;
  bool act_bf16, gen_bf16;
};

// Gates of one token, computed by one warp with lane = channel.
// Stabilized key, retention clamp, softplus step, soft injection cap and
// spectral clamp (paper summary, stability paragraph; "Why the Stability
// Controls Matter").
__device__ __forceinline__ void token_gates(float kt, float vv, float pa, float pb, float alpha,
                                            float eps, float& k_out, float& u_out, float& al_out,
                                            float& eta_out) {
  const float n2 = warp_sum(kt * kt);
  const float a = warp_sum(pa);
  const float beta = warp_sum(pb);
  const float k = kt / sqrtf(n2 + eps);
  const float kn2 = warp_sum(k * k);
  const float dkv = k - vv;
  const float d2 = warp_sum(dkv * dkv);
  const float gain = sqrtf(d2) * sqrtf(kn2);
  float sg;
  if (beta >= 0.f) {
    sg = 1.f / (1.f + expf(-beta));
  } else {
    const float e = expf(beta);
    sg = e / (1.f + e);
  }
  const float al = fminf(sg, alpha);
  const float eta0 = fmaxf(a, 0.f) + log1pf(expf(-fabsf(a)));
  const float z = eta0 * gain / (1.f - al);
  const float phi = (z < 1e-4f) ? (1.f - z * z * (1.f / 3.f)) : tanhf(z) / z;
  float eta = eta0 * phi;
  if (eta * kn2 > 2.f) eta = 2.f / kn2;
  k_out = k;
  u_out = (1.f + al) * k - vv;
  al_out = al;
  eta_out = eta;
}

__global__ void __launch_bounds__(kScanThreads)
srnl_scan_kernel(const ScanKernelArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ScanSmem& sm = *reinterpret_cast<ScanSmem*>(smem_raw);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int row = tid >> 2, cb = (tid & 3) * 8;  // this thread's slice of Q: row, cols cb..cb+7

  const int seq = blockIdx.x;                    // ((r * B + b) * heads + h)
  const int h = seq % a.heads;
  const int b = (seq / a.heads) % a.B;
  const int r = seq / (a.heads * a.B);
  const int N = a.H * a.W;
  const int L = (r < 2) ? a.Lrow : a.Lcol;
  const int64_t tok0 = (int64_t)b * N;           // first token row of this batch item
  const int ch0 = h * kD;

  const float* Gsrc = a.G + (int64_t)(r * a.heads + h) * kGen * kD;
  for (int i = tid; i < kGen * kD; i += kScanThreads) sm.G[i / kD][i % kD] = Gsrc[i];
  float mrow[kD];  // content-memory initial row `lane` (readout: y = M_mem0 z)
  {
    const float* Msrc = a.Mm + (int64_t)(r * a.heads + h) * kD * kD + lane * kD;
#pragma unroll
    for (int j = 0; j < kD; ++j) mrow[j] = Msrc[j];
  }
  const float scale = a.scales[r * a.C + ch0 + lane];

  float Qr[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) Qr[j] = (cb + j == row) ? 1.f : 0.f;
  __syncthreads();

  for (int c0 = 0; c0 < N; c0 += L) {
    const int Lc = min(L, N - c0);
    // ---- chunk boundary: generating states G Q_b (bf16-rounded on the bf16 path)
#pragma unroll
    for (int j = 0; j < 8; ++j) sm.Qb[row][cb + j] = Qr[j];
    __syncthreads();
    for (int m = warp; m < kGen; m += kScanThreads / 32) {
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < kD; ++i) acc = fmaf(sm.G[m][i], sm.Qb[i][lane], acc);
      sm.Hb[m][lane] = a.gen_bf16 ? round_bf16(acc) : acc;
    }
    __syncthreads();
    float hk[kD], hv[kD];
#pragma unroll
    for (int j = 0; j < kD; ++j) {
      hk[j] = sm.Hb[lane][j];
      hv[j] = sm.Hb[kD + lane][j];
    }
    const float ha = sm.Hb[2 * kD][lane];
    const float hb = sm.Hb[2 * kD + 1][lane];

    for (int s0 = 0; s0 < Lc; s0 += kSub) {
      const int T = min(kSub, Lc - s0);
      // ---- stage x and q of T tokens (route order)
      for (int idx = tid; idx < T * (kD / 4); idx += kScanThreads) {
        const int tt = idx >> 3, part = (idx & 7) * 4;
        const int p = route_pos(r, c0 + s0 + tt, a.H, a.W);
        const int64_t off = (tok0 + p) * a.C + ch0 + part;
        *reinterpret_cast<float4*>(&sm.x[tt][part]) = load4(a.x, off, a.act_bf16);
        *reinterpret_cast<float4*>(&sm.q[tt][part]) = load4(a.q, off, a.gen_bf16);
        if (part == 0) sm.pos[tt] = p;
      }
      __syncthreads();
      // ---- generation from the boundary states + gates, one warp per token
      for (int tt = warp; tt < T; tt += kScanThreads / 32) {
        float kt = 0.f, vv = 0.f;
#pragma unroll
        for (int j = 0; j < kD; ++j) {
          const float xj = sm.x[tt][j];
          kt = fmaf(hk[j], xj, kt);
          vv = fmaf(hv[j], xj, vv);
        }
        const float xl = sm.x[tt][lane];
        float k, u, al, eta;
        token_gates(kt, vv, ha * xl, hb * xl, a.alpha, a.eps, k, u, al, eta);
        sm.k[tt][lane] = k;
        sm.u[tt][lane] = u;
        if (lane == 0) sm.ae[tt] = make_float2(al, eta);
      }
      __syncthreads();
      // ---- token-order write of Q's rows and readout z_t = Q_t q_t
      for (int tt = 0; tt < T; ++tt) {
        const float4 u0 = *reinterpret_cast<const float4*>(&sm.u[tt][cb]);
        const float4 u1 = *reinterpret_cast<const float4*>(&sm.u[tt][cb + 4]);
        const float4 k0 = *reinterpret_cast<const float4*>(&sm.k[tt][cb]);
        const float4 k1 = *reinterpret_cast<const float4*>(&sm.k[tt][cb + 4]);
        const float4 q0 = *reinterpret_cast<const float4*>(&sm.q[tt][cb]);
        const float4 q1 = *reinterpret_cast<const float4*>(&sm.q[tt][cb + 4]);
        const float2 ae = sm.ae[tt];
        const float uu[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
        const float kk[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
        const float qq[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) s = fmaf(Qr[j], uu[j], s);
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        const float cs = ae.y * s;
#pragma unroll
        for (int j = 0; j < 8; ++j) Qr[j] = fmaf(ae.x, Qr[j], -cs * kk[j]);
        float z = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) z = fmaf(Qr[j], qq[j], z);
        z += __shfl_xor_sync(0xffffffffu, z, 1);
        z += __shfl_xor_sync(0xffffffffu, z, 2);
        if ((tid & 3) == 0) sm.z[tt][row] = z;
      }
      __syncthreads();
      // ---- readout y_t = M_mem0 z_t, scaled, written at the token's raster slot
      for (int tt = warp; tt < T; tt += kScanThreads / 32) {
        float y = 0.f;
#pragma unroll
        for (int j = 0; j < kD; ++j) y = fmaf(mrow[j], sm.z[tt][j], y);
        const int p = sm.pos[tt];
        a.yr[((int64_t)r * a.B * N + tok0 + p) * a.C + ch0 + lane] = scale * y;
      }
      __syncthreads();
    }
  }

  if (a.finals != nullptr) {
    // memories after the last token: [M_mem0; G] Q
#pragma unroll
    for (int j = 0; j < 8; ++j) sm.Qb[row][cb + j] = Qr[j];
    __syncthreads();
    float* dst = a.finals + (int64_t)seq * kStateFloats;
    const float* Msrc = a.Mm + (int64_t)(r * a.heads + h) * kD * kD;
    for (int m = warp; m < kMemRows; m += kScanThreads / 32) {
      float acc = 0.f;
      for (int i = 0; i < kD; ++i) {
        const float w = (m < kD) ? Msrc[m * kD + i] : sm.G[m - kD][i];
        acc = fmaf(w, sm.Qb[i][lane], acc);
      }
      dst[m * kD + lane] = acc;
    }
  }
}

// ---------------------------------------------------------------------------
// Fusion epilogue: y = yr0 + yr1 + yr2 + yr3 (fixed order), 8 channels per
// thread, 16-byte loads and stores.
// ---------------------------------------------------------------------------
__global__ void fuse_kernel(const float* __restrict__ yr, void* __restrict__ y, int64_t total,
                            bool act_bf16) {
  const int64_t i8 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (i8 >= total) return;
  float acc[8];
  {
    const float4 a = *reinterpret_cast<const float4*>(yr + i8);
    const float4 b = *reinterpret_cast<const float4*>(yr + i8 + 4);
    acc[0] = a.x; acc[1] = a.y; acc[2] = a.z; acc[3] = a.w;
    acc[4] = b.x; acc[5] = b.y; acc[6] = b.z; acc[7] = b.w;
  }
#pragma unroll
  for (int r = 1; r < 4; ++r) {
    const float4 a = *reinterpret_cast<const float4*>(yr + r * total + i8);
    const float4 b = *reinterpret_cast<const float4*>(yr + r * total + i8 + 4);
    acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
    acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
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
  return cudaFuncSetAttribute(srnl_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)sizeof(ScanSmem));
}

cudaError_t launch_query_projection(const ScanGeom& g, const ScanParamsDev& p, const void* x,
                                    void* q, cudaStream_t s) {
  const int64_t M = (int64_t)g.B * g.H * g.W;
  dim3 grid((unsigned)((M + kQpBM - 1) / kQpBM), (unsigned)((g.C + kQpBO - 1) / kQpBO));
  query_projection_kernel<<<grid, kQpThreads, 0, s>>>(x, p.Wq, q, M, g.C, g.act_bf16, g.gen_bf16);
  return cudaGetLastError();
}

cudaError_t launch_scan(const ScanGeom& g, const ScanParamsDev& p, const void* x, const void* q,
                        float* yr, float* finals, cudaStream_t s) {
  ScanKernelArgs a;
  a.x = x; a.q = q; a.yr = yr; a.finals = finals;
  a.G = p.G; a.Mm = p.Mm; a.scales = p.scales;
  a.B = g.B; a.H = g.H; a.W = g.W; a.C = g.C; a.heads = g.heads;
  a.Lrow = g.Lrow; a.Lcol = g.Lcol; a.alpha = g.alpha; a.eps = g.eps;
  a.act_bf16 = g.act_bf16; a.gen_bf16 = g.gen_bf16;
  const unsigned nseq = 4u * (unsigned)g.B * (unsigned)g.heads;
  srnl_scan_kernel<<<nseq, kScanThreads, sizeof(ScanSmem), s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_fuse(const ScanGeom& g, const float* yr, void* y, cudaStream_t s) {
  const int64_t total = (int64_t)g.B * g.H * g.W * g.C;
  const int64_t threads = total / 8;
  const int bs = 256;
  fuse_kernel<<<(unsigned)((threads + bs - 1) / bs), bs, 0, s>>>(yr, y, total, g.act_bf16);
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
