// SRNL four-direction chunked scan for head dim 64 (sm_100a), both precision paths.
//
// Method sources (web pages on VisionHOPE; no page prints an equation): "VisionHOPE" README,
// "SRNL and VisionHOPE operator" (head_dim up to 64); "VisionHOPE: Visual Backbones as
// Self-Modifying Learning Systems" (summary of arXiv 2609.33325), write-rule, stability and
// 2D-maps paragraphs; "VisionHOPE Model Overview: Architecture, Benchmarks, and Practical
// Limits", "Four-Directional Scanning and Spatial Chunking".
//
// Single-product form, as the 32-wide kernels: a sequence carries one 64 x 64 product Q of the
// transitions T_t = alpha_t I - eta_t u_t k_t^T; at a chunk start the boundary Q_b generates
// [k~ v a beta]_t = G (Q_b x_t) (G = [M_k0; M_v0; m_eta0; m_alpha0], 130 x 64) for the
// chunk's tokens; each row of Q is then written in token order, row <- alpha_t row -
// eta_t (row . u_t) k_t, and the readout is y_t = M_mem0 (Q_t q_t).
//
// One CTA per (route, batch, head) sequence, 256 threads.  Thread (row i = tid / 4) of Q owns the
// columns 16 m + 4 (tid % 4) + e (m, e = 0..3): the four lanes of a row read the shared token
// vectors at distinct banks.  The write is row-local, so the token loop needs no block
// barrier.  Per segment of up to kSeg tokens of a chunk: x and q staged block-wide;
// generation and the vector reductions with a warp per token; the scalar gates with a lane
// per token; the token loop (which also forms z_t = Q_t q_t); then the readout
// y_t = M_mem0 z_t with a warp per token, scaled by the route's fusion scales and stored
// at the token's raster position.  All arithmetic is fp32 (SIMT).  With bf16 generation the
// kernel applies that path's roundings: x, the boundary products w = Q_b x and G are rounded
// to bf16 before the generation product, and q arrives in bf16; the write and the readout
// stay fp32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "srnl_common.cuh"
#include "srnl_launch.h"
#include "srnl_umma.cuh"

namespace srnl {
namespace {

constexpr int kD64 = 64;
constexpr int kGen64 = 2 * kD64 + 2;   // 130 generating rows
constexpr int kThreads64 = 256;
constexpr int kWarps64 = kThreads64 / 32;
constexpr int kSeg64 = 24;             // tokens per segment
constexpr int kLd64 = kD64 + 4;        // row stride: 16-byte rows, conflict-free float4 row reads
constexpr int kRec64 = 2 * kD64 + 4;   // per-token record: k[64] u[64] alpha eta |k|^2 |k-v|^2
constexpr int kRk = 0, kRu = kD64, kRal = 2 * kD64, kReta = kRal + 1, kRkn2 = kRal + 2, kRne2 = kRal + 3;

struct Smem64 {
  alignas(16) float Qb[kD64][kLd64];
  alignas(16) float Gm[kGen64][kLd64];
  alignas(16) float Mm[kD64][kLd64];
  alignas(16) float rec[kSeg64][kRec64];
  alignas(16) float xs[kSeg64][kD64];
  alignas(16) float qv[kSeg64][kD64];
  alignas(16) float zs[kSeg64][kD64];
  alignas(16) float wh[kWarps64][kD64];
  alignas(16) float ab[kSeg64][2];     // a, beta per token
};
static_assert(sizeof(Smem64) <= 112 * 1024, "two CTAs per SM");

struct Args64 {
  const void* x;     // [B][N][C] act dtype (C = heads * 64)
  const void* q;     // [B][N][C] fp32, or bf16 with bf16 generation
  float* yr;         // [routes][B*N][C] scaled route partials at raster positions
  float* finals;     // [routes][B][heads][3*64*64 + 2*64] or nullptr
  unsigned long long* binds;
  const float* G;    // [routes][heads][130][64]
  const float* Mm;   // [routes][heads][64][64]
  const float* scales;
  int B, H, W, C, heads, Lrow, Lcol;
  float alpha, eps;
  bool act_bf16, gen_bf16, hard_cap;
};

// Dot product of a 16-byte-aligned shared row with a broadcast shared vector, n a multiple of
// 8; two accumulators, unrolled by 4 float4 pairs so that few loads are in flight at once.
template <int n>
__device__ __forceinline__ float dot64(const float* a, const float* b) {
  float s0 = 0.f, s1 = 0.f;
#pragma unroll 2
  for (int i = 0; i < n; i += 8) {
    const float4 x0 = *reinterpret_cast<const float4*>(a + i);
    const float4 y0 = *reinterpret_cast<const float4*>(b + i);
    const float4 x1 = *reinterpret_cast<const float4*>(a + i + 4);
    const float4 y1 = *reinterpret_cast<const float4*>(b + i + 4);
    s0 = fmaf(x0.x, y0.x, s0); s1 = fmaf(x1.x, y1.x, s1);
    s0 = fmaf(x0.y, y0.y, s0); s1 = fmaf(x1.y, y1.y, s1);
    s0 = fmaf(x0.z, y0.z, s0); s1 = fmaf(x1.z, y1.z, s1);
    s0 = fmaf(x0.w, y0.w, s0); s1 = fmaf(x1.w, y1.w, s1);
  }
  return s0 + s1;
}

__device__ __forceinline__ float load_act64(const void* base, int64_t idx, bool bf16) {
  if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[idx]);
  return reinterpret_cast<const float*>(base)[idx];
}

__device__ __forceinline__ float row4_sum(float v) {   // the 4 lanes of a row
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  return v;
}

__global__ void __launch_bounds__(kThreads64, 2) srnl_scan_d64_kernel(const Args64 A) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem64& sm = *reinterpret_cast<Smem64*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ri = tid >> 2;            // row of Q owned
  const int c0 = (tid & 3) * 4;       // columns owned: 16 m + c0 + e, m, e = 0..3
  const int seq = blockIdx.x;         // ((r * B + b) * heads + h)
  const int hh = seq % A.heads;
  const int b = (seq / A.heads) % A.B;
  const int r = seq / (A.heads * A.B);
  const int N = A.H * A.W;
  const int L = (r < 2) ? A.Lrow : A.Lcol;
  const int nc = (N + L - 1) / L;
  const int C = A.C, ch0 = hh * kD64;
  const int64_t tokbase = (int64_t)b * N;
  const int rh = r * A.heads + hh;

  for (int i = tid; i < kD64 * kD64; i += kThreads64) sm.Mm[i / kD64][i % kD64] = A.Mm[(size_t)rh * kD64 * kD64 + i];
  for (int i = tid; i < kGen64 * kD64; i += kThreads64) {
    const float gv = A.G[(size_t)rh * kGen64 * kD64 + i];
    sm.Gm[i / kD64][i % kD64] = A.gen_bf16 ? round_bf16(gv) : gv;
  }
  const float sc0 = A.scales[(size_t)r * C + ch0 + lane], sc1 = A.scales[(size_t)r * C + ch0 + 32 + lane];

  float Q[16];   // Q[4 m + e] = Q[ri][16 m + c0 + e]
#pragma unroll
  for (int c = 0; c < 16; ++c) Q[c] = (ri == 16 * (c >> 2) + c0 + (c & 3)) ? 1.f : 0.f;

  for (int c = 0; c < nc; ++c) {
    const int t0c = c * L, Lc = min(L, N - t0c);
    __syncthreads();
#pragma unroll
    for (int cc = 0; cc < 16; cc += 4)
      *reinterpret_cast<float4*>(&sm.Qb[ri][4 * cc + c0]) = make_float4(Q[cc], Q[cc + 1], Q[cc + 2], Q[cc + 3]);
    for (int s0 = 0; s0 < Lc; s0 += kSeg64) {
      const int T = min(kSeg64, Lc - s0);
      const int t0 = t0c + s0;
      __syncthreads();   // Q_b written; the previous segment's buffers are free
      for (int idx = tid; idx < T * kD64; idx += kThreads64) {
        const int tt = idx / kD64, j = idx % kD64;
        const int64_t o = (tokbase + route_pos(r, t0 + tt, A.H, A.W)) * C + ch0 + j;
        const float xv = load_act64(A.x, o, A.act_bf16);
        sm.xs[tt][j] = A.gen_bf16 ? round_bf16(xv) : xv;
        sm.qv[tt][j] = load_act64(A.q, o, A.gen_bf16);
      }
      __syncthreads();
      // generation and the vector reductions (warp per token; lane covers j and 32 + j)
      for (int tt = warp; tt < T; tt += kWarps64) {
        const float w0 = dot64<kD64>(sm.Qb[lane], sm.xs[tt]);              // w = Q_b x
        const float w1 = dot64<kD64>(sm.Qb[32 + lane], sm.xs[tt]);
        sm.wh[warp][lane] = A.gen_bf16 ? round_bf16(w0) : w0;
        sm.wh[warp][32 + lane] = A.gen_bf16 ? round_bf16(w1) : w1;
        __syncwarp();
        const float k0 = dot64<kD64>(sm.Gm[lane], sm.wh[warp]);
        const float k1 = dot64<kD64>(sm.Gm[32 + lane], sm.wh[warp]);
        const float v0 = dot64<kD64>(sm.Gm[kD64 + lane], sm.wh[warp]);
        const float v1 = dot64<kD64>(sm.Gm[kD64 + 32 + lane], sm.wh[warp]);
        const float ex = dot64<kD64>(sm.Gm[2 * kD64 + (lane & 1)], sm.wh[warp]);   // lanes 0/1: a / beta
        __syncwarp();
        const float inv = rsqrtf(warp_sum(k0 * k0 + k1 * k1) + A.eps);
        const float ka = k0 * inv, kb = k1 * inv;
        const float ea = ka - v0, eb = kb - v1;
        const float kn2 = warp_sum(ka * ka + kb * kb);
        const float ne2 = warp_sum(ea * ea + eb * eb);
        float* rc = sm.rec[tt];
        rc[kRk + lane] = ka;
        rc[kRk + 32 + lane] = kb;
        rc[kRu + lane] = v0;         // v until u is formed below
        rc[kRu + 32 + lane] = v1;
        if (lane == 0) { rc[kRkn2] = kn2; rc[kRne2] = ne2; sm.ab[tt][0] = ex; }
        if (lane == 1) sm.ab[tt][1] = ex;
      }
      __syncthreads();
      if (warp == 0) {   // scalar gates, one lane per token
        bool binds = false;
        if (lane < T) {
          float* rc = sm.rec[lane];
          float al, eta;
          binds = gate_scalars(rc[kRkn2], rc[kRne2], sm.ab[lane][0], sm.ab[lane][1], A.alpha, al, eta, A.hard_cap);
          rc[kRal] = al;
          rc[kReta] = eta;
        }
        if (A.binds != nullptr) count_binds(binds, A.binds);
      }
      __syncthreads();
      for (int idx = tid; idx < T * kD64; idx += kThreads64) {
        float* rc = sm.rec[idx / kD64];
        const int j = idx % kD64;
        rc[kRu + j] = (1.f + rc[kRal]) * rc[kRk + j] - rc[kRu + j];
      }
      __syncthreads();
      // token-order write on this thread's 16 entries of Q, then z_t = Q_t q_t
      for (int tt = 0; tt < T; ++tt) {
        const float* rc = sm.rec[tt];
        const float al = rc[kRal], eta = rc[kReta];
        float pr = 0.f;
#pragma unroll
        for (int cc = 0; cc < 16; cc += 4) {
          const float4 u = *reinterpret_cast<const float4*>(rc + kRu + 4 * cc + c0);
          pr = fmaf(Q[cc], u.x, pr);
          pr = fmaf(Q[cc + 1], u.y, pr);
          pr = fmaf(Q[cc + 2], u.z, pr);
          pr = fmaf(Q[cc + 3], u.w, pr);
        }
        const float ep = eta * row4_sum(pr);
        float z = 0.f;
#pragma unroll
        for (int cc = 0; cc < 16; cc += 4) {
          const float4 k = *reinterpret_cast<const float4*>(rc + kRk + 4 * cc + c0);
          const float4 qq = *reinterpret_cast<const float4*>(&sm.qv[tt][4 * cc + c0]);
          Q[cc] = fmaf(al, Q[cc], -ep * k.x);
          Q[cc + 1] = fmaf(al, Q[cc + 1], -ep * k.y);
          Q[cc + 2] = fmaf(al, Q[cc + 2], -ep * k.z);
          Q[cc + 3] = fmaf(al, Q[cc + 3], -ep * k.w);
          z = fmaf(Q[cc], qq.x, z);
          z = fmaf(Q[cc + 1], qq.y, z);
          z = fmaf(Q[cc + 2], qq.z, z);
          z = fmaf(Q[cc + 3], qq.w, z);
        }
        z = row4_sum(z);
        if ((tid & 3) == 0) sm.zs[tt][ri] = z;
      }
      __syncthreads();
      // readout y_t = M_mem0 z_t, scaled, at the token's raster position (warp per token)
      for (int tt = warp; tt < T; tt += kWarps64) {
        const float y0 = dot64<kD64>(sm.Mm[lane], sm.zs[tt]);
        const float y1 = dot64<kD64>(sm.Mm[32 + lane], sm.zs[tt]);
        const int64_t o = ((int64_t)r * A.B * N + tokbase + route_pos(r, t0 + tt, A.H, A.W)) * C + ch0;
        A.yr[o + lane] = sc0 * y0;
        A.yr[o + 32 + lane] = sc1 * y1;
      }
    }
  }
  if (A.finals == nullptr) return;
  // final memories X_0 Q: M_mem, M_k, M_v row-major, then m_eta, m_alpha
  __syncthreads();
#pragma unroll
  for (int cc = 0; cc < 16; cc += 4)
    *reinterpret_cast<float4*>(&sm.Qb[ri][4 * cc + c0]) = make_float4(Q[cc], Q[cc + 1], Q[cc + 2], Q[cc + 3]);
  __syncthreads();
  float* fo = A.finals + (size_t)seq * (3 * kD64 * kD64 + 2 * kD64);
  const int nrows = kD64 + kGen64;   // M_mem rows, then the 130 generating rows
  for (int e = tid; e < nrows * kD64; e += kThreads64) {
    const int row = e / kD64, col = e % kD64;
    const float* x0 = row < kD64 ? sm.Mm[row] : sm.Gm[row - kD64];
    float s = 0.f;
#pragma unroll 4
    for (int m = 0; m < kD64; ++m) s = fmaf(x0[m], sm.Qb[m][col], s);
    fo[e] = s;
  }
}

}  // namespace

cudaError_t prepare_scan_d64_kernel() {
  return cudaFuncSetAttribute(srnl_scan_d64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)sizeof(Smem64));
}

cudaError_t launch_scan_d64(const ScanGeom& g, const ScanParamsDev& p, const void* x, const void* q, float* yr,
                            float* finals, unsigned long long* binds, cudaStream_t s) {
  Args64 a;
  a.x = x; a.q = q; a.yr = yr; a.finals = finals; a.binds = binds;
  a.G = p.G; a.Mm = p.Mm; a.scales = p.scales;
  a.B = g.B; a.H = g.H; a.W = g.W; a.C = g.C; a.heads = g.heads; a.Lrow = g.Lrow; a.Lcol = g.Lcol;
  a.alpha = g.alpha; a.eps = g.eps; a.act_bf16 = g.act_bf16; a.gen_bf16 = g.gen_bf16; a.hard_cap = g.hard_cap;
  const unsigned nseq = (unsigned)g.routes * (unsigned)g.B * (unsigned)g.heads;
  srnl_scan_d64_kernel<<<nseq, kThreads64, sizeof(Smem64), s>>>(a);
  return cudaGetLastError();
}

}  // namespace srnl
