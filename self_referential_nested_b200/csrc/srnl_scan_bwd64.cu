// Backward pass of the SRNL scan for head dim 64 (sm_100a), fp32.
//
// Sources and the reverse-mode recurrence are those of srnl_scan_bwd.cu (32-wide heads): the
// forward in single-product form, a checkpoint pass, then chunks in reverse with the
// in-chunk states recomputed, the row-local reverse chain
//   dQ <- alpha_t dQ - eta_t (dQ k_t) u_t^T  (+ a_t q_t^T from the readout),
// per-warp partial sums of the token reductions, the gate backward (vector part with a warp
// per token, scalar part with a lane per token), the generation and readout adjoints and the
// rank-one parameter sums.
//
// 64-wide layout: one CTA of 256 threads per (route, batch, head) sequence (one CTA per SM).
// Thread (row i = tid / 4) of every 64 x 64 matrix owns the columns 16 m + 4 (tid % 4) + e
// (m, e = 0..3), so the four lanes of a row read shared token vectors at distinct banks; warp
// w owns rows 8 w .. 8 w + 7.  Row sums take two shuffles; a column sum over the warp's eight
// rows is a reduce-scatter of the thread's 16 values (14 shuffles) that leaves each lane two
// columns.  A warp working on one token covers components j and 32 + j with lane j.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <algorithm>

#include "srnl_bwd_common.cuh"
#include "srnl_common.cuh"
#include "srnl_launch.h"

namespace srnl {
namespace {

using bwd::load_act;

constexpr int D = 64;
constexpr int G6 = 2 * D + 2;            // generating rows: M_k, M_v, m_eta, m_alpha
constexpr int kThr = 256;
constexpr int kW = kThr / 32;
constexpr int kSeg6 = 16;                // tokens whose gate records sit in shared memory at once
constexpr int kSB6 = 8;                  // tokens per reverse sub-block
constexpr int kLd6 = D + 4;              // 16-byte rows, conflict-free float4 row reads
constexpr int kGt6 = G6 + 2;             // row stride of G^T (columns 130, 131 zero)
constexpr int kRec6 = 2 * D + 8;         // k[64] u[64] alpha eta s a beta |k|^2 |k-v|^2 pad
constexpr int kRk = 0, kRu = D, kRal = 2 * D, kReta = kRal + 1, kRs = kRal + 2, kRa = kRal + 3, kRb = kRal + 4,
              kRkn2 = kRal + 5, kRne2 = kRal + 6;
constexpr int kPart6 = 2 + 3 * D;        // per (token, warp): dalpha, p.w, du[64], dk[64], dq[64]
constexpr int kSeqPart6 = D * D + G6 * D + D;

struct Smem6 {
  alignas(16) float Mm[D][kLd6];
  alignas(16) float Gm[G6][kLd6];
  alignas(16) float GmT[D][kGt6];
  alignas(16) float Qb[D][kLd6];
  alignas(16) float rec[kSeg6][kRec6];
  alignas(16) float wh[kW][D];
  alignas(16) float sx[kSB6][D];
  alignas(16) float sq[kSB6][D];
  alignas(16) float sdo[kSB6][D];
  alignas(16) float sdy[kSB6][D];
  alignas(16) float sa[kSB6][D];
  alignas(16) float syq[kSB6][D];
  alignas(16) float sdh[kSB6][D];
  alignas(16) float sh[kSB6][D];
  alignas(16) float sdg[kSB6][kGt6];
  alignas(16) float part[kSB6][kW][kPart6];
  alignas(16) float sc[kSB6][8];
  alignas(16) float ds[kW][D];
};
static_assert(sizeof(Smem6) <= 227 * 1024, "one CTA per SM");
static_assert(offsetof(Smem6, sq) == offsetof(Smem6, sx) + sizeof(float) * kSB6 * D && 2 * kSB6 >= kSeg6,
              "the gate pass stages a segment's x over sx and sq");

struct Args6 {
  const void* x;
  const float* q;
  const void* dy;
  float *dxr, *dqr, *parts, *ckpt, *qs, *grec;
  const float *G, *Mm, *scales;
  int B, H, W, C, heads, Lrow, Lcol, max_chunks, Lmax;
  float alpha, eps;
  bool act_bf16, hard_cap;
};

template <int n>
__device__ __forceinline__ float dotv(const float* a, const float* b) {   // n a multiple of 4
  float s0 = 0.f, s1 = 0.f;
#pragma unroll 4
  for (int i = 0; i < n; i += 4) {
    const float4 x = *reinterpret_cast<const float4*>(a + i);
    const float4 y = *reinterpret_cast<const float4*>(b + i);
    s0 = fmaf(x.x, y.x, s0); s1 = fmaf(x.y, y.y, s1);
    s0 = fmaf(x.z, y.z, s0); s1 = fmaf(x.w, y.w, s1);
  }
  return s0 + s1;
}

// Column j of a [D][kLd6] shared matrix against a broadcast vector.
__device__ __forceinline__ float dotc(const float (*m)[kLd6], int j, const float* b) {
  float s0 = 0.f, s1 = 0.f;
#pragma unroll 4
  for (int i = 0; i < D; i += 4) {
    const float4 y = *reinterpret_cast<const float4*>(b + i);
    s0 = fmaf(m[i][j], y.x, s0); s1 = fmaf(m[i + 1][j], y.y, s1);
    s0 = fmaf(m[i + 2][j], y.z, s0); s1 = fmaf(m[i + 3][j], y.w, s1);
  }
  return s0 + s1;
}

__device__ __forceinline__ float row4(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  return v;
}

__device__ __forceinline__ float rows8(float v) {   // over the warp's 8 rows (lanes ^4, ^8, ^16)
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  v += __shfl_xor_sync(0xffffffffu, v, 8);
  v += __shfl_xor_sync(0xffffffffu, v, 16);
  return v;
}

// Reduce-scatter of the thread's 16 column values (index 4 m + e <-> column 16 m + c0 + e) over
// the warp's 8 rows; the lane ends with the sums of columns col0 and col0 + 1, where
// col0 = 16 (2 bit4 + bit3) + c0 + 2 bit2 (bits of the lane).
__device__ __forceinline__ void col8(const float (&c)[16], int lane, float& o0, float& o1) {
  const bool b4 = (lane >> 4) & 1, b3 = (lane >> 3) & 1, b2 = (lane >> 2) & 1;
  float h[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float keep = b4 ? c[8 + i] : c[i], send = b4 ? c[i] : c[8 + i];
    h[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
  float q4[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float keep = b3 ? h[4 + i] : h[i], send = b3 ? h[i] : h[4 + i];
    q4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float keep = b2 ? q4[2 + i] : q4[i], send = b2 ? q4[i] : q4[2 + i];
    (i == 0 ? o0 : o1) = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
}

// This thread's 16 entries of row i of a [64][64] global matrix (4 float4 at 16 m + c0).
__device__ __forceinline__ void ld16(const float* m, int i, int c0, float (&v)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 f = *reinterpret_cast<const float4*>(m + i * D + 16 * q + c0);
    v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
  }
}
__device__ __forceinline__ void st16(float* m, int i, int c0, const float (&v)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<float4*>(m + i * D + 16 * q + c0) = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}
__device__ __forceinline__ void to_qb(Smem6& sm, int i, int c0, const float (&v)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<float4*>(&sm.Qb[i][16 * q + c0]) = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}
__device__ __forceinline__ void from_qb(const Smem6& sm, int i, int c0, float (&v)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 f = *reinterpret_cast<const float4*>(&sm.Qb[i][16 * q + c0]);
    v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
  }
}
// Load the thread's 16 entries of a shared 64-vector (row of a [*][D] array).
__device__ __forceinline__ void vec16(const float* v64, int c0, float (&o)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 f = *reinterpret_cast<const float4*>(v64 + 16 * q + c0);
    o[4 * q] = f.x; o[4 * q + 1] = f.y; o[4 * q + 2] = f.z; o[4 * q + 3] = f.w;
  }
}

// One forward write on this thread's 16 entries: Q <- alpha Q - eta (Q u) k^T.
__device__ __forceinline__ void fwd_step(float (&Q)[16], const float* rc, int c0) {
  float u[16], k[16];
  vec16(rc + kRu, c0, u);
  vec16(rc + kRk, c0, k);
  float p0 = 0.f, p1 = 0.f;
#pragma unroll
  for (int v = 0; v < 16; v += 2) { p0 = fmaf(Q[v], u[v], p0); p1 = fmaf(Q[v + 1], u[v + 1], p1); }
  const float ep = rc[kReta] * row4(p0 + p1), al = rc[kRal];
#pragma unroll
  for (int v = 0; v < 16; ++v) Q[v] = fmaf(al, Q[v], -ep * k[v]);
}

// Gates of tokens [t0, t0 + T) into sm.rec (T <= kSeg6), as in the 32-wide kernel.
__device__ void gates_seg(Smem6& sm, const Args6& A, int r, int64_t tokbase, int ch0, int t0, int T, int tid) {
  float (*xs)[D] = reinterpret_cast<float (*)[D]>(&sm.sx[0][0]);
  const int warp = tid >> 5, lane = tid & 31;
  for (int idx = tid; idx < T * D; idx += kThr) {
    const int tt = idx / D, j = idx % D;
    xs[tt][j] = load_act(A.x, (tokbase + route_pos(r, t0 + tt, A.H, A.W)) * A.C + ch0 + j, A.act_bf16);
  }
  __syncthreads();
  for (int tt = warp; tt < T; tt += kW) {
    sm.wh[warp][lane] = dotv<D>(sm.Qb[lane], xs[tt]);
    sm.wh[warp][32 + lane] = dotv<D>(sm.Qb[32 + lane], xs[tt]);
    __syncwarp();
    const float k0 = dotv<D>(sm.Gm[lane], sm.wh[warp]), k1 = dotv<D>(sm.Gm[32 + lane], sm.wh[warp]);
    const float v0 = dotv<D>(sm.Gm[D + lane], sm.wh[warp]), v1 = dotv<D>(sm.Gm[D + 32 + lane], sm.wh[warp]);
    const float ex = dotv<D>(sm.Gm[2 * D + (lane & 1)], sm.wh[warp]);   // lanes 0/1: a / beta
    __syncwarp();
    const float s = sqrtf(warp_sum(k0 * k0 + k1 * k1) + A.eps);
    const float ka = k0 / s, kb = k1 / s;
    const float ea = ka - v0, eb = kb - v1;
    const float kn2 = warp_sum(ka * ka + kb * kb), ne2 = warp_sum(ea * ea + eb * eb);
    float* rc = sm.rec[tt];
    rc[kRk + lane] = ka; rc[kRk + 32 + lane] = kb;
    rc[kRu + lane] = v0; rc[kRu + 32 + lane] = v1;   // v until u is formed below
    if (lane == 0) { rc[kRs] = s; rc[kRa] = ex; rc[kRkn2] = kn2; rc[kRne2] = ne2; }
    if (lane == 1) rc[kRb] = ex;
  }
  __syncthreads();
  if (tid < T) {
    float* rc = sm.rec[tid];
    float al, eta;
    bwd::gate_scalars_f(rc[kRkn2], rc[kRne2], rc[kRa], rc[kRb], A.alpha, A.hard_cap, al, eta);
    rc[kRal] = al;
    rc[kReta] = eta;
  }
  __syncthreads();
  for (int idx = tid; idx < T * D; idx += kThr) {
    float* rc = sm.rec[idx / D];
    const int j = idx % D;
    rc[kRu + j] = (1.f + rc[kRal]) * rc[kRk + j] - rc[kRu + j];
  }
  __syncthreads();
}

__device__ __forceinline__ void copy4(float* dst, const float* src, int n4, int tid) {
  for (int i = tid; i < n4; i += kThr) reinterpret_cast<float4*>(dst)[i] = reinterpret_cast<const float4*>(src)[i];
}

__global__ void __launch_bounds__(kThr, 1) srnl_scan_backward64_kernel(const Args6 A) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem6& sm = *reinterpret_cast<Smem6*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ri = tid >> 2, c0 = (tid & 3) * 4;
  const int seq = blockIdx.x;
  const int hh = seq % A.heads;
  const int b = (seq / A.heads) % A.B;
  const int r = seq / (A.heads * A.B);
  const int N = A.H * A.W;
  const int L = (r < 2) ? A.Lrow : A.Lcol;
  const int nc = (N + L - 1) / L;
  const int C = A.C, ch0 = hh * D;
  const int64_t tokbase = (int64_t)b * N;
  const int rh = r * A.heads + hh;
  float* ckpt = A.ckpt + (size_t)seq * (A.max_chunks + 1) * (D * D);
  float* qs = A.qs + (size_t)seq * A.Lmax * (D * D);
  float* grec = A.grec + (size_t)seq * N * kRec6;
  // the lane's two columns after col8
  const int colA = 16 * (2 * ((lane >> 4) & 1) + ((lane >> 3) & 1)) + c0 + 2 * ((lane >> 2) & 1);

  for (int i = tid; i < D * D; i += kThr) sm.Mm[i / D][i % D] = A.Mm[(size_t)rh * D * D + i];
  for (int i = tid; i < G6 * D; i += kThr) {
    const float gv = A.G[(size_t)rh * G6 * D + i];
    sm.Gm[i / D][i % D] = gv;
    sm.GmT[i % D][i / D] = gv;
  }
  if (tid < D) { sm.GmT[tid][G6] = 0.f; sm.GmT[tid][G6 + 1] = 0.f; }
  if (tid < kSB6) { sm.sdg[tid][G6] = 0.f; sm.sdg[tid][G6 + 1] = 0.f; }
  for (int i = tid; i < kW * D; i += kThr) sm.ds[i / D][i % D] = 0.f;

  // ---------------- phase 1: forward chain, checkpoints, gate records
  float Qr[16];
#pragma unroll
  for (int v = 0; v < 16; ++v) Qr[v] = (ri == 16 * (v >> 2) + c0 + (v & 3)) ? 1.f : 0.f;
  for (int c = 0; c < nc; ++c) {
    st16(ckpt + (size_t)c * D * D, ri, c0, Qr);
    to_qb(sm, ri, c0, Qr);
    __syncthreads();
    const int t0c = c * L, Lc = min(L, N - t0c);
    for (int s0 = 0; s0 < Lc; s0 += kSeg6) {
      const int T = min(kSeg6, Lc - s0);
      gates_seg(sm, A, r, tokbase, ch0, t0c + s0, T, tid);
      copy4(grec + (size_t)(t0c + s0) * kRec6, sm.rec[0], T * kRec6 / 4, tid);
      for (int tt = 0; tt < T; ++tt) fwd_step(Qr, sm.rec[tt], c0);
      __syncthreads();
    }
  }
  st16(ckpt + (size_t)nc * D * D, ri, c0, Qr);

  // ---------------- phase 2: chunks in reverse
  float dQ[16], dM0[16], dQb[16], dG[3][16];
#pragma unroll
  for (int v = 0; v < 16; ++v) {
    dQ[v] = 0.f; dM0[v] = 0.f;
    dG[0][v] = 0.f; dG[1][v] = 0.f; dG[2][v] = 0.f;
  }
  const bool has_g2 = ri < 2;                 // third dG row: 128 + ri (rows 128, 129)

  for (int c = nc - 1; c >= 0; --c) {
    const int t0c = c * L, Lc = min(L, N - t0c);
    const int nseg = (Lc + kSeg6 - 1) / kSeg6;
    __syncthreads();
    ld16(ckpt + (size_t)c * D * D, ri, c0, Qr);
    to_qb(sm, ri, c0, Qr);
    __syncthreads();
    for (int sg = 0; sg < nseg; ++sg) {          // in-chunk states
      const int s0 = sg * kSeg6, T = min(kSeg6, Lc - s0);
      copy4(sm.rec[0], grec + (size_t)(t0c + s0) * kRec6, T * kRec6 / 4, tid);
      __syncthreads();
      for (int tt = 0; tt < T; ++tt) {
        fwd_step(Qr, sm.rec[tt], c0);
        st16(qs + (size_t)(s0 + tt) * D * D, ri, c0, Qr);
      }
      __syncthreads();
    }
    float Qt[16];
    ld16(ckpt + (size_t)(c + 1) * D * D, ri, c0, Qt);
#pragma unroll
    for (int v = 0; v < 16; ++v) dQb[v] = 0.f;
    for (int sg = nseg - 1; sg >= 0; --sg) {
      const int s0 = sg * kSeg6, T = min(kSeg6, Lc - s0);
      if (nseg > 1) {
        __syncthreads();
        copy4(sm.rec[0], grec + (size_t)(t0c + s0) * kRec6, T * kRec6 / 4, tid);
        __syncthreads();
      }
      for (int sb_end = T; sb_end > 0; sb_end -= kSB6) {
        const int sb0 = max(0, sb_end - kSB6), nsb = sb_end - sb0;
        for (int idx = tid; idx < nsb * D; idx += kThr) {
          const int tt = idx / D, j = idx % D;
          const int64_t o = (tokbase + route_pos(r, t0c + s0 + sb0 + tt, A.H, A.W)) * C + ch0 + j;
          sm.sx[tt][j] = load_act(A.x, o, A.act_bf16);
          sm.sq[tt][j] = A.q[o];
          const float g = load_act(A.dy, o, A.act_bf16);
          sm.sdo[tt][j] = g;
          sm.sdy[tt][j] = A.scales[(size_t)r * C + ch0 + j] * g;
        }
        __syncthreads();
        for (int tt = warp; tt < nsb; tt += kW) {   // a = M0^T dy
          sm.sa[tt][lane] = dotc(sm.Mm, lane, sm.sdy[tt]);
          sm.sa[tt][32 + lane] = dotc(sm.Mm, 32 + lane, sm.sdy[tt]);
        }
        __syncthreads();
        // reverse chain (no block barrier inside); Q_{t-1} is fetched one token ahead
        float qn[16];
        {
          const int jl0 = s0 + sb0 + nsb - 1;
          if (jl0 == 0) from_qb(sm, ri, c0, qn);
          else ld16(qs + (size_t)(jl0 - 1) * D * D, ri, c0, qn);
        }
        for (int tt = nsb - 1; tt >= 0; --tt) {
          const int jl = s0 + sb0 + tt;
          float Qm[16];
#pragma unroll
          for (int v = 0; v < 16; ++v) Qm[v] = qn[v];
          if (tt > 0) {
            if (jl - 1 == 0) from_qb(sm, ri, c0, qn);
            else ld16(qs + (size_t)(jl - 2) * D * D, ri, c0, qn);
          }
          const float* rc = sm.rec[sb0 + tt];
          float k[16], u[16], q[16];
          vec16(rc + kRk, c0, k);
          vec16(rc + kRu, c0, u);
          vec16(sm.sq[tt], c0, q);
          const float al = rc[kRal], eta = rc[kReta];
          const float ai = sm.sa[tt][ri];
          float w0 = 0.f, w1 = 0.f, p0 = 0.f, p1 = 0.f, y0 = 0.f, y1 = 0.f, a0 = 0.f, a1 = 0.f;
#pragma unroll
          for (int v = 0; v < 16; v += 2) {
            dQ[v] = fmaf(ai, q[v], dQ[v]);
            dQ[v + 1] = fmaf(ai, q[v + 1], dQ[v + 1]);
            w0 = fmaf(dQ[v], k[v], w0); w1 = fmaf(dQ[v + 1], k[v + 1], w1);
            p0 = fmaf(Qm[v], u[v], p0); p1 = fmaf(Qm[v + 1], u[v + 1], p1);
            y0 = fmaf(Qt[v], q[v], y0); y1 = fmaf(Qt[v + 1], q[v + 1], y1);
            a0 = fmaf(Qm[v], dQ[v], a0); a1 = fmaf(Qm[v + 1], dQ[v + 1], a1);
          }
          const float w = row4(w0 + w1), pp = row4(p0 + p1), yq = row4(y0 + y1);
          const float ta = rows8(row4(a0 + a1));
          const float tn = rows8(pp * w);
          float cv[16];
          float cu0, cu1, ck0, ck1, cq0, cq1;
#pragma unroll
          for (int v = 0; v < 16; ++v) cv[v] = Qm[v] * w;
          col8(cv, lane, cu0, cu1);
#pragma unroll
          for (int v = 0; v < 16; ++v) cv[v] = dQ[v] * pp;
          col8(cv, lane, ck0, ck1);
#pragma unroll
          for (int v = 0; v < 16; ++v) cv[v] = Qt[v] * ai;
          col8(cv, lane, cq0, cq1);
          float* pt = sm.part[tt][warp];
          pt[2 + colA] = cu0; pt[3 + colA] = cu1;
          pt[2 + D + colA] = ck0; pt[3 + D + colA] = ck1;
          pt[2 + 2 * D + colA] = cq0; pt[3 + 2 * D + colA] = cq1;
          if (lane == 0) { pt[0] = ta; pt[1] = tn; }
          if ((tid & 3) == 0) sm.syq[tt][ri] = yq;
          const float ew = eta * w;
#pragma unroll
          for (int v = 0; v < 16; ++v) {
            dQ[v] = fmaf(al, dQ[v], -ew * u[v]);
            Qt[v] = Qm[v];
          }
        }
        __syncthreads();
        // per token, vector part (warp per token; lane covers j and 32 + j)
        for (int tt = warp; tt < nsb; tt += kW) {
          const int t = t0c + s0 + sb0 + tt;
          const float* rc = sm.rec[sb0 + tt];
          float ta = 0.f, pw = 0.f, du0 = 0.f, du1 = 0.f, dk0 = 0.f, dk1 = 0.f, dq0 = 0.f, dq1 = 0.f;
#pragma unroll
          for (int w8 = 0; w8 < kW; ++w8) {
            const float* pt = sm.part[tt][w8];
            ta += pt[0]; pw += pt[1];
            du0 += pt[2 + lane]; du1 += pt[2 + 32 + lane];
            dk0 += pt[2 + D + lane]; dk1 += pt[2 + D + 32 + lane];
            dq0 += pt[2 + 2 * D + lane]; dq1 += pt[2 + 2 * D + 32 + lane];
          }
          const float al = rc[kRal], eta = rc[kReta];
          const float ka = rc[kRk + lane], kb = rc[kRk + 32 + lane];
          const float va = (1.f + al) * ka - rc[kRu + lane], vb = (1.f + al) * kb - rc[kRu + 32 + lane];
          du0 *= -eta; du1 *= -eta;
          const float ea = ka - va, eb = kb - vb;
          const float kdu = warp_sum(ka * du0 + kb * du1);
          const float kn2 = warp_sum(ka * ka + kb * kb);
          const float ne2 = warp_sum(ea * ea + eb * eb);
          sm.sdg[tt][lane] = -eta * dk0 + (1.f + al) * du0;
          sm.sdg[tt][32 + lane] = -eta * dk1 + (1.f + al) * du1;
          sm.sdg[tt][D + lane] = -du0;
          sm.sdg[tt][D + 32 + lane] = -du1;
          if (lane == 0) { float* s = sm.sc[tt]; s[0] = ta + kdu; s[1] = -pw; s[2] = kn2; s[3] = ne2; }
          const int64_t o = ((int64_t)r * A.B * N + tokbase + route_pos(r, t, A.H, A.W)) * C + ch0;
          A.dqr[o + lane] = dq0;
          A.dqr[o + 32 + lane] = dq1;
        }
        __syncthreads();
        if (tid < nsb) {
          const float* rc = sm.rec[sb0 + tid];
          bwd::gate_backward_scalars_f(sm.sc[tid], rc[kRal], rc[kRa], rc[kRb], A.alpha, A.hard_cap);
        }
        __syncthreads();
        for (int tt = warp; tt < nsb; tt += kW) {
          const int t = t0c + s0 + sb0 + tt;
          const float* rc = sm.rec[sb0 + tt];
          const float* scv = sm.sc[tt];
          const float al = rc[kRal], s = rc[kRs];
          const float ka = rc[kRk + lane], kb = rc[kRk + 32 + lane];
          const float ea = ka - ((1.f + al) * ka - rc[kRu + lane]);
          const float eb = kb - ((1.f + al) * kb - rc[kRu + 32 + lane]);
          const float dka = sm.sdg[tt][lane] + scv[4] * ea + scv[5] * ka;
          const float dkb = sm.sdg[tt][32 + lane] + scv[4] * eb + scv[5] * kb;
          const float dva = sm.sdg[tt][D + lane] - scv[4] * ea;
          const float dvb = sm.sdg[tt][D + 32 + lane] - scv[4] * eb;
          const float kdk = warp_sum(ka * dka + kb * dkb);
          sm.sdg[tt][lane] = (dka - ka * kdk) / s;        // k = k~ / s
          sm.sdg[tt][32 + lane] = (dkb - kb * kdk) / s;
          sm.sdg[tt][D + lane] = dva;
          sm.sdg[tt][D + 32 + lane] = dvb;
          if (lane == 0) { sm.sdg[tt][2 * D] = scv[6]; sm.sdg[tt][2 * D + 1] = scv[7]; }
          __syncwarp();
          const float dha = dotv<kGt6>(sm.GmT[lane], sm.sdg[tt]), dhb = dotv<kGt6>(sm.GmT[32 + lane], sm.sdg[tt]);
          const float hwa = dotv<D>(sm.Qb[lane], sm.sx[tt]), hwb = dotv<D>(sm.Qb[32 + lane], sm.sx[tt]);
          const float ya = dotv<D>(sm.Mm[lane], sm.syq[tt]), yb = dotv<D>(sm.Mm[32 + lane], sm.syq[tt]);
          sm.sdh[tt][lane] = dha; sm.sdh[tt][32 + lane] = dhb;
          sm.sh[tt][lane] = hwa; sm.sh[tt][32 + lane] = hwb;
          sm.ds[warp][lane] += sm.sdo[tt][lane] * ya;
          sm.ds[warp][32 + lane] += sm.sdo[tt][32 + lane] * yb;
          __syncwarp();
          const float dxa = dotc(sm.Qb, lane, sm.sdh[tt]), dxb = dotc(sm.Qb, 32 + lane, sm.sdh[tt]);
          const int64_t o = ((int64_t)r * A.B * N + tokbase + route_pos(r, t, A.H, A.W)) * C + ch0;
          A.dxr[o + lane] = dxa;
          A.dxr[o + 32 + lane] = dxb;
        }
        __syncthreads();
        // rank-one sums: dM0, dQ_b and dG in this thread's layout
        for (int tt = 0; tt < nsb; ++tt) {
          float yq[16], xv[16], hv[16];
          vec16(sm.syq[tt], c0, yq);
          vec16(sm.sx[tt], c0, xv);
          vec16(sm.sh[tt], c0, hv);
          const float dyi = sm.sdy[tt][ri], dhi = sm.sdh[tt][ri];
          const float g0 = sm.sdg[tt][ri], g1 = sm.sdg[tt][D + ri], g2 = has_g2 ? sm.sdg[tt][2 * D + ri] : 0.f;
#pragma unroll
          for (int v = 0; v < 16; ++v) {
            dM0[v] = fmaf(dyi, yq[v], dM0[v]);
            dQb[v] = fmaf(dhi, xv[v], dQb[v]);
            dG[0][v] = fmaf(g0, hv[v], dG[0][v]);
            dG[1][v] = fmaf(g1, hv[v], dG[1][v]);
            dG[2][v] = fmaf(g2, hv[v], dG[2][v]);
          }
        }
        __syncthreads();
      }
    }
#pragma unroll
    for (int v = 0; v < 16; ++v) dQ[v] += dQb[v];
  }

  // ---------------- per-sequence parameter partials: dM0 [64][64], dG [130][64], ds [64]
  float* pp = A.parts + (size_t)seq * kSeqPart6;
  st16(pp, ri, c0, dM0);
  float* pg = pp + D * D;
  st16(pg, ri, c0, dG[0]);
  st16(pg, D + ri, c0, dG[1]);
  if (has_g2) st16(pg, 2 * D + ri, c0, dG[2]);
  __syncthreads();
  if (warp == 0) {
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < kW; ++w8) { s0 += sm.ds[w8][lane]; s1 += sm.ds[w8][32 + lane]; }
    pp[D * D + G6 * D + lane] = s0;
    pp[D * D + G6 * D + 32 + lane] = s1;
  }
}

}  // namespace

cudaError_t prepare_backward64_kernel() {
  return cudaFuncSetAttribute(srnl_scan_backward64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)sizeof(Smem6));
}

cudaError_t launch_backward_scan64(const ScanGeom& g, const ScanParamsDev& p, const void* x, const float* q,
                                   const void* dy, float* ws, const BwdLayout& l, cudaStream_t s) {
  Args6 A;
  A.x = x; A.q = q; A.dy = dy;
  A.dxr = ws + l.dxr; A.dqr = ws + l.dqr; A.parts = ws + l.parts; A.ckpt = ws + l.ckpt; A.qs = ws + l.qs;
  A.grec = ws + l.grec;
  A.G = p.G; A.Mm = p.Mm; A.scales = p.scales;
  A.B = g.B; A.H = g.H; A.W = g.W; A.C = g.C; A.heads = g.heads; A.Lrow = g.Lrow; A.Lcol = g.Lcol;
  A.max_chunks = l.max_chunks; A.Lmax = l.Lmax;
  A.alpha = g.alpha; A.eps = g.eps; A.act_bf16 = g.act_bf16; A.hard_cap = g.hard_cap;
  const int nseq = g.routes * g.B * g.heads;
  srnl_scan_backward64_kernel<<<nseq, kThr, sizeof(Smem6), s>>>(A);
  return cudaGetLastError();
}

}  // namespace srnl
