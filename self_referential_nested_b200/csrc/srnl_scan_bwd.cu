// Backward pass of the SRNL four-direction chunked scan (sm_100a), fp32.
//
// Method sources (web pages on VisionHOPE; no page prints an equation, and none prints a
// backward pass): "VisionHOPE: Visual Backbones as Self-Modifying Learning Systems"
// (summary of arXiv 2609.33325), write-rule, stability and 2D-maps paragraphs;
// "VisionHOPE Model Overview: Architecture, Benchmarks, and Practical Limits",
// "Four-Directional Scanning and Spatial Chunking"; "VisionHOPE" README, "SRNL and
// VisionHOPE operator" (the layer is trained end to end inside a backbone).
//
// The forward in single-product form (every memory is its initial state times one d x d
// product Q_t of the transitions T_t = alpha_t I - eta_t u_t k_t^T, u_t = (1 + alpha_t) k_t - v_t):
//   generation  w_t = Q_b x_t, [k~ v a beta]_t = G w_t       (Q_b: Q at the chunk start)
//   write       Q_t = Q_{t-1} T_t
//   readout     y_t = M0 Q_t q_t
// Reverse mode, with dQ = dL/dQ_t carried backwards through the tokens:
//   readout     dQ += a_t q_t^T,  a_t = M0^T dy_t,   dq_t = Q_t^T a_t,   dM0 += dy_t (Q_t q_t)^T
//   write       w = dQ k_t, p = Q_{t-1} u_t:
//               dalpha_t = <Q_{t-1}, dQ>,  deta_t = -p.w,
//               du_t = -eta_t Q_{t-1}^T w,  dk_t = -eta_t dQ^T p,
//               dQ <- alpha_t dQ - eta_t w u_t^T                 (= dL/dQ_{t-1})
//   gates       chain rule through u, the spectral clamp, the soft cap (or hard clamp), the
//               softplus, the retention clamp and the key normalisation -> dgen_t (66)
//   generation  dh_t = G^T dgen_t, dx_t = Q_b^T dh_t, dG += dgen_t w_t^T,
//               and dQ_b += sum_t dh_t x_t^T joins dQ at the chunk start.
//
// The chain dQ <- alpha dQ - eta (dQ k) u^T + a q^T acts on each row of dQ independently, so
// the eight warps of a CTA run it without a block barrier per token; the forward chain
// Q <- alpha Q - eta (Q u) k^T likewise.  One CTA owns one (route, batch, head) sequence:
//   phase 1  forward chain over all chunks, saving Q at every chunk boundary (checkpoints);
//   phase 2  chunks in reverse: recompute the chunk's gates and its Q_t (into an
//            L2-resident scratch), then the reverse chain in sub-blocks of kSB tokens,
//            each followed by the per-token gate backward and the rank-one parameter sums.
// Thread layout of the 32 x 32 matrices: thread (row i = tid / 8, columns 4 (tid % 8) .. +3);
// warp w owns rows 4w .. 4w + 3.
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

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kSeg = 32;        // tokens whose gate records sit in shared memory at once
constexpr int kSB = 16;         // tokens per reverse sub-block
constexpr int kLd = kD + 4;     // row stride of 32-wide matrices: 16-byte rows, conflict-free
                                //   float4 row reads and scalar column reads
constexpr int kGtLd = kGen + 2; // row stride of G^T (68 = 4 mod 32: conflict-free float4 rows)
constexpr int kRec = 72;        // per-token gate record: k[32] u[32] alpha eta s a beta |k|^2 |k-v|^2
constexpr int kRk = 0, kRu = 32, kRal = 64, kReta = 65, kRs = 66, kRa = 67, kRb = 68, kRkn2 = 69, kRne2 = 70;
constexpr int kPart = 2 + 3 * kD;   // per (token, warp): dalpha, p.w, du[32], dk[32], dq[32]
constexpr int kGenLd = kGen + 2;

struct BwdSmem {
  alignas(16) float Mm[kD][kLd];            // M_mem0 of this (route, head)
  alignas(16) float Gm[kGen][kLd];          // generating initials G
  alignas(16) float GmT[kD][kGtLd];         // G transposed (columns 66, 67 zero)
  alignas(16) float Qb[kD][kLd];            // Q at the current chunk start
  alignas(16) float rec[kSeg][kRec];        // gates of the current segment
  alignas(16) float wh[kWarps][kD];         // per-warp scratch of the gate pass
  alignas(16) float sx[kSB][kD];            // reverse sub-block: x, q, dout, dy (scaled), a = M0^T dy,
  alignas(16) float sq[kSB][kD];            //   Q_t q_t, dh, h = Q_b x, dgen
  alignas(16) float sdo[kSB][kD];
  alignas(16) float sdy[kSB][kD];
  alignas(16) float sa[kSB][kD];
  alignas(16) float syq[kSB][kD];
  alignas(16) float sdh[kSB][kD];
  alignas(16) float sh[kSB][kD];
  alignas(16) float sdg[kSB][kGenLd];
  alignas(16) float part[kSB][kWarps][kPart];
  alignas(16) float sc[kSB][8];             // per-token scalars of the gate backward
  alignas(16) float ds[kWarps][kD];
};
static_assert(sizeof(BwdSmem) <= 112 * 1024, "two CTAs per SM");
static_assert(offsetof(BwdSmem, sq) == offsetof(BwdSmem, sx) + sizeof(float) * kSB * kD && 2 * kSB >= kSeg,
              "the gate pass stages a segment's x over sx and sq");

struct BwdArgs {
  const void* x;       // [B][N][C] act dtype (C = heads * 32)
  const float* q;      // [B][N][C] fp32
  const void* dy;      // [B][N][C] act dtype (upstream gradient of the fused output)
  float* dxr;          // [routes][B][N][C] route partials of dL/dx (generation path)
  float* dqr;          // [routes][B][N][C] route partials of dL/dq
  float* parts;        // [nseq][kSeqPart] dM0, dG, dscale partials per sequence
  float* ckpt;         // [nseq][max_chunks + 1][32 * 32]
  float* qs;           // [nseq][Lmax][32 * 32]
  float* grec;         // [nseq][N][kRec] gate records of every token (written by phase 1)
  const float* G;
  const float* Mm;
  const float* scales;
  int B, H, W, C, heads, Lrow, Lcol, routes, max_chunks, Lmax;
  float alpha, eps;
  bool act_bf16, hard_cap;
};

__device__ __forceinline__ float row8_sum(float v) {   // sum over the 8 lanes of a matrix row
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  return v;
}

// Sum four column values over the warp's four rows (lanes l, l^8, l^16, l^24); the lane ends
// with column 4 (lane % 8) + 2 bit4(lane) + bit3(lane).
__device__ __forceinline__ float col4_sum(float c0, float c1, float c2, float c3, int lane) {
  const bool b4 = (lane >> 4) & 1, b3 = (lane >> 3) & 1;
  const float s0 = b4 ? c0 : c2, s1 = b4 ? c1 : c3;
  const float r0 = __shfl_xor_sync(0xffffffffu, s0, 16);
  const float r1 = __shfl_xor_sync(0xffffffffu, s1, 16);
  const float k0 = (b4 ? c2 : c0) + r0, k1 = (b4 ? c3 : c1) + r1;
  const float s = b3 ? k0 : k1;
  return (b3 ? k1 : k0) + __shfl_xor_sync(0xffffffffu, s, 8);
}

// Dot product of a 16-byte-aligned shared row with a shared vector that every lane reads
// (broadcast), n a multiple of 4; two accumulators.
template <int n>
__device__ __forceinline__ float dot_vec(const float* a, const float* b) {
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int i = 0; i < n; i += 4) {
    const float4 x = *reinterpret_cast<const float4*>(a + i);
    const float4 y = *reinterpret_cast<const float4*>(b + i);
    float& acc = ((i >> 2) & 1) ? s1 : s0;
    acc = fmaf(x.x, y.x, acc);
    acc = fmaf(x.y, y.y, acc);
    acc = fmaf(x.z, y.z, acc);
    acc = fmaf(x.w, y.w, acc);
  }
  return s0 + s1;
}

// Column j of a shared matrix (row stride kLd, scalar reads) against a broadcast vector.
__device__ __forceinline__ float dot_col(const float (*m)[kLd], int j, const float* b) {
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int i = 0; i < kD; i += 4) {
    const float4 y = *reinterpret_cast<const float4*>(b + i);
    float& acc = ((i >> 2) & 1) ? s1 : s0;
    acc = fmaf(m[i][j], y.x, acc);
    acc = fmaf(m[i + 1][j], y.y, acc);
    acc = fmaf(m[i + 2][j], y.z, acc);
    acc = fmaf(m[i + 3][j], y.w, acc);
  }
  return s0 + s1;
}

// Copy n4 float4 values (16-byte aligned both sides) with the whole block.
__device__ __forceinline__ void block_copy4(float* dst, const float* src, int n4, int tid) {
  for (int i = tid; i < n4; i += kThreads)
    reinterpret_cast<float4*>(dst)[i] = reinterpret_cast<const float4*>(src)[i];
}

// Gates of tokens [t0, t0 + T) of the sequence into sm.rec (T <= kSeg), by all threads:
// the segment's x staged block-wide (over sx and sq), generation and the vector reductions
// with a warp per token, the scalar gates with a lane per token, then u = (1 + alpha) k - v.
// Q_b in sm.Qb.  Ends with a block barrier.
__device__ void gates_segment(BwdSmem& sm, const BwdArgs& A, int r, int64_t tokbase_b, int ch0, int t0, int T,
                              int tid) {
  float (*xs)[kD] = reinterpret_cast<float (*)[kD]>(&sm.sx[0][0]);   // kSeg rows: sx then sq
  const int warp = tid >> 5, lane = tid & 31;
  for (int idx = tid; idx < T * kD; idx += kThreads) {
    const int tt = idx >> 5;
    const int p = route_pos(r, t0 + tt, A.H, A.W);
    xs[tt][lane] = load_act(A.x, (tokbase_b + p) * A.C + ch0 + lane, A.act_bf16);
  }
  __syncthreads();
  for (int tt = warp; tt < T; tt += kWarps) {
    sm.wh[warp][lane] = dot_vec<kD>(sm.Qb[lane], xs[tt]);                 // w = Q_b x
    __syncwarp();
    const float kt = dot_vec<kD>(sm.Gm[lane], sm.wh[warp]);               // k~
    const float vv = dot_vec<kD>(sm.Gm[kD + lane], sm.wh[warp]);          // v
    const float ex = dot_vec<kD>(sm.Gm[2 * kD + (lane & 1)], sm.wh[warp]);  // lanes 0/1: a / beta
    __syncwarp();
    const float s = sqrtf(warp_sum(kt * kt) + A.eps);
    const float k = kt / s;
    const float e = k - vv;
    const float kn2 = warp_sum(k * k);
    const float ne2 = warp_sum(e * e);
    float* rc = sm.rec[tt];
    rc[kRk + lane] = k;
    rc[kRu + lane] = vv;   // v until u is formed below
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
  for (int idx = tid; idx < T * kD; idx += kThreads) {
    float* rc = sm.rec[idx >> 5];
    rc[kRu + lane] = (1.f + rc[kRal]) * rc[kRk + lane] - rc[kRu + lane];
  }
  __syncthreads();
}

__device__ __forceinline__ void load_row4(const float* m, int i, int j0, float (&v)[4]) {
  const float4 f = *reinterpret_cast<const float4*>(m + i * kD + j0);
  v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}
__device__ __forceinline__ void store_row4(float* m, int i, int j0, const float (&v)[4]) {
  *reinterpret_cast<float4*>(m + i * kD + j0) = make_float4(v[0], v[1], v[2], v[3]);
}

// One forward write on this thread's 4 entries of Q: Q <- alpha Q - eta (Q u) k^T.
__device__ __forceinline__ void forward_step(float (&Qr)[4], const float* rec, int j0) {
  const float4 u = *reinterpret_cast<const float4*>(rec + kRu + j0);
  const float4 k = *reinterpret_cast<const float4*>(rec + kRk + j0);
  const float al = rec[kRal], eta = rec[kReta];
  float pr = Qr[0] * u.x;
  pr = fmaf(Qr[1], u.y, pr);
  pr = fmaf(Qr[2], u.z, pr);
  pr = fmaf(Qr[3], u.w, pr);
  const float ep = eta * row8_sum(pr);
  Qr[0] = fmaf(al, Qr[0], -ep * k.x);
  Qr[1] = fmaf(al, Qr[1], -ep * k.y);
  Qr[2] = fmaf(al, Qr[2], -ep * k.z);
  Qr[3] = fmaf(al, Qr[3], -ep * k.w);
}

__global__ void __launch_bounds__(kThreads, 2) srnl_scan_backward_kernel(const BwdArgs A) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  BwdSmem& sm = *reinterpret_cast<BwdSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ri = tid >> 3;            // matrix row owned
  const int j0 = (tid & 7) * 4;       // first of the four columns owned
  const int seq = blockIdx.x;
  const int hh = seq % A.heads;
  const int b = (seq / A.heads) % A.B;
  const int r = seq / (A.heads * A.B);
  const int N = A.H * A.W;
  const int L = (r < 2) ? A.Lrow : A.Lcol;
  const int nc = (N + L - 1) / L;
  const int C = A.C, ch0 = hh * kD;
  const int64_t tokbase_b = (int64_t)b * N;
  const int rh = r * A.heads + hh;
  float* ckpt = A.ckpt + (size_t)seq * (A.max_chunks + 1) * (kD * kD);
  float* qs = A.qs + (size_t)seq * A.Lmax * (kD * kD);

  for (int idx = tid; idx < kD * kD; idx += kThreads) sm.Mm[idx / kD][idx % kD] = A.Mm[(size_t)rh * kD * kD + idx];
  for (int idx = tid; idx < kGen * kD; idx += kThreads) {
    const float gv = A.G[(size_t)rh * kGen * kD + idx];
    sm.Gm[idx / kD][idx % kD] = gv;
    sm.GmT[idx % kD][idx / kD] = gv;
  }
  if (tid < kD) { sm.GmT[tid][kGen] = 0.f; sm.GmT[tid][kGen + 1] = 0.f; }
  if (tid < kSB) { sm.sdg[tid][kGen] = 0.f; sm.sdg[tid][kGen + 1] = 0.f; }
  float* grec = A.grec + (size_t)seq * N * kRec;
  for (int idx = tid; idx < kWarps * kD; idx += kThreads) sm.ds[idx / kD][idx % kD] = 0.f;

  // ---------------- phase 1: forward chain, checkpoints at chunk starts
  float Qr[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) Qr[c] = (ri == j0 + c) ? 1.f : 0.f;
  for (int c = 0; c < nc; ++c) {
    store_row4(ckpt + (size_t)c * kD * kD, ri, j0, Qr);
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) sm.Qb[ri][j0 + cc] = Qr[cc];
    __syncthreads();
    const int c0 = c * L, Lc = min(L, N - c0);
    for (int s0 = 0; s0 < Lc; s0 += kSeg) {
      const int T = min(kSeg, Lc - s0);
      gates_segment(sm, A, r, tokbase_b, ch0, c0 + s0, T, tid);
      block_copy4(grec + (size_t)(c0 + s0) * kRec, sm.rec[0], T * kRec / 4, tid);
      for (int tt = 0; tt < T; ++tt) forward_step(Qr, sm.rec[tt], j0);
      __syncthreads();
    }
  }
  store_row4(ckpt + (size_t)nc * kD * kD, ri, j0, Qr);

  // ---------------- phase 2: chunks in reverse
  float dQ[4] = {0.f, 0.f, 0.f, 0.f}, dM0[4] = {0.f, 0.f, 0.f, 0.f}, dQb[4];
  float dG[3][4];
#pragma unroll
  for (int g = 0; g < 3; ++g)
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) dG[g][cc] = 0.f;
  const int gr2 = 2 * kD + ri;            // third dG row of this thread (rows 64, 65 only)
  const bool has_g2 = ri < 2;
  const float scale_l = A.scales[(size_t)r * C + ch0 + lane];

  for (int c = nc - 1; c >= 0; --c) {
    const int c0 = c * L, Lc = min(L, N - c0);
    const int nseg = (Lc + kSeg - 1) / kSeg;
    __syncthreads();
    load_row4(ckpt + (size_t)c * kD * kD, ri, j0, Qr);
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) sm.Qb[ri][j0 + cc] = Qr[cc];
    __syncthreads();
    // forward recompute of Q_t inside the chunk
    for (int sg = 0; sg < nseg; ++sg) {
      const int s0 = sg * kSeg, T = min(kSeg, Lc - s0);
      block_copy4(sm.rec[0], grec + (size_t)(c0 + s0) * kRec, T * kRec / 4, tid);
      __syncthreads();
      for (int tt = 0; tt < T; ++tt) {
        forward_step(Qr, sm.rec[tt], j0);
        store_row4(qs + (size_t)(s0 + tt) * kD * kD, ri, j0, Qr);
      }
      __syncthreads();
    }
    // reverse
    float Qt[4];
    load_row4(ckpt + (size_t)(c + 1) * kD * kD, ri, j0, Qt);
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) dQb[cc] = 0.f;
    for (int sg = nseg - 1; sg >= 0; --sg) {
      const int s0 = sg * kSeg, T = min(kSeg, Lc - s0);
      if (nseg > 1) {
        __syncthreads();
        block_copy4(sm.rec[0], grec + (size_t)(c0 + s0) * kRec, T * kRec / 4, tid);
        __syncthreads();
      }
      for (int sb_end = T; sb_end > 0; sb_end -= kSB) {
        const int sb0 = max(0, sb_end - kSB), nsb = sb_end - sb0;
        // stage x, q, dout, dy = scale * dout and a = M0^T dy (warp per token)
        for (int idx = tid; idx < nsb * kD; idx += kThreads) {
          const int tt = idx >> 5;
          const int t = c0 + s0 + sb0 + tt;
          const int64_t o = (tokbase_b + route_pos(r, t, A.H, A.W)) * C + ch0 + lane;
          sm.sx[tt][lane] = load_act(A.x, o, A.act_bf16);
          sm.sq[tt][lane] = A.q[o];
          const float g = load_act(A.dy, o, A.act_bf16);
          sm.sdo[tt][lane] = g;
          sm.sdy[tt][lane] = scale_l * g;
        }
        __syncthreads();
        for (int tt = warp; tt < nsb; tt += kWarps) sm.sa[tt][lane] = dot_col(sm.Mm, lane, sm.sdy[tt]);  // M0^T dy
        __syncthreads();
        // reverse chain over the sub-block (no block barrier inside)
        {
          float qn[4];
          const int jl0 = s0 + sb0 + nsb - 1;   // chunk-local index of the sub-block's last token
          if (jl0 == 0) {
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) qn[cc] = sm.Qb[ri][j0 + cc];
          } else {
            load_row4(qs + (size_t)(jl0 - 1) * kD * kD, ri, j0, qn);
          }
          for (int tt = nsb - 1; tt >= 0; --tt) {
            const int jl = s0 + sb0 + tt;        // chunk-local token index
            float Qm[4] = {qn[0], qn[1], qn[2], qn[3]};
            if (tt > 0) {                        // prefetch Q_{t-2} for the next token
              if (jl - 1 == 0) {
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) qn[cc] = sm.Qb[ri][j0 + cc];
              } else {
                load_row4(qs + (size_t)(jl - 2) * kD * kD, ri, j0, qn);
              }
            }
            const float* rc = sm.rec[sb0 + tt];
            const float4 k4 = *reinterpret_cast<const float4*>(rc + kRk + j0);
            const float4 u4 = *reinterpret_cast<const float4*>(rc + kRu + j0);
            const float4 q4 = *reinterpret_cast<const float4*>(&sm.sq[tt][j0]);
            const float al = rc[kRal], eta = rc[kReta];
            const float ai = sm.sa[tt][ri];
            dQ[0] = fmaf(ai, q4.x, dQ[0]);
            dQ[1] = fmaf(ai, q4.y, dQ[1]);
            dQ[2] = fmaf(ai, q4.z, dQ[2]);
            dQ[3] = fmaf(ai, q4.w, dQ[3]);
            float w = dQ[0] * k4.x, pp = Qm[0] * u4.x, yq = Qt[0] * q4.x, ta = Qm[0] * dQ[0];
            w = fmaf(dQ[1], k4.y, w); pp = fmaf(Qm[1], u4.y, pp); yq = fmaf(Qt[1], q4.y, yq); ta = fmaf(Qm[1], dQ[1], ta);
            w = fmaf(dQ[2], k4.z, w); pp = fmaf(Qm[2], u4.z, pp); yq = fmaf(Qt[2], q4.z, yq); ta = fmaf(Qm[2], dQ[2], ta);
            w = fmaf(dQ[3], k4.w, w); pp = fmaf(Qm[3], u4.w, pp); yq = fmaf(Qt[3], q4.w, yq); ta = fmaf(Qm[3], dQ[3], ta);
            w = row8_sum(w);
            pp = row8_sum(pp);
            yq = row8_sum(yq);
            ta = row8_sum(ta);
            float tn = pp * w;
            ta += __shfl_xor_sync(0xffffffffu, ta, 8);
            tn += __shfl_xor_sync(0xffffffffu, tn, 8);
            ta += __shfl_xor_sync(0xffffffffu, ta, 16);
            tn += __shfl_xor_sync(0xffffffffu, tn, 16);
            const float cu = col4_sum(Qm[0] * w, Qm[1] * w, Qm[2] * w, Qm[3] * w, lane);
            const float ck = col4_sum(dQ[0] * pp, dQ[1] * pp, dQ[2] * pp, dQ[3] * pp, lane);
            const float cq = col4_sum(Qt[0] * ai, Qt[1] * ai, Qt[2] * ai, Qt[3] * ai, lane);
            float* pt = sm.part[tt][warp];
            const int col = j0 + ((lane >> 4) & 1) * 2 + ((lane >> 3) & 1);
            pt[2 + col] = cu;
            pt[2 + kD + col] = ck;
            pt[2 + 2 * kD + col] = cq;
            if (lane == 0) { pt[0] = ta; pt[1] = tn; }
            if ((tid & 7) == 0) sm.syq[tt][ri] = yq;
            const float ew = eta * w;
            dQ[0] = fmaf(al, dQ[0], -ew * u4.x);
            dQ[1] = fmaf(al, dQ[1], -ew * u4.y);
            dQ[2] = fmaf(al, dQ[2], -ew * u4.z);
            dQ[3] = fmaf(al, dQ[3], -ew * u4.w);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) Qt[cc] = Qm[cc];
          }
        }
        __syncthreads();
        // per token, vector part (warp per token): partial sums over the warps, the write's
        // gradients of k and v, and the reductions the scalar gate backward needs
        for (int tt = warp; tt < nsb; tt += kWarps) {
          const int t = c0 + s0 + sb0 + tt;
          const float* rc = sm.rec[sb0 + tt];
          float ta = 0.f, pw = 0.f, du = 0.f, dkT = 0.f, dq = 0.f;
#pragma unroll
          for (int w8 = 0; w8 < kWarps; ++w8) {
            const float* pt = sm.part[tt][w8];
            ta += pt[0];
            pw += pt[1];
            du += pt[2 + lane];
            dkT += pt[2 + kD + lane];
            dq += pt[2 + 2 * kD + lane];
          }
          const float al = rc[kRal], eta = rc[kReta];
          const float k = rc[kRk + lane];
          const float v = (1.f + al) * k - rc[kRu + lane];
          du *= -eta;                                  // du = -eta Q_{t-1}^T w
          const float e = k - v;
          const float kdu = warp_sum(k * du);          // u = (1 + alpha) k - v
          const float kn2 = warp_sum(k * k);
          const float ne2 = warp_sum(e * e);
          sm.sdg[tt][lane] = -eta * dkT + (1.f + al) * du;
          sm.sdg[tt][kD + lane] = -du;
          if (lane == 0) {
            float* sc = sm.sc[tt];
            sc[0] = ta + kdu;
            sc[1] = -pw;
            sc[2] = kn2;
            sc[3] = ne2;
          }
          A.dqr[((int64_t)r * A.B * N + tokbase_b + route_pos(r, t, A.H, A.W)) * C + ch0 + lane] = dq;
        }
        __syncthreads();
        if (tid < nsb) {   // lane per token
          const float* rc = sm.rec[sb0 + tid];
          bwd::gate_backward_scalars_f(sm.sc[tid], rc[kRal], rc[kRa], rc[kRb], A.alpha, A.hard_cap);
        }
        __syncthreads();
        // per token, the rest (warp per token): dk~, then the generation and readout adjoints
        for (int tt = warp; tt < nsb; tt += kWarps) {
          const int t = c0 + s0 + sb0 + tt;
          const float* rc = sm.rec[sb0 + tt];
          const float* sc = sm.sc[tt];
          const float al = rc[kRal], s = rc[kRs];
          const float k = rc[kRk + lane];
          const float e = k - ((1.f + al) * k - rc[kRu + lane]);
          const float dk = sm.sdg[tt][lane] + sc[4] * e + sc[5] * k;
          const float dv = sm.sdg[tt][kD + lane] - sc[4] * e;
          sm.sdg[tt][lane] = (dk - k * warp_sum(k * dk)) / s;   // k = k~ / s
          sm.sdg[tt][kD + lane] = dv;
          if (lane == 0) { sm.sdg[tt][2 * kD] = sc[6]; sm.sdg[tt][2 * kD + 1] = sc[7]; }
          __syncwarp();
          const float dh = dot_vec<kGtLd>(sm.GmT[lane], sm.sdg[tt]);   // (G^T dgen)_lane
          const float hw = dot_vec<kD>(sm.Qb[lane], sm.sx[tt]);         // (Q_b x)_lane
          const float y = dot_vec<kD>(sm.Mm[lane], sm.syq[tt]);         // (M0 Q_t q)_lane
          sm.sdh[tt][lane] = dh;
          sm.sh[tt][lane] = hw;
          sm.ds[warp][lane] += sm.sdo[tt][lane] * y;
          __syncwarp();
          const float dx = dot_col(sm.Qb, lane, sm.sdh[tt]);             // (Q_b^T dh)_lane
          A.dxr[((int64_t)r * A.B * N + tokbase_b + route_pos(r, t, A.H, A.W)) * C + ch0 + lane] = dx;
        }
        __syncthreads();
        // rank-one sums of the sub-block: dM0, dQ_b and dG in this thread's layout
        for (int tt = 0; tt < nsb; ++tt) {
          const float4 yq4 = *reinterpret_cast<const float4*>(&sm.syq[tt][j0]);
          const float4 x4 = *reinterpret_cast<const float4*>(&sm.sx[tt][j0]);
          const float4 h4 = *reinterpret_cast<const float4*>(&sm.sh[tt][j0]);
          const float dyi = sm.sdy[tt][ri], dhi = sm.sdh[tt][ri];
          dM0[0] = fmaf(dyi, yq4.x, dM0[0]); dM0[1] = fmaf(dyi, yq4.y, dM0[1]);
          dM0[2] = fmaf(dyi, yq4.z, dM0[2]); dM0[3] = fmaf(dyi, yq4.w, dM0[3]);
          dQb[0] = fmaf(dhi, x4.x, dQb[0]); dQb[1] = fmaf(dhi, x4.y, dQb[1]);
          dQb[2] = fmaf(dhi, x4.z, dQb[2]); dQb[3] = fmaf(dhi, x4.w, dQb[3]);
          const float g0 = sm.sdg[tt][ri], g1 = sm.sdg[tt][kD + ri], g2 = has_g2 ? sm.sdg[tt][gr2] : 0.f;
          dG[0][0] = fmaf(g0, h4.x, dG[0][0]); dG[0][1] = fmaf(g0, h4.y, dG[0][1]);
          dG[0][2] = fmaf(g0, h4.z, dG[0][2]); dG[0][3] = fmaf(g0, h4.w, dG[0][3]);
          dG[1][0] = fmaf(g1, h4.x, dG[1][0]); dG[1][1] = fmaf(g1, h4.y, dG[1][1]);
          dG[1][2] = fmaf(g1, h4.z, dG[1][2]); dG[1][3] = fmaf(g1, h4.w, dG[1][3]);
          dG[2][0] = fmaf(g2, h4.x, dG[2][0]); dG[2][1] = fmaf(g2, h4.y, dG[2][1]);
          dG[2][2] = fmaf(g2, h4.z, dG[2][2]); dG[2][3] = fmaf(g2, h4.w, dG[2][3]);
        }
        __syncthreads();
      }
    }
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) dQ[cc] += dQb[cc];
  }

  // ---------------- per-sequence parameter partials
  float* pp = A.parts + (size_t)seq * kSeqPart;
  store_row4(pp, ri, j0, dM0);
  float* pg = pp + kD * kD;
  store_row4(pg, ri, j0, dG[0]);
  store_row4(pg, kD + ri, j0, dG[1]);
  if (has_g2) store_row4(pg, gr2, j0, dG[2]);
  __syncthreads();
  if (warp == 0) {
    float s = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < kWarps; ++w8) s += sm.ds[w8][lane];
    pp[kD * kD + kGen * kD + lane] = s;
  }
}

// ---------------------------------------------------------------- combine kernels
// dq[p][c] = sum_r dqr[r][p][c]  (route order r = 0..3)
__global__ void sum_routes_kernel(const float* __restrict__ src, float* __restrict__ dst, int64_t n4, int routes) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 acc = reinterpret_cast<const float4*>(src)[i];
    for (int r = 1; r < routes; ++r) {
      const float4 v = reinterpret_cast<const float4*>(src)[(int64_t)r * n4 + i];
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    reinterpret_cast<float4*>(dst)[i] = acc;
  }
}

// dx[p][c] = sum_r dxr[r][p][c] + sum_o dq[p][o] W_q[o][c]: a 64 x 64 output tile per block,
// 256 threads with 4 x 4 outputs each, K in steps of 32.
constexpr int kGT = 64, kGK = 32;
__global__ void __launch_bounds__(256) dx_gemm_kernel(const float* __restrict__ dq, const float* __restrict__ Wq,
                                                      const float* __restrict__ dxr, void* dx, int64_t M, int C,
                                                      int routes, bool out_bf16) {
  __shared__ float As[kGK][kGT + 4];   // As[k][m] = dq[m0 + m][k0 + k]
  __shared__ float Bs[kGK][kGT + 4];   // Bs[k][n] = Wq[k0 + k][n0 + n]
  const int tid = threadIdx.x, tm = tid >> 4, tn = tid & 15;
  const int64_t m0 = (int64_t)blockIdx.x * kGT;
  const int n0 = blockIdx.y * kGT;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < C; k0 += kGK) {
    for (int idx = tid; idx < kGT * kGK; idx += 256) {
      const int m = idx / kGK, k = idx % kGK;
      As[k][m] = (m0 + m < M) ? dq[(m0 + m) * C + k0 + k] : 0.f;
      const int kb = idx / kGT, nb = idx % kGT;
      Bs[kb][nb] = (n0 + nb < C) ? Wq[(int64_t)(k0 + kb) * C + n0 + nb] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kGK; ++k) {
      float a[4], bb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[k][tm * 4 + i]; bb[i] = Bs[k][tn * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
    __syncthreads();
  }
  const int64_t MC = M * C;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + tm * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tn * 4 + j;
      if (n >= C) continue;
      float v = 0.f;
      for (int r = 0; r < routes; ++r) v += dxr[(int64_t)r * MC + m * C + n];
      v += acc[i][j];
      if (out_bf16) reinterpret_cast<__nv_bfloat16*>(dx)[m * C + n] = __float2bfloat16_rn(v);
      else reinterpret_cast<float*>(dx)[m * C + n] = v;
    }
  }
}

// Split-K partials of dW_q[o][c] = sum_p dq[p][o] x[p][c]: block (tile, split) sums tokens
// [split * per, (split + 1) * per).
__global__ void __launch_bounds__(256) dwq_partial_kernel(const float* __restrict__ dq, const void* x, bool x_bf16,
                                                          float* __restrict__ part, int64_t M, int C, int64_t per) {
  __shared__ float As[kGK][kGT + 4];   // As[p][o]
  __shared__ float Bs[kGK][kGT + 4];   // Bs[p][c]
  const int tid = threadIdx.x, tm = tid >> 4, tn = tid & 15;
  const int tiles_n = (C + kGT - 1) / kGT;
  const int o0 = (blockIdx.x / tiles_n) * kGT, c0 = (blockIdx.x % tiles_n) * kGT;
  const int64_t p_begin = (int64_t)blockIdx.y * per;
  const int64_t p_end = p_begin + per < M ? p_begin + per : M;
  float acc[4][4] = {};
  for (int64_t pk = p_begin; pk < p_end; pk += kGK) {
    for (int idx = tid; idx < kGT * kGK; idx += 256) {
      const int kk = idx / kGT, n = idx % kGT;
      const int64_t p = pk + kk;
      const bool okp = p < p_end;
      As[kk][n] = (okp && o0 + n < C) ? dq[p * C + o0 + n] : 0.f;
      float xv = 0.f;
      if (okp && c0 + n < C) xv = load_act(x, p * C + c0 + n, x_bf16);
      Bs[kk][n] = xv;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kGK; ++k) {
      float a[4], bb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[k][tm * 4 + i]; bb[i] = Bs[k][tn * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* dst = part + (size_t)blockIdx.y * C * C;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int o = o0 + tm * 4 + i;
    if (o >= C) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = c0 + tn * 4 + j;
      if (c < C) dst[(size_t)o * C + c] = acc[i][j];
    }
  }
}

// Sum the split-K partials in split order and unpad to the caller's [C][C].
__global__ void dwq_reduce_kernel(const float* __restrict__ part, int nsplit, int Cp, int heads, int ud, int hd,
                                  float* __restrict__ out) {
  const int Cu = heads * ud;
  const int64_t n = (int64_t)Cu * Cu;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int o = (int)(i / Cu), c = (int)(i % Cu);
    const int op = (o / ud) * hd + o % ud, cp = (c / ud) * hd + c % ud;
    float s = 0.f;
    for (int k = 0; k < nsplit; ++k) s += part[(size_t)k * Cp * Cp + (size_t)op * Cp + cp];
    out[i] = s;
  }
}

// Sum the per-sequence partials over the batch (in batch order) and unpad: one thread per
// output element of dM_mem0, dM_k0, dM_v0, dm_eta0, dm_alpha0 and dscales.  A sequence's partials
// (stride seq_part) are dM0 [hd][hd], dG [2 hd + 2][hd] (M_k, M_v, m_eta, m_alpha rows) and ds [hd].
__global__ void param_reduce_kernel(const float* __restrict__ parts, int routes, int B, int heads, int ud, int hd,
                                    size_t seq_part, BwdGrads out) {
  const int nm = ud * ud;
  const int per_rh = 3 * nm + 2 * ud + ud;      // M_mem, M_k, M_v, m_eta, m_alpha, scales
  const int64_t total = (int64_t)routes * heads * per_rh;
  const int hh2 = hd * hd;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int rh = (int)(i / per_rh), e = (int)(i % per_rh);
    const int r = rh / heads, hh = rh % heads;
    int src;      // offset inside a sequence's partial block
    float* dst;
    if (e < nm) { src = (e / ud) * hd + e % ud; dst = out.M_mem0 ? out.M_mem0 + (size_t)rh * nm + e : nullptr; }
    else if (e < 2 * nm) { const int f = e - nm; src = hh2 + (f / ud) * hd + f % ud;
      dst = out.M_k0 ? out.M_k0 + (size_t)rh * nm + f : nullptr; }
    else if (e < 3 * nm) { const int f = e - 2 * nm; src = hh2 + (hd + f / ud) * hd + f % ud;
      dst = out.M_v0 ? out.M_v0 + (size_t)rh * nm + f : nullptr; }
    else if (e < 3 * nm + ud) { const int f = e - 3 * nm; src = hh2 + 2 * hh2 + f;
      dst = out.m_eta0 ? out.m_eta0 + (size_t)rh * ud + f : nullptr; }
    else if (e < 3 * nm + 2 * ud) { const int f = e - 3 * nm - ud; src = hh2 + 2 * hh2 + hd + f;
      dst = out.m_alpha0 ? out.m_alpha0 + (size_t)rh * ud + f : nullptr; }
    else { const int f = e - 3 * nm - 2 * ud; src = hh2 + (2 * hd + 2) * hd + f;
      dst = out.scales ? out.scales + (size_t)r * heads * ud + hh * ud + f : nullptr; }
    if (dst == nullptr) continue;
    float s = 0.f;
    for (int b = 0; b < B; ++b) s += parts[((size_t)(r * B + b) * heads + hh) * seq_part + src];
    *dst = s;
  }
}

// Sequence layer: dx = dxr (+ dqr when x is also the query), dq = dqr, in the act dtype.
__global__ void seq_combine_kernel(const float* __restrict__ dxr, const float* __restrict__ dqr, void* dx, void* dq,
                                   int64_t n, bool add_q, bool bf16) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float gq = dqr[i];
    const float gx = dxr[i] + (add_q ? gq : 0.f);
    if (bf16) {
      reinterpret_cast<__nv_bfloat16*>(dx)[i] = __float2bfloat16_rn(gx);
      if (dq != nullptr) reinterpret_cast<__nv_bfloat16*>(dq)[i] = __float2bfloat16_rn(gq);
    } else {
      reinterpret_cast<float*>(dx)[i] = gx;
      if (dq != nullptr) reinterpret_cast<float*>(dq)[i] = gq;
    }
  }
}

}  // namespace

size_t backward_workspace_floats(const ScanGeom& g, BwdLayout* lay) {
  const int N = g.H * g.W;
  const int nseq = g.routes * g.B * g.heads;
  const int hd = g.hd;
  const size_t hd2 = (size_t)hd * hd;
  int maxc = 0, Lmax = 0;
  for (int r = 0; r < g.routes; ++r) {
    const int L = r < 2 ? g.Lrow : g.Lcol;
    maxc = max(maxc, (N + L - 1) / L);
    Lmax = max(Lmax, min(L, N));
  }
  const size_t act = (size_t)g.B * N * g.C;
  BwdLayout l;
  l.max_chunks = maxc;
  l.Lmax = Lmax;
  l.hd = hd;
  l.rec = 2 * hd + 8;
  l.seq_part = hd2 + (size_t)(2 * hd + 2) * hd + hd;
  const int tiles = ((g.C + kGT - 1) / kGT) * ((g.C + kGT - 1) / kGT);
  const int64_t M = (int64_t)g.B * N;
  l.nsplit = (int)std::min<int64_t>(std::max<int64_t>(1, 296 / tiles), (M + kGK - 1) / kGK);
  size_t off = 0;
  l.dxr = off;  off += (size_t)g.routes * act;
  l.dqr = off;  off += (size_t)g.routes * act;
  l.dq = off;   off += act;
  l.parts = off; off += (size_t)nseq * l.seq_part;
  l.ckpt = off; off += (size_t)nseq * (maxc + 1) * hd2;
  l.qs = off;   off += (size_t)nseq * Lmax * hd2;
  l.grec = off; off += (size_t)nseq * N * l.rec;
  l.dwq = off;  off += (size_t)l.nsplit * g.C * g.C;
  l.total = off;
  if (lay) *lay = l;
  return off;
}

cudaError_t prepare_backward_kernel() {
  return cudaFuncSetAttribute(srnl_scan_backward_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)sizeof(BwdSmem));
}

static BwdArgs backward_args(const ScanGeom& g, const ScanParamsDev& p, const void* x, const float* q,
                             const void* dy, float* ws, const BwdLayout& l) {
  BwdArgs A;
  A.x = x; A.q = q; A.dy = dy;
  A.dxr = ws + l.dxr; A.dqr = ws + l.dqr; A.parts = ws + l.parts; A.ckpt = ws + l.ckpt; A.qs = ws + l.qs;
  A.grec = ws + l.grec;
  A.G = p.G; A.Mm = p.Mm; A.scales = p.scales;
  A.B = g.B; A.H = g.H; A.W = g.W; A.C = g.C; A.heads = g.heads; A.Lrow = g.Lrow; A.Lcol = g.Lcol;
  A.routes = g.routes; A.max_chunks = l.max_chunks; A.Lmax = l.Lmax;
  A.alpha = g.alpha; A.eps = g.eps; A.act_bf16 = g.act_bf16; A.hard_cap = g.hard_cap;
  return A;
}

cudaError_t launch_backward_scan(const ScanGeom& g, const ScanParamsDev& p, const void* x, const float* q,
                                 const void* dy, float* ws, cudaStream_t s) {
  BwdLayout l;
  backward_workspace_floats(g, &l);
  if (g.hd == 64) return launch_backward_scan64(g, p, x, q, dy, ws, l, s);
  const BwdArgs A = backward_args(g, p, x, q, dy, ws, l);
  const int nseq = g.routes * g.B * g.heads;
  srnl_scan_backward_kernel<<<nseq, kThreads, sizeof(BwdSmem), s>>>(A);
  return cudaGetLastError();
}

cudaError_t launch_backward_combine(const ScanGeom& g, const ScanParamsDev& p, int ud, const void* x, float* ws,
                                    void* dx, const BwdGrads& out, float* dwq_out, cudaStream_t s) {
  BwdLayout l;
  backward_workspace_floats(g, &l);
  const int N = g.H * g.W;
  const int64_t M = (int64_t)g.B * N;
  const int64_t n4 = M * g.C / 4;
  cudaError_t e;
  sum_routes_kernel<<<(unsigned)std::min<int64_t>((n4 + 255) / 256, 148 * 16), 256, 0, s>>>(ws + l.dqr, ws + l.dq, n4,
                                                                                           g.routes);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  dim3 gx((unsigned)((M + kGT - 1) / kGT), (unsigned)((g.C + kGT - 1) / kGT));
  dx_gemm_kernel<<<gx, 256, 0, s>>>(ws + l.dq, p.Wq, ws + l.dxr, dx, M, g.C, g.routes, g.act_bf16);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (dwq_out != nullptr) {
    const int tiles = ((g.C + kGT - 1) / kGT) * ((g.C + kGT - 1) / kGT);
    int64_t per = (M + l.nsplit - 1) / l.nsplit;
    per = (per + kGK - 1) / kGK * kGK;
    dwq_partial_kernel<<<dim3(tiles, l.nsplit), 256, 0, s>>>(ws + l.dq, x, g.act_bf16, ws + l.dwq, M, g.C, per);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t nout = (int64_t)g.heads * ud * g.heads * ud;
    dwq_reduce_kernel<<<(unsigned)std::min<int64_t>((nout + 255) / 256, 4096), 256, 0, s>>>(
        ws + l.dwq, l.nsplit, g.C, g.heads, ud, l.hd, dwq_out);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const int64_t nparam = (int64_t)g.routes * g.heads * (3 * ud * ud + 3 * ud);
  param_reduce_kernel<<<(unsigned)std::min<int64_t>((nparam + 255) / 256, 4096), 256, 0, s>>>(
      ws + l.parts, g.routes, g.B, g.heads, ud, l.hd, l.seq_part, out);
  return cudaGetLastError();
}

cudaError_t launch_backward_seq_combine(const ScanGeom& g, int ud, float* ws, void* dx, void* dq, bool add_q,
                                        const BwdGrads& out, cudaStream_t s) {
  BwdLayout l;
  backward_workspace_floats(g, &l);
  const int64_t n = (int64_t)g.B * g.H * g.W * g.C;
  seq_combine_kernel<<<(unsigned)std::min<int64_t>((n + 255) / 256, 148 * 16), 256, 0, s>>>(
      ws + l.dxr, ws + l.dqr, dx, dq, n, add_q, g.act_bf16);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t nparam = (int64_t)g.routes * g.heads * (3 * ud * ud + 3 * ud);
  param_reduce_kernel<<<(unsigned)std::min<int64_t>((nparam + 255) / 256, 4096), 256, 0, s>>>(
      ws + l.parts, g.routes, g.B, g.heads, ud, l.hd, l.seq_part, out);
  return cudaGetLastError();
}

}  // namespace srnl
