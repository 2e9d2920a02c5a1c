// SRNL four-direction chunked scan, fp32-generation path (sm_100a): the token-order
// write one token at a time.
//
// Method sources (web pages on VisionHOPE; no page prints an equation):
//   "VisionHOPE: Visual Backbones as Self-Modifying Learning Systems" (summary
//   of arXiv 2609.33325) - write-rule, stability and 2D-maps paragraphs;
//   "VisionHOPE Model Overview: Architecture, Benchmarks, and Practical
//   Limits" - "Four-Directional Scanning and Spatial Chunking" and "Why the
//   Stability Controls Matter"; "VisionHOPE" README - "SRNL and VisionHOPE
//   operator".
//
// Single-product form.  Each write right-multiplies all five memories by the
// same T_t = alpha_t I - eta_t u_t k_t^T (u_t = (1 + alpha_t) k_t - v_t), so
// every memory is its initial state times one d x d product Q_t, and a
// sequence carries only Q:
//   boundary generation  w_t = Q_b x_t,  [k~ v a beta]_t = G w_t
//                        (G = [M_k0; M_v0; m_eta0; m_alpha0], 66 x 32)
//   token-order write    row <- alpha_t row - eta_t s_t k_t,  s_t = row . u_t
//   readout              y_t = M_mem0 z_t,  z_t = Q_t q_t
// The write keeps two tokens of lookahead: with c1_t = k_t . u_{t+1} and
// c2_t = k_t . u_{t+2} (shared by all rows),
//   s_{t+2} = alpha_{t+1} (alpha_t (row_{t-1} . u_{t+2}) - eta_t c2_t s_t) - eta_{t+1} c1_{t+1} s_{t+1}
// so each row's dot-product reduction has two tokens of slack before it is used.
//
// This kernel serves the fp32 generation path: boundary products and generation run
// on the SIMT pipes in fp32, and every step of the write is an fp32 FMA, so its
// results follow the sequential recurrence to fp32 rounding.  (The bf16 generation
// path runs the chunkwise kernel in srnl_scan_tc.cu.)
//
// One CTA owns one (route, batch, head) sequence; 192 threads:
//   warps 0-3  rows of Q: four lanes per row, 8 columns per lane; the token
//              loop above; z_t (bf16 hi/lo) into the readout operand tile
//   warps 4-5  one thread per token (TMEM lanes 0..63): gates, lookahead
//              coefficients, readout y from TMEM, and asynchronous copies of the
//              next stage
// The readout y = z M_mem0^T runs on the tensor cores (tcgen05, z and M_mem0 as bf16
// hi + lo, three products, fp32 accumulate in TMEM).
// Tokens are staged kStage at a time; a chunk longer than kStage spans several
// stages that all generate from the chunk's boundary Q_b.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "srnl_common.cuh"
#include "srnl_launch.h"
#include "srnl_scan.h"
#include "srnl_umma.cuh"

namespace srnl {
namespace {

constexpr int kThreads = 192;
constexpr int kRowWarps = 4;
constexpr int kTokThreads = 64;   // warps 4-5
constexpr int kPad = 36;          // padded fp32 row stride for per-token rows written row-wise
constexpr int kGenStride = 68;    // padded stride of the SIMT generation rows (66 outputs)
constexpr int kMmma = kUmmaM;     // MMA M; tokens occupy rows 0..63 (TMEM lanes of warps 4-5)
constexpr uint32_t kTmemCols = 32;
constexpr uint32_t kColY = 0;     // TMEM columns of the readout accumulator

struct alignas(128) Smem {
  struct {
    alignas(16) float x[2][kStage][kD];           // x head slices (source dtype), double buffer
    alignas(16) float w[kStage][kPad];            // w_t = Q_b x_t
    alignas(16) float gen[kStage][kGenStride];    // [k~ v a beta]
    alignas(16) float qb[kD][kPad];               // Q_b
  } simt;
  alignas(128) unsigned char zh[kMmma * 64];      // z_t bf16 high part (row t), K = row of Q
  alignas(128) unsigned char zl[kMmma * 64];      // z_t bf16 low part
  alignas(128) unsigned char mh[kD * 64];         // M_mem0 bf16 high part (row = output channel)
  alignas(128) unsigned char ml[kD * 64];         // M_mem0 bf16 low part
  alignas(16) float q[2][kStage][kD];             // q head slices (fp32), double buffer
  alignas(16) float k[kStage][kPad];              // normalised keys
  alignas(16) float u[kStage + 2][kPad];          // u = (1 + alpha) k - v (two padding rows)
  alignas(16) float4 ae[kStage + 2];              // (alpha, eta, eta c1, eta c2)
  alignas(16) float qfin[kD][kD + 1];             // final-state staging
  alignas(16) float scale[kD];                    // fusion scales of this head's channels
  alignas(8) unsigned long long mbar_y;           // readout MMA completion
  uint32_t tmem_base;
  int wait_failed;
};
static_assert(sizeof(Smem) <= 113 * 1024, "two CTAs per SM");

struct Args {
  const void* x;
  const void* q;
  float* yr;
  float* finals;
  int* err;
  unsigned long long* binds;  // hard-clamp activations (nullptr: not counted)
  const float* G;
  const float* Mm;
  const float* scales;
  int B, H, W, C, heads, Lrow, Lcol;
  float alpha, eps;
  bool act_bf16;  // q is fp32 on this path
  bool hard_cap;
};

// Token warps: asynchronous copies of a stage's q (fp32) and x (source dtype) head slices.
__device__ __forceinline__ void prefetch_stage(Smem& sm, int buf, const StageInfo& si, const Args& a,
                                               int r, int64_t tok0, int ch0, int ht) {
  for (int idx = ht; idx < si.T * 8; idx += kTokThreads) {
    const int tt = idx >> 3, part = idx & 7;
    const int p = route_pos(r, si.t0 + tt, a.H, a.W);
    const char* src = reinterpret_cast<const char*>(a.q) + ((tok0 + p) * a.C + ch0) * 4 + part * 16;
    cp_async16(reinterpret_cast<char*>(sm.q[buf][tt]) + part * 16, src);
  }
  const int xe = a.act_bf16 ? 2 : 4;
  const int xparts = kD * xe / 16;
  for (int idx = ht; idx < si.T * xparts; idx += kTokThreads) {
    const int tt = idx / xparts, part = idx - tt * xparts;
    const int p = route_pos(r, si.t0 + tt, a.H, a.W);
    const char* src = reinterpret_cast<const char*>(a.x) + ((tok0 + p) * a.C + ch0) * xe + part * 16;
    cp_async16(reinterpret_cast<char*>(sm.simt.x[buf][tt]) + part * 16, src);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// Token warps: y_t = (readout accumulator row) scaled, stored at the token's raster slot.
__device__ __forceinline__ void readout_from_tmem(Smem& sm, uint32_t tmem_lane, const StageInfo& si,
                                                  const Args& a, int r, int64_t tok0, int ch0, int gt) {
  float y[kD];
  SRNL_LD16(y, tmem_lane + kColY);
  SRNL_LD16(y + 16, tmem_lane + kColY + 16);
  tmem_wait_ld();
  if (gt < si.T) {
    const int p = route_pos(r, si.t0 + gt, a.H, a.W);
    float* dst = a.yr + ((int64_t)r * a.B * a.H * a.W + tok0 + p) * a.C + ch0;
#pragma unroll
    for (int i = 0; i < kD; i += 4)
      *reinterpret_cast<float4*>(dst + i) =
          make_float4(sm.scale[i] * y[i], sm.scale[i + 1] * y[i + 1], sm.scale[i + 2] * y[i + 2],
                      sm.scale[i + 3] * y[i + 3]);
  }
}

__global__ void __launch_bounds__(kThreads, 2) srnl_scan_sequential_kernel(const Args a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const bool is_row = warp < kRowWarps;          // warps 0-3: rows of Q
  const bool is_tok = !is_row;                   // warps 4-5: tokens (TMEM lanes 0..63)
  const int row = (tid >> 2) & 31, cq = tid & 3, cb = cq * 8;  // row lanes
  const int gt = tid - kRowWarps * 32;           // token lanes: token gt of the stage

  const int seq = blockIdx.x;  // ((r * B + b) * heads + h)
  const int h = seq % a.heads;
  const int b = (seq / a.heads) % a.B;
  const int r = seq / (a.heads * a.B);
  const int N = a.H * a.W;
  const int L = (r < 2) ? a.Lrow : a.Lcol;
  const int64_t tok0 = (int64_t)b * N;
  const int ch0 = h * kD;
  const float* Gsrc = a.G + (int64_t)(r * a.heads + h) * kGen * kD;
  const float* Msrc = a.Mm + (int64_t)(r * a.heads + h) * kD * kD;

  // ---- one-time set-up
  if (tid == 0) {
    sm.wait_failed = 0;
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.mbar_y)));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&sm.tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  for (int i = tid; i < kD * kD; i += kThreads) {
    const int o = i / kD, kk = i % kD;
    store_split(sm.mh, sm.ml, o, kk, Msrc[i]);  // readout B operand
    sm.simt.qb[o][kk] = (o == kk) ? 1.f : 0.f;  // Q_b = I
  }
  if (tid < kD) sm.scale[tid] = a.scales[r * a.C + ch0 + tid];
  if (tid < 2) {  // the lookahead reads two rows past the stage: keep them inert
    sm.ae[kStage + tid] = make_float4(1.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kD; ++i) sm.u[kStage + tid][i] = 0.f;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");

  // row state: this lane's 8 columns of row `row` (identity at the start)
  float2 qr[4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
    qr[j] = f2((cb + 2 * j == row) ? 1.f : 0.f, (cb + 2 * j + 1 == row) ? 1.f : 0.f);

  const int nst = num_stages(N, L);
  if (is_tok && nst > 0) {
    prefetch_stage(sm, 0, stage_info(0, N, L), a, r, tok0, ch0, gt);
    cp_async_wait_all();
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = sm.tmem_base;
  const uint32_t tmem_lane = tmem + ((uint32_t)(32 * (warp & 3)) << 16);  // this warp's TMEM lanes
  const uint32_t idesc_y = idesc_bf16(kD);

  uint32_t phase_y = 0;
  bool y_pending = false;  // a readout MMA was issued and not yet consumed
  for (int st = 0; st < nst; ++st) {
    const int cur = st & 1;
    const StageInfo si = stage_info(st, N, L);
    const int T = si.T;
    // ---- generation: w = x Q_b^T, [k~ v a beta] = w G^T, gates, lookahead coefficients
    {
      // SIMT: boundary products (all threads: lane = row, warp = token group), then generation
      {
        float2 qv[16];
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
          const float4 v = *reinterpret_cast<const float4*>(&sm.simt.qb[lane][2 * j]);
          qv[j] = f2(v.x, v.y);
          qv[j + 1] = f2(v.z, v.w);
        }
#pragma unroll 1
        for (int tt = warp; tt < T; tt += kThreads / 32) {
          float2 acc = f2(0.f, 0.f), acc2 = f2(0.f, 0.f);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float2 xv[4];
            load8(sm.simt.x[cur][tt], 8 * j, a.act_bf16, xv);
            acc = __ffma2_rn(qv[4 * j], xv[0], acc);
            acc2 = __ffma2_rn(qv[4 * j + 1], xv[1], acc2);
            acc = __ffma2_rn(qv[4 * j + 2], xv[2], acc);
            acc2 = __ffma2_rn(qv[4 * j + 3], xv[3], acc2);
          }
          sm.simt.w[tt][lane] = (acc.x + acc.y) + (acc2.x + acc2.y);
        }
      }
      __syncthreads();
      {
        const int m = tid & 63;  // m < 32 -> k~, else v
        float grow[kD];
#pragma unroll
        for (int j = 0; j < kD; j += 4) {
          const float4 g4 = __ldg(reinterpret_cast<const float4*>(Gsrc + m * kD + j));
          grow[j] = g4.x; grow[j + 1] = g4.y; grow[j + 2] = g4.z; grow[j + 3] = g4.w;
        }
#pragma unroll 1
        for (int tt = tid >> 6; tt < T; tt += kThreads / 64) sm.simt.gen[tt][m] = dot32(grow, sm.simt.w[tt]);
      }
      __syncthreads();
      bool binds = false;
      if (is_tok && gt < T) {
        float kt[kD], vv[kD], ga = 0.f, gb = 0.f;
        const float* wt = sm.simt.w[gt];
#pragma unroll
        for (int i = 0; i < kD; ++i) {
          kt[i] = sm.simt.gen[gt][i];
          vv[i] = sm.simt.gen[gt][kD + i];
          ga = fmaf(Gsrc[2 * kD * kD + i], wt[i], ga);
          gb = fmaf(Gsrc[2 * kD * kD + kD + i], wt[i], gb);
        }
        float al, eta;
        binds = gates_row(kt, vv, ga, gb, a.alpha, a.eps, al, eta, a.hard_cap);
        store_row(sm.k[gt], kt);
        store_row(sm.u[gt], vv);
        sm.ae[gt] = make_float4(al, eta, 0.f, 0.f);
      }
      if (is_tok && a.hard_cap) count_binds(binds, a.binds);
    }
    if (is_tok && T > 0) {
      tok_bar();
      // lookahead coefficients eta_t (k_t . u_{t+1}) and eta_t (k_t . u_{t+2}); padding rows
      if (gt < T) {
        float kt[kD];
#pragma unroll
        for (int i = 0; i < kD; i += 4) {
          const float4 v = *reinterpret_cast<const float4*>(&sm.k[gt][i]);
          kt[i] = v.x; kt[i + 1] = v.y; kt[i + 2] = v.z; kt[i + 3] = v.w;
        }
        const float eta = sm.ae[gt].y;
        const float c1 = (gt + 1 < T) ? dot32(kt, sm.u[gt + 1]) : 0.f;
        const float c2 = (gt + 2 < T) ? dot32(kt, sm.u[gt + 2]) : 0.f;
        sm.ae[gt].z = eta * c1;
        sm.ae[gt].w = eta * c2;
      } else if (gt < T + 2) {
        sm.ae[gt] = make_float4(1.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < kD; ++i) sm.u[gt][i] = 0.f;
      }
    }
    __syncthreads();
    // ---- token-order write (row warps) | readout + prefetch (token warps)
    if (is_row) {
      if (y_pending) mbar_wait(&sm.mbar_y, phase_y, &sm.wait_failed);  // z tiles free again
      if (T > 0) {
        float2 uv[4];
        load8f(sm.u[0] + cb, uv);
        float s0 = quad_sum(dot8v(qr, uv));
        load8f(sm.u[1] + cb, uv);
        float4 ae_c = sm.ae[0];
        float s1 = fmaf(ae_c.x, quad_sum(dot8v(qr, uv)), -ae_c.z * s0);
        // one token of the write; operands of token tt (k, q, u_{tt+2}) in registers
        auto step = [&](int tt, const float2 (&kc)[4], const float2 (&qc)[4], const float2 (&un)[4],
                        const float4& ae_t, const float4& ae_n) {
          const float pp = dot8v(qr, un);  // row_{t-1} . u_{t+2}
          const float cs = ae_t.y * s0;
          const float2 al2 = f2(ae_t.x, ae_t.x), ncs = f2(-cs, -cs);
          qr[0] = __ffma2_rn(ncs, kc[0], __fmul2_rn(al2, qr[0]));
          qr[1] = __ffma2_rn(ncs, kc[1], __fmul2_rn(al2, qr[1]));
          qr[2] = __ffma2_rn(ncs, kc[2], __fmul2_rn(al2, qr[2]));
          qr[3] = __ffma2_rn(ncs, kc[3], __fmul2_rn(al2, qr[3]));
          const float zt = quad_sum(dot8v(qr, qc));
          if (cq == 0) store_split(sm.zh, sm.zl, tt, row, zt);
          // s_{t+2} = alpha_{t+1} (alpha_t P - eta_t c2_t s_t) - eta_{t+1} c1_{t+1} s_{t+1}
          const float s2 = fmaf(ae_n.x, fmaf(ae_t.x, quad_sum(pp), -ae_t.w * s0), -ae_n.z * s1);
          s0 = s1;
          s1 = s2;
        };
        float2 ka[4], qa_[4], ua[4], kb[4], qb_[4], ub[4];
        load8f(sm.k[0] + cb, ka);
        load8f(sm.q[cur][0] + cb, qa_);
        load8f(sm.u[2] + cb, ua);
#pragma unroll 1
        for (int tt = 0; tt < T; tt += 2) {
          // tokens tt (operands a) and tt + 1 (operands b); rows past T are inert or unused
          const int t1 = tt + 1 < kStage ? tt + 1 : tt;
          const float4 ae_1 = sm.ae[tt + 1];
          load8f(sm.k[t1] + cb, kb);
          load8f(sm.q[cur][t1] + cb, qb_);
          load8f(sm.u[tt + 3] + cb, ub);
          step(tt, ka, qa_, ua, ae_c, ae_1);
          if (tt + 1 >= T) break;
          const int t2 = tt + 2 < kStage ? tt + 2 : tt;
          ae_c = sm.ae[tt + 2];
          load8f(sm.k[t2] + cb, ka);
          load8f(sm.q[cur][t2] + cb, qa_);
          load8f(sm.u[tt + 4 < kStage + 2 ? tt + 4 : kStage + 1] + cb, ua);
          step(tt + 1, kb, qb_, ub, ae_1, ae_c);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      const StageInfo nx = stage_info(st + 1, N, L);
      if (st + 1 < nst && nx.chunk_start) {  // next stage opens a chunk: publish Q_b
        *reinterpret_cast<float4*>(&sm.simt.qb[row][cb]) = make_float4(qr[0].x, qr[0].y, qr[1].x, qr[1].y);
        *reinterpret_cast<float4*>(&sm.simt.qb[row][cb + 4]) = make_float4(qr[2].x, qr[2].y, qr[3].x, qr[3].y);
      }
    } else {
      if (y_pending) {  // readout of the previous stage
        mbar_wait(&sm.mbar_y, phase_y, &sm.wait_failed);
        readout_from_tmem(sm, tmem_lane, stage_info(st - 1, N, L), a, r, tok0, ch0, gt);
      }
      if (st + 1 < nst) prefetch_stage(sm, cur ^ 1, stage_info(st + 1, N, L), a, r, tok0, ch0, gt);
      cp_async_wait_all();
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (y_pending) {
      phase_y ^= 1u;
      y_pending = false;
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    // ---- readout MMA of this stage: y = z M_mem0^T (3-term bf16 split)
    if (T > 0) {
      if (tid == kRowWarps * 32) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t zh = smem_u32(sm.zh), zl = smem_u32(sm.zl);
        const uint32_t mh = smem_u32(sm.mh), ml = smem_u32(sm.ml);
        mma_k32(tmem + kColY, zh, mh, idesc_y, false);
        mma_k32(tmem + kColY, zh, ml, idesc_y, true);
        mma_k32(tmem + kColY, zl, mh, idesc_y, true);
        mma_commit(&sm.mbar_y);
      }
      y_pending = true;
    }
  }
  if (y_pending && is_tok) {
    mbar_wait(&sm.mbar_y, phase_y, &sm.wait_failed);
    readout_from_tmem(sm, tmem_lane, stage_info(nst - 1, N, L), a, r, tok0, ch0, gt);
  }

  __syncthreads();
  if (sm.wait_failed && tid == 0) atomicExch(a.err, SRNL_E_TIMEOUT);

  if (a.finals != nullptr) {
    // memories after the last token: [M_mem0; G] Q
    if (is_row) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sm.qfin[row][cb + 2 * j] = qr[j].x;
        sm.qfin[row][cb + 2 * j + 1] = qr[j].y;
      }
    }
    __syncthreads();
    float* dst = a.finals + (int64_t)seq * kStateFloats;
    for (int mm = warp; mm < kMemRows; mm += kThreads / 32) {
      const float* src = (mm < kD) ? (Msrc + mm * kD) : (Gsrc + (mm - kD) * kD);
      float acc = 0.f;
      for (int i = 0; i < kD; ++i) acc = fmaf(src[i], sm.qfin[i][lane], acc);
      dst[mm * kD + lane] = acc;
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

}  // namespace

cudaError_t prepare_scan_kernels() {
  const cudaError_t e = cudaFuncSetAttribute(srnl_scan_sequential_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Smem));
  if (e != cudaSuccess) return e;
  return prepare_scan_chunkwise_kernel();
}

cudaError_t launch_scan(const ScanGeom& g, const ScanParamsDev& p, const void* x, const void* q,
                        float* yr, float* finals, int* err, unsigned long long* binds, cudaStream_t s) {
  if (g.hd == 64) return launch_scan_d64(g, p, x, q, yr, finals, binds, s);
  if (g.gen_bf16) return launch_scan_chunkwise(g, p, x, q, yr, finals, err, binds, s);
  Args a;
  a.x = x; a.q = q; a.yr = yr; a.finals = finals; a.err = err;
  a.G = p.G; a.Mm = p.Mm; a.scales = p.scales;
  a.B = g.B; a.H = g.H; a.W = g.W; a.C = g.C; a.heads = g.heads;
  a.Lrow = g.Lrow; a.Lcol = g.Lcol; a.alpha = g.alpha; a.eps = g.eps;
  a.act_bf16 = g.act_bf16;
  a.hard_cap = g.hard_cap; a.binds = binds;
  const unsigned nseq = (unsigned)g.routes * (unsigned)g.B * (unsigned)g.heads;
  srnl_scan_sequential_kernel<<<nseq, kThreads, sizeof(Smem), s>>>(a);
  return cudaGetLastError();
}

}  // namespace srnl
