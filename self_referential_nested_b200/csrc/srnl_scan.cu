// SRNL four-direction chunked scan: the sequence kernel (sm_100a).
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
//   token-order write    row <- alpha_t row - eta_t (row . u_t) k_t  (per row of Q)
//   readout              y_t = M_mem0 (Q_t q_t)
//
// One CTA owns one (route, batch, head) sequence; 256 threads:
//   warps 0-3  Q rows (4 lanes x 8 columns per row): boundary products w_t,
//              then the token loop with one token of lookahead
//                s_{t+1} = alpha_t (row_{t-1} . u_{t+1}) - eta_t s_t (k_t . u_{t+1})
//              so the row . u reduction is off the per-token dependency chain;
//   warps 0-1  also the gates, one thread per token;
//   warps 4-7  readout of the previous stage (y = M_mem0 z, scaled, stored at
//              the raster slot) and prefetch of the next stage's x, q.
// Tokens are staged kStage at a time; a chunk longer than kStage spans several
// stages that all generate from the chunk's boundary Q_b.
//
// Generation contraction G w_t: on the bf16 path a tcgen05 MMA (A = w rounded
// to bf16, 128 x 32, K-major; B = G in bf16, 80 x 32, K-major; D fp32 in TMEM,
// one TMEM lane per token), issued by one thread and completed through an
// mbarrier; on the fp32 path a SIMT product with G held in registers.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "srnl_common.cuh"
#include "srnl_launch.h"
#include "srnl_scan.h"

namespace srnl {
namespace {

constexpr int kThreads = 256;
constexpr int kRowThreads = 128;
constexpr int kStage = 64;       // tokens staged per pass
constexpr int kGroup = 4;        // tokens per block of the row update
constexpr int kPad = 36;         // padded fp32 row stride for per-token rows written row-wise
constexpr int kGenStride = 68;   // padded stride of the SIMT generation rows (66 outputs)
constexpr int kNmma = 80;        // MMA N: 66 generated outputs padded to a multiple of 16
constexpr int kMmma = 128;       // MMA M: token rows (kStage used)
constexpr uint32_t kTmemCols = 128;
constexpr long long kWaitLimit = 1ll << 20;  // mbarrier polls before giving up

struct alignas(128) Smem {
  union {
    struct {                                      // bf16 path (tensor cores)
      alignas(128) unsigned char a[kMmma * 64];   // w_t in bf16, UMMA K-major, no swizzle
      alignas(128) unsigned char b[kNmma * 64];   // G in bf16, UMMA K-major, no swizzle
    } tc;
    struct {                                      // fp32 path (SIMT)
      alignas(16) float w[kStage][kPad];          // w_t = Q_b x_t
      alignas(16) float gen[kStage][kGenStride];  // [k~ v a beta]
    } simt;
    alignas(16) float qfin[kD][kD + 1];           // final-state staging (after the scan)
  } g;
  alignas(16) float qb[kD][kPad];                 // boundary product Q_b of the current chunk
  alignas(16) float mm[kD][kPad];                 // content-memory initial state M_mem0
  alignas(16) float x[2][kStage][kD];             // x head slices, route order, source dtype
  alignas(16) float q[2][kStage][kD];             // q head slices, route order, source dtype
  alignas(16) float k[kStage][kPad];              // normalised keys
  alignas(16) float u[kStage][kPad];              // u = (1 + alpha) k - v
  alignas(16) float z[2][kStage][kD];             // z_t = Q_t q_t, double buffer
  alignas(16) float2 ae[kStage];                  // (alpha_t, eta_t)
  alignas(16) float tbl[kStage / kGroup][32];     // per 4-token group: A_prev[4] A[4] W[4] P[6] N[10] A_G
  alignas(8) unsigned long long mbar;
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
  const float* G;
  const float* Mm;
  const float* scales;
  int B, H, W, C, heads, Lrow, Lcol;
  float alpha, eps;
  bool act_bf16, q_bf16;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// UMMA shared-memory descriptor: K-major, no swizzle, core matrices of 8 rows x 16 B,
// K-adjacent core matrices 128 B apart (LBO), 8-row groups 512 B apart (SBO).
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) |
         ((uint64_t)(512u >> 4) << 32) | (1ull << 46);
}

// Byte offset of element (row, k) of a [rows x 32] bf16 K-major operand tile.
__device__ __forceinline__ uint32_t umma_off(int row, int k) {
  return (uint32_t)((row >> 3) * 512 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2);
}

// Instruction descriptor: kind::f16, A = B = bf16, D = f32, both K-major, M = 128, N = 80.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kNmma >> 3) << 17) |
                            ((uint32_t)(kMmma >> 4) << 24);

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// 8 consecutive activations from shared memory (fp32, or bf16 stored in the same row).
__device__ __forceinline__ void load8(const float* row, int c, bool bf16, float2 (&v)[4]) {
  if (bf16) {
    const uint4 raw = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(row) + c);
    v[0] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
    v[1] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
    v[2] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.z));
    v[3] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.w));
  } else {
    const float4 a = *reinterpret_cast<const float4*>(row + c);
    const float4 b = *reinterpret_cast<const float4*>(row + c + 4);
    v[0] = f2(a.x, a.y); v[1] = f2(a.z, a.w); v[2] = f2(b.x, b.y); v[3] = f2(b.z, b.w);
  }
}

__device__ __forceinline__ void load8f(const float* p, float2 (&v)[4]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = f2(a.x, a.y); v[1] = f2(a.z, a.w); v[2] = f2(b.x, b.y); v[3] = f2(b.z, b.w);
}

__device__ __forceinline__ float dot8v(const float2 (&r)[4], const float2 (&v)[4]) {
  float2 acc = __fmul2_rn(r[0], v[0]);
  float2 acc2 = __fmul2_rn(r[2], v[2]);
  acc = __ffma2_rn(r[1], v[1], acc);
  acc2 = __ffma2_rn(r[3], v[3], acc2);
  return (acc.x + acc.y) + (acc2.x + acc2.y);
}

__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  return v;
}

// Gates of one token from its generated row (k~[32], v[32], a, beta): kt becomes the
// stabilized key and vv becomes u.  Stabilized key, retention clamp, softplus step,
// soft injection cap, spectral clamp.
__device__ __forceinline__ void gates_row(float (&kt)[kD], float (&vv)[kD], float a, float beta,
                                          float alpha_max, float eps, float& al, float& eta) {
  float n0 = 0.f, n1 = 0.f, n2 = 0.f, n3 = 0.f;
#pragma unroll
  for (int i = 0; i < kD; i += 4) {
    n0 = fmaf(kt[i], kt[i], n0);
    n1 = fmaf(kt[i + 1], kt[i + 1], n1);
    n2 = fmaf(kt[i + 2], kt[i + 2], n2);
    n3 = fmaf(kt[i + 3], kt[i + 3], n3);
  }
  const float inv = 1.f / sqrtf(((n0 + n1) + (n2 + n3)) + eps);
  float k0 = 0.f, k1 = 0.f, d0 = 0.f, d1 = 0.f;
#pragma unroll
  for (int i = 0; i < kD; i += 2) {
    const float ka = kt[i] * inv, kb = kt[i + 1] * inv;
    kt[i] = ka;
    kt[i + 1] = kb;
    k0 = fmaf(ka, ka, k0);
    k1 = fmaf(kb, kb, k1);
    const float da = ka - vv[i], db = kb - vv[i + 1];
    d0 = fmaf(da, da, d0);
    d1 = fmaf(db, db, d1);
  }
  const float kn2 = k0 + k1;
  const float gain = sqrtf(d0 + d1) * sqrtf(kn2);
  float sg;
  if (beta >= 0.f) {
    sg = 1.f / (1.f + expf(-beta));
  } else {
    const float e = expf(beta);
    sg = e / (1.f + e);
  }
  al = fminf(sg, alpha_max);
  const float eta0 = fmaxf(a, 0.f) + log1pf(expf(-fabsf(a)));
  const float zc = eta0 * gain / (1.f - al);
  const float phi = (zc < 1e-4f) ? (1.f - zc * zc * (1.f / 3.f)) : tanhf(zc) / zc;
  eta = eta0 * phi;
  if (eta * kn2 > 2.f) eta = 2.f / kn2;
#pragma unroll
  for (int i = 0; i < kD; ++i) vv[i] = (1.f + al) * kt[i] - vv[i];
}

__device__ __forceinline__ void store_row(float* dst, const float (&v)[kD]) {
#pragma unroll
  for (int i = 0; i < kD; i += 4)
    *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
}

// Stage `idx` of the sequence: tokens [t0, t0 + T) in route order.
struct StageInfo {
  int t0, T, chunk_start;
};

__device__ __forceinline__ StageInfo stage_info(int idx, int N, int L) {
  const int per = (L + kStage - 1) / kStage;  // stages per chunk
  const int c = idx / per, s = idx - c * per;
  StageInfo si;
  const int c0 = c * L;
  const int Lc = min(L, N - c0);
  si.t0 = c0 + s * kStage;
  si.T = max(0, min(kStage, Lc - s * kStage));
  si.chunk_start = (s == 0);
  return si;
}

__device__ __forceinline__ int num_stages(int N, int L) {
  const int per = (L + kStage - 1) / kStage;
  const int chunks = (N + L - 1) / L;
  return chunks * per;  // trailing stages of a short last chunk may be empty (T = 0)
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}

// Helpers (warps 4-7): asynchronous copy of a stage's x and q head slices (source dtype).
__device__ __forceinline__ void prefetch_stage(Smem& sm, int buf, const StageInfo& si, const Args& a,
                                               int r, int64_t tok0, int ch0, int h128) {
  const int xe = a.act_bf16 ? 2 : 4, qe = a.q_bf16 ? 2 : 4;
  const int xparts = kD * xe / 16, qparts = kD * qe / 16;  // 16-byte pieces per token slice
  for (int idx = h128; idx < si.T * xparts; idx += 128) {
    const int tt = idx / xparts, part = idx - tt * xparts;
    const int p = route_pos(r, si.t0 + tt, a.H, a.W);
    const char* src = reinterpret_cast<const char*>(a.x) + ((tok0 + p) * a.C + ch0) * xe + part * 16;
    cp_async16(reinterpret_cast<char*>(sm.x[buf][tt]) + part * 16, src);
  }
  for (int idx = h128; idx < si.T * qparts; idx += 128) {
    const int tt = idx / qparts, part = idx - tt * qparts;
    const int p = route_pos(r, si.t0 + tt, a.H, a.W);
    const char* src = reinterpret_cast<const char*>(a.q) + ((tok0 + p) * a.C + ch0) * qe + part * 16;
    cp_async16(reinterpret_cast<char*>(sm.q[buf][tt]) + part * 16, src);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Helpers: y_t = M_mem0 z_t for a finished stage, scaled, stored at the raster slot.
__device__ __forceinline__ void readout_stage(const Smem& sm, int buf, const StageInfo& si, float scale,
                                              const Args& a, int r, int64_t tok0, int ch0, int hw,
                                              int lane) {
  const int T = si.T;
  const int64_t base = (int64_t)r * a.B * a.H * a.W;
  const float* mrow = sm.mm[lane];
  for (int tt = hw; tt < T; tt += 4) {
    const float* zt = sm.z[buf][tt];
    float y0 = 0.f, y1 = 0.f;
#pragma unroll
    for (int j = 0; j < kD; j += 4) {
      const float4 za = *reinterpret_cast<const float4*>(zt + j);
      const float4 ma = *reinterpret_cast<const float4*>(mrow + j);
      y0 = fmaf(ma.x, za.x, y0);
      y1 = fmaf(ma.y, za.y, y1);
      y0 = fmaf(ma.z, za.z, y0);
      y1 = fmaf(ma.w, za.w, y1);
    }
    const int p = route_pos(r, si.t0 + tt, a.H, a.W);
    a.yr[(base + tok0 + p) * a.C + ch0 + lane] = scale * (y0 + y1);
  }
}

template <bool kTC>
__global__ void __launch_bounds__(kThreads, 2) srnl_scan2_kernel(const Args a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const bool is_row = tid < kRowThreads;
  const int row = (tid >> 2) & 31, cq = tid & 3, cb = cq * 8;  // row threads' slice of Q
  const int h128 = tid - kRowThreads;                          // helper index (warps 4-7)
  const int hw = warp - 4;

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
    if (kTC) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.mbar)));
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
  }
  if (kTC) {
    if (warp == 0) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(&sm.tmem_base)),
                   "r"(kTmemCols));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    // B operand: G in bf16 (rows 66..79 zero)
    for (int i = tid; i < kNmma * kD; i += kThreads) {
      const int n = i / kD, kk = i % kD;
      const float v = n < kGen ? Gsrc[n * kD + kk] : 0.f;
      *reinterpret_cast<__nv_bfloat16*>(sm.g.tc.b + umma_off(n, kk)) = __float2bfloat16_rn(v);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  for (int i = tid; i < kD * kD; i += kThreads) {
    sm.mm[i / kD][i % kD] = Msrc[i];
    sm.qb[i / kD][i % kD] = (i / kD == i % kD) ? 1.f : 0.f;
  }
  const float scale = is_row ? 0.f : a.scales[r * a.C + ch0 + lane];

  // row state: this thread's slice of Q (identity at the start)
  float2 qr[4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
    qr[j] = f2((cb + 2 * j == row) ? 1.f : 0.f, (cb + 2 * j + 1 == row) ? 1.f : 0.f);

  const int nst = num_stages(N, L);
  if (!is_row && nst > 0) {
    prefetch_stage(sm, 0, stage_info(0, N, L), a, r, tok0, ch0, h128);
    cp_async_wait_all();
  }
  if (kTC) asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (kTC) asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = kTC ? sm.tmem_base : 0u;

  uint32_t phase = 0;
  for (int st = 0; st < nst; ++st) {
    const int cur = st & 1;
    const StageInfo si = stage_info(st, N, L);
    const int T = si.T;
    // ---- P1: boundary products w_t = Q_b x_t (all threads: lane = row, warp = token group)
    {
      float2 qv[16];
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        const float4 v = *reinterpret_cast<const float4*>(&sm.qb[lane][2 * j]);
        qv[j] = f2(v.x, v.y);
        qv[j + 1] = f2(v.z, v.w);
      }
#pragma unroll 1
      for (int tt = warp; tt < T; tt += kThreads / 32) {
        float2 acc = f2(0.f, 0.f), acc2 = f2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float2 xv[4];
          load8(sm.x[cur][tt], 8 * j, a.act_bf16, xv);
          acc = __ffma2_rn(qv[4 * j], xv[0], acc);
          acc2 = __ffma2_rn(qv[4 * j + 1], xv[1], acc2);
          acc = __ffma2_rn(qv[4 * j + 2], xv[2], acc);
          acc2 = __ffma2_rn(qv[4 * j + 3], xv[3], acc2);
        }
        const float w = (acc.x + acc.y) + (acc2.x + acc2.y);
        if (kTC)
          *reinterpret_cast<__nv_bfloat16*>(sm.g.tc.a + umma_off(tt, lane)) = __float2bfloat16_rn(w);
        else
          sm.g.simt.w[tt][lane] = w;
      }
      if (kTC) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();
    // ---- P2: generation [k~ v a beta]_t = G w_t, then gates (one thread per token)
    if (kTC) {
      if (tid == 0 && T > 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t a0 = smem_u32(sm.g.tc.a), b0 = smem_u32(sm.g.tc.b);
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          const uint64_t ad = umma_desc(a0 + ks * 256), bd = umma_desc(b0 + ks * 256);
          asm volatile(
              "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
              "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem),
              "l"(ad), "l"(bd), "r"(kIdesc), "r"(ks));
        }
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_u32(&sm.mbar))
                     : "memory");
      }
      if (warp < 2 && T > 0) {
        // bounded wait for the MMA (skipped once a wait has failed)
        uint32_t done = sm.wait_failed;
        long long polls = 0;
        while (!done) {
          asm volatile(
              "{\n\t.reg .pred P1;\n\tmbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
              "selp.b32 %0, 1, 0, P1;\n\t}\n"
              : "=r"(done)
              : "r"(smem_u32(&sm.mbar)), "r"(phase)
              : "memory");
          if (!done && ++polls > kWaitLimit) {
            sm.wait_failed = 1;
            break;
          }
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        float kt[kD], vv[kD];
        const uint32_t ta = tmem + ((uint32_t)(warp * 32) << 16);
#define SRNL_LD16(dst, col)                                                                         \
  asm volatile(                                                                                     \
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, " \
      "[%16];"                                                                                      \
      : "=f"(dst[0]), "=f"(dst[1]), "=f"(dst[2]), "=f"(dst[3]), "=f"(dst[4]), "=f"(dst[5]),         \
        "=f"(dst[6]), "=f"(dst[7]), "=f"(dst[8]), "=f"(dst[9]), "=f"(dst[10]), "=f"(dst[11]),       \
        "=f"(dst[12]), "=f"(dst[13]), "=f"(dst[14]), "=f"(dst[15])                                  \
      : "r"(ta + (col)))
        SRNL_LD16(kt, 0);
        SRNL_LD16((kt + 16), 16);
        SRNL_LD16(vv, 32);
        SRNL_LD16((vv + 16), 48);
        float ab0, ab1;
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];"
                     : "=f"(ab0), "=f"(ab1)
                     : "r"(ta + 64u));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
#undef SRNL_LD16
        const int tt = tid;
        if (tt < T) {
          float al, eta;
          gates_row(kt, vv, ab0, ab1, a.alpha, a.eps, al, eta);
          store_row(sm.k[tt], kt);
          store_row(sm.u[tt], vv);
          sm.ae[tt] = make_float2(al, eta);
        }
      }
      phase ^= (T > 0) ? 1u : 0u;
    } else {
      // SIMT: thread (m = tid & 63, token group tid >> 6) computes k~ (m < 32) and v (m >= 32)
      const int m = tid & 63;
      float grow[kD];
#pragma unroll
      for (int j = 0; j < kD; j += 4) {
        const float4 g4 = __ldg(reinterpret_cast<const float4*>(Gsrc + m * kD + j));
        grow[j] = g4.x; grow[j + 1] = g4.y; grow[j + 2] = g4.z; grow[j + 3] = g4.w;
      }
#pragma unroll 1
      for (int tt = tid >> 6; tt < T; tt += 4) {
        const float* wt = sm.g.simt.w[tt];
        float2 acc = f2(0.f, 0.f), acc2 = f2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < kD; j += 4) {
          const float4 wv = *reinterpret_cast<const float4*>(wt + j);
          acc = __ffma2_rn(f2(grow[j], grow[j + 1]), f2(wv.x, wv.y), acc);
          acc2 = __ffma2_rn(f2(grow[j + 2], grow[j + 3]), f2(wv.z, wv.w), acc2);
        }
        sm.g.simt.gen[tt][m] = (acc.x + acc.y) + (acc2.x + acc2.y);
      }
      __syncthreads();
      if (tid < T) {
        const int tt = tid;
        float kt[kD], vv[kD];
        float av = 0.f, bv = 0.f;
        const float* wt = sm.g.simt.w[tt];
#pragma unroll
        for (int i = 0; i < kD; ++i) {
          kt[i] = sm.g.simt.gen[tt][i];
          vv[i] = sm.g.simt.gen[tt][kD + i];
          av = fmaf(Gsrc[2 * kD * kD + i], wt[i], av);
          bv = fmaf(Gsrc[2 * kD * kD + kD + i], wt[i], bv);
        }
        float al, eta;
        gates_row(kt, vv, av, bv, a.alpha, a.eps, al, eta);
        store_row(sm.k[tt], kt);
        store_row(sm.u[tt], vv);
        sm.ae[tt] = make_float2(al, eta);
      }
    }
    __syncthreads();
    // ---- P3: tables of each 4-token block (one thread per token; padded tokens are inert)
    {
      const int Tp = (T + kGroup - 1) & ~(kGroup - 1);
      if (tid >= T && tid < Tp) {  // pad to whole blocks: alpha = 1, eta = 0, k = u = 0
        sm.ae[tid] = make_float2(1.f, 0.f);
#pragma unroll
        for (int i = 0; i < kD; i += 4) {
          *reinterpret_cast<float4*>(&sm.k[tid][i]) = make_float4(0.f, 0.f, 0.f, 0.f);
          *reinterpret_cast<float4*>(&sm.u[tid][i]) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      __syncthreads();
      if (tid < Tp) {
        const int g0 = tid & ~(kGroup - 1), i = tid & (kGroup - 1);
        float al[kGroup], et[kGroup];
#pragma unroll
        for (int m = 0; m < kGroup; ++m) {
          const float2 v = sm.ae[g0 + m];
          al[m] = v.x;
          et[m] = v.y;
        }
        // decay products D(j, t) = prod_{m = j+1 .. t} alpha_m (1 when j >= t)
        auto decay = [&](int j, int t) {
          float d = 1.f;
#pragma unroll
          for (int m = 0; m < kGroup; ++m)
            if (m > j && m <= t) d *= al[m];
          return d;
        };
        float* tb = sm.tbl[g0 / kGroup];
        tb[i] = decay(-1, i - 1);            // A_{t-1} (block-relative)
        tb[4 + i] = decay(-1, i);            // A_t
        tb[8 + i] = decay(i, kGroup - 1) * et[i];  // W_j = (A_G / A_j) eta_j
        if (i == 0) tb[28] = decay(-1, kGroup - 1);
        float2 uv[4], qv[4], kv[4];
        const float* ut = sm.u[tid];
#pragma unroll
        for (int j = 0; j < kGroup; ++j) {
          if (j > i) break;
          const float* kj = sm.k[g0 + j];
          float ku = 0.f, kq = 0.f;
#pragma unroll
          for (int c = 0; c < kD; c += 8) {
            load8f(kj + c, kv);
            load8f(ut + c, uv);
            load8(sm.q[cur][tid], c, a.q_bf16, qv);
            ku += dot8v(kv, uv);
            kq += dot8v(kv, qv);
          }
          if (j < i) tb[12 + i * (i - 1) / 2 + j] = decay(j, i - 1) * et[j] * ku;  // P(t, j)
          tb[18 + i * (i + 1) / 2 + j] = decay(j, i) * et[j] * kq;                // N(t, j)
        }
      }
    }
    __syncthreads();
    // ---- P4: token-order write (row threads) | readout + prefetch (helpers)
    if (is_row) {
      const int ng = (T + kGroup - 1) / kGroup;
#pragma unroll 1
      for (int gi = 0; gi < ng; ++gi) {
        const int t0 = gi * kGroup;
        // operands of the block, all loads issued before use
        float4 U[kGroup][2], Qr[kGroup][2];
#pragma unroll
        for (int j = 0; j < kGroup; ++j) {
          U[j][0] = *reinterpret_cast<const float4*>(sm.u[t0 + j] + cb);
          U[j][1] = *reinterpret_cast<const float4*>(sm.u[t0 + j] + cb + 4);
          if (a.q_bf16) {
            Qr[j][0] = *reinterpret_cast<const float4*>(reinterpret_cast<const __nv_bfloat16*>(sm.q[cur][t0 + j]) + cb);
          } else {
            Qr[j][0] = *reinterpret_cast<const float4*>(sm.q[cur][t0 + j] + cb);
            Qr[j][1] = *reinterpret_cast<const float4*>(sm.q[cur][t0 + j] + cb + 4);
          }
        }
        // b_j = r . u_j and e_j = r . q_j (partial over this lane's 8 columns)
        float bp[kGroup], ep[kGroup];
#pragma unroll
        for (int j = 0; j < kGroup; ++j) {
          float2 v[4] = {f2(U[j][0].x, U[j][0].y), f2(U[j][0].z, U[j][0].w), f2(U[j][1].x, U[j][1].y),
                         f2(U[j][1].z, U[j][1].w)};
          bp[j] = dot8v(qr, v);
          if (a.q_bf16) {
            const uint4 raw = *reinterpret_cast<const uint4*>(&Qr[j][0]);
            v[0] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
            v[1] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
            v[2] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.z));
            v[3] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.w));
          } else {
            v[0] = f2(Qr[j][0].x, Qr[j][0].y); v[1] = f2(Qr[j][0].z, Qr[j][0].w);
            v[2] = f2(Qr[j][1].x, Qr[j][1].y); v[3] = f2(Qr[j][1].z, Qr[j][1].w);
          }
          ep[j] = dot8v(qr, v);
        }
        // block tables and keys, loaded while the reductions run
        const float* tb = sm.tbl[gi];
        const float4 Ap = *reinterpret_cast<const float4*>(tb);
        const float4 Aa = *reinterpret_cast<const float4*>(tb + 4);
        const float4 Wv = *reinterpret_cast<const float4*>(tb + 8);
        const float4 P0 = *reinterpret_cast<const float4*>(tb + 12);   // P10 P20 P21 P30
        const float4 P1 = *reinterpret_cast<const float4*>(tb + 16);   // P31 P32 N00 N10
        const float4 N0 = *reinterpret_cast<const float4*>(tb + 20);   // N11 N20 N21 N22
        const float4 N1 = *reinterpret_cast<const float4*>(tb + 24);   // N30 N31 N32 N33
        const float AG = tb[28];
        float4 K[kGroup][2];
#pragma unroll
        for (int j = 0; j < kGroup; ++j) {
          K[j][0] = *reinterpret_cast<const float4*>(sm.k[t0 + j] + cb);
          K[j][1] = *reinterpret_cast<const float4*>(sm.k[t0 + j] + cb + 4);
        }
        // interleaved quad reductions
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
          float tb_[kGroup], te_[kGroup];
#pragma unroll
          for (int j = 0; j < kGroup; ++j) {
            tb_[j] = __shfl_xor_sync(0xffffffffu, bp[j], o);
            te_[j] = __shfl_xor_sync(0xffffffffu, ep[j], o);
          }
#pragma unroll
          for (int j = 0; j < kGroup; ++j) {
            bp[j] += tb_[j];
            ep[j] += te_[j];
          }
        }
        // s_t = A_{t-1} b_t - sum_{j<t} P(t,j) s_j
        const float s0 = Ap.x * bp[0];
        const float s1 = fmaf(-P0.x, s0, Ap.y * bp[1]);
        const float s2 = fmaf(-P0.z, s1, fmaf(-P0.y, s0, Ap.z * bp[2]));
        const float s3 = fmaf(-P1.y, s2, fmaf(-P1.x, s1, fmaf(-P0.w, s0, Ap.w * bp[3])));
        // z_t = A_t e_t - sum_{j<=t} N(t,j) s_j; lane cq stores token t0 + cq
        float zs;
        if (cq == 0) zs = fmaf(-P1.z, s0, Aa.x * ep[0]);
        else if (cq == 1) zs = fmaf(-N0.x, s1, fmaf(-P1.w, s0, Aa.y * ep[1]));
        else if (cq == 2) zs = fmaf(-N0.w, s2, fmaf(-N0.z, s1, fmaf(-N0.y, s0, Aa.z * ep[2])));
        else zs = fmaf(-N1.w, s3, fmaf(-N1.z, s2, fmaf(-N1.y, s1, fmaf(-N1.x, s0, Aa.w * ep[3]))));
        if (t0 + cq < T) sm.z[cur][t0 + cq][row] = zs;
        // r <- A_G r - sum_j W_j s_j k_j
        const float c0 = Wv.x * s0, c1 = Wv.y * s1, c2 = Wv.z * s2, c3 = Wv.w * s3;
        const float2 ag = f2(AG, AG), n0 = f2(-c0, -c0), n1 = f2(-c1, -c1), n2 = f2(-c2, -c2),
                     n3 = f2(-c3, -c3);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          float2 v = __fmul2_rn(ag, qr[2 * h2]);
          v = __ffma2_rn(n0, f2(K[0][h2].x, K[0][h2].y), v);
          v = __ffma2_rn(n1, f2(K[1][h2].x, K[1][h2].y), v);
          v = __ffma2_rn(n2, f2(K[2][h2].x, K[2][h2].y), v);
          qr[2 * h2] = __ffma2_rn(n3, f2(K[3][h2].x, K[3][h2].y), v);
          float2 w = __fmul2_rn(ag, qr[2 * h2 + 1]);
          w = __ffma2_rn(n0, f2(K[0][h2].z, K[0][h2].w), w);
          w = __ffma2_rn(n1, f2(K[1][h2].z, K[1][h2].w), w);
          w = __ffma2_rn(n2, f2(K[2][h2].z, K[2][h2].w), w);
          qr[2 * h2 + 1] = __ffma2_rn(n3, f2(K[3][h2].z, K[3][h2].w), w);
        }
      }
      const StageInfo nx = stage_info(st + 1, N, L);
      if (st + 1 < nst && nx.chunk_start) {  // next stage opens a chunk: publish Q_b
        *reinterpret_cast<float4*>(&sm.qb[row][cb]) = make_float4(qr[0].x, qr[0].y, qr[1].x, qr[1].y);
        *reinterpret_cast<float4*>(&sm.qb[row][cb + 4]) = make_float4(qr[2].x, qr[2].y, qr[3].x, qr[3].y);
      }
    } else {
      if (st + 1 < nst) prefetch_stage(sm, cur ^ 1, stage_info(st + 1, N, L), a, r, tok0, ch0, h128);
      if (st > 0) readout_stage(sm, cur ^ 1, stage_info(st - 1, N, L), scale, a, r, tok0, ch0, hw, lane);
      cp_async_wait_all();
    }
    __syncthreads();
  }
  if (!is_row && nst > 0)
    readout_stage(sm, (nst - 1) & 1, stage_info(nst - 1, N, L), scale, a, r, tok0, ch0, hw, lane);

  if (sm.wait_failed && tid == 0) atomicExch(a.err, SRNL_E_TIMEOUT);

  if (a.finals != nullptr) {
    // memories after the last token: [M_mem0; G] Q
    __syncthreads();
    if (is_row) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sm.g.qfin[row][cb + 2 * j] = qr[j].x;
        sm.g.qfin[row][cb + 2 * j + 1] = qr[j].y;
      }
    }
    __syncthreads();
    float* dst = a.finals + (int64_t)seq * kStateFloats;
    for (int mm = warp; mm < kMemRows; mm += kThreads / 32) {
      const float* src = (mm < kD) ? (Msrc + mm * kD) : (Gsrc + (mm - kD) * kD);
      float acc = 0.f;
      for (int i = 0; i < kD; ++i) acc = fmaf(src[i], sm.g.qfin[i][lane], acc);
      dst[mm * kD + lane] = acc;
    }
  }
  if (kTC) {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
  }
}

}  // namespace

cudaError_t prepare_scan_kernels() {
  cudaError_t e = cudaFuncSetAttribute(srnl_scan2_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sizeof(Smem));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(srnl_scan2_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)sizeof(Smem));
}

cudaError_t launch_scan(const ScanGeom& g, const ScanParamsDev& p, const void* x, const void* q,
                        float* yr, float* finals, int* err, cudaStream_t s) {
  Args a;
  a.x = x; a.q = q; a.yr = yr; a.finals = finals; a.err = err;
  a.G = p.G; a.Mm = p.Mm; a.scales = p.scales;
  a.B = g.B; a.H = g.H; a.W = g.W; a.C = g.C; a.heads = g.heads;
  a.Lrow = g.Lrow; a.Lcol = g.Lcol; a.alpha = g.alpha; a.eps = g.eps;
  a.act_bf16 = g.act_bf16; a.q_bf16 = g.gen_bf16;
  const unsigned nseq = 4u * (unsigned)g.B * (unsigned)g.heads;
  if (g.gen_bf16)
    srnl_scan2_kernel<true><<<nseq, kThreads, sizeof(Smem), s>>>(a);
  else
    srnl_scan2_kernel<false><<<nseq, kThreads, sizeof(Smem), s>>>(a);
  return cudaGetLastError();
}

}  // namespace srnl
