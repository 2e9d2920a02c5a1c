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
//   readout              y_t = M_mem0 z_t,  z_t = Q_t q_t
// Inside a block of 4 tokens the write is applied in closed form: with
// A_t = alpha_1..alpha_t (block-relative),
//   s_t = row_{t-1} . u_t = A_{t-1} (row_0 . u_t) - sum_{j<t} (A_{t-1}/A_j) eta_j (k_j . u_t) s_j
//   z_t = row_t . q_t     = A_t (row_0 . q_t)     - sum_{j<=t} (A_t/A_j) eta_j (k_j . q_t) s_j
//   row_4 = A_4 row_0 - sum_j (A_4/A_j) eta_j s_j k_j
// which is the token-order recurrence reorganised (same terms, exact).
//
// One CTA owns one (route, batch, head) sequence; 192 threads:
//   warps 0-1  rows of Q: each lane holds 8 columns of two rows (rows rp and
//              rp + 16), runs the block recursion and writes z_t (bf16 hi/lo)
//   warps 2-3  one thread per token (TMEM lanes 64..127): gates from the
//              generation MMA, the block tables, and the readout y from TMEM
//   warps 4-5  asynchronous copies of the next stage's x and q
//   all        boundary products w_t (SIMT)
// Tensor cores (tcgen05, fp32 accumulate in TMEM):
//   generation  [k~ v a beta] = w G^T     A = w (bf16), B = G (bf16), N = 80
//               (bf16 path; the fp32 path runs this product on the SIMT pipes)
//   readout     y = z M_mem0^T            3-term bf16 split of z and M_mem0
//               (z_hi M_hi + z_hi M_lo + z_lo M_hi), about fp32 accuracy
// Tokens are staged kStage at a time; a chunk longer than kStage spans several
// stages that all generate from the chunk's boundary Q_b.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "srnl_common.cuh"
#include "srnl_launch.h"
#include "srnl_scan.h"

namespace srnl {
namespace {

constexpr int kThreads = 192;
constexpr int kCopyThreads = 64;  // warps 4-5
constexpr int kStage = 64;       // tokens staged per pass
constexpr int kGroup = 4;        // tokens per block of the row update
constexpr int kPad = 36;         // padded fp32 row stride for per-token rows written row-wise
constexpr int kGenStride = 68;   // padded stride of the SIMT generation rows (66 outputs)
constexpr int kNgen = 80;        // generation MMA N: 66 outputs padded to a multiple of 16
constexpr int kNy = 32;          // readout MMA N
constexpr int kMmma = 128;       // MMA M; tokens occupy rows 64..127 (TMEM lanes of warps 2-3)
constexpr int kTok0 = 64;        // first MMA row / TMEM lane holding a token
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kColGen = 0;  // TMEM columns of the generation accumulator
constexpr uint32_t kColY = 96;   // TMEM columns of the readout accumulator
constexpr long long kWaitLimit = 1ll << 20;  // mbarrier polls before giving up

struct alignas(128) Smem {
  union {
    struct {                                      // bf16 path (tensor-core generation)
      alignas(128) unsigned char a[kMmma * 64];   // w_t in bf16 (row 64 + t), K-major, no swizzle
      alignas(128) unsigned char b[kNgen * 64];   // G in bf16
    } tc;
    struct {                                      // fp32 path (SIMT generation)
      alignas(16) float w[kStage][kPad];          // w_t = Q_b x_t
      alignas(16) float gen[kStage][kGenStride];  // [k~ v a beta]
    } simt;
    alignas(16) float qfin[kD][kD + 1];           // final-state staging (after the scan)
  } g;
  alignas(128) unsigned char zh[kMmma * 64];      // z_t bf16 high part (row 64 + t), K = row of Q
  alignas(128) unsigned char zl[kMmma * 64];      // z_t bf16 low part
  alignas(128) unsigned char mh[kNy * 64];        // M_mem0 bf16 high part (row = output channel)
  alignas(128) unsigned char ml[kNy * 64];        // M_mem0 bf16 low part
  alignas(16) float qb[kD][kPad];                 // boundary product Q_b of the current chunk
  alignas(16) float x[2][kStage][kD];             // x head slices, route order, source dtype
  alignas(16) float q[2][kStage][kD];             // q head slices, route order, source dtype
  alignas(16) float k[kStage][kPad];              // normalised keys
  alignas(16) float u[kStage][kPad];              // u = (1 + alpha) k - v
  alignas(16) float2 ae[kStage];                  // (alpha_t, eta_t)
  alignas(16) float tbl[kStage / kGroup][32];     // per block: A_prev[4] A[4] W[4] P[6] N[10] A_G
  alignas(16) float scale[kD];                    // fusion scales of this head's channels
  alignas(8) unsigned long long mbar_g;           // generation MMA completion
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

// Instruction descriptor: kind::f16, A = B = bf16, D = f32, both K-major, M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kMmma >> 4) << 24);
}

// D[tmem] (+)= A B^T over K = 32 (two K = 16 steps).
__device__ __forceinline__ void mma_k32(uint32_t tmem, uint32_t a_smem, uint32_t b_smem, uint32_t idesc,
                                        bool accumulate) {
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    const uint64_t ad = umma_desc(a_smem + ks * 256), bd = umma_desc(b_smem + ks * 256);
    const uint32_t acc = (accumulate || ks > 0) ? 1u : 0u;
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem),
        "l"(ad), "l"(bd), "r"(idesc), "r"(acc));
  }
}

__device__ __forceinline__ void mma_commit(unsigned long long* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Bounded wait on an mbarrier phase; records a failure instead of hanging.
__device__ __forceinline__ void mbar_wait(unsigned long long* bar, uint32_t phase, int* failed) {
  uint32_t done = *reinterpret_cast<volatile int*>(failed);
  long long polls = 0;
  while (!done) {
    asm volatile(
        "{\n\t.reg .pred P1;\n\tmbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, P1;\n\t}\n"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(phase)
        : "memory");
    if (!done && ++polls > kWaitLimit) {
      *failed = 1;
      break;
    }
  }
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void store_bf16(unsigned char* tile, int row, int k, float v) {
  *reinterpret_cast<__nv_bfloat16*>(tile + umma_off(row, k)) = __float2bfloat16_rn(v);
}

// v ~ hi + lo with hi, lo bf16 (hi = round(v), lo = round(v - hi)).
__device__ __forceinline__ void store_split(unsigned char* th, unsigned char* tl, int row, int k, float v) {
  const __nv_bfloat16 hi = __float2bfloat16_rn(v);
  *reinterpret_cast<__nv_bfloat16*>(th + umma_off(row, k)) = hi;
  *reinterpret_cast<__nv_bfloat16*>(tl + umma_off(row, k)) = __float2bfloat16_rn(v - __bfloat162float(hi));
}

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

__device__ __forceinline__ float dot32(const float (&a)[kD], const float* b) {
  float2 acc = f2(0.f, 0.f), acc2 = f2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < kD; i += 4) {
    const float4 v = *reinterpret_cast<const float4*>(b + i);
    acc = __ffma2_rn(f2(a[i], a[i + 1]), f2(v.x, v.y), acc);
    acc2 = __ffma2_rn(f2(a[i + 2], a[i + 3]), f2(v.z, v.w), acc2);
  }
  return (acc.x + acc.y) + (acc2.x + acc2.y);
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

// Warps 4-5: asynchronous copy of a stage's x and q head slices (source dtype).
__device__ __forceinline__ void prefetch_stage(Smem& sm, int buf, const StageInfo& si, const Args& a,
                                               int r, int64_t tok0, int ch0, int hc) {
  const int xe = a.act_bf16 ? 2 : 4, qe = a.q_bf16 ? 2 : 4;
  const int xparts = kD * xe / 16, qparts = kD * qe / 16;  // 16-byte pieces per token slice
  for (int idx = hc; idx < si.T * xparts; idx += kCopyThreads) {
    const int tt = idx / xparts, part = idx - tt * xparts;
    const int p = route_pos(r, si.t0 + tt, a.H, a.W);
    const char* src = reinterpret_cast<const char*>(a.x) + ((tok0 + p) * a.C + ch0) * xe + part * 16;
    cp_async16(reinterpret_cast<char*>(sm.x[buf][tt]) + part * 16, src);
  }
  for (int idx = hc; idx < si.T * qparts; idx += kCopyThreads) {
    const int tt = idx / qparts, part = idx - tt * qparts;
    const int p = route_pos(r, si.t0 + tt, a.H, a.W);
    const char* src = reinterpret_cast<const char*>(a.q) + ((tok0 + p) * a.C + ch0) * qe + part * 16;
    cp_async16(reinterpret_cast<char*>(sm.q[buf][tt]) + part * 16, src);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

#define SRNL_LD16(dst, addr)                                                                          \
  asm volatile(                                                                                       \
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, " \
      "[%16];"                                                                                        \
      : "=f"((dst)[0]), "=f"((dst)[1]), "=f"((dst)[2]), "=f"((dst)[3]), "=f"((dst)[4]),               \
        "=f"((dst)[5]), "=f"((dst)[6]), "=f"((dst)[7]), "=f"((dst)[8]), "=f"((dst)[9]),               \
        "=f"((dst)[10]), "=f"((dst)[11]), "=f"((dst)[12]), "=f"((dst)[13]), "=f"((dst)[14]),          \
        "=f"((dst)[15])                                                                               \
      : "r"(addr))

// Warps 2-3: y_t = (readout accumulator row) scaled, stored at the token's raster slot.
__device__ __forceinline__ void readout_from_tmem(Smem& sm, uint32_t tmem, const StageInfo& si,
                                                  const Args& a, int r, int64_t tok0, int ch0, int gw,
                                                  int gt) {
  float y[kD];
  const uint32_t ta = tmem + ((uint32_t)(kTok0 + 32 * gw) << 16) + kColY;
  SRNL_LD16(y, ta);
  SRNL_LD16(y + 16, ta + 16);
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
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

template <bool kTC>
__global__ void __launch_bounds__(kThreads, 2) srnl_scan2_kernel(const Args a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const bool is_row = warp < 2;                  // warps 0-1: rows of Q
  const bool is_gate = warp == 2 || warp == 3;   // warps 2-3: tokens (TMEM lanes 64..127)
  const bool is_copy = warp >= 4;                // warps 4-5: prefetch
  const int cq = lane & 3, cb = cq * 8;          // row lanes: column block
  const int ra = (lane >> 2) + 8 * (warp & 1);   // row lanes: rows ra and ra + 16
  const int rb = ra + 16;
  const int gw = warp - 2, gt = tid - 64;        // token lanes: token gt of the stage
  const int hc = tid - 128;

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
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.mbar_g)));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.mbar_y)));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&sm.tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (kTC) {  // B operand of the generation MMA: G in bf16 (rows 66..79 zero)
    for (int i = tid; i < kNgen * kD; i += kThreads) {
      const int n = i / kD, kk = i % kD;
      store_bf16(sm.g.tc.b, n, kk, n < kGen ? Gsrc[n * kD + kk] : 0.f);
    }
  }
  for (int i = tid; i < kD * kD; i += kThreads) {  // readout B operand: M_mem0 hi/lo; Q_b = I
    const int o = i / kD, kk = i % kD;
    store_split(sm.mh, sm.ml, o, kk, Msrc[i]);
    sm.qb[o][kk] = (o == kk) ? 1.f : 0.f;
  }
  if (tid < kD) sm.scale[tid] = a.scales[r * a.C + ch0 + tid];
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");

  // row state: 8 columns of rows ra and rb (identity at the start)
  float2 qa[4], qz[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    qa[j] = f2((cb + 2 * j == ra) ? 1.f : 0.f, (cb + 2 * j + 1 == ra) ? 1.f : 0.f);
    qz[j] = f2((cb + 2 * j == rb) ? 1.f : 0.f, (cb + 2 * j + 1 == rb) ? 1.f : 0.f);
  }

  const int nst = num_stages(N, L);
  if (is_copy && nst > 0) {
    prefetch_stage(sm, 0, stage_info(0, N, L), a, r, tok0, ch0, hc);
    cp_async_wait_all();
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = sm.tmem_base;
  const uint32_t idesc_gen = idesc_bf16(kNgen), idesc_y = idesc_bf16(kNy);

  uint32_t phase_g = 0, phase_y = 0;
  bool y_pending = false;  // a readout MMA was issued and not yet consumed
  for (int st = 0; st < nst; ++st) {
    const int cur = st & 1;
    const StageInfo si = stage_info(st, N, L);
    const int T = si.T;
    const int Tp = (T + kGroup - 1) & ~(kGroup - 1);
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
          store_bf16(sm.g.tc.a, kTok0 + tt, lane, w);
        else
          sm.g.simt.w[tt][lane] = w;
      }
      if (kTC) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();
    // ---- P2: generation, gates and block tables (token lanes)
    if (!kTC) {
      // SIMT generation: thread (m = tid & 63, token group tid >> 6), m < 32 -> k~, else v
      const int m = tid & 63;
      float grow[kD];
#pragma unroll
      for (int j = 0; j < kD; j += 4) {
        const float4 g4 = __ldg(reinterpret_cast<const float4*>(Gsrc + m * kD + j));
        grow[j] = g4.x; grow[j + 1] = g4.y; grow[j + 2] = g4.z; grow[j + 3] = g4.w;
      }
#pragma unroll 1
      for (int tt = tid >> 6; tt < T; tt += kThreads / 64) sm.g.simt.gen[tt][m] = dot32(grow, sm.g.simt.w[tt]);
      __syncthreads();
    } else if (tid == 64 && T > 0) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      mma_k32(tmem + kColGen, smem_u32(sm.g.tc.a), smem_u32(sm.g.tc.b), idesc_gen, false);
      mma_commit(&sm.mbar_g);
    }
    if (is_gate && T > 0) {
      float kt[kD], vv[kD];
      float ga = 0.f, gb = 0.f;
      if (kTC) {
        mbar_wait(&sm.mbar_g, phase_g, &sm.wait_failed);
        const uint32_t ta = tmem + ((uint32_t)(kTok0 + 32 * gw) << 16) + kColGen;
        SRNL_LD16(kt, ta);
        SRNL_LD16(kt + 16, ta + 16);
        SRNL_LD16(vv, ta + 32);
        SRNL_LD16(vv + 16, ta + 48);
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];"
                     : "=f"(ga), "=f"(gb)
                     : "r"(ta + 64u));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      } else if (gt < T) {
        const float* wt = sm.g.simt.w[gt];
#pragma unroll
        for (int i = 0; i < kD; ++i) {
          kt[i] = sm.g.simt.gen[gt][i];
          vv[i] = sm.g.simt.gen[gt][kD + i];
          ga = fmaf(Gsrc[2 * kD * kD + i], wt[i], ga);
          gb = fmaf(Gsrc[2 * kD * kD + kD + i], wt[i], gb);
        }
      }
      float al = 1.f, eta = 0.f;
      if (gt < T) {
        gates_row(kt, vv, ga, gb, a.alpha, a.eps, al, eta);
      } else {  // pad to whole blocks: alpha = 1, eta = 0, k = u = 0 (inert tokens)
#pragma unroll
        for (int i = 0; i < kD; ++i) kt[i] = vv[i] = 0.f;
      }
      if (gt < Tp) {
        store_row(sm.k[gt], kt);
        store_row(sm.u[gt], vv);
        sm.ae[gt] = make_float2(al, eta);
      }
      __syncwarp();
      // tables of this token's block: P(t, j) = (A_{t-1}/A_j) eta_j (k_j . u_t),
      // N(t, j) = (A_t/A_j) eta_j (k_j . q_t), W_j = (A_G/A_j) eta_j, A_{t-1}, A_t, A_G
      if (gt < Tp) {
        const int g0 = gt & ~(kGroup - 1), i = gt & (kGroup - 1);
        float alb[kGroup], etb[kGroup];
#pragma unroll
        for (int m = 0; m < kGroup; ++m) {
          const float2 v = sm.ae[g0 + m];
          alb[m] = v.x;
          etb[m] = v.y;
        }
        auto decay = [&](int j, int t) {  // prod_{m = j+1 .. t} alpha_m
          float d = 1.f;
#pragma unroll
          for (int m = 0; m < kGroup; ++m)
            if (m > j && m <= t) d *= alb[m];
          return d;
        };
        float qt[kD];
        if (gt < T) {
#pragma unroll
          for (int c = 0; c < kD; c += 8) {
            float2 qv2[4];
            load8(sm.q[cur][gt], c, a.q_bf16, qv2);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              qt[c + 2 * e] = qv2[e].x;
              qt[c + 2 * e + 1] = qv2[e].y;
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < kD; ++c) qt[c] = 0.f;
        }
        float* tb = sm.tbl[g0 / kGroup];
        tb[i] = decay(-1, i - 1);
        tb[4 + i] = decay(-1, i);
        tb[8 + i] = decay(i, kGroup - 1) * etb[i];
        if (i == 0) tb[28] = decay(-1, kGroup - 1);
#pragma unroll
        for (int j = 0; j < kGroup; ++j) {
          if (j > i) break;
          const float* kj = sm.k[g0 + j];
          if (j < i) tb[12 + i * (i - 1) / 2 + j] = decay(j, i - 1) * etb[j] * dot32(vv, kj);
          tb[18 + i * (i + 1) / 2 + j] = decay(j, i) * etb[j] * dot32(qt, kj);
        }
      }
    }
    if (kTC) phase_g ^= (T > 0) ? 1u : 0u;
    __syncthreads();
    // ---- P4: rows | readout of the previous stage | prefetch of the next stage
    if (is_row) {
      if (y_pending) mbar_wait(&sm.mbar_y, phase_y, &sm.wait_failed);  // z tiles free again
      const int ng = Tp / kGroup;
#pragma unroll 1
      for (int gi = 0; gi < ng; ++gi) {
        const int t0 = gi * kGroup;
        // partial dots over this lane's 8 columns: b (row . u), e (row . q), rows ra and rb
        float pb[2][kGroup], pe[2][kGroup];
#pragma unroll
        for (int j = 0; j < kGroup; ++j) {
          float2 v[4];
          load8f(sm.u[t0 + j] + cb, v);
          pb[0][j] = dot8v(qa, v);
          pb[1][j] = dot8v(qz, v);
          load8(sm.q[cur][t0 + j], cb, a.q_bf16, v);
          pe[0][j] = dot8v(qa, v);
          pe[1][j] = dot8v(qz, v);
        }
        // interleaved reductions over the 4 lanes of a row
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
          float tb_[2][kGroup], te_[2][kGroup];
#pragma unroll
          for (int rr = 0; rr < 2; ++rr)
#pragma unroll
            for (int j = 0; j < kGroup; ++j) {
              tb_[rr][j] = __shfl_xor_sync(0xffffffffu, pb[rr][j], o);
              te_[rr][j] = __shfl_xor_sync(0xffffffffu, pe[rr][j], o);
            }
#pragma unroll
          for (int rr = 0; rr < 2; ++rr)
#pragma unroll
            for (int j = 0; j < kGroup; ++j) {
              pb[rr][j] += tb_[rr][j];
              pe[rr][j] += te_[rr][j];
            }
        }
        const float* tb = sm.tbl[gi];
        const float4 Ap = *reinterpret_cast<const float4*>(tb);
        const float4 Aa = *reinterpret_cast<const float4*>(tb + 4);
        const float4 Wv = *reinterpret_cast<const float4*>(tb + 8);
        const float4 P0 = *reinterpret_cast<const float4*>(tb + 12);   // P10 P20 P21 P30
        const float4 P1 = *reinterpret_cast<const float4*>(tb + 16);   // P31 P32 N00 N10
        const float4 N0 = *reinterpret_cast<const float4*>(tb + 20);   // N11 N20 N21 N22
        const float4 N1 = *reinterpret_cast<const float4*>(tb + 24);   // N30 N31 N32 N33
        const float AG = tb[28];
        float sv[2][kGroup];
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const float* bp = pb[rr];
          const float* ep = pe[rr];
          // s_t = A_{t-1} b_t - sum_{j<t} P(t,j) s_j
          const float s0 = Ap.x * bp[0];
          const float s1 = fmaf(-P0.x, s0, Ap.y * bp[1]);
          const float s2 = fmaf(-P0.z, s1, fmaf(-P0.y, s0, Ap.z * bp[2]));
          const float s3 = fmaf(-P1.y, s2, fmaf(-P1.x, s1, fmaf(-P0.w, s0, Ap.w * bp[3])));
          // z_t = A_t e_t - sum_{j<=t} N(t,j) s_j; lane cq handles token t0 + cq
          float zs;
          if (cq == 0) zs = fmaf(-P1.z, s0, Aa.x * ep[0]);
          else if (cq == 1) zs = fmaf(-N0.x, s1, fmaf(-P1.w, s0, Aa.y * ep[1]));
          else if (cq == 2) zs = fmaf(-N0.w, s2, fmaf(-N0.z, s1, fmaf(-N0.y, s0, Aa.z * ep[2])));
          else zs = fmaf(-N1.w, s3, fmaf(-N1.z, s2, fmaf(-N1.y, s1, fmaf(-N1.x, s0, Aa.w * ep[3]))));
          if (t0 + cq < T) store_split(sm.zh, sm.zl, kTok0 + t0 + cq, rr ? rb : ra, zs);
          sv[rr][0] = s0; sv[rr][1] = s1; sv[rr][2] = s2; sv[rr][3] = s3;
        }
        // row <- A_G row - sum_j W_j s_j k_j (both rows, one key vector at a time)
        {
          const float2 ag = f2(AG, AG);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            qa[e] = __fmul2_rn(ag, qa[e]);
            qz[e] = __fmul2_rn(ag, qz[e]);
          }
          const float wv[kGroup] = {Wv.x, Wv.y, Wv.z, Wv.w};
#pragma unroll
          for (int j = 0; j < kGroup; ++j) {
            float2 kv[4];
            load8f(sm.k[t0 + j] + cb, kv);
            const float ca = -wv[j] * sv[0][j], cz = -wv[j] * sv[1][j];
            const float2 na = f2(ca, ca), nz = f2(cz, cz);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              qa[e] = __ffma2_rn(na, kv[e], qa[e]);
              qz[e] = __ffma2_rn(nz, kv[e], qz[e]);
            }
          }
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      const StageInfo nx = stage_info(st + 1, N, L);
      if (st + 1 < nst && nx.chunk_start) {  // next stage opens a chunk: publish Q_b
        *reinterpret_cast<float4*>(&sm.qb[ra][cb]) = make_float4(qa[0].x, qa[0].y, qa[1].x, qa[1].y);
        *reinterpret_cast<float4*>(&sm.qb[ra][cb + 4]) = make_float4(qa[2].x, qa[2].y, qa[3].x, qa[3].y);
        *reinterpret_cast<float4*>(&sm.qb[rb][cb]) = make_float4(qz[0].x, qz[0].y, qz[1].x, qz[1].y);
        *reinterpret_cast<float4*>(&sm.qb[rb][cb + 4]) = make_float4(qz[2].x, qz[2].y, qz[3].x, qz[3].y);
      }
    } else if (is_gate) {
      if (y_pending) {  // readout of the previous stage
        mbar_wait(&sm.mbar_y, phase_y, &sm.wait_failed);
        readout_from_tmem(sm, tmem, stage_info(st - 1, N, L), a, r, tok0, ch0, gw, gt);
      }
    } else {
      if (st + 1 < nst) prefetch_stage(sm, cur ^ 1, stage_info(st + 1, N, L), a, r, tok0, ch0, hc);
      cp_async_wait_all();
    }
    if (y_pending) {
      phase_y ^= 1u;
      y_pending = false;
    }
    __syncthreads();
    // ---- readout MMA of this stage: y = z M_mem0^T (3-term bf16 split)
    if (T > 0) {
      if (tid == 64) {
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
  if (y_pending && is_gate) {
    mbar_wait(&sm.mbar_y, phase_y, &sm.wait_failed);
    readout_from_tmem(sm, tmem, stage_info(nst - 1, N, L), a, r, tok0, ch0, gw, gt);
  }

  __syncthreads();
  if (sm.wait_failed && tid == 0) atomicExch(a.err, SRNL_E_TIMEOUT);

  if (a.finals != nullptr) {
    // memories after the last token: [M_mem0; G] Q
    if (is_row) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sm.g.qfin[ra][cb + 2 * j] = qa[j].x;
        sm.g.qfin[ra][cb + 2 * j + 1] = qa[j].y;
        sm.g.qfin[rb][cb + 2 * j] = qz[j].x;
        sm.g.qfin[rb][cb + 2 * j + 1] = qz[j].y;
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
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}
#undef SRNL_LD16

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
