// Device helpers shared by the SRNL scan kernels (sm_100a): tcgen05 operand
// descriptors and issue, bounded mbarrier waits, bf16 hi/lo splits, the per-token
// gates and the stage bookkeeping.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "srnl_common.cuh"

namespace srnl {
namespace {

constexpr int kStage = 64;                   // tokens staged per pass
constexpr int kUmmaM = 128;                  // M of every tcgen05.mma issued here
constexpr long long kWaitLimit = 1ll << 20;              // mbarrier polls before giving up,
constexpr unsigned long long kWaitNs = 2000000000ull;    // or 2 s of wall time, whichever first

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// UMMA shared-memory descriptor: K-major, no swizzle, core matrices of 8 rows x 16 B,
// K-adjacent core matrices 128 B apart (LBO), 8-row groups 512 B apart (SBO).
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) |
         ((uint64_t)(512u >> 4) << 32) | (1ull << 46);
}

// The same descriptor with other strides: K-adjacent core matrices lbo bytes apart, 8-row
// groups sbo bytes apart (both multiples of 16).
__device__ __forceinline__ uint64_t umma_desc_strided(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Byte offset of element (row, k) of a [rows x 32] bf16 K-major operand tile.
__host__ __device__ __forceinline__ uint32_t umma_off(int row, int k) {
  return (uint32_t)((row >> 3) * 512 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2);
}

// Instruction descriptor: kind::f16, A = B = bf16, D = f32, both K-major, M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kUmmaM >> 4) << 24);
}

// D[tmem] (+)= A B^T over one K = 16 step.
__device__ __forceinline__ void mma_k16(uint32_t tmem, uint32_t a_smem, uint32_t b_smem, uint32_t idesc,
                                        bool accumulate) {
  const uint64_t ad = umma_desc(a_smem), bd = umma_desc(b_smem);
  const uint32_t acc = accumulate ? 1u : 0u;
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem),
      "l"(ad), "l"(bd), "r"(idesc), "r"(acc));
}

// D[tmem] (+)= A B^T over K = 32 (two K = 16 steps; the second core-matrix pair is 256 B on).
__device__ __forceinline__ void mma_k32(uint32_t tmem, uint32_t a_smem, uint32_t b_smem, uint32_t idesc,
                                        bool accumulate) {
  mma_k16(tmem, a_smem, b_smem, idesc, accumulate);
  mma_k16(tmem, a_smem + 256, b_smem + 256, idesc, true);
}

// D[tmem] (+)= A B^T over one K = 16 step, with explicit descriptors.
__device__ __forceinline__ void mma_k16_desc(uint32_t tmem, uint64_t ad, uint64_t bd, uint32_t idesc, bool accumulate) {
  const uint32_t acc = accumulate ? 1u : 0u;
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem),
      "l"(ad), "l"(bd), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_commit(unsigned long long* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Bounded wait on an mbarrier phase; records a failure instead of hanging.
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for `phase` of an mbarrier, bounded: after kWaitLimit polls or limit_ns of wall time
// (the clock is read only once 256 polls have failed, so a normal wait never reads it) the
// wait gives up and sets *failed, which later waits see and return at once.
__device__ __forceinline__ void mbar_wait(unsigned long long* bar, uint32_t phase, int* failed,
                                          unsigned long long limit_ns = kWaitNs) {
  uint32_t done = *reinterpret_cast<volatile int*>(failed);
  long long polls = 0;
  unsigned long long t0 = 0;
  while (!done) {
    asm volatile(
        "{\n\t.reg .pred P1;\n\tmbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, P1;\n\t}\n"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(phase)
        : "memory");
    if (!done && (++polls & 255) == 0) {
      if (polls == 256) t0 = global_ns();
      if (polls > kWaitLimit || global_ns() - t0 > limit_ns) {
        *failed = 1;
        break;
      }
    }
  }
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tok_bar() {  // named barrier 1: the two token warps (64 threads)
  asm volatile("bar.sync 1, 64;" ::: "memory");
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

__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  return v;
}

// Gate scalars of one token from ||k||^2 (stabilized key), ||k - v||^2, a and beta:
// retention clamp, softplus step, injection cap (soft, or the hard clamp), spectral clamp.
// Returns whether the hard clamp is active (eta0 g > 1 - alpha_t); false for the soft cap.
__device__ __forceinline__ bool gate_scalars(float kn2, float dk2, float a, float beta, float alpha_max,
                                             float& al, float& eta, bool hard) {
  const float gain = sqrtf(dk2 * kn2);
  const float eb = __expf(-fabsf(beta));  // sigmoid without overflow
  const float sg = (beta >= 0.f) ? __fdividef(1.f, 1.f + eb) : __fdividef(eb, 1.f + eb);
  al = fminf(sg, alpha_max);
  const float eta0 = fmaxf(a, 0.f) + log1pf(__expf(-fabsf(a)));
  bool binds = false;
  if (hard) {
    binds = eta0 * gain > 1.f - al;
    eta = binds ? __fdividef(1.f - al, gain) : eta0;
  } else {
    const float zc = __fdividef(eta0 * gain, 1.f - al);
    const float phi = (zc < 1e-4f) ? (1.f - zc * zc * (1.f / 3.f)) : __fdividef(tanhf(zc), zc);
    eta = eta0 * phi;
  }
  if (eta * kn2 > 2.f) eta = __fdividef(2.f, kn2);
  return binds;
}

// Gates of one token from its generated row (k~[32], v[32], a, beta): kt becomes the
// stabilized key and vv becomes u.
__device__ __forceinline__ bool gates_row(float (&kt)[kD], float (&vv)[kD], float a, float beta,
                                          float alpha_max, float eps, float& al, float& eta, bool hard) {
  float n0 = 0.f, n1 = 0.f, n2 = 0.f, n3 = 0.f;
#pragma unroll
  for (int i = 0; i < kD; i += 4) {
    n0 = fmaf(kt[i], kt[i], n0);
    n1 = fmaf(kt[i + 1], kt[i + 1], n1);
    n2 = fmaf(kt[i + 2], kt[i + 2], n2);
    n3 = fmaf(kt[i + 3], kt[i + 3], n3);
  }
  const float inv = rsqrtf(((n0 + n1) + (n2 + n3)) + eps);
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
  const bool binds = gate_scalars(k0 + k1, d0 + d1, a, beta, alpha_max, al, eta, hard);
#pragma unroll
  for (int i = 0; i < kD; ++i) vv[i] = (1.f + al) * kt[i] - vv[i];
  return binds;
}

// Warp-wide count of active hard clamps, one atomic per warp (all lanes call it).
__device__ __forceinline__ void count_binds(bool binds, unsigned long long* counter) {
  const unsigned m = __ballot_sync(0xffffffffu, binds);
  if (counter != nullptr && (threadIdx.x & 31) == 0 && m != 0u) atomicAdd(counter, (unsigned long long)__popc(m));
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

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

}  // namespace
}  // namespace srnl
