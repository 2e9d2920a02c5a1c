// The VisionHOPE residual block around the SRNL operator (sm_100a), bf16 activations.
//
// Sources (web pages on VisionHOPE; none prints the block's equations):
//   "VisionHOPE: Visual Backbones as Self-Modifying Learning Systems", 2D-maps paragraph: a
//   standard two-branch residual, depthwise conv for local context, SRNL for long range, then
//   an FFN.  "VisionHOPE Model Overview", "Four-Directional Scanning and Spatial Chunking": the
//   residual blocks also hold projections, normalization, depthwise convolution and a
//   feed-forward network.  "VisionHOPE" README, "SRNL and VisionHOPE operator": the block keeps
//   the feature map's shape and mixer_dim sets its internal width.
// Reading (m = mixer_dim, channels-last):
//   u   = LN1(x) W_in^T + b_in                        [B, H, W, m]
//   mix = DWConv3x3(u) + operator(u)
//   y   = x + mix W_out^T + b_out
//   out = y + GELU(LN2(y) W_1^T + b_1) W_2^T + b_2    hidden width 4 dim
//
// Kernels: a warp-per-token LayerNorm; one tcgen05 GEMM (128-token tiles, K streamed in two
// 64-wide stages through shared memory, fp32 accumulate in TMEM, epilogue bias [+ GELU]
// [+ residual] to bf16) for the four projections; the depthwise convolution fused with the
// sum of the two branches; the operator through its own handle (srnl_scan_forward).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <string>
#include <vector>

#include "srnl_common.cuh"
#include "srnl_internal.h"
#include "srnl_launch.h"
#include "srnl_scan.h"
#include "srnl_umma.cuh"

namespace srnl {
namespace {

// ------------------------------------------------------------------ LayerNorm
// out[t][c] = (x[t][c] - mean_t) / sqrt(var_t + eps) * g[c] + b[c]; one warp per token,
// fp32 statistics (two passes over the values held in registers), bf16 in and out.
template <int PER>   // channels per lane: dim / 32
__global__ void layer_norm_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ g,
                                  const float* __restrict__ b, __nv_bfloat16* __restrict__ out, int64_t M,
                                  float eps) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= M) return;
  constexpr int D = 32 * PER;
  const __nv_bfloat16* row = x + t * D;
  float v[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) v[i] = __bfloat162float(row[i * 32 + lane]);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) s += v[i];
  const float mean = warp_sum(s) * (1.f / D);
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) q = fmaf(v[i] - mean, v[i] - mean, q);
  const float inv = rsqrtf(warp_sum(q) * (1.f / D) + eps);
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int c = i * 32 + lane;
    out[t * D + c] = __float2bfloat16_rn((v[i] - mean) * inv * g[c] + b[c]);
  }
}

// ------------------------------------------------------------------ GEMM on tcgen05
// out[M][N] = epi(A[M][K] W[N][K]^T): bias[n], then GELU (exact, v Phi(v)) when gelu, then
// + res[m][n] when res is given; bf16 out.  A CTA owns 128 rows x Nt columns (Nt = N or a
// 128 / 256 slice of it); K (a multiple of 32) streams through two shared-memory stages of up
// to 64 columns, loaded with 16-byte cp.async into K-major operand sub-tiles of 32, while the
// tensor cores work on the other stage.
constexpr int kGemmThreads = 128;
constexpr int kKc = 64;                  // K columns per stage
constexpr int kASub = kUmmaM * 64;      // [128 x 32] bf16 sub-tile

struct GemmTile {
  int Nt;
  uint32_t cols;
  size_t smem;
};

GemmTile gemm_tile(int N) {
  GemmTile t{0, 0, 0};
  if (N <= 0 || N % 16 != 0) return t;
  if (N <= 256) t.Nt = N;
  else if (N % 256 == 0) t.Nt = 256;
  else if (N % 128 == 0) t.Nt = 128;
  else return t;
  t.cols = 32;
  while ((int)t.cols < t.Nt) t.cols <<= 1;
  const size_t stage = 2 * (size_t)kASub + 2 * (size_t)t.Nt * 64;   // A and B for 64 columns of K
  t.smem = 2 * stage + 64;
  // at most 512 / cols CTAs per SM, so their TMEM allocations always fit
  const size_t floor_bytes = (size_t)228 * 1024 * t.cols / 512 - 1024;
  if (t.smem < floor_bytes) t.smem = floor_bytes;
  return t;
}

__device__ __forceinline__ float gelu_f(float v) { return 0.5f * v * (1.f + erff(v * 0.70710678118654752f)); }

__global__ void __launch_bounds__(kGemmThreads) gemm_tc_kernel(
    const __nv_bfloat16* __restrict__ A, const __nv_bfloat16* __restrict__ Wt, const float* __restrict__ bias,
    const __nv_bfloat16* __restrict__ res, __nv_bfloat16* __restrict__ out, int64_t M, int N, int K, int Nt,
    uint32_t cols, int gelu, int* err) {
  extern __shared__ __align__(128) unsigned char smem[];
  const size_t stage_bytes = 2 * (size_t)kASub + 2 * (size_t)Nt * 64;
  unsigned long long* mbar = reinterpret_cast<unsigned long long*>(smem + 2 * stage_bytes);   // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mbar + 2);
  int* failed = reinterpret_cast<int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t m0 = (int64_t)blockIdx.x * kUmmaM;
  const int n0 = blockIdx.y * Nt;
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    *failed = 0;
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&mbar[0])));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&mbar[1])));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  const uint32_t idesc = idesc_bf16(Nt);
  const int nkc = (K + kKc - 1) / kKc;
  uint32_t phase[2] = {0u, 0u};
  for (int kc = 0; kc < nkc; ++kc) {
    const int st = kc & 1;
    unsigned char* As = smem + st * stage_bytes;
    unsigned char* Bs = As + 2 * kASub;
    if (kc >= 2) {   // the MMAs of chunk kc - 2 have finished reading this stage
      mbar_wait(&mbar[st], phase[st], failed);
      phase[st] ^= 1u;
    }
    const int k0 = kc * kKc;
    const int runs = (K - k0 >= kKc) ? 8 : 4;   // 16-byte runs per row in this chunk (64 or 32 columns)
    for (int idx = tid; idx < kUmmaM * runs; idx += kGemmThreads) {
      const int row = idx / runs, k = (idx - row * runs) * 8;
      unsigned char* dst = As + (k >> 5) * kASub + umma_off(row, k & 31);
      if (m0 + row < M) cp_async16(dst, A + (m0 + row) * K + k0 + k);
      else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
    for (int idx = tid; idx < Nt * runs; idx += kGemmThreads) {
      const int o = idx / runs, k = (idx - o * runs) * 8;
      cp_async16(Bs + (k >> 5) * (Nt * 64) + umma_off(o, k & 31), Wt + (int64_t)(n0 + o) * K + k0 + k);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    cp_async_wait_all();
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (tid == 0) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      mma_k32(tmem, smem_u32(As), smem_u32(Bs), idesc, kc > 0);
      if (runs == 8) mma_k32(tmem, smem_u32(As + kASub), smem_u32(Bs + Nt * 64), idesc, true);
      mma_commit(&mbar[st]);
    }
  }
  // wait for the last chunk's products (the commit of chunk nkc - 1 covers every earlier MMA)
  {
    const int st = (nkc - 1) & 1;
    mbar_wait(&mbar[st], phase[st], failed);
  }
  const uint32_t lane_addr = tmem + ((uint32_t)(32 * warp) << 16);
  const int64_t row = m0 + tid;
  for (int n = 0; n < Nt; n += 16) {
    float v[16];
    SRNL_LD16(v, lane_addr + (uint32_t)n);
    tmem_wait_ld();
    if (row < M) {
      const int c0 = n0 + n;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        v[i] += bias[c0 + i];
        if (gelu) v[i] = gelu_f(v[i]);
      }
      if (res != nullptr) {
        const uint4* rp = reinterpret_cast<const uint4*>(res + row * N + c0);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint4 raw = rp[h];
          const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[i]));
            v[8 * h + 2 * i] += f.x;
            v[8 * h + 2 * i + 1] += f.y;
          }
        }
      }
      uint32_t pk[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const __nv_bfloat162 bb = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        pk[i] = *reinterpret_cast<const uint32_t*>(&bb);
      }
      uint4* dst = reinterpret_cast<uint4*>(out + row * N + c0);
      dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (tid == 0 && *failed) atomicExch(err, SRNL_E_TIMEOUT);
  if (warp == 0) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(cols));
  }
}

// ------------------------------------------------------------------ depthwise conv + branch sum
// mix[b][i][j][c] = dw_b[c] + sum_{di, dj} dw_w[c][di + 1][dj + 1] u[b][i + di][j + dj][c]
//                   + glob[b][i][j][c]     (zero padding); one thread per token and 8 channels.
__global__ void dwconv_add_kernel(const __nv_bfloat16* __restrict__ u, const __nv_bfloat16* __restrict__ glob,
                                  const float* __restrict__ w, const float* __restrict__ bias,
                                  __nv_bfloat16* __restrict__ mix, int B, int H, int W, int m) {
  const int groups = m / 8;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)B * H * W * groups;
  if (idx >= total) return;
  const int g = (int)(idx % groups);
  const int64_t tok = idx / groups;
  const int j = (int)(tok % W);
  const int i = (int)((tok / W) % H);
  const int64_t b = tok / ((int64_t)H * W);
  const int c0 = g * 8;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = bias[c0 + e];
#pragma unroll
  for (int di = -1; di <= 1; ++di) {
    const int ii = i + di;
    if (ii < 0 || ii >= H) continue;
#pragma unroll
    for (int dj = -1; dj <= 1; ++dj) {
      const int jj = j + dj;
      if (jj < 0 || jj >= W) continue;
      const uint4 raw = *reinterpret_cast<const uint4*>(u + (((b * H + ii) * W + jj) * m + c0));
      const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
        acc[2 * e] = fmaf(w[(c0 + 2 * e) * 9 + (di + 1) * 3 + (dj + 1)], f.x, acc[2 * e]);
        acc[2 * e + 1] = fmaf(w[(c0 + 2 * e + 1) * 9 + (di + 1) * 3 + (dj + 1)], f.y, acc[2 * e + 1]);
      }
    }
  }
  const uint4 graw = *reinterpret_cast<const uint4*>(glob + tok * m + c0);
  const uint32_t g4[4] = {graw.x, graw.y, graw.z, graw.w};
  uint32_t pk[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&g4[e]));
    const __nv_bfloat162 o = __floats2bfloat162_rn(acc[2 * e] + f.x, acc[2 * e + 1] + f.y);
    pk[e] = *reinterpret_cast<const uint32_t*>(&o);
  }
  *reinterpret_cast<uint4*>(mix + tok * m + c0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
}

cudaError_t launch_layer_norm(const void* x, const float* g, const float* b, void* out, int64_t M, int dim,
                              float eps, cudaStream_t s) {
  const unsigned blocks = (unsigned)((M + 7) / 8);
  const auto* xi = static_cast<const __nv_bfloat16*>(x);
  auto* o = static_cast<__nv_bfloat16*>(out);
  if (dim % 32 != 0) return cudaErrorInvalidValue;
  switch (dim / 32) {
#define SRNL_LN_CASE(n) \
  case n: layer_norm_kernel<n><<<blocks, 256, 0, s>>>(xi, g, b, o, M, eps); break;
    SRNL_LN_CASE(1) SRNL_LN_CASE(2) SRNL_LN_CASE(3) SRNL_LN_CASE(4) SRNL_LN_CASE(5) SRNL_LN_CASE(6)
    SRNL_LN_CASE(7) SRNL_LN_CASE(8) SRNL_LN_CASE(9) SRNL_LN_CASE(10) SRNL_LN_CASE(11) SRNL_LN_CASE(12)
    SRNL_LN_CASE(13) SRNL_LN_CASE(14) SRNL_LN_CASE(15) SRNL_LN_CASE(16)
#undef SRNL_LN_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_gemm(const void* A, const void* Wt, const float* bias, const void* res, void* out, int64_t M,
                        int N, int K, bool gelu, int* err, cudaStream_t s) {
  const GemmTile t = gemm_tile(N);
  if (t.Nt == 0 || K <= 0 || K % 32 != 0) return cudaErrorInvalidValue;
  dim3 grid((unsigned)((M + kUmmaM - 1) / kUmmaM), (unsigned)(N / t.Nt));
  gemm_tc_kernel<<<grid, kGemmThreads, t.smem, s>>>(
      static_cast<const __nv_bfloat16*>(A), static_cast<const __nv_bfloat16*>(Wt), bias,
      static_cast<const __nv_bfloat16*>(res), static_cast<__nv_bfloat16*>(out), M, N, K, t.Nt, t.cols, gelu ? 1 : 0,
      err);
  return cudaGetLastError();
}

cudaError_t launch_dwconv_add(const void* u, const void* glob, const float* w, const float* bias, void* mix, int B,
                              int H, int W, int m, cudaStream_t s) {
  const int64_t total = (int64_t)B * H * W * (m / 8);
  dwconv_add_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(u), static_cast<const __nv_bfloat16*>(glob), w, bias,
      static_cast<__nv_bfloat16*>(mix), B, H, W, m);
  return cudaGetLastError();
}

}  // namespace
}  // namespace srnl

// ------------------------------------------------------------------ C ABI
struct srnl_block {
  srnl_block_config cfg{};
  int device = 0;
  srnl_scan* op = nullptr;   // the operator at width mixer_dim
  // packed parameters: bf16 weights, fp32 vectors
  void *W_in = nullptr, *W_out = nullptr, *W_1 = nullptr, *W_2 = nullptr;
  float *ln1_g = nullptr, *ln1_b = nullptr, *b_in = nullptr, *dw_w = nullptr, *dw_b = nullptr;
  float *b_out = nullptr, *ln2_g = nullptr, *ln2_b = nullptr, *b_1 = nullptr, *b_2 = nullptr;
  // workspace (bf16): normalised input, u, operator output, branch sum, first residual, hidden
  void *xn = nullptr, *u = nullptr, *glob = nullptr, *mix = nullptr, *y1 = nullptr, *hid = nullptr;
  int* dev_err = nullptr;
  std::string err;
};

namespace {

srnl_status block_fail(srnl_block* h, srnl_status st, const std::string& msg) {
  if (h != nullptr) h->err = msg;
  srnl::set_thread_error(msg);
  return st;
}

void block_free(srnl_block* h) {
  void* ptrs[] = {h->W_in, h->W_out, h->W_1, h->W_2, h->ln1_g, h->ln1_b, h->b_in, h->dw_w, h->dw_b, h->b_out,
                  h->ln2_g, h->ln2_b, h->b_1, h->b_2, h->xn, h->u, h->glob, h->mix, h->y1, h->hid, h->dev_err};
  for (void* p : ptrs)
    if (p != nullptr) cudaFree(p);
  if (h->op != nullptr) srnl_scan_destroy(h->op);
}

cudaError_t upload_f32(float** dst, const float* src, size_t n) {
  cudaError_t e = cudaMalloc(dst, n * sizeof(float));
  if (e == cudaSuccess) e = cudaMemcpy(*dst, src, n * sizeof(float), cudaMemcpyHostToDevice);
  return e;
}

cudaError_t upload_bf16(void** dst, const float* src, size_t n) {
  std::vector<__nv_bfloat16> tmp(n);
  for (size_t i = 0; i < n; ++i) tmp[i] = __float2bfloat16_rn(src[i]);
  cudaError_t e = cudaMalloc(dst, n * sizeof(__nv_bfloat16));
  if (e == cudaSuccess) e = cudaMemcpy(*dst, tmp.data(), n * sizeof(__nv_bfloat16), cudaMemcpyHostToDevice);
  return e;
}

}  // namespace

extern "C" {

srnl_status srnl_block_create(srnl_block** out, const srnl_block_config* cfg, const srnl_block_params* p) {
  srnl::set_thread_error("");
  if (out == nullptr || cfg == nullptr || p == nullptr) return block_fail(nullptr, SRNL_E_INVAL, "NULL argument");
  *out = nullptr;
  const srnl_block_config& c = *cfg;
  if (c.B <= 0 || c.H <= 0 || c.W <= 0) return block_fail(nullptr, SRNL_E_INVAL, "B, H and W must be positive");
  if (c.dim <= 0 || c.dim % 32 != 0 || c.dim > 512)
    return block_fail(nullptr, SRNL_E_UNSUPPORTED, "dim must be a multiple of 32, at most 512");
  if (c.mixer_dim <= 0 || c.mixer_dim % 32 != 0 || c.mixer_dim > 512)
    return block_fail(nullptr, SRNL_E_UNSUPPORTED, "mixer_dim must be a multiple of 32, at most 512");
  if (c.head_dim <= 0 || c.mixer_dim % c.head_dim != 0)
    return block_fail(nullptr, SRNL_E_INVAL, "mixer_dim must be a multiple of head_dim");
  if (!(c.ln_eps > 0.f)) return block_fail(nullptr, SRNL_E_INVAL, "ln_eps must be positive");
  if (c.act_dtype != SRNL_BF16) return block_fail(nullptr, SRNL_E_UNSUPPORTED, "the block takes bf16 activations");
  const float* need[] = {p->ln1_g, p->ln1_b, p->W_in, p->b_in, p->dw_w, p->dw_b, p->W_out, p->b_out,
                         p->ln2_g, p->ln2_b, p->W_1, p->b_1, p->W_2, p->b_2};
  for (const float* q : need)
    if (q == nullptr) return block_fail(nullptr, SRNL_E_INVAL, "a block parameter pointer is NULL");
  srnl_scan_config oc{};
  oc.B = c.B; oc.H = c.H; oc.W = c.W; oc.C = c.mixer_dim; oc.heads = c.mixer_dim / c.head_dim; oc.d = c.head_dim;
  oc.alpha = c.alpha; oc.eps = c.eps; oc.chunk_row = c.chunk_row; oc.chunk_col = c.chunk_col;
  oc.act_dtype = SRNL_BF16; oc.gen_dtype = c.gen_dtype; oc.injection_cap = c.injection_cap;
  srnl_block* h = new srnl_block();
  h->cfg = c;
  cudaGetDevice(&h->device);
  srnl_status st = srnl_scan_create(&h->op, &oc, &p->op);
  if (st != SRNL_OK) {
    const std::string msg = std::string("operator: ") + srnl_scan_last_error(nullptr);
    delete h;
    return block_fail(nullptr, st, msg);
  }
  const size_t D = c.dim, m = c.mixer_dim, hid = 4 * D;
  const size_t M = (size_t)c.B * c.H * c.W;
  cudaError_t e = cudaSuccess;
  if (e == cudaSuccess) e = upload_bf16(&h->W_in, p->W_in, m * D);
  if (e == cudaSuccess) e = upload_bf16(&h->W_out, p->W_out, D * m);
  if (e == cudaSuccess) e = upload_bf16(&h->W_1, p->W_1, hid * D);
  if (e == cudaSuccess) e = upload_bf16(&h->W_2, p->W_2, D * hid);
  if (e == cudaSuccess) e = upload_f32(&h->ln1_g, p->ln1_g, D);
  if (e == cudaSuccess) e = upload_f32(&h->ln1_b, p->ln1_b, D);
  if (e == cudaSuccess) e = upload_f32(&h->b_in, p->b_in, m);
  if (e == cudaSuccess) e = upload_f32(&h->dw_w, p->dw_w, m * 9);
  if (e == cudaSuccess) e = upload_f32(&h->dw_b, p->dw_b, m);
  if (e == cudaSuccess) e = upload_f32(&h->b_out, p->b_out, D);
  if (e == cudaSuccess) e = upload_f32(&h->ln2_g, p->ln2_g, D);
  if (e == cudaSuccess) e = upload_f32(&h->ln2_b, p->ln2_b, D);
  if (e == cudaSuccess) e = upload_f32(&h->b_1, p->b_1, hid);
  if (e == cudaSuccess) e = upload_f32(&h->b_2, p->b_2, D);
  const size_t bf = sizeof(__nv_bfloat16);
  if (e == cudaSuccess) e = cudaMalloc(&h->xn, M * D * bf);
  if (e == cudaSuccess) e = cudaMalloc(&h->u, M * m * bf);
  if (e == cudaSuccess) e = cudaMalloc(&h->glob, M * m * bf);
  if (e == cudaSuccess) e = cudaMalloc(&h->mix, M * m * bf);
  if (e == cudaSuccess) e = cudaMalloc(&h->y1, M * D * bf);
  if (e == cudaSuccess) e = cudaMalloc(&h->hid, M * hid * bf);
  if (e == cudaSuccess) e = cudaMalloc(&h->dev_err, sizeof(int));
  if (e == cudaSuccess) e = cudaMemset(h->dev_err, 0, sizeof(int));
  if (e == cudaSuccess) e = srnl::prepare_block_kernels();
  if (e != cudaSuccess) {
    const std::string msg = std::string("block create: ") + cudaGetErrorString(e);
    block_free(h);
    delete h;
    return block_fail(nullptr, e == cudaErrorMemoryAllocation ? SRNL_E_NOMEM : SRNL_E_CUDA, msg);
  }
  *out = h;
  return SRNL_OK;
}

srnl_status srnl_block_forward(srnl_block* h, const void* x, void* y, void* stream) {
  if (h == nullptr) return block_fail(nullptr, SRNL_E_INVAL, "handle is NULL");
  h->err.clear();
  if (x == nullptr || y == nullptr) return block_fail(h, SRNL_E_INVAL, "x or y is NULL");
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(y) & 15u))
    return block_fail(h, SRNL_E_INVAL, "x and y must be 16-byte aligned");
  const srnl_block_config& c = h->cfg;
  const int64_t M = (int64_t)c.B * c.H * c.W;
  const size_t bytes = (size_t)M * c.dim * 2;
  {
    const uintptr_t xa = reinterpret_cast<uintptr_t>(x), ya = reinterpret_cast<uintptr_t>(y);
    if (xa < ya + bytes && ya < xa + bytes) return block_fail(h, SRNL_E_INVAL, "x and y overlap");
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = c.dim, m = c.mixer_dim, hid = 4 * c.dim;
  cudaError_t e = srnl::launch_layer_norm(x, h->ln1_g, h->ln1_b, h->xn, M, D, c.ln_eps, s);
  if (e == cudaSuccess) e = srnl::launch_gemm(h->xn, h->W_in, h->b_in, nullptr, h->u, M, m, D, false, h->dev_err, s);
  if (e != cudaSuccess) return block_fail(h, SRNL_E_CUDA, std::string("block launch: ") + cudaGetErrorString(e));
  srnl_status st = srnl_scan_forward(h->op, h->u, h->glob, nullptr, stream);
  if (st != SRNL_OK) return block_fail(h, st, std::string("operator: ") + srnl_scan_last_error(h->op));
  e = srnl::launch_dwconv_add(h->u, h->glob, h->dw_w, h->dw_b, h->mix, c.B, c.H, c.W, m, s);
  if (e == cudaSuccess) e = srnl::launch_gemm(h->mix, h->W_out, h->b_out, x, h->y1, M, D, m, false, h->dev_err, s);
  if (e == cudaSuccess) e = srnl::launch_layer_norm(h->y1, h->ln2_g, h->ln2_b, h->xn, M, D, c.ln_eps, s);
  if (e == cudaSuccess) e = srnl::launch_gemm(h->xn, h->W_1, h->b_1, nullptr, h->hid, M, hid, D, true, h->dev_err, s);
  if (e == cudaSuccess) e = srnl::launch_gemm(h->hid, h->W_2, h->b_2, h->y1, y, M, D, hid, false, h->dev_err, s);
  if (e != cudaSuccess) return block_fail(h, SRNL_E_CUDA, std::string("block launch: ") + cudaGetErrorString(e));
  return SRNL_OK;
}

srnl_status srnl_block_device_status(srnl_block* h) {
  if (h == nullptr) return block_fail(nullptr, SRNL_E_INVAL, "handle is NULL");
  int v = 0;
  const cudaError_t e = cudaMemcpy(&v, h->dev_err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return block_fail(h, SRNL_E_CUDA, std::string("status read: ") + cudaGetErrorString(e));
  if (v != 0) return block_fail(h, static_cast<srnl_status>(v), "a bounded in-kernel wait gave up");
  return srnl_scan_device_status(h->op);
}

const char* srnl_block_last_error(const srnl_block* h) {
  return h != nullptr ? h->err.c_str() : srnl_scan_last_error(nullptr);
}

void srnl_block_destroy(srnl_block* h) {
  if (h == nullptr) return;
  int prev = -1;
  if (cudaGetDevice(&prev) == cudaSuccess && prev != h->device) cudaSetDevice(h->device);
  cudaDeviceSynchronize();
  block_free(h);
  if (prev >= 0 && prev != h->device) cudaSetDevice(prev);
  delete h;
}

}  // extern "C"

namespace srnl {
cudaError_t prepare_block_kernels() {
  return cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
}
}  // namespace srnl
