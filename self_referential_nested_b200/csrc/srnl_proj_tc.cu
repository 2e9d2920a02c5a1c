// Query projection q = x W_q^T on the tensor cores (bf16 activations and bf16 W_q, fp32
// accumulate, bf16 q).  The projection is the one dense contraction outside the scan that
// all four routes share ("VisionHOPE: Visual Backbones as Self-Modifying Learning Systems",
// caveats paragraph: the query projection sits outside the recurrent loop).
//
// One CTA computes a 128-token x Nc-channel tile: x rows and W_q rows are copied with
// cp.async straight into UMMA K-major operand tiles (K = C in sub-tiles of 32), one
// thread issues C / 16 tcgen05.mma into TMEM, and the four warps drain their 32 TMEM lanes
// (one token each), round to bf16 and store 16-byte runs of q.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "srnl_common.cuh"
#include "srnl_launch.h"
#include "srnl_scan.h"
#include "srnl_umma.cuh"

namespace srnl {
namespace {

constexpr int kPjThreads = 128;  // four warps: TMEM lanes 0..127 = the tile's tokens
constexpr int kPjSub = kUmmaM * 64;  // one [128 x 32] bf16 operand sub-tile

struct ProjTile {
  int Nc;          // output channels per CTA
  uint32_t cols;   // TMEM columns allocated (power of two >= Nc)
  size_t smem;     // dynamic shared memory per CTA
};

// Output-channel tile for C: the whole row when C <= 256, else 128-channel tiles
// (C a multiple of 128).  Nc = 0: no tensor-core tiling for this C.
ProjTile proj_tile(int C) {
  ProjTile t{0, 0, 0};
  if (C % 32 != 0 || C <= 0) return t;
  if (C <= 256) t.Nc = C;
  else if (C % 128 == 0) t.Nc = 128;
  else return t;
  t.cols = 32;
  while ((int)t.cols < t.Nc) t.cols <<= 1;
  const size_t nk = (size_t)C / 32;
  const size_t need = nk * kPjSub + nk * (size_t)t.Nc * 64 + 64;
  // at most 512 / cols CTAs per SM: their TMEM allocations always fit
  const size_t floor_bytes = (size_t)228 * 1024 * t.cols / 512 - 1024;
  t.smem = need > floor_bytes ? need : floor_bytes;
  if (t.smem > (size_t)227 * 1024) t = ProjTile{0, 0, 0};  // operand panels do not fit
  return t;
}

__global__ void __launch_bounds__(kPjThreads) query_projection_tc_kernel(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ wq, __nv_bfloat16* __restrict__ q,
    int64_t M, int C, int Nc, uint32_t cols, int* err) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int nk = C / 32;
  unsigned char* A = smem;                                   // nk sub-tiles of [128 x 32]
  unsigned char* Bt = smem + (size_t)nk * kPjSub;            // nk sub-tiles of [Nc x 32]
  unsigned long long* mbar = reinterpret_cast<unsigned long long*>(Bt + (size_t)nk * Nc * 64);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mbar + 1);
  int* failed = reinterpret_cast<int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t m0 = (int64_t)blockIdx.x * kUmmaM;
  const int n0 = blockIdx.y * Nc;
  const int c8n = C / 8;  // 16-byte runs per row

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    *failed = 0;
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(mbar)));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int idx = tid; idx < kUmmaM * c8n; idx += kPjThreads) {
    const int row = idx / c8n, k = (idx - row * c8n) * 8;
    unsigned char* dst = A + (k >> 5) * kPjSub + umma_off(row, k & 31);
    if (m0 + row < M) cp_async16(dst, x + (m0 + row) * C + k);
    else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
  }
  for (int idx = tid; idx < Nc * c8n; idx += kPjThreads) {
    const int o = idx / c8n, k = (idx - o * c8n) * 8;
    cp_async16(Bt + (k >> 5) * (Nc * 64) + umma_off(o, k & 31), wq + (int64_t)(n0 + o) * C + k);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  cp_async_wait_all();
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  if (tid == 0) {
    const uint32_t idesc = idesc_bf16(Nc);
    for (int kk = 0; kk < nk; ++kk)
      mma_k32(tmem, smem_u32(A + kk * kPjSub), smem_u32(Bt + (size_t)kk * Nc * 64), idesc, kk > 0);
    mma_commit(mbar);
  }
  mbar_wait(mbar, 0u, failed);
  // drain: thread = token (TMEM lane), 16 channels per load
  const uint32_t lane_addr = tmem + ((uint32_t)(32 * warp) << 16);
  const int64_t row = m0 + tid;
  for (int n = 0; n < Nc; n += 16) {
    float v[16];
    SRNL_LD16(v, lane_addr + (uint32_t)n);
    tmem_wait_ld();
    if (row < M) {
      uint32_t pk[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        pk[i] = *reinterpret_cast<const uint32_t*>(&b);
      }
      uint4* dst = reinterpret_cast<uint4*>(q + row * C + n0 + n);
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

// Persistent, pipelined variant for C <= 128 (the whole output row in one tile): each CTA
// loads W_q once, then walks 128-token tiles with two x stages and two TMEM buffers, so that
// tile i + 2 loads and tile i + 1 multiplies while tile i drains:
//   iteration i:  wait x(i + 1), issue MMA(i + 1) -> TMEM buffer (i + 1) & 1
//                 wait MMA(i); load x(i + 2) into the stage tile i used
//                 drain tile i from TMEM buffer i & 1 to bf16 rows in shared memory, in q's own
//                 layout, and write them back with one bulk copy (the tile's rows are
//                 contiguous in q), instead of 16-byte stores that scatter over 32 rows
constexpr int kPpStages = 2;

__global__ void __launch_bounds__(kPjThreads) query_projection_tc_pipelined_kernel(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ wq, __nv_bfloat16* __restrict__ q,
    int64_t M, int C, int* err) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int nk = C / 32;
  const size_t stage_bytes = (size_t)nk * kPjSub;
  unsigned char* Bt = smem;                                          // nk sub-tiles of [C x 32]
  unsigned char* Xs = smem + (size_t)nk * C * 64;                    // kPpStages x nk sub-tiles
  unsigned char* Os = Xs + kPpStages * stage_bytes;                  // [128][C] bf16 output rows
  unsigned long long* mbar = reinterpret_cast<unsigned long long*>(Os + (size_t)kUmmaM * C * 2);   // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mbar + 2);
  int* failed = reinterpret_cast<int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t ntiles = (M + kUmmaM - 1) / kUmmaM;
  const int64_t first = blockIdx.x;
  const int64_t count = first < ntiles ? (ntiles - 1 - first) / gridDim.x + 1 : 0;
  const int c8n = C / 8;
  uint32_t cols = 32;
  while ((int)cols < 2 * C) cols <<= 1;

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
  auto load_x = [&](int64_t i) {   // tile number i of this CTA into stage i & 1 (one cp.async group)
    const int64_t m0 = (first + i * gridDim.x) * kUmmaM;
    unsigned char* A = Xs + (i & 1) * stage_bytes;
    for (int idx = tid; idx < kUmmaM * c8n; idx += kPjThreads) {
      const int row = idx / c8n, k = (idx - row * c8n) * 8;
      unsigned char* dst = A + (k >> 5) * kPjSub + umma_off(row, k & 31);
      if (m0 + row < M) cp_async16(dst, x + (m0 + row) * C + k);
      else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  auto issue_mma = [&](int64_t i, uint32_t tmem) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const unsigned char* A = Xs + (i & 1) * stage_bytes;
    const uint32_t idesc = idesc_bf16(C);
    for (int kk = 0; kk < nk; ++kk)
      mma_k32(tmem + (uint32_t)((i & 1) * C), smem_u32(A + kk * kPjSub), smem_u32(Bt + (size_t)kk * C * 64), idesc,
              kk > 0);
    mma_commit(&mbar[i & 1]);
  };
  // W_q and the first tile (one group), the second tile (another)
  for (int idx = tid; idx < C * c8n; idx += kPjThreads) {
    const int o = idx / c8n, k = (idx - o * c8n) * 8;
    cp_async16(Bt + (k >> 5) * (C * 64) + umma_off(o, k & 31), wq + (int64_t)o * C + k);
  }
  if (count > 0) load_x(0);
  else asm volatile("cp.async.commit_group;" ::: "memory");
  if (count > 1) load_x(1);
  else asm volatile("cp.async.commit_group;" ::: "memory");
  asm volatile("cp.async.wait_group 1;" ::: "memory");   // W_q and tile 0
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  const uint32_t tmem = *tmem_slot;
  if (tid == 0 && count > 0) issue_mma(0, tmem);
  const uint32_t lane_addr = tmem + ((uint32_t)(32 * warp) << 16);
  for (int64_t i = 0; i < count; ++i) {
    if (i + 1 < count) {   // tile i + 1 is loaded: multiply it while tile i drains
      asm volatile("cp.async.wait_group 0;" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncthreads();
      if (tid == 0) issue_mma(i + 1, tmem);
    }
    mbar_wait(&mbar[i & 1], (uint32_t)((i >> 1) & 1), failed);
    if (i + 2 < count) load_x(i + 2);   // stage i & 1 is free: MMA(i) has completed
    if (i > 0) {   // the previous tile's bulk store has finished reading the output rows
      if (tid == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      __syncthreads();
    }
    const int64_t m0 = (first + i * gridDim.x) * kUmmaM;
    for (int n = 0; n < C; n += 16) {
      float v[16];
      SRNL_LD16(v, lane_addr + (uint32_t)((i & 1) * C + n));
      tmem_wait_ld();
      uint32_t pk[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
        pk[e] = *reinterpret_cast<const uint32_t*>(&b);
      }
      uint4* dst = reinterpret_cast<uint4*>(Os + ((size_t)tid * C + n) * 2);
      dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the rows, before the bulk copy reads them
    __syncthreads();
    if (tid == 0) {
      const int64_t rows = (M - m0 < kUmmaM) ? (M - m0) : kUmmaM;
      asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(q + m0 * C),
                   "r"(smem_u32(Os)), "r"((uint32_t)(rows * C * 2))
                   : "memory");
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
  }
  if (tid == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");   // q written before the kernel ends
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (tid == 0 && *failed) atomicExch(err, SRNL_E_TIMEOUT);
  if (warp == 0) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(cols));
  }
}

size_t pipelined_smem(int C) {
  const size_t nk = (size_t)C / 32;
  return nk * C * 64 + kPpStages * nk * kPjSub + (size_t)kUmmaM * C * 2 + 64;
}

}  // namespace

bool query_projection_tc_supported(const ScanGeom& g) {
  return g.act_bf16 && g.gen_bf16 && proj_tile(g.C).Nc > 0;
}

cudaError_t prepare_projection_kernel() {
  cudaError_t e = cudaFuncSetAttribute(query_projection_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       227 * 1024);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(query_projection_tc_pipelined_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             227 * 1024);
  return e;
}

cudaError_t launch_query_projection_tc(const ScanGeom& g, const ScanParamsDev& p, const void* x, void* q,
                                       int* err, cudaStream_t s) {
  const int64_t M = (int64_t)g.B * g.H * g.W;
  if (g.C <= 128) {
    // persistent: TMEM (2 C columns, rounded up to a power of two) and shared memory bound the
    // CTAs per SM; every SM holds up to two, each walking several tiles
    uint32_t cols = 32;
    while ((int)cols < 2 * g.C) cols <<= 1;
    const int per_sm_tmem = 512 / (int)cols;
    const size_t sm_bytes = pipelined_smem(g.C);
    const int per_sm_smem = (int)((size_t)(228 * 1024) / (sm_bytes + 1024));
    // two per SM measured best at S1 (20.9 us, against 22.4 with three and 24.7 with one)
    const int per_sm = std::max(1, std::min(std::min(per_sm_tmem, per_sm_smem), 2));
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t ntiles = (M + kUmmaM - 1) / kUmmaM;
    const int64_t grid = std::min<int64_t>(ntiles, (int64_t)sms * per_sm);
    // shared memory sized so that at most per_sm CTAs share an SM (their TMEM always fits)
    const size_t smem = std::max(sm_bytes, (size_t)(228 * 1024) / per_sm - 1024);
    query_projection_tc_pipelined_kernel<<<(unsigned)grid, kPjThreads, smem, s>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(p.Wqb),
        static_cast<__nv_bfloat16*>(q), M, g.C, err);
    return cudaGetLastError();
  }
  const ProjTile t = proj_tile(g.C);
  dim3 grid((unsigned)((M + kUmmaM - 1) / kUmmaM), (unsigned)(g.C / t.Nc));
  query_projection_tc_kernel<<<grid, kPjThreads, t.smem, s>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(p.Wqb),
      static_cast<__nv_bfloat16*>(q), M, g.C, t.Nc, t.cols, err);
  return cudaGetLastError();
}

}  // namespace srnl
