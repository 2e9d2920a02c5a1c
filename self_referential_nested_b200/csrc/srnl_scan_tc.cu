// SRNL four-direction chunked scan, bf16-generation path (sm_100a): the token-order
// write in chunkwise form on the tensor cores.
//
// Method sources (web pages on VisionHOPE; no page prints an equation):
//   "VisionHOPE: Visual Backbones as Self-Modifying Learning Systems" (summary
//   of arXiv 2609.33325) - write-rule, stability and 2D-maps paragraphs;
//   "VisionHOPE Model Overview: Architecture, Benchmarks, and Practical
//   Limits" - "Four-Directional Scanning and Spatial Chunking"; "VisionHOPE"
//   README - "SRNL and VisionHOPE operator".
//
// Single-product form: every write right-multiplies all memories by
// T_t = alpha_t I - eta_t u_t k_t^T (u_t = (1 + alpha_t) k_t - v_t), so a sequence
// carries one d x d product Q, generation reads w_t = Q_b x_t (Q_b: Q at the chunk
// boundary) and the readout is y_t = M_mem0 Q_t q_t.
//
// Chunkwise write.  Inside a stage (up to 64 tokens of one chunk) all gates are
// known before the first write, because generation only reads the boundary state.
// For one row rho of Q (rho_s: the row at stage start) and the base-2 prefix
// Lambda_t = sum_{m <= t} log2 alpha_m (Lambda_{-1} = 0), g(j, t) = 2^(Lambda_t - Lambda_j):
//   rho_t = 2^Lambda_t rho_s - sum_{j <= t} g(j, t) eta_j s_j k_j,   s_t = rho_{t-1} . u_t
// hence the s_t of every row solve one unit lower-triangular system that all rows share,
//   s_t + sum_{j < t} A[t][j] s_j = 2^Lambda_{t-1} (rho_s . u_t),  A[t][j] = g(j, t-1) eta_j (u_t . k_j),
// and the readout and the stage-end rows are products:
//   z_t   = 2^Lambda_t (rho_s . q_t) - sum_{j <= t} g(j, t) eta_j (q_t . k_j) s_j
//   rho_e = 2^Lambda_{T-1} rho_s - sum_j g(j, T-1) eta_j s_j k_j.
// Only ratios g <= 1 of the retention products appear, so nothing overflows when a
// retention gate is tiny.
//
// One CTA owns one (route, batch, head) sequence; 192 threads.  Warp w runs on SMSP w % 4
// and reads TMEM lanes 32 (w % 4) .. + 31, which fixes who can drain which accumulator rows:
//   warps 0-1  solve warps: -A from TMEM lanes 0..63 (warp 0 its diagonal 32 x 32 block; warp 1
//              its diagonal block and, factored at the split point 31, the columns below 32,
//              also written as the coupling operand A_21); warp 0 then solves the stage's
//              triangular system with one row of Q per lane (tokens 0..31, the tensor-core
//              coupling, tokens 32..) and forms the stage-end Q; warp 1 issues the next
//              stage's TMA boxes during the gates
//   warps 2-3  readout warps: half of the gate vector work (tokens repeated in TMEM lanes
//              64..127), the readout coefficients from lanes 64..127 during -A and the solve,
//              z_t and the Y product of the previous stage
//   warps 4-5  token warps: boundary products and generation, the gate scalars, the
//              retention prefix, the other half of the gate vector work, the right-hand sides,
//              y_t of the previous stage, and the next stage's x and q out of the TMA staging
// Tensor-core products per stage (tcgen05, M = 128, fp32 accumulate in TMEM; an fp32
// operand is split into bf16 hi + lo and a product of two such takes three MMAs):
//   W    [x] Q_b^T                      N = 32   w_t = Q_b x_t
//   Gen  [w] G^T                        N = 80   [k~ v a beta]_t
//   M1   [u; q] [k; Q_s]^T              N = 96   u.k, Q_s u, q.k, Q_s q
//   C    (-S_1) (-A_21)^T               N = 32   the first 32 tokens' share of the others' solve
//   Z    [Kd^T; -; Mz^T] (-S)^T         N = 32   stage-end correction and z_t - 2^Lambda_t Q_s q_t
//   Y    [z] M_mem0^T                   N = 32   y_t
// TMEM holds two 128-column halves; consecutive stages alternate, so the readout of
// one stage overlaps the generation of the next.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "srnl_common.cuh"
#include "srnl_launch.h"
#include "srnl_scan.h"
#include "srnl_umma.cuh"

namespace srnl {
namespace {

constexpr int kThreadsTc = 192;
constexpr int kTile = kUmmaM * 64;      // 128 rows x 32 bf16: one K = 32 operand tile
// The Z product's A operand tiles space their K-adjacent core matrices 144 B apart (not 128):
// the scalar column stores of Kd^T (lanes = consecutive K) then fall in distinct banks.
constexpr uint32_t kZCore = 144;                       // LBO: K-adjacent core matrices
constexpr uint32_t kZGroup = 4 * kZCore;               // SBO: 8-row groups (576 B)
constexpr int kTileZ = (kUmmaM / 8) * kZGroup;         // 9216 B per K = 32 sub-tile
constexpr int kB1Rows = 96;             // M1 B operand: 64 keys + 32 rows of Q_s
constexpr uint32_t kTmemColsTc = 256;   // two halves of 128 columns
constexpr uint32_t kColM1 = 0;          // W, Gen, M1 and Y accumulate from column 0 of a half
constexpr uint32_t kColZ0 = 64;         // M1 columns 64..95: Q_s u_t / Q_s q_t
constexpr uint32_t kColZ = 96;          // Z accumulator

struct alignas(128) TcSmem {
  // x tile (token t in rows t and 64 + t); after the W product it holds w in bf16
  alignas(128) unsigned char xa[kTile];
  // M1 A operand: rows 0..63 u_t, rows 64..127 q_t (bf16, exact: its low part stays zero)
  alignas(128) unsigned char a1h[kTile];
  alignas(128) unsigned char a1l[kTile];
  // M1 B operand: rows 0..63 k_j, rows 64..95 Q_s (row r, K = column)
  alignas(128) unsigned char b1h[kB1Rows * 64];
  alignas(128) unsigned char b1l[kB1Rows * 64];
  // Z A operand, K halves j < 32 and j >= 32: rows 0..31 Kd^T, rows 32..63 free,
  // rows 64..127 Mz^T.  Rows 32..63 hold the right-hand sides b^T during the solve.
  alignas(128) unsigned char zah[2][kTileZ];
  alignas(128) unsigned char zal[2][kTileZ];
  // Z B operand: -S (row r, K = token j)
  alignas(128) unsigned char zbh[2][kD * 64];
  alignas(128) unsigned char zbl[2][kD * 64];
  // Y A operand: z_t rows 0..63; the MMA's rows 64..127 read the next 4 KB (unused lanes)
  alignas(128) unsigned char yah[64 * 64];
  alignas(128) unsigned char yal[64 * 64];
  // the other head's 32 channels of the stage's x rows (rows 0..63), the second K half of the
  // in-kernel query product when it is fused (its M = 128 read continues into mh / ml)
  alignas(128) unsigned char xo[64 * 64];
  alignas(128) unsigned char mh[kD * 64];      // M_mem0 hi (row = output channel)
  alignas(128) unsigned char ml[kD * 64];      // M_mem0 lo
  alignas(128) unsigned char gb[80 * 64];      // G in bf16 (rows 66..79 zero)
  // Q_b hi and lo (the W product's B operand when a chunk spans several stages); when every
  // chunk fits one stage they are unused and, with the query product fused, hold this head's
  // 32 rows of W_q in bf16 (K = channels 0..31 in qbh, 32..63 in qbl)
  alignas(128) unsigned char qbh[kD * 64];
  alignas(128) unsigned char qbl[kD * 64];
  alignas(16) float qsT[kD][kD + 1];            // Q_s transposed, fp32 (column c in row c)
  alignas(16) float lam[kStage];                // Lambda_t (log2 retention prefix)
  alignas(16) float eta[kStage];
  alignas(16) float cf32[32];                   // 2^(Lambda_31 - Lambda_j) eta_j for j < 32
  alignas(16) float scale[kD];
  alignas(16) float4 gpart[kStage];            // readout-warp halves of ||k~||^2, k~.v, ||v||^2
  alignas(16) float4 gpar[kStage];             // gate scalars: 1/||k~||, alpha, g(t, T-1) eta, live
  float wsum;                                   // prefix of the first token warp
  alignas(8) unsigned long long mbar_w, mbar_g, mbar_1, mbar_z, mbar_y, mbar_c, mbar_x, mbar_q;
  uint32_t tmem_base;
  int wait_failed;
};
static_assert(sizeof(TcSmem) <= 113 * 1024, "two CTAs per SM");
static_assert(offsetof(TcSmem, yal) + 2 * 64 * 64 <= sizeof(TcSmem), "Y operand rows 64..127 stay in bounds");
static_assert(offsetof(TcSmem, xo) + 2 * 64 * 64 <= sizeof(TcSmem), "query operand rows 64..127 stay in bounds");
static_assert(offsetof(TcSmem, qbl) == offsetof(TcSmem, qbh) + kD * 64, "W_q slice halves");
static_assert(offsetof(TcSmem, a1l) == offsetof(TcSmem, a1h) + kTile, "A pieces");
static_assert(offsetof(TcSmem, b1h) == offsetof(TcSmem, a1h) + 2 * kTile, "A pieces");
static_assert(offsetof(TcSmem, b1l) == offsetof(TcSmem, b1h) + kB1Rows * 64, "A pieces");
static_assert(offsetof(TcSmem, zal) == offsetof(TcSmem, zah) + 2 * kTileZ, "b pieces");

struct TcArgs {
  const void* x;
  const __nv_bfloat16* q;
  float* yr;
  float* finals;
  int* err;
  unsigned long long* binds;  // hard-clamp activations (nullptr: not counted)
  const float* G;
  const float* Mm;
  const float* scales;
  int B, H, W, C, heads, Lrow, Lcol;
  float alpha, eps;
  bool act_bf16;
  bool hard_cap;
  const __nv_bfloat16* Wqb;   // W_q [C][C] in bf16 (read when fuse_q)
  bool fuse_q;                // q computed here from full-width x rows (C = 64, chunks <= 64)
};

// Tensor maps of the bf16 activations and queries, [B][H][W][C]: "row" views tokens as one
// dimension (B*H*W tokens of C channels; a stage of a row route is consecutive tokens) and
// "col" as [B*H][W][C] (a stage of a column route is one column j: consecutive i at stride
// W*C).  Boxes are 32 channels (one head) by 64 tokens.
struct TcMaps {
  CUtensorMap xr, xc, qr, qc;
  uint32_t box_bytes_r, box_bytes_c;   // bytes of one x box (= one q box) per orientation
  int box_ch;                          // channels per x box: 32 (one head), or C with the fused query
};

// -A[t][j] for j in [16p, 16p + 16) lives in the first 4 KB of a1h, a1l, b1h, b1l
// (p = 0..3): the u and k rows of M1, dead between M1 and the next stage's gates.
__device__ __forceinline__ float* neg_a_row(TcSmem& sm, int j) {
  const int p = j >> 4;
  unsigned char* base = p < 2 ? sm.a1h + p * kTile : sm.b1h + (p - 2) * (kB1Rows * 64);
  return reinterpret_cast<float*>(base) + (j & 15) * kStage;
}

__device__ __forceinline__ const float* neg_a_col(const TcSmem& sm, int j) {
  const int p = j >> 4;
  const unsigned char* base = p < 2 ? sm.a1h + p * kTile : sm.b1h + (p - 2) * (kB1Rows * 64);
  return reinterpret_cast<const float*>(base) + (j & 15) * kStage;
}

// b^T[r][t] (right-hand sides) in rows 32..63 of the four Z A sub-tiles, 64 floats per row r.
// The 16-byte chunks of a row are permuted by r & 7 (rhs_chunk), so that the solve warp's
// lanes r reading the same chunk index hit distinct banks.
__device__ __forceinline__ float* rhs_row(TcSmem& sm, int r) {
  return reinterpret_cast<float*>(&sm.zah[0][0] + (r >> 3) * kTileZ + 4 * kZGroup) + (r & 7) * kStage;
}
static_assert(8 * kStage * 4 <= 4 * (int)kZGroup, "right-hand sides fit in rows 32..63 of a Z A sub-tile");

// Byte offset of element (row, k) of a Z A sub-tile (the padded layout above).
__device__ __forceinline__ uint32_t zoff(int row, int k) {
  return (uint32_t)((row >> 3) * kZGroup + (k >> 3) * kZCore + (row & 7) * 16 + (k & 7) * 2);
}

// Offset in floats of chunk i (tokens 4i .. 4i + 3) in row r of the right-hand sides.
__device__ __forceinline__ int rhs_chunk(int r, int i) { return (i ^ (r & 7)) << 2; }

// 8 fp32 values -> bf16 hi and lo, each one 16-byte core-matrix row.
__device__ __forceinline__ void split8(const float* v, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 bh = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    const float2 fh = __bfloat1622float2(bh);
    const __nv_bfloat162 bl = __floats2bfloat162_rn(v[2 * i] - fh.x, v[2 * i + 1] - fh.y);
    h[i] = *reinterpret_cast<const uint32_t*>(&bh);
    l[i] = *reinterpret_cast<const uint32_t*>(&bl);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Row `row` (32 fp32 values) of a K = 32 operand tile, as bf16 hi and lo.
__device__ __forceinline__ void store_row_split(unsigned char* th, unsigned char* tl, int row, const float* v) {
#pragma unroll
  for (int c = 0; c < kD; c += 8) {
    uint4 hi, lo;
    split8(v + c, hi, lo);
    *reinterpret_cast<uint4*>(th + umma_off(row, c)) = hi;
    *reinterpret_cast<uint4*>(tl + umma_off(row, c)) = lo;
  }
}

// 2^x on the MUFU (ex2.approx.ftz): the retention ratios g(j, t) <= 1 need no more, and a
// ratio below 2^-126 is a decay to zero.
__device__ __forceinline__ float exp2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Columns [c0, c0 + 16) of row `row` of a K = 32 operand tile, as bf16 hi and lo.
__device__ __forceinline__ void store_half_split(unsigned char* th, unsigned char* tl, int row, int c0,
                                                 const float* v) {
#pragma unroll
  for (int c = 0; c < 16; c += 8) {
    uint4 hi, lo;
    split8(v + c, hi, lo);
    *reinterpret_cast<uint4*>(th + umma_off(row, c0 + c)) = hi;
    *reinterpret_cast<uint4*>(tl + umma_off(row, c0 + c)) = lo;
  }
}

__device__ __forceinline__ void named_bar_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Forward substitution of one row of the stage's shared unit lower-triangular system over the
// tokens [BASE, BASE + TB), on the lane that owns the row: b[i] holds the right-hand side of
// token BASE + i, already reduced by every earlier token's contribution, and leaves as its
// solution s.  No value crosses lanes: the columns of -A are read with broadcast loads (every
// lane of the warp reads the same address).  Blocks of 4 columns J:
//   - the 4 x 4 diagonal block is solved in registers (s_j = b_j, then the later b of the block);
//   - the next block's 4 right-hand sides take block J's contribution first (the chain);
//   - the remaining rows take it afterwards, off the chain.
// The -A values the chain needs (the next block's diagonal block and its coupling to block J)
// are loaded one block ahead.  TB is a multiple of 8; past the stage's tokens the right-hand
// sides and the columns of A are zero, so those s stay zero.
template <int TB>
__device__ __forceinline__ void solve_block(const TcSmem& sm, float (&b)[TB], int BASE) {
  constexpr int NB = TB / 4;
  // dg[i] = -A[j0 .. j0 + 3][j0 + i] (i = 0..2): the diagonal block of block J (rows as a float4)
  // cp[i] = -A[j0 + 4 .. j0 + 7][j0 + i] (i = 0..3): block J's columns on the next block's rows
  float4 dg[3], cp[4];
#pragma unroll
  for (int i = 0; i < 3; ++i) dg[i] = *reinterpret_cast<const float4*>(neg_a_col(sm, BASE + i) + BASE);
  if (NB > 1) {
#pragma unroll
    for (int i = 0; i < 4; ++i) cp[i] = *reinterpret_cast<const float4*>(neg_a_col(sm, BASE + i) + BASE + 4);
  }
#pragma unroll
  for (int J = 0; J < NB; ++J) {
    const int j0 = 4 * J;   // local index; the token is BASE + j0
    b[j0 + 1] = fmaf(dg[0].y, b[j0], b[j0 + 1]);
    b[j0 + 2] = fmaf(dg[0].z, b[j0], b[j0 + 2]);
    b[j0 + 3] = fmaf(dg[0].w, b[j0], b[j0 + 3]);
    b[j0 + 2] = fmaf(dg[1].z, b[j0 + 1], b[j0 + 2]);
    b[j0 + 3] = fmaf(dg[1].w, b[j0 + 1], b[j0 + 3]);
    b[j0 + 3] = fmaf(dg[2].w, b[j0 + 2], b[j0 + 3]);
    if (J + 1 < NB) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 s2 = f2(b[j0 + i], b[j0 + i]);
        const float2 lo = __ffma2_rn(f2(cp[i].x, cp[i].y), s2, f2(b[j0 + 4], b[j0 + 5]));
        const float2 hi = __ffma2_rn(f2(cp[i].z, cp[i].w), s2, f2(b[j0 + 6], b[j0 + 7]));
        b[j0 + 4] = lo.x; b[j0 + 5] = lo.y; b[j0 + 6] = hi.x; b[j0 + 7] = hi.y;
      }
#pragma unroll
      for (int i = 0; i < 3; ++i)
        dg[i] = *reinterpret_cast<const float4*>(neg_a_col(sm, BASE + j0 + 4 + i) + BASE + j0 + 4);
      if (J + 2 < NB) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          cp[i] = *reinterpret_cast<const float4*>(neg_a_col(sm, BASE + j0 + 4 + i) + BASE + j0 + 8);
      }
#pragma unroll
      for (int t4 = J + 2; t4 < NB; ++t4) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 av = *reinterpret_cast<const float4*>(neg_a_col(sm, BASE + j0 + i) + BASE + 4 * t4);
          const float2 s2 = f2(b[j0 + i], b[j0 + i]);
          const float2 lo = __ffma2_rn(f2(av.x, av.y), s2, f2(b[4 * t4], b[4 * t4 + 1]));
          const float2 hi = __ffma2_rn(f2(av.z, av.w), s2, f2(b[4 * t4 + 2], b[4 * t4 + 3]));
          b[4 * t4] = lo.x; b[4 * t4 + 1] = lo.y; b[4 * t4 + 2] = hi.x; b[4 * t4 + 3] = hi.y;
        }
      }
    }
  }
}

// Right-hand sides of tokens [BASE, BASE + TB) of row r from shared memory.
template <int TB>
__device__ __forceinline__ void load_rhs(TcSmem& sm, int r, float (&b)[TB], int BASE) {
  const float* src = rhs_row(sm, r);
#pragma unroll
  for (int i = 0; i < TB / 4; ++i) {
    const float4 v = *reinterpret_cast<const float4*>(src + rhs_chunk(r, BASE / 4 + i));
    b[4 * i] = v.x; b[4 * i + 1] = v.y; b[4 * i + 2] = v.z; b[4 * i + 3] = v.w;
  }
}

// -S of tokens [BASE, BASE + 32) of row r into the Z B operand (row r, K = token), one
// core-matrix row per 8 tokens, hi and lo; zeros past TB (the Z product contracts over all 64).
template <int TB>
__device__ __forceinline__ void store_neg_s(TcSmem& sm, int r, const float (&b)[TB], int BASE) {
#pragma unroll
  for (int g8 = 0; g8 < 4; ++g8) {
    uint4 hi = make_uint4(0u, 0u, 0u, 0u), lo = hi;
    if (8 * g8 < TB) {
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = -b[8 * g8 + i];
      split8(v, hi, lo);
    }
    *reinterpret_cast<uint4*>(sm.zbh[BASE / 32] + umma_off(r, 8 * g8)) = hi;
    *reinterpret_cast<uint4*>(sm.zbl[BASE / 32] + umma_off(r, 8 * g8)) = lo;
  }
}

// Zeros for -S of tokens [BASE, BASE + 32) of row r (tokens past the stage).
__device__ __forceinline__ void store_neg_s_zero(TcSmem& sm, int r, int BASE) {
#pragma unroll
  for (int g8 = 0; g8 < 4; ++g8) {
    *reinterpret_cast<uint4*>(sm.zbh[BASE / 32] + umma_off(r, 8 * g8)) = make_uint4(0u, 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(sm.zbl[BASE / 32] + umma_off(r, 8 * g8)) = make_uint4(0u, 0u, 0u, 0u);
  }
}

// Tokens [BASE, BASE + 32) of row r (BASE = 0 or 32): right-hand sides (reduced by the coupling
// c of the first 32 tokens when BASE = 32), solve, -S.  Both halves run the same instance, so
// the code fetched for the first half serves the second.
template <int TB>
__device__ __forceinline__ void solve_half(TcSmem& sm, int r, int BASE, const float* c) {
  float b[TB];
  load_rhs<TB>(sm, r, b, BASE);
  if (c != nullptr) {
#pragma unroll
    for (int i = 0; i < TB; ++i) b[i] -= c[i];
  }
  solve_block<TB>(sm, b, BASE);
  store_neg_s<TB>(sm, r, b, BASE);
}

// One token's scaled route partial (32 channels of one head) at element offset `off` of the
// partial buffer: bf16 when the activations are bf16 (the fusion's output precision), else fp32.
__device__ __forceinline__ void store_partial(float* yr, int64_t off, const float* scale, const float (&y)[kD],
                                              bool bf16) {
  if (bf16) {
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(yr) + off);
#pragma unroll
    for (int i = 0; i < kD; i += 8) {
      uint32_t w4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(scale[i + 2 * e] * y[i + 2 * e], scale[i + 2 * e + 1] * y[i + 2 * e + 1]);
        w4[e] = *reinterpret_cast<const uint32_t*>(&b);
      }
      dst[i / 8] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
  } else {
    float* dst = yr + off;
#pragma unroll
    for (int i = 0; i < kD; i += 4)
      *reinterpret_cast<float4*>(dst + i) =
          make_float4(scale[i] * y[i], scale[i + 1] * y[i + 1], scale[i + 2] * y[i + 2], scale[i + 3] * y[i + 3]);
  }
}

// Number of stages that hold tokens: only the last chunk can be short.
__device__ __forceinline__ int live_stages(int N, int L) {
  const int per = (L + kStage - 1) / kStage;
  const int chunks = (N + L - 1) / L;
  const int last = N - (chunks - 1) * L;
  return (chunks - 1) * per + (last + kStage - 1) / kStage;
}

// Token warps: asynchronous copies of a stage's x head slices (into rows t and 64 + t of the
// x tile; fp32 activations are rounded to bf16) and q head slices (into rows 64.. of the M1 A tile).
__device__ __forceinline__ void tc_prefetch(TcSmem& sm, const StageInfo& si, const TcArgs& a, int r,
                                            int64_t tok0, int ch0, int ht) {
  for (int idx = ht; idx < si.T * 4; idx += 64) {
    const int tt = idx >> 2, part = idx & 3;
    const int p = route_pos(r, si.t0 + tt, a.H, a.W);
    const __nv_bfloat16* src = a.q + (tok0 + p) * a.C + ch0 + part * 8;
    cp_async16(sm.a1h + umma_off(64 + tt, part * 8), src);
  }
  if (a.act_bf16) {
    for (int idx = ht; idx < si.T * 4; idx += 64) {
      const int tt = idx >> 2, part = idx & 3;
      const int p = route_pos(r, si.t0 + tt, a.H, a.W);
      const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(a.x) + (tok0 + p) * a.C + ch0 + part * 8;
      cp_async16(sm.xa + umma_off(tt, part * 8), src);
      cp_async16(sm.xa + umma_off(64 + tt, part * 8), src);
    }
  } else {
    for (int idx = ht; idx < si.T * 4; idx += 64) {
      const int tt = idx >> 2, part = idx & 3;
      const int p = route_pos(r, si.t0 + tt, a.H, a.W);
      const float* src = reinterpret_cast<const float*>(a.x) + (tok0 + p) * a.C + ch0 + part * 8;
      const float4 v0 = *reinterpret_cast<const float4*>(src);
      const float4 v1 = *reinterpret_cast<const float4*>(src + 4);
      const __nv_bfloat162 b0 = __floats2bfloat162_rn(v0.x, v0.y), b1 = __floats2bfloat162_rn(v0.z, v0.w);
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(v1.x, v1.y), b3 = __floats2bfloat162_rn(v1.z, v1.w);
      uint4 raw;
      raw.x = *reinterpret_cast<const uint32_t*>(&b0); raw.y = *reinterpret_cast<const uint32_t*>(&b1);
      raw.z = *reinterpret_cast<const uint32_t*>(&b2); raw.w = *reinterpret_cast<const uint32_t*>(&b3);
      *reinterpret_cast<uint4*>(sm.xa + umma_off(tt, part * 8)) = raw;
      *reinterpret_cast<uint4*>(sm.xa + umma_off(64 + tt, part * 8)) = raw;
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// One thread: the stage's x and q boxes into the staging area (the Y operand tiles, dead
// between the Y product's completion and the next z), completing on mbar_x.  A box holds the
// orientation's chunk length rounded up to 8 tokens, at most 64.  Row routes load from the
// stage's lowest raster index p_lo on; column routes the rows of column j from i_lo on.  Boxes may run past the image or the tensor (the rest is unused; TMA
// fills what lies outside the tensor with zeros).  Coordinates: channels ch0 (a multiple of
// 32, so 64-byte aligned), then tokens; never negative.
__device__ __forceinline__ void tma_stage(TcSmem& sm, const TcMaps& m, const StageInfo& si, int r, int b, int ch0,
                                          int H, int W) {
  const uint32_t bar = smem_u32(&sm.mbar_x);
  const uint32_t box = r < 2 ? m.box_bytes_r : m.box_bytes_c;
  const bool full = m.box_ch != kD;   // the fused query: full-width x rows, no q box
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(full ? box : 2 * box)
               : "memory");
  if (full) ch0 = 0;
  const int t_lo = (r & 1) ? si.t0 + si.T - 1 : si.t0;      // route token at the lowest address
  const int p = route_pos(r, t_lo, H, W);
  if (r < 2) {
    const int c1 = b * H * W + p;
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(sm.yah)), "l"(reinterpret_cast<uint64_t>(&m.xr)), "r"(ch0), "r"(c1), "r"(bar)
        : "memory");
    if (!full)
      asm volatile(
          "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
              smem_u32(sm.yal)), "l"(reinterpret_cast<uint64_t>(&m.qr)), "r"(ch0), "r"(c1), "r"(bar)
          : "memory");
  } else {
    const int i = p / W, j = p - i * W;
    const int c2 = b * H + i;
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
            smem_u32(sm.yah)), "l"(reinterpret_cast<uint64_t>(&m.xc)), "r"(ch0), "r"(j), "r"(c2), "r"(bar)
        : "memory");
    if (!full)
      asm volatile(
          "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
              smem_u32(sm.yal)), "l"(reinterpret_cast<uint64_t>(&m.qc)), "r"(ch0), "r"(j), "r"(c2), "r"(bar)
          : "memory");
  }
}

// Whether a stage's tokens form one box: always on the row routes (consecutive raster
// indices); on the column routes when they lie in one column (the default chunks are whole
// columns; an overridden chunk length may cross a column boundary, and such a stage is
// copied token by token instead).  The reverse column route walks the same columns.
__device__ __forceinline__ bool stage_is_box(const StageInfo& si, int r, int H) {
  return r < 2 || si.t0 / H == (si.t0 + si.T - 1) / H;
}

// Token warps (ht = 0..63): the staged boxes (64-byte rows, ascending raster order) into the
// operand tiles in route order: x into rows t and 64 + t of the x tile, q into rows 64 + t of
// the M1 A tile (with the fused query: the other head's x channels into xo instead), for the
// stage's T tokens (the rows past them keep earlier tokens, which every
// consumer masks).  Reverse routes read the box backwards.
__device__ __forceinline__ void unstage(TcSmem& sm, const StageInfo& si, int r, int ht, bool fused, int h) {
  if (fused) {   // full-width rows (128 B): this head's channels to the x tile, the other head's to xo
    for (int idx = ht; idx < si.T * 4; idx += 64) {
      const int t = idx >> 2, part = idx & 3;
      const int row = (r & 1) ? si.T - 1 - t : t;
      const uint4 own = *reinterpret_cast<const uint4*>(sm.yah + row * 128 + h * 64 + part * 16);
      const uint4 oth = *reinterpret_cast<const uint4*>(sm.yah + row * 128 + (1 - h) * 64 + part * 16);
      *reinterpret_cast<uint4*>(sm.xa + umma_off(t, part * 8)) = own;
      *reinterpret_cast<uint4*>(sm.xa + umma_off(64 + t, part * 8)) = own;
      *reinterpret_cast<uint4*>(sm.xo + umma_off(t, part * 8)) = oth;
    }
    return;
  }
  for (int idx = ht; idx < si.T * 4; idx += 64) {
    const int t = idx >> 2, part = idx & 3;
    const int row = (r & 1) ? si.T - 1 - t : t;
    const uint4 xv = *reinterpret_cast<const uint4*>(sm.yah + row * 64 + part * 16);
    const uint4 qv = *reinterpret_cast<const uint4*>(sm.yal + row * 64 + part * 16);
    *reinterpret_cast<uint4*>(sm.xa + umma_off(t, part * 8)) = xv;
    *reinterpret_cast<uint4*>(sm.xa + umma_off(64 + t, part * 8)) = xv;
    *reinterpret_cast<uint4*>(sm.a1h + umma_off(64 + t, part * 8)) = qv;
  }
}

// Token warps (ht = 0..63), fused query only: q_t = x_t W_q[h]^T for the staged stage (x of
// channels 0..31 and 32..63 as the two K halves, this head's W_q rows in the Q_b tiles), on the
// tensor cores into 32 columns of TMEM (lanes = tokens), then rounded to bf16 into rows 64 + t
// of the M1 A tile, as the separate projection kernel would have left them.  The K order
// (channels 0..31 first) is the projection kernel's.  query_issue starts the product;
// query_drain waits for it and stores q, so other work can sit between the two.
__device__ __forceinline__ void query_issue(TcSmem& sm, uint32_t tmem, uint32_t col, int h, int ht) {
  fence_async_smem();
  tc_fence_before();
  tok_bar();
  if (ht == 0) {
    tc_fence_after();
    const uint32_t lo = smem_u32(h == 0 ? sm.xa : sm.xo), hi = smem_u32(h == 0 ? sm.xo : sm.xa);
    mma_k32(tmem + col, lo, smem_u32(sm.qbh), idesc_bf16(32), false);
    mma_k32(tmem + col, hi, smem_u32(sm.qbl), idesc_bf16(32), true);
    mma_commit(&sm.mbar_q);
  }
}

__device__ __forceinline__ void query_drain(TcSmem& sm, uint32_t tmem_lane, uint32_t col, int T, int ht,
                                            uint32_t& qpar) {
  mbar_wait(&sm.mbar_q, qpar, &sm.wait_failed);
  qpar ^= 1u;
  float qv[kD];
  SRNL_LD16(qv, tmem_lane + col);
  SRNL_LD16(qv + 16, tmem_lane + col + 16);
  tmem_wait_ld();
  if (ht < T) {
#pragma unroll
    for (int c = 0; c < kD; c += 8) {
      uint32_t w4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(qv[c + 2 * e], qv[c + 2 * e + 1]);
        w4[e] = *reinterpret_cast<const uint32_t*>(&b2);
      }
      *reinterpret_cast<uint4*>(sm.a1h + umma_off(64 + ht, c)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
  }
  fence_async_smem();
}

__global__ void __launch_bounds__(kThreadsTc, 2) srnl_scan_chunkwise_kernel(const TcArgs a,
                                                                       const __grid_constant__ TcMaps maps) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  TcSmem& sm = *reinterpret_cast<TcSmem*>(smem_raw);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const bool is_s = warp < 2;                  // solve warps (TMEM lanes 0..63)
  const bool is_r = warp == 2 || warp == 3;    // readout warps (TMEM lanes 64..127)
  const bool is_k = warp >= 4;                 // token warps (TMEM lanes 0..63)

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

  // ---- set-up: zero the operand tiles, constants, Q_s = Q_b = I
  {
    uint4* z = reinterpret_cast<uint4*>(&sm);
    const int n16 = (int)(offsetof(TcSmem, qsT) / 16);
    for (int i = tid; i < n16; i += kThreadsTc) z[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_async_smem();   // the zeros land before any tensor copy into the same tiles
  }
  if (tid == 0) {
    sm.wait_failed = 0;
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.mbar_w)));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.mbar_g)));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.mbar_1)));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.mbar_z)));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.mbar_y)));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.mbar_c)));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.mbar_x)));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.mbar_q)));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&sm.tmem_base)),
                 "r"(kTmemColsTc));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  __syncthreads();
  for (int i = tid; i < kD * kD; i += kThreadsTc) {
    const int o = i / kD, kk = i % kD;
    store_split(sm.mh, sm.ml, o, kk, Msrc[i]);
    const float e = (o == kk) ? 1.f : 0.f;
    if (!a.fuse_q) store_split(sm.qbh, sm.qbl, o, kk, e);   // fused: the tiles hold W_q instead
    store_split(sm.b1h, sm.b1l, 64 + o, kk, e);
    sm.qsT[o][kk] = e;
  }
  for (int i = tid; i < 80 * kD; i += kThreadsTc) {
    const int n = i / kD, kk = i % kD;
    store_bf16(sm.gb, n, kk, n < kGen ? Gsrc[n * kD + kk] : 0.f);
  }
  if (tid < kD) sm.scale[tid] = a.scales[r * a.C + ch0 + tid];

  const int nst = live_stages(N, L);
  if (tid == 32 && a.act_bf16) {   // the tensor maps into the descriptor cache before first use
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.xr)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.xc)) : "memory");
    if (!a.fuse_q) {   // with the fused query the q maps are not encoded
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.qr)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.qc)) : "memory");
    }
  }
  uint32_t xpar = 0;   // phase of mbar_x (token warps)
  uint32_t qpar = 0;   // phase of mbar_q (token warps)
  if (is_k && nst > 0) {
    const StageInfo s0 = stage_info(0, N, L);
    if (a.fuse_q) {   // this head's W_q rows (bf16), K halves in qbh / qbl
      for (int i = tid - 128; i < kD * 64; i += 64) {
        const int o = i >> 6, k = i & 63;
        *reinterpret_cast<__nv_bfloat16*>((k < 32 ? sm.qbh : sm.qbl) + umma_off(o, k & 31)) =
            a.Wqb[(int64_t)(ch0 + o) * a.C + k];
      }
    }
    if (a.act_bf16 && stage_is_box(s0, r, a.H)) {
      if (tid == 128) tma_stage(sm, maps, s0, r, b, ch0, a.H, a.W);
      mbar_wait(&sm.mbar_x, xpar, &sm.wait_failed);
      xpar ^= 1u;
      unstage(sm, s0, r, tid - 128, a.fuse_q, h);
      if (a.fuse_q) {
        query_issue(sm, sm.tmem_base, 32u, h, tid - 128);
        query_drain(sm, sm.tmem_base + ((uint32_t)(32 * (warp & 3)) << 16), 32u, s0.T, tid - 128, qpar);
      }
    } else {
      tc_prefetch(sm, s0, a, r, tok0, ch0, tid - 128);
      cp_async_wait_all();
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = sm.tmem_base;
  const uint32_t tmem_lane = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
  const uint32_t idesc32 = idesc_bf16(32), idesc80 = idesc_bf16(80), idesc96 = idesc_bf16(96);
  // A chunk within one stage makes every stage open a chunk: Q_b is then Q_s, and W reads
  // its operand from rows 64..95 of the M1 B tiles.
  const bool qb_is_qs = L <= kStage;
  const uint32_t wb_hi = qb_is_qs ? smem_u32(sm.b1h) + 64 * 64 : smem_u32(sm.qbh);
  const uint32_t wb_lo = qb_is_qs ? smem_u32(sm.b1l) + 64 * 64 : smem_u32(sm.qbl);

  // readout warps: the stage whose z / y is still to be produced
  uint32_t cpar = 0;   // phase of mbar_c (warp 0)
  bool pend = false;
  StageInfo pst{0, 0, 0};
  uint32_t phb = 0;
  float ct_pend = 0.f;

  for (int ne = 0; ne < nst; ++ne) {
    const StageInfo si = stage_info(ne, N, L);
    const int T = si.T;
    const uint32_t hb = (uint32_t)(ne & 1) * 128u;
    const uint32_t par = (uint32_t)(ne & 1);

    // ---- (A) generation.  Token warps: boundary products, generation, the gate scalars and
    // the retention prefix.  Readout warps: z and the Y product of the previous stage.  Both
    // then share every token's key / value columns (the generation tile repeats the tokens in
    // rows 64..127, so the readout warps find them in their own TMEM lanes).
    if (is_k || is_r) {
      const int t = is_k ? tid - 128 : tid - 64;  // token (TMEM lane t, or 64 + t)
      const int c0 = is_k ? 0 : 16;               // this thread's half of the key and value columns
      if (is_k) {
        if (t == 0) {
          tc_fence_after();
          mma_k32(tmem + hb + kColM1, smem_u32(sm.xa), wb_hi, idesc32, false);
          mma_k32(tmem + hb + kColM1, smem_u32(sm.xa), wb_lo, idesc32, true);
          mma_commit(&sm.mbar_w);
        }
        mbar_wait(&sm.mbar_w, par, &sm.wait_failed);
        float wv[kD];
        SRNL_LD16(wv, tmem_lane + hb + kColM1);
        SRNL_LD16(wv + 16, tmem_lane + hb + kColM1 + 16);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < kD; c += 8) {
          const __nv_bfloat162 b0 = __floats2bfloat162_rn(wv[c], wv[c + 1]);
          const __nv_bfloat162 b1 = __floats2bfloat162_rn(wv[c + 2], wv[c + 3]);
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(wv[c + 4], wv[c + 5]);
          const __nv_bfloat162 b3 = __floats2bfloat162_rn(wv[c + 6], wv[c + 7]);
          uint4 raw;
          raw.x = *reinterpret_cast<const uint32_t*>(&b0); raw.y = *reinterpret_cast<const uint32_t*>(&b1);
          raw.z = *reinterpret_cast<const uint32_t*>(&b2); raw.w = *reinterpret_cast<const uint32_t*>(&b3);
          *reinterpret_cast<uint4*>(sm.xa + umma_off(t, c)) = raw;
          *reinterpret_cast<uint4*>(sm.xa + umma_off(64 + t, c)) = raw;
        }
        fence_async_smem();
        tc_fence_before();
        tok_bar();
        if (t == 0) {
          tc_fence_after();
          mma_k32(tmem + hb + kColM1, smem_u32(sm.xa), smem_u32(sm.gb), idesc80, false);
          mma_commit(&sm.mbar_g);
        }
      } else if (pend) {  // z and the Y product of the previous stage
        mbar_wait(&sm.mbar_z, (uint32_t)((ne - 1) & 1), &sm.wait_failed);
        float z0[kD], zm[kD];
        SRNL_LD16(z0, tmem_lane + phb + kColZ0);
        SRNL_LD16(z0 + 16, tmem_lane + phb + kColZ0 + 16);
        SRNL_LD16(zm, tmem_lane + phb + kColZ);
        SRNL_LD16(zm + 16, tmem_lane + phb + kColZ + 16);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < kD; ++i) z0[i] = fmaf(ct_pend, z0[i], zm[i]);
        store_row_split(sm.yah, sm.yal, t, z0);
        fence_async_smem();
        tc_fence_before();
        named_bar(4, 64);
        if (t == 0) {
          tc_fence_after();
          mma_k32(tmem + phb + kColM1, smem_u32(sm.yah), smem_u32(sm.mh), idesc32, false);
          mma_k32(tmem + phb + kColM1, smem_u32(sm.yah), smem_u32(sm.ml), idesc32, true);
          mma_k32(tmem + phb + kColM1, smem_u32(sm.yal), smem_u32(sm.mh), idesc32, true);
          mma_commit(&sm.mbar_y);
        }
      }
      mbar_wait(&sm.mbar_g, par, &sm.wait_failed);
      float kt[16], vv[16], ga = 0.f, gbeta = 0.f;
      SRNL_LD16(kt, tmem_lane + hb + kColM1 + c0);
      SRNL_LD16(vv, tmem_lane + hb + kColM1 + 32 + c0);
      if (is_k)
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];"
                     : "=f"(ga), "=f"(gbeta)
                     : "r"(tmem_lane + hb + kColM1 + 64u));
      tmem_wait_ld();
      float nk0 = 0.f, nk1 = 0.f, kv0 = 0.f, kv1 = 0.f, nv0 = 0.f, nv1 = 0.f;
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        nk0 = fmaf(kt[i], kt[i], nk0); nk1 = fmaf(kt[i + 1], kt[i + 1], nk1);
        kv0 = fmaf(kt[i], vv[i], kv0); kv1 = fmaf(kt[i + 1], vv[i + 1], kv1);
        nv0 = fmaf(vv[i], vv[i], nv0); nv1 = fmaf(vv[i + 1], vv[i + 1], nv1);
      }
      if (is_r) sm.gpart[t] = make_float4(nk0 + nk1, kv0 + kv1, nv0 + nv1, 0.f);
      named_bar(6, 128);  // warps 2-5
      if (is_k) {
        const float4 o = sm.gpart[t];
        const float nk = (nk0 + nk1) + o.x, kv = (kv0 + kv1) + o.y, nv = (nv0 + nv1) + o.z;
        const bool live = t < T;
        float l2a = 0.f, et = 0.f, al = 1.f, inv = 0.f;
        bool binds = false;
        if (live) {
          inv = rsqrtf(nk + a.eps);
          // ||k||^2 and ||k - v||^2 of the stabilized key k = inv k~
          const float kn2 = nk * inv * inv;
          const float dk2 = fmaxf(fmaf(inv, fmaf(-2.f, kv, inv * nk), nv), 0.f);
          binds = gate_scalars(kn2, dk2, ga, gbeta, a.alpha, al, et, a.hard_cap);
          l2a = fmaxf(log2f(al), -126.f);  // a retention that underflows acts as 2^-126
        }
        if (a.hard_cap) count_binds(binds, a.binds);
        sm.eta[t] = et;
        // inclusive prefix of log2 alpha over the stage
        float pre = l2a;
#pragma unroll
        for (int o2 = 1; o2 < 32; o2 <<= 1) {
          const float v = __shfl_up_sync(0xffffffffu, pre, o2);
          if (lane >= o2) pre += v;
        }
        if (t == 31) sm.wsum = pre;
        tok_bar();
        if (t >= 32) pre += sm.wsum;
        sm.lam[t] = pre;
        tok_bar();
        const float gk = live ? exp2_fast(sm.lam[T - 1] - pre) * et : 0.f;
        sm.gpar[t] = make_float4(inv, al, gk, live ? 1.f : 0.f);
        if (t < 32) sm.cf32[t] = exp2_fast(sm.lam[31] - pre) * et;   // 2^(Lambda_31 - Lambda_t) eta_t
      }
      named_bar(7, 128);
      {
        const float4 gp = sm.gpar[t];  // (1/||k~||, alpha, g(t, T-1) eta_t, live)
        const float up = 1.f + gp.y;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          kt[i] *= gp.x;                                  // k_t (zero past the stage)
          vv[i] = gp.w != 0.f ? up * kt[i] - vv[i] : 0.f;  // u_t
        }
        store_half_split(sm.a1h, sm.a1l, t, c0, vv);
        store_half_split(sm.b1h, sm.b1l, t, c0, kt);
        // Kd^T[c][j] = g(j, T-1) eta_j k_j[c]: column j = t, rows c0..c0 + 15 of Z A
        unsigned char* zh = sm.zah[t >> 5];
        unsigned char* zl = sm.zal[t >> 5];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float v = gp.z * kt[c];
          const __nv_bfloat16 hi = __float2bfloat16_rn(v);
          *reinterpret_cast<__nv_bfloat16*>(zh + zoff(c0 + c, t & 31)) = hi;
          *reinterpret_cast<__nv_bfloat16*>(zl + zoff(c0 + c, t & 31)) = __float2bfloat16_rn(v - __bfloat162float(hi));
        }
      }
      fence_async_smem();
    } else if (tid == 32 && ne + 1 < nst) {
      // warp 1 is idle here: the next stage's x and q boxes, as soon as the Y product (issued
      // by the readout warps for the previous stage) has finished reading the staging area
      const StageInfo sn = stage_info(ne + 1, N, L);
      if (a.act_bf16 && stage_is_box(sn, r, a.H)) {
        if (pend) mbar_wait(&sm.mbar_y, (uint32_t)((ne - 1) & 1), &sm.wait_failed);
        tma_stage(sm, maps, sn, r, b, ch0, a.H, a.W);
      }
    }
    tc_fence_before();
    __syncthreads();
    // ---- (C) M1 = [u; q] [k; Q_s]^T
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ah = smem_u32(sm.a1h), al = smem_u32(sm.a1l);
      const uint32_t bh = smem_u32(sm.b1h), bl = smem_u32(sm.b1l);
      mma_k32(tmem + hb + kColM1, ah, bh, idesc96, false);
      mma_k32(tmem + hb + kColM1, ah, bl, idesc96, true);
      mma_k32(tmem + hb + kColM1, al, bh, idesc96, true);
      mma_commit(&sm.mbar_1);
    }
    // ---- (D) -A and the right-hand sides (solve and token warps) | readout coefficients
    // (readout warps) | then the token warps copy the next stage and store y of the previous one
    if (is_s) {
      // -A (warps 0 and 1; thread = token t = TMEM lane).  Columns j < 32 of tokens t >= 32
      // (warp 1) lie below the split point 31 <= t - 1, so
      // g(j, t - 1) = 2^(Lambda_{t-1} - Lambda_31) 2^(Lambda_31 - Lambda_j) with both factors <= 1:
      // one exp2 per thread and the precomputed column factors.  The diagonal 32 x 32 blocks take
      // one exp2 per element.  Columns j >= 32 of tokens t < 32 are above the diagonal; the solve
      // never reads them, so nobody writes them.  A short stage (T <= 32) is solved over tokens
      // below 8 ceil(T / 8) only: warp 1 has nothing to write, and warp 0 skips columns 16..31
      // when T <= 16 (the rows of dead tokens the solve does read are written as zeros).
      mbar_wait(&sm.mbar_1, par, &sm.wait_failed);
      const int t = tid;
      const bool live = t < T;
      const float lp = (t > 0 && live) ? sm.lam[t - 1] : 0.f;  // Lambda_{t-1}
      float g[32];
      if (warp == 1 && T > 32) {
        SRNL_LD16(g, tmem_lane + hb + kColM1);
        SRNL_LD16(g + 16, tmem_lane + hb + kColM1 + 16);
        tmem_wait_ld();
        const float rf = live ? exp2_fast(lp - sm.lam[31]) : 0.f;
#pragma unroll
        for (int jb = 0; jb < 32; jb += 16) {
          float cv[16];
#pragma unroll
          for (int i = 0; i < 16; i += 4) {
            const float4 c4 = *reinterpret_cast<const float4*>(&sm.cf32[jb + i]);
            cv[i] = c4.x; cv[i + 1] = c4.y; cv[i + 2] = c4.z; cv[i + 3] = c4.w;
          }
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = -rf * cv[i] * g[jb + i];
#pragma unroll
          for (int i = 0; i < 16; ++i) neg_a_row(sm, jb + i)[t] = v[i];
          // the same block as the coupling product's B operand: row t - 32, K = j, bf16 hi + lo
          store_half_split(sm.b1h, sm.b1l, 64 + (t - 32), jb, v);
        }
        fence_async_smem();
      }
      const int j0 = 32 * warp;   // the diagonal block: columns [32 w, 32 w + 32)
      const int jb_end = (warp == 1) ? (T > 32 ? 32 : 0) : (T > 16 ? 32 : 16);
      if (jb_end > 0) {
        SRNL_LD16(g, tmem_lane + hb + kColM1 + j0);
        SRNL_LD16(g + 16, tmem_lane + hb + kColM1 + j0 + 16);
        tmem_wait_ld();
      }
#pragma unroll
      for (int jb = 0; jb < 32; jb += 16) {
        if (jb >= jb_end) break;
        // the block's Lambda_j and eta_j first: the stores below may alias them
        float lv[16], ev[16], v[16];
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          const float4 lj = *reinterpret_cast<const float4*>(&sm.lam[j0 + jb + i]);
          const float4 ej = *reinterpret_cast<const float4*>(&sm.eta[j0 + jb + i]);
          lv[i] = lj.x; lv[i + 1] = lj.y; lv[i + 2] = lj.z; lv[i + 3] = lj.w;
          ev[i] = ej.x; ev[i + 1] = ej.y; ev[i + 2] = ej.z; ev[i + 3] = ej.w;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i)
          v[i] = (live && j0 + jb + i < t) ? -exp2_fast(lp - lv[i]) * ev[i] * g[jb + i] : 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) neg_a_row(sm, j0 + jb + i)[t] = v[i];
      }
    } else if (is_k && (warp == 4 || T > 32)) {
      // the right-hand sides b^T[r][t] = 2^Lambda_{t-1} (Q_s u_t)[r] (token warps; the solve of a
      // stage of at most 32 tokens reads none of warp 5's)
      mbar_wait(&sm.mbar_1, par, &sm.wait_failed);
      const int t = tid - 128;
      const bool live = t < T;
      float bv[kD];
      SRNL_LD16(bv, tmem_lane + hb + kColZ0);
      SRNL_LD16(bv + 16, tmem_lane + hb + kColZ0 + 16);
      tmem_wait_ld();
      const float cp = (live && t > 0) ? exp2_fast(sm.lam[t - 1]) : (live ? 1.f : 0.f);
#pragma unroll
      for (int i = 0; i < kD; ++i) rhs_row(sm, i)[rhs_chunk(i, t >> 2) + (t & 3)] = cp * bv[i];
    }
    if (is_k) {
      const int gt = tid - 128;
      named_bar_arrive(5, 128);  // this half of A and the right-hand sides are written
      const StageInfo sn = stage_info(ne + 1 < nst ? ne + 1 : ne, N, L);
      const bool next_box = a.act_bf16 && ne + 1 < nst && stage_is_box(sn, r, a.H);
      if (!next_box && ne + 1 < nst) tc_prefetch(sm, sn, a, r, tok0, ch0, gt);
      // the next stage's boxes (issued during the gates) into the operand tiles, which the Gen
      // and M1 products have finished reading; with the fused query, its product starts here,
      // into columns 32..63 of the next stage's TMEM half, and runs beside the y drain below
      // (columns 0..31 of that half)
      const uint32_t qcol = (uint32_t)((ne + 1) & 1) * 128u + 32u;
      if (next_box) {
        mbar_wait(&sm.mbar_x, xpar, &sm.wait_failed);
        xpar ^= 1u;
        unstage(sm, sn, r, gt, a.fuse_q, h);
        if (a.fuse_q) query_issue(sm, tmem, qcol, h, gt);
      }
      if (pend) {  // y of the previous stage: the Y product was issued in (A)
        mbar_wait(&sm.mbar_y, (uint32_t)((ne - 1) & 1), &sm.wait_failed);
        float y[kD];
        SRNL_LD16(y, tmem_lane + phb + kColM1);
        SRNL_LD16(y + 16, tmem_lane + phb + kColM1 + 16);
        tmem_wait_ld();
        if (gt < pst.T) {
          const int p = route_pos(r, pst.t0 + gt, a.H, a.W);
          store_partial(a.yr, ((int64_t)r * a.B * N + tok0 + p) * a.C + ch0, sm.scale, y, a.act_bf16);
        }
      }
      if (next_box) {
        if (a.fuse_q) query_drain(sm, tmem_lane, qcol, sn.T, gt, qpar);
      } else {
        cp_async_wait_all();
      }
      fence_async_smem();
    } else if (is_r) {
      mbar_wait(&sm.mbar_1, par, &sm.wait_failed);
      const int t = tid - 64;
      const bool live = t < T;
      const float lt = live ? sm.lam[t] : 0.f;
      // as for -A: columns j < 32 of tokens t >= 32 (warp 3) factor at the split point 31 <= t;
      // columns j >= 32 of tokens t < 32 (warp 2) are zero.  A rolled loop over 16-column
      // blocks keeps the code small (instruction fetch is shared by every SM on the GPU).
      const float rf = (warp == 3 && live) ? exp2_fast(lt - sm.lam[31]) : 0.f;
#pragma unroll 1
      for (int jb = 0; jb < kStage; jb += 16) {
        float v[16];
        if ((warp == 2 && jb >= 32) || jb >= T || (warp == 3 && T <= 32)) {   // all zero
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = 0.f;
        } else {
          float g[16];
          SRNL_LD16(g, tmem_lane + hb + kColM1 + jb);
          tmem_wait_ld();
          const bool fac = warp == 3 && jb < 32;
#pragma unroll
          for (int i = 0; i < 16; i += 4) {
            const float4 lj = *reinterpret_cast<const float4*>(&sm.lam[jb + i]);
            const float4 ej = *reinterpret_cast<const float4*>(&sm.eta[jb + i]);
            const float4 c4 = *reinterpret_cast<const float4*>(&sm.cf32[(jb + i) & 31]);
            const float lv[4] = {lj.x, lj.y, lj.z, lj.w}, ev[4] = {ej.x, ej.y, ej.z, ej.w};
            const float cv[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
              v[i + e] = fac ? rf * cv[e] * g[i + e]
                             : ((live && jb + i + e <= t) ? exp2_fast(lt - lv[e]) * ev[e] * g[i + e] : 0.f);
          }
        }
        unsigned char* th = sm.zah[jb >> 5];
        unsigned char* tl = sm.zal[jb >> 5];
#pragma unroll
        for (int c = 0; c < 16; c += 8) {
          uint4 hi, lo;
          split8(v + c, hi, lo);
          *reinterpret_cast<uint4*>(th + zoff(64 + t, (jb & 31) + c)) = hi;
          *reinterpret_cast<uint4*>(tl + zoff(64 + t, (jb & 31) + c)) = lo;
        }
      }
      fence_async_smem();
      ct_pend = live ? exp2_fast(lt) : 0.f;
    }
    // ---- forward substitution (warp 0): lane r owns row r of Q (solve_rows), then writes -S.
    if (warp == 0) {
      named_bar(5, 128);  // A and the right-hand sides (the token warps arrive without waiting)
      if (T > 32) {
        solve_half<32>(sm, lane, 0, nullptr);
      } else {
        switch ((T + 7) >> 3) {   // the smallest multiple of 8 tokens that covers the stage
          case 1: solve_half<8>(sm, lane, 0, nullptr); break;
          case 2: solve_half<16>(sm, lane, 0, nullptr); break;
          case 3: solve_half<24>(sm, lane, 0, nullptr); break;
          default: solve_half<32>(sm, lane, 0, nullptr); break;
        }
      }
      if (T > 32) {
        // the coupling of tokens 32.. to the first 32: C[r][t'] = sum_{j < 32} S[r][j] A[32 + t'][j]
        // = (-S_1)(-A_21)^T on the tensor cores (A_21 as bf16 hi + lo in rows 64..95 of the M1 B
        // tiles, written by warp 1), into the Z columns, which the Z product overwrites later
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          tc_fence_after();
          const uint32_t sh = smem_u32(sm.zbh[0]), sl = smem_u32(sm.zbl[0]);
          const uint32_t ah = smem_u32(sm.b1h) + 64 * 64, al = smem_u32(sm.b1l) + 64 * 64;
          mma_k32(tmem + hb + kColZ, sh, ah, idesc32, false);
          mma_k32(tmem + hb + kColZ, sh, al, idesc32, true);
          mma_k32(tmem + hb + kColZ, sl, ah, idesc32, true);
          mma_commit(&sm.mbar_c);
        }
        mbar_wait(&sm.mbar_c, cpar, &sm.wait_failed);
        cpar ^= 1u;
        float c[32];
        SRNL_LD16(c, tmem + hb + kColZ);
        SRNL_LD16(c + 16, tmem + hb + kColZ + 16);
        tmem_wait_ld();
        solve_half<32>(sm, lane, 32, c);
      } else {
        store_neg_s_zero(sm, lane, 32);
      }
      fence_async_smem();
    } else if (warp == 1) {
      named_bar(5, 128);
    }
    // ---- (E) Z = [Kd^T; -; Mz^T] (-S)^T
    if (!is_k) {
      tc_fence_before();
      named_bar(3, 128);
      if (tid == 0) {
        tc_fence_after();
        // K steps of 16 tokens up to the stage's last token: past it -S is zero
        const int nk16 = (T + 15) >> 4;
        for (int st16 = 0; st16 < nk16; ++st16) {
          const int kk = st16 >> 1, k16 = st16 & 1;   // A steps 2 padded core matrices, B 2 plain ones
          const uint32_t ao = k16 * 2 * kZCore, bo = k16 * 256;
          const uint64_t ah = umma_desc_strided(smem_u32(sm.zah[kk]) + ao, kZCore, kZGroup);
          const uint64_t al = umma_desc_strided(smem_u32(sm.zal[kk]) + ao, kZCore, kZGroup);
          const uint64_t bh = umma_desc(smem_u32(sm.zbh[kk]) + bo), bl = umma_desc(smem_u32(sm.zbl[kk]) + bo);
          mma_k16_desc(tmem + hb + kColZ, ah, bh, idesc32, st16 > 0);
          mma_k16_desc(tmem + hb + kColZ, ah, bl, idesc32, true);
          mma_k16_desc(tmem + hb + kColZ, al, bh, idesc32, true);
        }
        mma_commit(&sm.mbar_z);
      }
    }
    // ---- (F) stage-end Q (warp 0: lane = column c)
    if (warp == 0) {
      mbar_wait(&sm.mbar_z, par, &sm.wait_failed);
      float qc[kD];
      SRNL_LD16(qc, tmem_lane + hb + kColZ);
      SRNL_LD16(qc + 16, tmem_lane + hb + kColZ + 16);
      tmem_wait_ld();
      const float cT = exp2_fast(sm.lam[T - 1]);
      float* col = sm.qsT[lane];
#pragma unroll
      for (int i = 0; i < kD; ++i) col[i] = fmaf(cT, col[i], qc[i]);
      __syncwarp();
      // lane = row r of Q_s: operand rows (hi/lo) of M1 and, at a chunk boundary, of W
      float row[kD];
#pragma unroll
      for (int c = 0; c < kD; ++c) row[c] = sm.qsT[c][lane];
      store_row_split(sm.b1h, sm.b1l, 64 + lane, row);
      if (!qb_is_qs && ne + 1 < nst && stage_info(ne + 1, N, L).chunk_start)
        store_row_split(sm.qbh, sm.qbl, lane, row);
      fence_async_smem();
    }
    pend = true;
    pst = si;
    phb = hb;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  // ---- the last stage's z, Y product and y
  if (is_r && pend) {
    const int t = tid - 64;
    mbar_wait(&sm.mbar_z, (uint32_t)((nst - 1) & 1), &sm.wait_failed);
    float z0[kD], zm[kD];
    SRNL_LD16(z0, tmem_lane + phb + kColZ0);
    SRNL_LD16(z0 + 16, tmem_lane + phb + kColZ0 + 16);
    SRNL_LD16(zm, tmem_lane + phb + kColZ);
    SRNL_LD16(zm + 16, tmem_lane + phb + kColZ + 16);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < kD; ++i) z0[i] = fmaf(ct_pend, z0[i], zm[i]);
    store_row_split(sm.yah, sm.yal, t, z0);
    fence_async_smem();
    tc_fence_before();
    named_bar(4, 64);
    if (t == 0) {
      tc_fence_after();
      mma_k32(tmem + phb + kColM1, smem_u32(sm.yah), smem_u32(sm.mh), idesc32, false);
      mma_k32(tmem + phb + kColM1, smem_u32(sm.yah), smem_u32(sm.ml), idesc32, true);
      mma_k32(tmem + phb + kColM1, smem_u32(sm.yal), smem_u32(sm.mh), idesc32, true);
      mma_commit(&sm.mbar_y);
    }
  }
  if (is_k && pend) {
    const int gt = tid - 128;
    mbar_wait(&sm.mbar_y, (uint32_t)((nst - 1) & 1), &sm.wait_failed);
    float y[kD];
    SRNL_LD16(y, tmem_lane + phb + kColM1);
    SRNL_LD16(y + 16, tmem_lane + phb + kColM1 + 16);
    tmem_wait_ld();
    if (gt < pst.T) {
      const int p = route_pos(r, pst.t0 + gt, a.H, a.W);
      store_partial(a.yr, ((int64_t)r * a.B * N + tok0 + p) * a.C + ch0, sm.scale, y, a.act_bf16);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (sm.wait_failed && tid == 0) atomicExch(a.err, SRNL_E_TIMEOUT);

  if (a.finals != nullptr) {
    // memories after the last token: [M_mem0; G] Q  (Q[i][c] = qsT[c][i])
    float* dst = a.finals + (int64_t)seq * kStateFloats;
    for (int mm = warp; mm < kMemRows; mm += kThreadsTc / 32) {
      const float* src = (mm < kD) ? (Msrc + mm * kD) : (Gsrc + (mm - kD) * kD);
      float acc = 0.f;
      for (int i = 0; i < kD; ++i) acc = fmaf(src[i], sm.qsT[lane][i], acc);
      dst[mm * kD + lane] = acc;
    }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemColsTc));
  }
}

}  // namespace

cudaError_t prepare_scan_chunkwise_kernel() {
  return cudaFuncSetAttribute(srnl_scan_chunkwise_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)sizeof(TcSmem));
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

// The driver's tensor-map encoder, looked up once through the runtime (no link to libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// Row view: [B*H*W][C]; column view: [B*H][W][C].  bf16, boxes of box_ch channels x box_r (row
// view) or box_c (column view) tokens.
bool encode_maps(const void* base, int B, int H, int W, int C, int box_ch, int box_r, int box_c, CUtensorMap* row,
                 CUtensorMap* col) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint32_t estr[3] = {1, 1, 1};
  const cuuint64_t rdim[2] = {(cuuint64_t)C, (cuuint64_t)B * H * W};
  const cuuint64_t rstr[1] = {(cuuint64_t)C * 2};
  const cuuint32_t rbox[2] = {(cuuint32_t)box_ch, (cuuint32_t)box_r};
  CUresult e = enc(row, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), rdim, rstr, rbox, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (e != CUDA_SUCCESS) return false;
  const cuuint64_t cdim[3] = {(cuuint64_t)C, (cuuint64_t)W, (cuuint64_t)B * H};
  const cuuint64_t cstr[2] = {(cuuint64_t)C * 2, (cuuint64_t)W * C * 2};
  const cuuint32_t cbox[3] = {(cuuint32_t)box_ch, 1, (cuuint32_t)box_c};
  e = enc(col, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), cdim, cstr, cbox, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return e == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_scan_chunkwise(const ScanGeom& g, const ScanParamsDev& p, const void* x, const void* q,
                                  float* yr, float* finals, int* err, unsigned long long* binds,
                                  cudaStream_t s) {
  TcArgs a;
  a.x = x; a.q = static_cast<const __nv_bfloat16*>(q); a.yr = yr; a.finals = finals; a.err = err;
  a.G = p.G; a.Mm = p.Mm; a.scales = p.scales;
  a.B = g.B; a.H = g.H; a.W = g.W; a.C = g.C; a.heads = g.heads;
  a.Lrow = g.Lrow; a.Lcol = g.Lcol; a.alpha = g.alpha; a.eps = g.eps;
  a.act_bf16 = g.act_bf16;
  a.hard_cap = g.hard_cap; a.binds = binds;
  a.Wqb = static_cast<const __nv_bfloat16*>(p.Wqb);
  a.fuse_q = scan_fuses_query(g, p);
  const unsigned nseq = (unsigned)g.routes * (unsigned)g.B * (unsigned)g.heads;
  TcMaps maps;
  memset(&maps, 0, sizeof(maps));
  if (g.act_bf16) {
    // a stage holds at most min(L, 64) tokens: the box covers that, rounded up to 8
    const int box_r = std::min(kStage, (g.Lrow + 7) / 8 * 8), box_c = std::min(kStage, (g.Lcol + 7) / 8 * 8);
    const bool fuse = scan_fuses_query(g, p);
    maps.box_ch = fuse ? g.C : kD;   // the fused query reads full-width x rows (128 B) and no q
    maps.box_bytes_r = (uint32_t)box_r * maps.box_ch * 2;
    maps.box_bytes_c = (uint32_t)box_c * maps.box_ch * 2;
    if (!encode_maps(x, g.B, g.H, g.W, g.C, maps.box_ch, box_r, box_c, &maps.xr, &maps.xc) ||
        (!fuse && !encode_maps(q, g.B, g.H, g.W, g.C, kD, box_r, box_c, &maps.qr, &maps.qc)))
      return cudaErrorInvalidValue;
  }
  srnl_scan_chunkwise_kernel<<<nseq, kThreadsTc, sizeof(TcSmem), s>>>(a, maps);
  return cudaGetLastError();
}

}  // namespace srnl
