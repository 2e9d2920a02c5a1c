// Internal launch interface between the C ABI (srnl_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "srnl_common.cuh"

namespace srnl {

struct ScanGeom {
  int B, H, W, C, heads;
  int Lrow, Lcol;    // resolved chunk lengths (> 0)
  int routes = 4;    // 4: the image operator; 1: a sequence (H = 1, route r0 only)
  float alpha, eps;
  bool act_bf16;     // x / y element type
  bool gen_bf16;     // generation + projection operands in bf16
  bool hard_cap = false;  // hard injection clamp instead of the soft cap
  int hd = 32;       // kernel head width: 32 (heads of d <= 32, zero-padded) or 64
};

struct ScanParamsDev {
  const float* Wq;      // [C][C] (bf16-rounded values when gen_bf16)
  const void* Wqb;      // [C][C] W_q as bf16 (bf16 path), else nullptr
  const float* G;       // [4][heads][kGen][kD]  generating initials per route/head
  const float* Mm;      // [4][heads][kD][kD]    content-memory initials
  const float* scales;  // [4][C]
};

// q[B*N][C] = x W_q^T ; q is fp32 or bf16 (gen_bf16).  bf16 activations with a bf16 W_q
// run on the tensor cores; `err` (device int) receives SRNL_E_TIMEOUT if a bounded wait
// gives up.
cudaError_t launch_query_projection(const ScanGeom& g, const ScanParamsDev& p, const void* x,
                                    void* q, int* err, cudaStream_t s);
bool query_projection_tc_supported(const ScanGeom& g);
cudaError_t launch_query_projection_tc(const ScanGeom& g, const ScanParamsDev& p, const void* x, void* q,
                                       int* err, cudaStream_t s);

// Route partials yr[4][B*N][C] (already scaled by the fusion scales; fp32, or bf16 when
// partials_bf16(g)),
// optional final states.
// `err` (device int) receives SRNL_E_TIMEOUT if a bounded in-kernel wait gives up.
// `binds` (device counter or nullptr) accumulates the tokens on which the hard clamp acts.
cudaError_t launch_scan(const ScanGeom& g, const ScanParamsDev& p, const void* x, const void* q,
                        float* yr, float* finals, int* err, unsigned long long* binds, cudaStream_t s);

// Whether launch_scan computes the queries itself (the chunkwise kernel on bf16 activations
// and generation, two 32-wide heads (C = 64), the operator's four routes, chunks that fit one
// stage and column chunks that stay inside a column): each stage's full-width x rows arrive by
// TMA and one tensor-core product gives q, so launch_query_projection is skipped and its q
// buffer is not read.
inline bool scan_fuses_query(const ScanGeom& g, const ScanParamsDev& p) {
  return g.act_bf16 && g.gen_bf16 && g.hd == 32 && g.C == 64 && g.routes == 4 && p.Wqb != nullptr &&
         g.Lrow <= 64 && g.Lcol <= 64 && g.Lcol <= g.H && g.H % g.Lcol == 0;
}

// Whether launch_scan writes the route partials in bf16: the chunkwise kernel (bf16 generation,
// 32-wide heads) with bf16 activations writes them in the output's precision; every other
// path writes fp32.  The buffer is sized for fp32 either way.
inline bool partials_bf16(const ScanGeom& g) { return g.gen_bf16 && g.act_bf16 && g.hd == 32; }

// y = yr[0] + ... + yr[routes - 1] in act dtype, summed in fp32 in route order.
cudaError_t launch_fuse(const ScanGeom& g, const float* yr, void* y, cudaStream_t s);

cudaError_t launch_route_index(int route, int H, int W, int32_t* out, cudaStream_t s);
// Head dims below 32 run as zero-padded 32-wide heads (exact: the padded rows and columns of
// every memory stay zero).  pad: [n][heads*d] -> [n][heads*32]; unpad: the reverse; states:
// [S][3*32*32 + 2*32] -> [S][3*d*d + 2*d] (the top-left blocks).  elt: bytes per element.
cudaError_t launch_pad_heads(const void* src, void* dst, int64_t n, int heads, int d, int elt, cudaStream_t s);
cudaError_t launch_unpad_heads(const void* src, void* dst, int64_t n, int heads, int d, int elt, cudaStream_t s);
cudaError_t launch_unpad_states(const float* src, float* dst, int64_t S, int d, cudaStream_t s);
// dst[i] = src[i] converted between bf16 and fp32 (src_bf16: bf16 -> fp32, else fp32 -> bf16).
cudaError_t launch_convert(const void* src, bool src_bf16, void* dst, int64_t n, cudaStream_t s);
cudaError_t launch_gather(const ScanGeom& g, int route, const void* x, void* xr, cudaStream_t s);

// The chunkwise tensor-core scan (bf16 generation); launch_scan dispatches to it.
cudaError_t launch_scan_chunkwise(const ScanGeom& g, const ScanParamsDev& p, const void* x, const void* q,
                                  float* yr, float* finals, int* err, unsigned long long* binds,
                                  cudaStream_t s);

// ---- backward (fp32 arithmetic; see srnl_scan_bwd.cu)
constexpr int kSeqPart = kD * kD + (2 * kD + 2) * kD + kD;   // dM0, dG, dscale partials per sequence
struct BwdGrads {      // device outputs in the caller's (unpadded) layouts; nullptr skips one
  float* scales;       // [routes][heads * d]
  float* M_mem0;       // [routes][heads][d][d]
  float* M_k0;
  float* M_v0;
  float* m_eta0;       // [routes][heads][d]
  float* m_alpha0;
};
struct BwdLayout {     // float offsets of the backward workspace
  size_t dxr, dqr, dq, parts, ckpt, qs, grec, dwq, total;
  int max_chunks, Lmax, nsplit;
  int hd;              // head width of the kernels (32 or 64)
  int rec;             // floats per token gate record (2 hd + 8)
  size_t seq_part;     // floats of parameter partials per sequence: hd^2 + (2 hd + 2) hd + hd
};
// Floats of backward workspace for the geometry (and the layout when lay != nullptr).
size_t backward_workspace_floats(const ScanGeom& g, BwdLayout* lay);
// Gradient of sum(dy * y) for the forward y(x, params) of geometry g (32-wide padded heads,
// ud = the caller's head dim), in two launches.  x, dy, dx: [B][N][C] act dtype (padded);
// q: the fp32 query projection of x; ws: backward_workspace_floats(g) floats.
// launch_backward_scan: the per-sequence reverse scan (route partials of dx and dq, and
// per-sequence parameter partials, into ws).  launch_backward_combine: dx = sum of the route
// partials + dq W_q, dW_q (dwq_out [heads*ud]^2, or nullptr) and the batch-ordered
// parameter reductions into `out`.
cudaError_t launch_backward_scan(const ScanGeom& g, const ScanParamsDev& p, const void* x, const float* q,
                                 const void* dy, float* ws, cudaStream_t s);
cudaError_t launch_backward_combine(const ScanGeom& g, const ScanParamsDev& p, int ud, const void* x, float* ws,
                                    void* dx, const BwdGrads& out, float* dwq_out, cudaStream_t s);
// Sequence layer (routes = 1): dx = the generation partial (+ the query partial when x is also
// the query, add_q), dq = the query partial (nullptr skips it), both in the act dtype, and the
// parameter reductions into `out` (out.scales ignored).  ws: the workspace after
// launch_backward_scan.
cudaError_t launch_backward_seq_combine(const ScanGeom& g, int ud, float* ws, void* dx, void* dq, bool add_q,
                                        const BwdGrads& out, cudaStream_t s);
// Float offset of the region launch_backward_scan leaves free (B*N*C floats; the sequence
// layer stages fp32 queries there).
inline size_t backward_free_region(const ScanGeom& g) { BwdLayout l; backward_workspace_floats(g, &l); return l.dq; }
cudaError_t prepare_backward_kernel();
// The 64-wide reverse scan (head dim 64); launch_backward_scan dispatches to it when g.hd == 64.
cudaError_t launch_backward_scan64(const ScanGeom& g, const ScanParamsDev& p, const void* x, const float* q,
                                   const void* dy, float* ws, const BwdLayout& l, cudaStream_t s);
cudaError_t prepare_backward64_kernel();

// Head dim 64 (SIMT, both precision paths); launch_scan dispatches to it when g.hd == 64.
// finals: [routes][B][heads][3*64*64 + 2*64] or nullptr.
cudaError_t launch_scan_d64(const ScanGeom& g, const ScanParamsDev& p, const void* x, const void* q, float* yr,
                            float* finals, unsigned long long* binds, cudaStream_t s);
cudaError_t prepare_scan_d64_kernel();

cudaError_t prepare_block_kernels();  // the residual block's GEMM (dynamic smem)
cudaError_t prepare_kernels();       // one-time function attributes (dynamic smem)
cudaError_t prepare_scan_kernels();
cudaError_t prepare_scan_chunkwise_kernel();
cudaError_t prepare_projection_kernel();

}  // namespace srnl
