// C ABI of the standalone SRNL layer on sequences ("VisionHOPE" README, section "SRNL and
// VisionHOPE operator": [batch, tokens, dim] in and out, optional queries, 64-token chunks
// by default, an incomplete final chunk allowed, a new sequence on every call).
//
// A sequence is the image scan's route 0 on a 1 x T map with no fusion: the same scan
// kernels run with one route, the fusion kernel reduces to a cast of the single partial
// (scale 1), and the queries come from the caller instead of a projection.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "srnl_common.cuh"
#include "srnl_internal.h"
#include "srnl_launch.h"
#include "srnl_scan.h"

struct srnl_seq {
  srnl_seq_config cfg{};
  srnl::ScanGeom geom{};
  int device = 0;
  float* G = nullptr;       // [1][heads][66][32] generating initials
  float* Mm = nullptr;      // [1][heads][32][32] content-memory initials
  float* scales = nullptr;  // [1][D] ones
  void* qbuf = nullptr;     // queries in the generation dtype when it differs from act_dtype
  float* yr = nullptr;      // [1][B*T][D] fp32 partial
  int* dev_err = nullptr;
  unsigned long long* binds = nullptr;  // hard-clamp activations of the last forward
  // head dims below 32 run zero-padded to 32: padded copies of x, q, y and the final states
  void* x_pad = nullptr;
  void* q_pad = nullptr;
  void* y_pad = nullptr;
  float* fin_pad = nullptr;
  // backward (allocated on first use): workspace and padded dy / dx / dq for d < 32
  float* bws = nullptr;
  void* dy_pad = nullptr;
  void* dx_pad = nullptr;
  void* dq_pad = nullptr;
  std::string err;
};

namespace {

thread_local std::string g_seq_create_error;

srnl_status seq_fail(srnl_seq* h, srnl_status st, const std::string& msg) {
  if (h != nullptr) h->err = msg; else g_seq_create_error = msg;
  return st;
}

srnl_status seq_cuda_fail(srnl_seq* h, cudaError_t e, const char* what) {
  return seq_fail(h, e == cudaErrorMemoryAllocation ? SRNL_E_NOMEM : SRNL_E_CUDA,
                  std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")");
}

void seq_free(srnl_seq* h) {
  void* ptrs[] = {h->G, h->Mm, h->scales, h->qbuf, h->yr, h->dev_err, h->binds, h->x_pad, h->q_pad, h->y_pad,
                  h->fin_pad, h->bws, h->dy_pad, h->dx_pad, h->dq_pad};
  for (void* p : ptrs)
    if (p != nullptr) cudaFree(p);
  h->G = h->Mm = h->scales = h->yr = nullptr;
  h->qbuf = nullptr;
  h->dev_err = nullptr;
  h->binds = nullptr;
  h->x_pad = h->q_pad = h->y_pad = nullptr;
  h->fin_pad = nullptr;
  h->bws = nullptr;
  h->dy_pad = h->dx_pad = h->dq_pad = nullptr;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap(const void* a, const void* b, size_t n) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + n && y < x + n;
}

}  // namespace

extern "C" {

srnl_status srnl_seq_create(srnl_seq** out, const srnl_seq_config* cfg, const srnl_seq_params* prm) {
  if (out == nullptr) return seq_fail(nullptr, SRNL_E_INVAL, "out is NULL");
  *out = nullptr;
  if (cfg == nullptr || prm == nullptr) return seq_fail(nullptr, SRNL_E_INVAL, "cfg or params is NULL");
  if (prm->M_mem0 == nullptr || prm->M_k0 == nullptr || prm->M_v0 == nullptr || prm->m_eta0 == nullptr ||
      prm->m_alpha0 == nullptr)
    return seq_fail(nullptr, SRNL_E_INVAL, "a parameter pointer is NULL");
  if (cfg->B <= 0 || cfg->T <= 0 || cfg->D <= 0 || cfg->heads <= 0 || cfg->d <= 0)
    return seq_fail(nullptr, SRNL_E_INVAL, "B, T, D, heads and d must be positive");
  if (cfg->chunk < 0) return seq_fail(nullptr, SRNL_E_INVAL, "chunk must be >= 0 (0 = 64)");
  // the rest of the checks are those of a 1 x T image
  srnl_scan_config sc{};
  sc.B = cfg->B; sc.H = 1; sc.W = cfg->T; sc.C = cfg->D; sc.heads = cfg->heads; sc.d = cfg->d;
  sc.alpha = cfg->alpha; sc.eps = cfg->eps;
  sc.chunk_row = sc.chunk_col = cfg->chunk > 0 ? cfg->chunk : 64;
  sc.act_dtype = cfg->act_dtype; sc.gen_dtype = cfg->gen_dtype;
  sc.injection_cap = cfg->injection_cap;
  srnl_status st = srnl::validate_scan_config(&sc);
  if (st != SRNL_OK) {
    return seq_fail(nullptr, st, std::string("invalid sequence config: ") + srnl_scan_last_error(nullptr));
  }
  srnl_seq* h = new (std::nothrow) srnl_seq;
  if (h == nullptr) return seq_fail(nullptr, SRNL_E_NOMEM, "host allocation failed");
  h->cfg = *cfg;
  cudaError_t e = cudaGetDevice(&h->device);
  if (e != cudaSuccess) { st = seq_cuda_fail(nullptr, e, "cudaGetDevice"); delete h; return st; }

  // kernels run 32-wide heads (64-wide for head dim 64); a smaller head dim is zero-padded to
  // 32 (exact)
  const int d = cfg->d == 64 ? 64 : srnl::kD, ud = cfg->d, nh = cfg->heads, Dp = nh * d;
  const int gen = 2 * d + 2;   // generating rows: M_k, M_v, m_eta, m_alpha
  const bool padded = ud != d;
  srnl::ScanGeom& g = h->geom;
  g.B = cfg->B; g.H = 1; g.W = cfg->T; g.C = Dp; g.heads = nh;
  g.Lrow = g.Lcol = sc.chunk_row;
  g.alpha = cfg->alpha; g.eps = cfg->eps;
  g.act_bf16 = cfg->act_dtype == SRNL_BF16;
  g.gen_bf16 = cfg->gen_dtype == SRNL_BF16;
  g.routes = 1;
  g.hard_cap = cfg->injection_cap == SRNL_CAP_HARD;
  g.hd = d;

  std::vector<float> G((size_t)nh * gen * d, 0.f), Mm((size_t)nh * d * d, 0.f);
  for (int hh = 0; hh < nh; ++hh) {
    float* dst = G.data() + (size_t)hh * gen * d;
    float* mdst = Mm.data() + (size_t)hh * d * d;
    const size_t mo = (size_t)hh * ud * ud, vo = (size_t)hh * ud;
    for (int i = 0; i < ud; ++i) {
      for (int j = 0; j < ud; ++j) {
        dst[i * d + j] = prm->M_k0[mo + (size_t)i * ud + j];
        dst[(d + i) * d + j] = prm->M_v0[mo + (size_t)i * ud + j];
        mdst[i * d + j] = prm->M_mem0[mo + (size_t)i * ud + j];
      }
      dst[2 * d * d + i] = prm->m_eta0[vo + i];
      dst[2 * d * d + d + i] = prm->m_alpha0[vo + i];
    }
  }
  const std::vector<float> ones((size_t)Dp, 1.f);
  const size_t tokens = (size_t)cfg->B * cfg->T;
  const size_t n_mm = Mm.size();
  const size_t qbuf_bytes = g.act_bf16 != g.gen_bf16 ? tokens * Dp * (g.gen_bf16 ? 2 : 4) : 0;
  const size_t pad_bytes = padded ? tokens * Dp * (g.act_bf16 ? 2 : 4) : 0;
  const size_t fin_pad_bytes = padded ? (size_t)cfg->B * nh * srnl::kStateFloats * sizeof(float) : 0;
  struct { void** p; size_t n; } allocs[] = {
      {(void**)&h->G, G.size() * sizeof(float)}, {(void**)&h->Mm, n_mm * sizeof(float)},
      {(void**)&h->scales, ones.size() * sizeof(float)}, {&h->qbuf, qbuf_bytes},
      {(void**)&h->yr, tokens * Dp * sizeof(float)}, {(void**)&h->dev_err, sizeof(int)},
      {(void**)&h->binds, sizeof(unsigned long long)}, {&h->x_pad, pad_bytes}, {&h->q_pad, pad_bytes},
      {&h->y_pad, pad_bytes}, {(void**)&h->fin_pad, fin_pad_bytes}};
  for (auto& a : allocs) {
    if (a.n == 0) continue;
    e = cudaMalloc(a.p, a.n);
    if (e != cudaSuccess) { st = seq_cuda_fail(nullptr, e, "cudaMalloc"); seq_free(h); delete h; return st; }
  }
  struct { void* dst; const void* src; size_t n; } copies[] = {
      {h->G, G.data(), G.size() * sizeof(float)}, {h->Mm, Mm.data(), n_mm * sizeof(float)},
      {h->scales, ones.data(), ones.size() * sizeof(float)}};
  for (auto& cp : copies) {
    e = cudaMemcpy(cp.dst, cp.src, cp.n, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) { st = seq_cuda_fail(nullptr, e, "cudaMemcpy (params)"); seq_free(h); delete h; return st; }
  }
  e = cudaMemset(h->dev_err, 0, sizeof(int));
  if (e == cudaSuccess) e = cudaMemset(h->binds, 0, sizeof(unsigned long long));
  if (e == cudaSuccess) e = srnl::prepare_kernels();
  if (e != cudaSuccess) { st = seq_cuda_fail(nullptr, e, "set-up"); seq_free(h); delete h; return st; }
  *out = h;
  return SRNL_OK;
}

srnl_status srnl_seq_forward(srnl_seq* h, const void* x, const void* q, void* y, float* final_states,
                             void* stream) {
  if (h == nullptr) return SRNL_E_INVAL;
  h->err.clear();
  if (x == nullptr || y == nullptr) return seq_fail(h, SRNL_E_INVAL, "x or y is NULL");
  if (!aligned16(x) || !aligned16(y) || (q != nullptr && !aligned16(q)) ||
      (final_states != nullptr && !aligned16(final_states)))
    return seq_fail(h, SRNL_E_INVAL, "x, q, y and final_states must be 16-byte aligned");
  const srnl::ScanGeom& g = h->geom;
  const size_t n = (size_t)g.B * g.W * g.C;  // padded element count
  const size_t bytes = (size_t)g.B * g.W * h->cfg.D * (g.act_bf16 ? 2 : 4);
  if (overlap(x, y, bytes) || (q != nullptr && overlap(q, y, bytes)))
    return seq_fail(h, SRNL_E_INVAL, "y overlaps x or q");
  int cur = -1;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return seq_cuda_fail(h, e, "cudaGetDevice");
  if (cur != h->device) return seq_fail(h, SRNL_E_INVAL, "the current device is not the handle's device");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool padded = h->cfg.d < srnl::kD;
  const int elt = g.act_bf16 ? 2 : 4;
  const int64_t tokens = (int64_t)g.B * g.W;
  const void* qk = q != nullptr ? q : x;
  void* yk = y;
  float* fk = final_states;
  if (padded) {  // heads of d < 32 channels run as zero-padded 32-wide heads
    e = srnl::launch_pad_heads(x, h->x_pad, tokens, g.heads, h->cfg.d, elt, s);
    if (e == cudaSuccess && q != nullptr) e = srnl::launch_pad_heads(q, h->q_pad, tokens, g.heads, h->cfg.d, elt, s);
    if (e != cudaSuccess) return seq_cuda_fail(h, e, "head padding launch");
    qk = q != nullptr ? h->q_pad : h->x_pad;
    x = h->x_pad;
    yk = h->y_pad;
    if (final_states != nullptr) fk = h->fin_pad;
  }
  if (g.act_bf16 != g.gen_bf16) {  // queries in the generation dtype
    e = srnl::launch_convert(qk, g.act_bf16, h->qbuf, (int64_t)n, s);
    if (e != cudaSuccess) return seq_cuda_fail(h, e, "query conversion launch");
    qk = h->qbuf;
  }
  const srnl::ScanParamsDev p{nullptr, nullptr, h->G, h->Mm, h->scales};
  if (g.hard_cap && (e = cudaMemsetAsync(h->binds, 0, sizeof(unsigned long long), s)) != cudaSuccess)
    return seq_cuda_fail(h, e, "counter reset");
  e = srnl::launch_scan(g, p, x, qk, h->yr, fk, h->dev_err, h->binds, s);
  if (e != cudaSuccess) return seq_cuda_fail(h, e, "scan launch");
  e = srnl::launch_fuse(g, h->yr, yk, s);
  if (e != cudaSuccess) return seq_cuda_fail(h, e, "output launch");
  if (padded) {
    e = srnl::launch_unpad_heads(h->y_pad, y, tokens, g.heads, h->cfg.d, elt, s);
    if (e == cudaSuccess && final_states != nullptr)
      e = srnl::launch_unpad_states(h->fin_pad, final_states, (int64_t)g.B * g.heads, h->cfg.d, s);
    if (e != cudaSuccess) return seq_cuda_fail(h, e, "head unpadding launch");
  }
  return SRNL_OK;
}

srnl_status srnl_seq_backward(srnl_seq* h, const void* x, const void* q, const void* dy, void* dx, void* dq,
                              const srnl_seq_grads* grads, void* stream) {
  if (h == nullptr) return SRNL_E_INVAL;
  h->err.clear();
  if (x == nullptr || dy == nullptr || dx == nullptr) return seq_fail(h, SRNL_E_INVAL, "x, dy or dx is NULL");
  if (q == nullptr && dq != nullptr) return seq_fail(h, SRNL_E_INVAL, "dq needs separate queries q");
  if (!aligned16(x) || !aligned16(dy) || !aligned16(dx) || (q != nullptr && !aligned16(q)) ||
      (dq != nullptr && !aligned16(dq)))
    return seq_fail(h, SRNL_E_INVAL, "x, q, dy, dx and dq must be 16-byte aligned");
  const srnl::ScanGeom& g = h->geom;
  const size_t bytes = (size_t)g.B * g.W * h->cfg.D * (g.act_bf16 ? 2 : 4);
  const void* ins[] = {x, q, dy};
  for (const void* in : ins)
    if (in != nullptr && (overlap(in, dx, bytes) || (dq != nullptr && overlap(in, dq, bytes))))
      return seq_fail(h, SRNL_E_INVAL, "dx or dq overlaps an input");
  if (dq != nullptr && overlap(dx, dq, bytes)) return seq_fail(h, SRNL_E_INVAL, "dx and dq overlap");
  if (g.gen_bf16) return seq_fail(h, SRNL_E_UNSUPPORTED, "the backward pass is built for gen_dtype SRNL_F32 handles");
  int cur = -1;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return seq_cuda_fail(h, e, "cudaGetDevice");
  if (cur != h->device) return seq_fail(h, SRNL_E_INVAL, "the current device is not the handle's device");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool padded = h->cfg.d < srnl::kD;
  const int elt = g.act_bf16 ? 2 : 4;
  const int64_t tokens = (int64_t)g.B * g.W;
  const size_t pbytes = (size_t)tokens * g.C * elt;
  if (h->bws == nullptr) {  // all or nothing: a failed allocation leaves none of the four
    void* got[4] = {nullptr, nullptr, nullptr, nullptr};
    e = cudaMalloc(&got[0], srnl::backward_workspace_floats(g, nullptr) * sizeof(float));
    for (int i = 1; i < 4 && padded && e == cudaSuccess; ++i) e = cudaMalloc(&got[i], pbytes);
    if (e != cudaSuccess) {
      for (void* q : got)
        if (q != nullptr) cudaFree(q);
      return seq_cuda_fail(h, e, "cudaMalloc (backward workspace)");
    }
    h->bws = static_cast<float*>(got[0]);
    h->dy_pad = got[1];
    h->dx_pad = got[2];
    h->dq_pad = got[3];
  }
  const void* qk = q != nullptr ? q : x;
  if (padded) {
    e = srnl::launch_pad_heads(x, h->x_pad, tokens, g.heads, h->cfg.d, elt, s);
    if (e == cudaSuccess && q != nullptr) e = srnl::launch_pad_heads(q, h->q_pad, tokens, g.heads, h->cfg.d, elt, s);
    if (e == cudaSuccess) e = srnl::launch_pad_heads(dy, h->dy_pad, tokens, g.heads, h->cfg.d, elt, s);
    if (e != cudaSuccess) return seq_cuda_fail(h, e, "head padding launch");
    qk = q != nullptr ? h->q_pad : h->x_pad;
    x = h->x_pad;
    dy = h->dy_pad;
  }
  const float* q32 = static_cast<const float*>(qk);
  if (g.act_bf16) {  // the backward reads fp32 queries
    float* qf = h->bws + srnl::backward_free_region(g);
    e = srnl::launch_convert(qk, true, qf, tokens * g.C, s);
    if (e != cudaSuccess) return seq_cuda_fail(h, e, "query conversion launch");
    q32 = qf;
  }
  const srnl::ScanParamsDev p{nullptr, nullptr, h->G, h->Mm, h->scales};
  e = srnl::launch_backward_scan(g, p, x, q32, dy, h->bws, s);
  if (e != cudaSuccess) return seq_cuda_fail(h, e, "backward scan launch");
  srnl::BwdGrads out{};
  if (grads != nullptr) out = srnl::BwdGrads{nullptr, grads->M_mem0, grads->M_k0, grads->M_v0, grads->m_eta0, grads->m_alpha0};
  void* dxk = padded ? h->dx_pad : dx;
  void* dqk = dq == nullptr ? nullptr : (padded ? h->dq_pad : dq);
  e = srnl::launch_backward_seq_combine(g, h->cfg.d, h->bws, dxk, dqk, q == nullptr, out, s);
  if (e != cudaSuccess) return seq_cuda_fail(h, e, "backward combine launch");
  if (padded) {
    e = srnl::launch_unpad_heads(h->dx_pad, dx, tokens, g.heads, h->cfg.d, elt, s);
    if (e == cudaSuccess && dq != nullptr) e = srnl::launch_unpad_heads(h->dq_pad, dq, tokens, g.heads, h->cfg.d, elt, s);
    if (e != cudaSuccess) return seq_cuda_fail(h, e, "head unpadding launch");
  }
  return SRNL_OK;
}

srnl_status srnl_seq_device_status(srnl_seq* h) {
  if (h == nullptr) return SRNL_E_INVAL;
  int v = 0;
  const cudaError_t e = cudaMemcpy(&v, h->dev_err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return seq_cuda_fail(h, e, "status read");
  if (v != 0) {
    h->err = "a bounded in-kernel wait gave up";
    return static_cast<srnl_status>(v);
  }
  return SRNL_OK;
}

srnl_status srnl_seq_cap_count(srnl_seq* h, unsigned long long* count) {
  if (h == nullptr || count == nullptr) return SRNL_E_INVAL;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(count, h->binds, sizeof(unsigned long long), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return seq_cuda_fail(h, e, "counter read");
  return SRNL_OK;
}

const char* srnl_seq_last_error(const srnl_seq* h) {
  return h != nullptr ? h->err.c_str() : g_seq_create_error.c_str();
}

void srnl_seq_destroy(srnl_seq* h) {
  if (h == nullptr) return;
  int prev = -1;
  cudaGetDevice(&prev);
  if (prev != h->device) cudaSetDevice(h->device);
  cudaDeviceSynchronize();
  seq_free(h);
  if (prev >= 0 && prev != h->device) cudaSetDevice(prev);
  delete h;
}

}  // extern "C"
