// C ABI of the SRNL four-direction scan (declared in include/srnl_scan.h).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "srnl_common.cuh"
#include "srnl_internal.h"
#include "srnl_launch.h"
#include "srnl_scan.h"

struct srnl_scan {
  srnl_scan_config cfg{};
  srnl::ScanGeom geom{};
  int device = 0;
  // packed parameters (device)
  float* Wq = nullptr;
  void* Wqb = nullptr;       // W_q in bf16 (bf16 path only)
  float* G = nullptr;
  float* Mm = nullptr;
  float* scales = nullptr;
  // workspace (device)
  void* q = nullptr;        // [B*N][C] fp32 or bf16
  float* yr = nullptr;      // [4][B*N][C] fp32 route partials
  void* x_stage = nullptr;  // staging for srnl_scan_forward_host (slot 0 of the pipeline)
  void* y_stage = nullptr;
  // pipelined host-buffer forwards: a second staging slot, one copy stream per direction and
  // the events that order slot reuse (created on first use)
  void* x_stage1 = nullptr;
  void* y_stage1 = nullptr;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t h2d_done[2] = {}, fwd_done[2] = {}, d2h_done[2] = {};
  bool slot_used[2] = {false, false};
  int slot = 0;
  int* dev_err = nullptr;   // device status word written by the scan kernel
  unsigned long long* binds = nullptr;  // hard-clamp activations of the last forward
  // head dims below 32 run zero-padded to 32: padded copies of x, y and the final states
  void* x_pad = nullptr;
  void* y_pad = nullptr;
  float* fin_pad = nullptr;
  // backward pass (allocated on first use): workspace and padded dy / dx for d < 32
  float* bws = nullptr;
  void* dy_pad = nullptr;
  void* dx_pad = nullptr;
  size_t ws_bytes = 0;
  // optional stage timing: a ring of event sets, 4 events per forward
  std::vector<cudaEvent_t> ev;
  int ring = 0;        // sets in the ring (0 = timing off)
  int recorded = 0;    // forwards recorded in the current window
  std::string err;
};

namespace {

thread_local std::string g_create_error;

srnl_status fail(srnl_scan* h, srnl_status st, const std::string& msg) {
  if (h != nullptr) h->err = msg; else g_create_error = msg;
  return st;
}

srnl_status cuda_fail(srnl_scan* h, cudaError_t e, const char* what) {
  std::string msg = std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
  return fail(h, e == cudaErrorMemoryAllocation ? SRNL_E_NOMEM : SRNL_E_CUDA, msg);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

float bf16_round_host(float v) {
  return __bfloat162float(__float2bfloat16_rn(v));
}

size_t act_bytes(const srnl_scan_config& c) {
  return (size_t)c.B * c.H * c.W * c.C * (c.act_dtype == SRNL_BF16 ? 2 : 4);
}

void free_all(srnl_scan* h) {
  void* ptrs[] = {h->Wq, h->Wqb, h->G, h->Mm, h->scales, h->q, h->yr, h->x_stage, h->y_stage, h->dev_err, h->binds,
                  h->x_pad, h->y_pad, h->fin_pad, h->x_stage1, h->y_stage1, h->bws, h->dy_pad, h->dx_pad};
  for (void* p : ptrs)
    if (p != nullptr) cudaFree(p);
  h->Wq = h->G = h->Mm = h->scales = nullptr;
  h->Wqb = nullptr;
  h->q = h->x_stage = h->y_stage = nullptr;
  h->yr = nullptr;
  h->dev_err = nullptr;
  h->binds = nullptr;
  h->x_pad = h->y_pad = nullptr;
  h->fin_pad = nullptr;
  h->x_stage1 = h->y_stage1 = nullptr;
  h->bws = nullptr;
  h->dy_pad = h->dx_pad = nullptr;
  for (int k = 0; k < 2; ++k) {
    cudaEvent_t* evs[] = {&h->h2d_done[k], &h->fwd_done[k], &h->d2h_done[k]};
    for (cudaEvent_t* e : evs)
      if (*e != nullptr) { cudaEventDestroy(*e); *e = nullptr; }
  }
  if (h->h2d != nullptr) { cudaStreamDestroy(h->h2d); h->h2d = nullptr; }
  if (h->d2h != nullptr) { cudaStreamDestroy(h->d2h); h->d2h = nullptr; }
}

srnl_status validate_config(const srnl_scan_config* c) {
  if (c->B <= 0 || c->H <= 0 || c->W <= 0 || c->C <= 0 || c->heads <= 0 || c->d <= 0)
    return fail(nullptr, SRNL_E_INVAL, "B, H, W, C, heads and d must be positive");
  if ((int64_t)c->heads * c->d != c->C)
    return fail(nullptr, SRNL_E_INVAL, "C must equal heads * d");
  if (c->d != 4 && c->d != 8 && c->d != 16 && c->d != srnl::kD && c->d != 64)
    return fail(nullptr, SRNL_E_UNSUPPORTED, "head dim d must be 4, 8, 16, 32 or 64");
  if (!(c->alpha > 0.f && c->alpha < 1.f))
    return fail(nullptr, SRNL_E_INVAL, "alpha must lie in (0, 1)");
  if (!(c->eps > 0.f) || !std::isfinite(c->eps))
    return fail(nullptr, SRNL_E_INVAL, "eps must be positive and finite");
  if (c->chunk_row < 0 || c->chunk_col < 0)
    return fail(nullptr, SRNL_E_INVAL, "chunk lengths must be >= 0 (0 = full rows/columns)");
  if ((c->act_dtype != SRNL_F32 && c->act_dtype != SRNL_BF16) ||
      (c->gen_dtype != SRNL_F32 && c->gen_dtype != SRNL_BF16))
    return fail(nullptr, SRNL_E_INVAL, "act_dtype and gen_dtype must be SRNL_F32 or SRNL_BF16");
  if (c->injection_cap != SRNL_CAP_SOFT && c->injection_cap != SRNL_CAP_HARD)
    return fail(nullptr, SRNL_E_INVAL, "injection_cap must be SRNL_CAP_SOFT or SRNL_CAP_HARD");
  const int64_t N = (int64_t)c->H * c->W;
  if (N > (int64_t)1 << 30) return fail(nullptr, SRNL_E_INVAL, "H*W too large");
  if ((int64_t)4 * c->B * c->heads > (int64_t)INT32_MAX)
    return fail(nullptr, SRNL_E_INVAL, "4*B*heads too large");
  if ((int64_t)c->B * N * c->C > ((int64_t)1 << 40))
    return fail(nullptr, SRNL_E_INVAL, "B*H*W*C too large");
  return SRNL_OK;
}

}  // namespace

namespace srnl {
srnl_status validate_scan_config(const srnl_scan_config* cfg) { return validate_config(cfg); }
void set_thread_error(const std::string& msg) { g_create_error = msg; }
}  // namespace srnl

extern "C" {

const char* srnl_status_string(int status) {
  switch (status) {
    case SRNL_OK: return "SRNL_OK";
    case SRNL_E_INVAL: return "SRNL_E_INVAL";
    case SRNL_E_UNSUPPORTED: return "SRNL_E_UNSUPPORTED";
    case SRNL_E_CUDA: return "SRNL_E_CUDA";
    case SRNL_E_NOMEM: return "SRNL_E_NOMEM";
    case SRNL_E_TIMEOUT: return "SRNL_E_TIMEOUT";
    default: return "SRNL_E_UNKNOWN";
  }
}

const char* srnl_scan_last_error(const srnl_scan* h) {
  return h != nullptr ? h->err.c_str() : g_create_error.c_str();
}

srnl_status srnl_scan_create(srnl_scan** out, const srnl_scan_config* cfg,
                             const srnl_scan_params* prm) {
  g_create_error.clear();
  if (out == nullptr) return fail(nullptr, SRNL_E_INVAL, "out is NULL");
  *out = nullptr;
  if (cfg == nullptr || prm == nullptr) return fail(nullptr, SRNL_E_INVAL, "cfg or params is NULL");
  if (prm->W_q == nullptr || prm->scales == nullptr || prm->M_mem0 == nullptr ||
      prm->M_k0 == nullptr || prm->M_v0 == nullptr || prm->m_eta0 == nullptr ||
      prm->m_alpha0 == nullptr)
    return fail(nullptr, SRNL_E_INVAL, "a parameter pointer is NULL");
  srnl_status st = validate_config(cfg);
  if (st != SRNL_OK) return st;

  srnl_scan* h = new (std::nothrow) srnl_scan();
  if (h == nullptr) return fail(nullptr, SRNL_E_NOMEM, "host allocation failed");
  h->cfg = *cfg;
  cudaError_t e = cudaGetDevice(&h->device);
  if (e != cudaSuccess) { st = cuda_fail(nullptr, e, "cudaGetDevice"); delete h; return st; }

  const srnl_scan_config& c = h->cfg;
  // kernels run 32-wide heads (64-wide for head dim 64); a smaller head dim is zero-padded to
  // 32 (exact: the padded rows and columns of every memory and transition stay zero)
  const int d = c.d == 64 ? 64 : srnl::kD, ud = c.d, nh = c.heads, Cp = nh * d;
  const int gen = 2 * d + 2;   // generating rows: M_k, M_v, m_eta, m_alpha
  const bool padded = ud != d;
  srnl::ScanGeom& g = h->geom;
  g.B = c.B; g.H = c.H; g.W = c.W; g.C = Cp; g.heads = nh;
  g.Lrow = c.chunk_row > 0 ? c.chunk_row : c.W;
  g.Lcol = c.chunk_col > 0 ? c.chunk_col : c.H;
  g.alpha = c.alpha; g.eps = c.eps;
  g.act_bf16 = c.act_dtype == SRNL_BF16;
  g.gen_bf16 = c.gen_dtype == SRNL_BF16;
  g.hard_cap = c.injection_cap == SRNL_CAP_HARD;
  g.hd = d;

  // ---- pack parameters on the host, then upload
  std::vector<float> Wq((size_t)Cp * Cp, 0.f);
  for (int o = 0; o < c.C; ++o)
    for (int i = 0; i < c.C; ++i) {
      const float w = prm->W_q[(size_t)o * c.C + i];
      Wq[(size_t)((o / ud) * d + o % ud) * Cp + (i / ud) * d + i % ud] = g.gen_bf16 ? bf16_round_host(w) : w;
    }
  std::vector<__nv_bfloat16> Wqb(g.gen_bf16 ? Wq.size() : 0);
  for (size_t i = 0; i < Wqb.size(); ++i) Wqb[i] = __float2bfloat16_rn(Wq[i]);  // exact: already rounded
  std::vector<float> G((size_t)4 * nh * gen * d, 0.f), Mm((size_t)4 * nh * d * d, 0.f);
  for (int r = 0; r < 4; ++r)
    for (int hh = 0; hh < nh; ++hh) {
      float* dst = G.data() + ((size_t)r * nh + hh) * gen * d;
      float* mdst = Mm.data() + ((size_t)r * nh + hh) * d * d;
      const size_t mo = ((size_t)r * nh + hh) * ud * ud, vo = ((size_t)r * nh + hh) * ud;
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
  std::vector<float> scales((size_t)4 * Cp, 0.f);
  for (int r = 0; r < 4; ++r)
    for (int ch = 0; ch < c.C; ++ch) scales[(size_t)r * Cp + (ch / ud) * d + ch % ud] = prm->scales[(size_t)r * c.C + ch];
  const size_t n_mm = Mm.size(), n_sc = scales.size();
  const size_t tokens = (size_t)c.B * c.H * c.W;
  const size_t q_bytes = tokens * Cp * (g.gen_bf16 ? 2 : 4);
  const size_t yr_bytes = 4 * tokens * Cp * sizeof(float);
  const size_t stage_bytes = act_bytes(c);
  const size_t pad_bytes = padded ? tokens * Cp * (g.act_bf16 ? 2 : 4) : 0;
  const size_t fin_pad_bytes = padded ? (size_t)4 * c.B * nh * srnl::kStateFloats * sizeof(float) : 0;

  struct { void** p; size_t n; } allocs[] = {
      {(void**)&h->Wq, Wq.size() * sizeof(float)}, {(void**)&h->G, G.size() * sizeof(float)},
      {(void**)&h->Mm, n_mm * sizeof(float)},      {(void**)&h->scales, n_sc * sizeof(float)},
      {&h->q, q_bytes},                            {(void**)&h->yr, yr_bytes},
      {&h->x_stage, stage_bytes},                  {&h->y_stage, stage_bytes},
      {(void**)&h->dev_err, sizeof(int)},          {&h->Wqb, Wqb.size() * sizeof(__nv_bfloat16)},
      {(void**)&h->binds, sizeof(unsigned long long)}, {&h->x_pad, pad_bytes}, {&h->y_pad, pad_bytes},
      {(void**)&h->fin_pad, fin_pad_bytes}};
  for (auto& a : allocs) {
    if (a.n == 0) continue;
    e = cudaMalloc(a.p, a.n);
    if (e != cudaSuccess) {
      st = cuda_fail(nullptr, e, "cudaMalloc");
      free_all(h); delete h; return st;
    }
  }
  h->ws_bytes = q_bytes + yr_bytes + 2 * stage_bytes + 2 * pad_bytes + fin_pad_bytes;
  struct { void* dst; const void* src; size_t n; } copies[] = {
      {h->Wq, Wq.data(), Wq.size() * sizeof(float)}, {h->G, G.data(), G.size() * sizeof(float)},
      {h->Mm, Mm.data(), n_mm * sizeof(float)},      {h->scales, scales.data(), n_sc * sizeof(float)},
      {h->Wqb, Wqb.data(), Wqb.size() * sizeof(__nv_bfloat16)}};
  for (auto& cp : copies) {
    if (cp.n == 0) continue;
    e = cudaMemcpy(cp.dst, cp.src, cp.n, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) { st = cuda_fail(nullptr, e, "cudaMemcpy (params)"); free_all(h); delete h; return st; }
  }
  e = cudaMemset(h->dev_err, 0, sizeof(int));
  if (e == cudaSuccess) e = cudaMemset(h->binds, 0, sizeof(unsigned long long));
  if (e != cudaSuccess) { st = cuda_fail(nullptr, e, "cudaMemset (status)"); free_all(h); delete h; return st; }
  e = srnl::prepare_kernels();
  if (e != cudaSuccess) { st = cuda_fail(nullptr, e, "kernel attributes"); free_all(h); delete h; return st; }
  *out = h;
  return SRNL_OK;
}

static srnl_status run_forward(srnl_scan* h, const void* x, void* y, float* finals, cudaStream_t s) {
  srnl::ScanParamsDev p{h->Wq, h->Wqb, h->G, h->Mm, h->scales};
  cudaError_t e;
  cudaEvent_t* ev = h->ring > 0 ? &h->ev[(size_t)(h->recorded % h->ring) * 4] : nullptr;
  if (ev && (e = cudaEventRecord(ev[0], s)) != cudaSuccess) return cuda_fail(h, e, "event record");
  const bool padded = h->cfg.d < srnl::kD;
  const int elt = h->geom.act_bf16 ? 2 : 4;
  const int64_t tokens = (int64_t)h->geom.B * h->geom.H * h->geom.W;
  if (padded) {  // heads of d < 32 channels run as zero-padded 32-wide heads
    e = srnl::launch_pad_heads(x, h->x_pad, tokens, h->geom.heads, h->cfg.d, elt, s);
    if (e != cudaSuccess) return cuda_fail(h, e, "head padding launch");
    x = h->x_pad;
  }
  float* fk = padded && finals != nullptr ? h->fin_pad : finals;
  void* yk = padded ? h->y_pad : y;
  if (!srnl::scan_fuses_query(h->geom, p)) {   // otherwise the scan forms q itself
    e = srnl::launch_query_projection(h->geom, p, x, h->q, h->dev_err, s);
    if (e != cudaSuccess) return cuda_fail(h, e, "query projection launch");
  }
  if (ev && (e = cudaEventRecord(ev[1], s)) != cudaSuccess) return cuda_fail(h, e, "event record");
  if (h->geom.hard_cap && (e = cudaMemsetAsync(h->binds, 0, sizeof(unsigned long long), s)) != cudaSuccess)
    return cuda_fail(h, e, "counter reset");
  e = srnl::launch_scan(h->geom, p, x, h->q, h->yr, fk, h->dev_err, h->binds, s);
  if (e != cudaSuccess) return cuda_fail(h, e, "scan launch");
  if (ev && (e = cudaEventRecord(ev[2], s)) != cudaSuccess) return cuda_fail(h, e, "event record");
  e = srnl::launch_fuse(h->geom, h->yr, yk, s);
  if (e != cudaSuccess) return cuda_fail(h, e, "fusion launch");
  if (padded) {
    e = srnl::launch_unpad_heads(h->y_pad, y, tokens, h->geom.heads, h->cfg.d, elt, s);
    if (e == cudaSuccess && finals != nullptr)
      e = srnl::launch_unpad_states(h->fin_pad, finals, (int64_t)4 * h->geom.B * h->geom.heads, h->cfg.d, s);
    if (e != cudaSuccess) return cuda_fail(h, e, "head unpadding launch");
  }
  if (ev) {
    if ((e = cudaEventRecord(ev[3], s)) != cudaSuccess) return cuda_fail(h, e, "event record");
    ++h->recorded;
  }
  return SRNL_OK;
}

static srnl_status check_device(srnl_scan* h) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(h, e, "cudaGetDevice");
  if (dev != h->device)
    return fail(h, SRNL_E_INVAL, "current CUDA device differs from the handle's device");
  return SRNL_OK;
}

srnl_status srnl_scan_forward(srnl_scan* h, const void* x, void* y, float* final_states, void* stream) {
  if (h == nullptr) return fail(nullptr, SRNL_E_INVAL, "handle is NULL");
  h->err.clear();
  if (x == nullptr || y == nullptr) return fail(h, SRNL_E_INVAL, "x or y is NULL");
  if (!aligned16(x) || !aligned16(y)) return fail(h, SRNL_E_INVAL, "x and y must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(final_states) & 3u) != 0)
    return fail(h, SRNL_E_INVAL, "final_states must be 4-byte aligned");
  const size_t n = act_bytes(h->cfg);
  const uintptr_t xa = reinterpret_cast<uintptr_t>(x), ya = reinterpret_cast<uintptr_t>(y);
  if (xa < ya + n && ya < xa + n) return fail(h, SRNL_E_INVAL, "x and y overlap");
  srnl_status st = check_device(h);
  if (st != SRNL_OK) return st;
  return run_forward(h, x, y, final_states, static_cast<cudaStream_t>(stream));
}

static bool overlaps(const void* a, const void* b, size_t n) {
  const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return pa < pb + n && pb < pa + n;
}

srnl_status srnl_scan_backward(srnl_scan* h, const void* x, const void* dy, void* dx,
                               const srnl_scan_grads* grads, void* stream) {
  if (h == nullptr) return fail(nullptr, SRNL_E_INVAL, "handle is NULL");
  h->err.clear();
  if (x == nullptr || dy == nullptr || dx == nullptr) return fail(h, SRNL_E_INVAL, "x, dy or dx is NULL");
  if (!aligned16(x) || !aligned16(dy) || !aligned16(dx))
    return fail(h, SRNL_E_INVAL, "x, dy and dx must be 16-byte aligned");
  const size_t n = act_bytes(h->cfg);
  if (overlaps(dx, x, n) || overlaps(dx, dy, n)) return fail(h, SRNL_E_INVAL, "dx overlaps x or dy");
  if (h->geom.gen_bf16)
    return fail(h, SRNL_E_UNSUPPORTED, "the backward pass is built for gen_dtype SRNL_F32 handles");
  if (grads != nullptr) {
    const float* gp[] = {grads->W_q, grads->scales, grads->M_mem0, grads->M_k0, grads->M_v0, grads->m_eta0,
                         grads->m_alpha0};
    for (const float* q : gp)
      if ((reinterpret_cast<uintptr_t>(q) & 3u) != 0) return fail(h, SRNL_E_INVAL, "gradient buffers must be 4-byte aligned");
  }
  srnl_status st = check_device(h);
  if (st != SRNL_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool padded = h->cfg.d < srnl::kD;
  const int elt = h->geom.act_bf16 ? 2 : 4;
  const int64_t tokens = (int64_t)h->geom.B * h->geom.H * h->geom.W;
  cudaError_t e;
  if (h->bws == nullptr) {  // all or nothing: a failed allocation leaves none of the three
    const size_t nb = srnl::backward_workspace_floats(h->geom, nullptr) * sizeof(float);
    const size_t pb = padded ? (size_t)tokens * h->geom.C * elt : 0;
    void* ws = nullptr;
    void* dyp = nullptr;
    void* dxp = nullptr;
    e = cudaMalloc(&ws, nb);
    if (e == cudaSuccess && padded) e = cudaMalloc(&dyp, pb);
    if (e == cudaSuccess && padded) e = cudaMalloc(&dxp, pb);
    if (e != cudaSuccess) {
      void* got[] = {ws, dyp, dxp};
      for (void* q : got)
        if (q != nullptr) cudaFree(q);
      return cuda_fail(h, e, "cudaMalloc (backward workspace)");
    }
    h->bws = static_cast<float*>(ws);
    h->dy_pad = dyp;
    h->dx_pad = dxp;
    h->ws_bytes += nb + 2 * pb;
  }
  if (padded) {
    e = srnl::launch_pad_heads(x, h->x_pad, tokens, h->geom.heads, h->cfg.d, elt, s);
    if (e == cudaSuccess) e = srnl::launch_pad_heads(dy, h->dy_pad, tokens, h->geom.heads, h->cfg.d, elt, s);
    if (e != cudaSuccess) return cuda_fail(h, e, "head padding launch");
    x = h->x_pad;
    dy = h->dy_pad;
  }
  srnl::ScanParamsDev p{h->Wq, nullptr, h->G, h->Mm, h->scales};
  cudaEvent_t* ev = h->ring > 0 ? &h->ev[(size_t)(h->recorded % h->ring) * 4] : nullptr;
  if (ev && (e = cudaEventRecord(ev[0], s)) != cudaSuccess) return cuda_fail(h, e, "event record");
  e = srnl::launch_query_projection(h->geom, p, x, h->q, h->dev_err, s);
  if (e != cudaSuccess) return cuda_fail(h, e, "query projection launch");
  if (ev && (e = cudaEventRecord(ev[1], s)) != cudaSuccess) return cuda_fail(h, e, "event record");
  srnl::BwdGrads out{};
  float* dwq = nullptr;
  if (grads != nullptr) {
    out = srnl::BwdGrads{grads->scales, grads->M_mem0, grads->M_k0, grads->M_v0, grads->m_eta0, grads->m_alpha0};
    dwq = grads->W_q;
  }
  e = srnl::launch_backward_scan(h->geom, p, x, static_cast<const float*>(h->q), dy, h->bws, s);
  if (e != cudaSuccess) return cuda_fail(h, e, "backward scan launch");
  if (ev && (e = cudaEventRecord(ev[2], s)) != cudaSuccess) return cuda_fail(h, e, "event record");
  void* dxk = padded ? h->dx_pad : dx;
  e = srnl::launch_backward_combine(h->geom, p, h->cfg.d, x, h->bws, dxk, out, dwq, s);
  if (e != cudaSuccess) return cuda_fail(h, e, "backward combine launch");
  if (padded && (e = srnl::launch_unpad_heads(h->dx_pad, dx, tokens, h->geom.heads, h->cfg.d, elt, s)) != cudaSuccess)
    return cuda_fail(h, e, "head unpadding launch");
  if (ev) {
    if ((e = cudaEventRecord(ev[3], s)) != cudaSuccess) return cuda_fail(h, e, "event record");
    ++h->recorded;
  }
  return SRNL_OK;
}

srnl_status srnl_scan_forward_host(srnl_scan* h, const void* x_host, void* y_host, void* stream) {
  if (h == nullptr) return fail(nullptr, SRNL_E_INVAL, "handle is NULL");
  h->err.clear();
  if (x_host == nullptr || y_host == nullptr) return fail(h, SRNL_E_INVAL, "x or y is NULL");
  srnl_status st = check_device(h);
  if (st != SRNL_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t n = act_bytes(h->cfg);
  cudaError_t e = cudaMemcpyAsync(h->x_stage, x_host, n, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(h, e, "host-to-device copy");
  st = run_forward(h, h->x_stage, h->y_stage, nullptr, s);
  if (st != SRNL_OK) return st;
  e = cudaMemcpyAsync(y_host, h->y_stage, n, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(h, e, "device-to-host copy");
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(h, e, "stream synchronize");
  return SRNL_OK;
}

static srnl_status pipeline_setup(srnl_scan* h) {
  if (h->h2d != nullptr) return SRNL_OK;
  const size_t n = act_bytes(h->cfg);
  cudaError_t e = cudaMalloc(&h->x_stage1, n);
  if (e == cudaSuccess) e = cudaMalloc(&h->y_stage1, n);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->h2d, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->d2h, cudaStreamNonBlocking);
  for (int k = 0; k < 2 && e == cudaSuccess; ++k) {
    cudaEvent_t* evs[] = {&h->h2d_done[k], &h->fwd_done[k], &h->d2h_done[k]};
    for (cudaEvent_t* ev : evs)
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  }
  if (e != cudaSuccess) {  // all or nothing: release what was created, so a later call starts over
    if (h->x_stage1 != nullptr) cudaFree(h->x_stage1);
    if (h->y_stage1 != nullptr) cudaFree(h->y_stage1);
    h->x_stage1 = h->y_stage1 = nullptr;
    for (int k = 0; k < 2; ++k) {
      cudaEvent_t* evs[] = {&h->h2d_done[k], &h->fwd_done[k], &h->d2h_done[k]};
      for (cudaEvent_t* ev : evs)
        if (*ev != nullptr) { cudaEventDestroy(*ev); *ev = nullptr; }
    }
    if (h->d2h != nullptr) { cudaStreamDestroy(h->d2h); h->d2h = nullptr; }
    if (h->h2d != nullptr) { cudaStreamDestroy(h->h2d); h->h2d = nullptr; }
    return cuda_fail(h, e, "pipeline set-up");
  }
  h->ws_bytes += 2 * n;
  return SRNL_OK;
}

srnl_status srnl_scan_forward_host_async(srnl_scan* h, const void* x_host, void* y_host, void* stream) {
  if (h == nullptr) return fail(nullptr, SRNL_E_INVAL, "handle is NULL");
  h->err.clear();
  if (x_host == nullptr || y_host == nullptr) return fail(h, SRNL_E_INVAL, "x or y is NULL");
  srnl_status st = check_device(h);
  if (st != SRNL_OK) return st;
  st = pipeline_setup(h);
  if (st != SRNL_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t n = act_bytes(h->cfg);
  const int k = h->slot;
  h->slot ^= 1;
  void* xs = k == 0 ? h->x_stage : h->x_stage1;
  void* ys = k == 0 ? h->y_stage : h->y_stage1;
  cudaError_t e = cudaSuccess;
  // the slot's x buffer is free once the forward that last read it has run
  if (h->slot_used[k]) e = cudaStreamWaitEvent(h->h2d, h->fwd_done[k], 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(xs, x_host, n, cudaMemcpyHostToDevice, h->h2d);
  if (e == cudaSuccess) e = cudaEventRecord(h->h2d_done[k], h->h2d);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, h->h2d_done[k], 0);
  // its y buffer is free once the copy that last read it is done
  if (e == cudaSuccess && h->slot_used[k]) e = cudaStreamWaitEvent(s, h->d2h_done[k], 0);
  if (e != cudaSuccess) return cuda_fail(h, e, "pipelined host-to-device copy");
  st = run_forward(h, xs, ys, nullptr, s);
  if (st != SRNL_OK) return st;
  e = cudaEventRecord(h->fwd_done[k], s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(h->d2h, h->fwd_done[k], 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(y_host, ys, n, cudaMemcpyDeviceToHost, h->d2h);
  if (e == cudaSuccess) e = cudaEventRecord(h->d2h_done[k], h->d2h);
  if (e != cudaSuccess) return cuda_fail(h, e, "pipelined device-to-host copy");
  h->slot_used[k] = true;
  return SRNL_OK;
}

srnl_status srnl_scan_host_join(srnl_scan* h, void* stream) {
  if (h == nullptr) return fail(nullptr, SRNL_E_INVAL, "handle is NULL");
  for (int k = 0; k < 2; ++k)
    if (h->slot_used[k]) {
      const cudaError_t e = cudaStreamWaitEvent(static_cast<cudaStream_t>(stream), h->d2h_done[k], 0);
      if (e != cudaSuccess) return cuda_fail(h, e, "cudaStreamWaitEvent");
    }
  return SRNL_OK;
}

srnl_status srnl_scan_host_sync(srnl_scan* h) {
  if (h == nullptr) return fail(nullptr, SRNL_E_INVAL, "handle is NULL");
  if (h->d2h == nullptr) return SRNL_OK;
  const cudaError_t e = cudaStreamSynchronize(h->d2h);
  if (e != cudaSuccess) return cuda_fail(h, e, "cudaStreamSynchronize");
  return SRNL_OK;
}

srnl_status srnl_scan_route_index(const srnl_scan* hc, int route, int32_t* out, void* stream) {
  srnl_scan* h = const_cast<srnl_scan*>(hc);
  if (h == nullptr) return fail(nullptr, SRNL_E_INVAL, "handle is NULL");
  h->err.clear();
  if (out == nullptr) return fail(h, SRNL_E_INVAL, "out is NULL");
  if (route < 0 || route > 3) return fail(h, SRNL_E_INVAL, "route must be 0..3");
  cudaError_t e = srnl::launch_route_index(route, h->geom.H, h->geom.W, out, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(h, e, "route index launch");
  return SRNL_OK;
}

srnl_status srnl_scan_gather(const srnl_scan* hc, int route, const void* x, void* xr, void* stream) {
  srnl_scan* h = const_cast<srnl_scan*>(hc);
  if (h == nullptr) return fail(nullptr, SRNL_E_INVAL, "handle is NULL");
  h->err.clear();
  if (x == nullptr || xr == nullptr) return fail(h, SRNL_E_INVAL, "x or xr is NULL");
  if (!aligned16(x) || !aligned16(xr)) return fail(h, SRNL_E_INVAL, "x and xr must be 16-byte aligned");
  if (route < 0 || route > 3) return fail(h, SRNL_E_INVAL, "route must be 0..3");
  srnl::ScanGeom ug = h->geom;  // the caller's layout (C = heads * d)
  ug.C = h->cfg.C;
  cudaError_t e = srnl::launch_gather(ug, route, x, xr, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(h, e, "gather launch");
  return SRNL_OK;
}

srnl_status srnl_scan_enable_stage_timing(srnl_scan* h, int n) {
  if (h == nullptr) return fail(nullptr, SRNL_E_INVAL, "handle is NULL");
  h->err.clear();
  if (n < 0 || n > 1024) return fail(h, SRNL_E_INVAL, "ring size must be in [0, 1024]");
  for (cudaEvent_t ev : h->ev) cudaEventDestroy(ev);
  h->ev.clear();
  h->ring = 0;
  h->recorded = 0;
  if (n == 0) return SRNL_OK;
  h->ev.assign((size_t)n * 4, nullptr);
  for (auto& ev : h->ev) {
    cudaError_t e = cudaEventCreate(&ev);
    if (e != cudaSuccess) {
      for (cudaEvent_t x : h->ev)
        if (x != nullptr) cudaEventDestroy(x);
      h->ev.clear();
      return cuda_fail(h, e, "cudaEventCreate");
    }
  }
  h->ring = n;
  return SRNL_OK;
}

srnl_status srnl_scan_stage_times(srnl_scan* h, float* ms_out, int* count) {
  if (h == nullptr) return fail(nullptr, SRNL_E_INVAL, "handle is NULL");
  h->err.clear();
  if (ms_out == nullptr) return fail(h, SRNL_E_INVAL, "ms_out is NULL");
  if (h->ring == 0 || h->recorded == 0) return fail(h, SRNL_E_INVAL, "stage timing is off or no forward ran");
  const int n = h->recorded < h->ring ? h->recorded : h->ring;
  double acc[3] = {0.0, 0.0, 0.0};
  for (int k = 0; k < n; ++k) {
    cudaEvent_t* ev = &h->ev[(size_t)k * 4];
    cudaError_t e = cudaEventSynchronize(ev[3]);
    if (e != cudaSuccess) return cuda_fail(h, e, "cudaEventSynchronize");
    for (int i = 0; i < 3; ++i) {
      float ms = 0.f;
      e = cudaEventElapsedTime(&ms, ev[i], ev[i + 1]);
      if (e != cudaSuccess) return cuda_fail(h, e, "cudaEventElapsedTime");
      acc[i] += ms;
    }
  }
  for (int i = 0; i < 3; ++i) ms_out[i] = (float)(acc[i] / n);
  if (count != nullptr) *count = n;
  h->recorded = 0;
  return SRNL_OK;
}

srnl_status srnl_scan_device_status(srnl_scan* h) {
  if (h == nullptr) return fail(nullptr, SRNL_E_INVAL, "handle is NULL");
  h->err.clear();
  int v = 0;
  cudaError_t e = cudaMemcpy(&v, h->dev_err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(h, e, "status read");
  if (v != 0) return fail(h, static_cast<srnl_status>(v), "a bounded in-kernel wait gave up");
  return SRNL_OK;
}

srnl_status srnl_scan_cap_count(srnl_scan* h, unsigned long long* count) {
  if (h == nullptr || count == nullptr) return SRNL_E_INVAL;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(count, h->binds, sizeof(unsigned long long), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(h, e, "counter read");
  return SRNL_OK;
}

size_t srnl_scan_workspace_bytes(const srnl_scan* h) { return h != nullptr ? h->ws_bytes : 0; }

void srnl_scan_destroy(srnl_scan* h) {
  if (h == nullptr) return;
  int prev = -1;
  if (cudaGetDevice(&prev) == cudaSuccess && prev != h->device) cudaSetDevice(h->device);
  cudaDeviceSynchronize();
  for (cudaEvent_t ev : h->ev)
    if (ev != nullptr) cudaEventDestroy(ev);
  h->ev.clear();
  free_all(h);
  if (prev >= 0 && prev != h->device) cudaSetDevice(prev);
  delete h;
}

}  // extern "C"
