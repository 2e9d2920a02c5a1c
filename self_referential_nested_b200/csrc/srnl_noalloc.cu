// srnl_scan_forward_noalloc: the forward pass without any device allocation.
//
// For callers that must not call cudaMalloc: code hosted by a framework that
// owns all device memory through its own pool (a raw cudaMalloc bypasses its
// accounting and can fail or fragment the pool), and latency-critical loops
// where cudaMalloc may synchronise the device and take unbounded time.
//
// The scratch the forward needs (repacked parameters, the projected queries
// and the four scaled route partials) lives in one file-scope __device__ array
// of kNoallocScratchBytes.  Every GPU that loads this library holds that array
// until the process exits.  In host code the array's name is only a host-side
// stand-in, so its device address is looked up with cudaGetSymbolAddress once
// per device, on the first call made with that device current, and cached.
//
// All calls share the array and it keeps the last call's contents.  Only the
// status word at its start must begin at zero, and every call clears it first
// (an asynchronous memset on the caller's stream); every other byte a call
// reads is written earlier in the same call (pack, projection, scan in that
// order on the caller's stream).  srnl_scan_noalloc_status reads the word back.
// Calls that overlap on the GPU (for example on two streams) race on the array.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <string>

#include "srnl_common.cuh"
#include "srnl_internal.h"
#include "srnl_launch.h"
#include "srnl_scan.h"

namespace {

constexpr size_t kNoallocScratchBytes = SRNL_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array for the current device.  Set up once per device, with
// that device current: the array's address, and the kernels' one-time function attributes.
srnl_status scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    srnl::set_thread_error(std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    return SRNL_E_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    srnl::set_thread_error("device ordinal out of range for the no-allocation scratch table");
    return SRNL_E_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      srnl::set_thread_error(std::string("cudaGetSymbolAddress(scratch): ") + cudaGetErrorString(e));
      return SRNL_E_CUDA;
    }
    e = srnl::prepare_kernels();
    if (e != cudaSuccess) {
      srnl::set_thread_error(std::string("kernel attributes: ") + cudaGetErrorString(e));
      return SRNL_E_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SRNL_OK;
}

size_t round_up(size_t n) { return (n + 255) & ~size_t(255); }

// A pointer the kernels may read or write on the current device: device memory of this
// device, or managed memory.  Host memory (pageable, pinned or mapped) is refused.
bool on_this_device(const void* p, int dev) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();   // reset the runtime's last error after the failed query
    return false;
  }
  if (a.type == cudaMemoryTypeManaged) return true;
  return a.type == cudaMemoryTypeDevice && a.device == dev;
}

// W_q copy (bf16-rounded on the bf16 path, plus a bf16 copy for the tensor-core projection)
// and G = [M_k0; M_v0; m_eta0; m_alpha0] per (route, head), the layouts the kernels read.
__global__ void noalloc_pack_kernel(const float* __restrict__ Wq_src, float* __restrict__ Wq_dst,
                                    __nv_bfloat16* __restrict__ Wqb_dst,
                                    int64_t n_wq, bool round_bf16_wq, const float* __restrict__ Mk,
                                    const float* __restrict__ Mv, const float* __restrict__ me,
                                    const float* __restrict__ ma, float* __restrict__ G,
                                    int64_t n_g) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n_wq) {
    const float w = Wq_src[i];
    Wq_dst[i] = round_bf16_wq ? srnl::round_bf16(w) : w;
    if (Wqb_dst != nullptr) Wqb_dst[i] = __float2bfloat16_rn(w);
  }
  if (i < n_g) {
    constexpr int per = srnl::kGen * srnl::kD;
    const int64_t rh = i / per;
    const int rem = (int)(i - rh * per);
    const int m = rem / srnl::kD, j = rem % srnl::kD;
    float v;
    if (m < srnl::kD) v = Mk[(rh * srnl::kD + m) * srnl::kD + j];
    else if (m < 2 * srnl::kD) v = Mv[(rh * srnl::kD + (m - srnl::kD)) * srnl::kD + j];
    else if (m == 2 * srnl::kD) v = me[rh * srnl::kD + j];
    else v = ma[rh * srnl::kD + j];
    G[i] = v;
  }
}

}  // namespace

extern "C" srnl_status srnl_scan_forward_noalloc(const srnl_scan_config* cfg,
                                                 const srnl_scan_params* p, const void* x,
                                                 void* y, void* stream) {
  srnl::set_thread_error("");
  if (cfg == nullptr || p == nullptr) {
    srnl::set_thread_error("cfg or params is NULL");
    return SRNL_E_INVAL;
  }
  if (p->W_q == nullptr || p->scales == nullptr || p->M_mem0 == nullptr || p->M_k0 == nullptr ||
      p->M_v0 == nullptr || p->m_eta0 == nullptr || p->m_alpha0 == nullptr) {
    srnl::set_thread_error("a parameter pointer is NULL");
    return SRNL_E_INVAL;
  }
  srnl_status st = srnl::validate_scan_config(cfg);
  if (st != SRNL_OK) return st;
  if (cfg->d != srnl::kD) {
    srnl::set_thread_error("the no-allocation forward is built for head dim d = 32 only");
    return SRNL_E_UNSUPPORTED;
  }
  if (x == nullptr || y == nullptr) {
    srnl::set_thread_error("x or y is NULL");
    return SRNL_E_INVAL;
  }
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(y) & 15u)) {
    srnl::set_thread_error("x and y must be 16-byte aligned");
    return SRNL_E_INVAL;
  }
  {
    // the kernels read every parameter array as fp32 scalars or float4 rows of 4-aligned
    // starts; a pointer that is not 4-byte aligned would fault on the device
    const void* ps[7] = {p->W_q, p->scales, p->M_mem0, p->M_k0, p->M_v0, p->m_eta0, p->m_alpha0};
    for (const void* q : ps)
      if (reinterpret_cast<uintptr_t>(q) & 3u) {
        srnl::set_thread_error("every parameter pointer must be 4-byte aligned (fp32 arrays)");
        return SRNL_E_INVAL;
      }
  }
  const bool act_bf16 = cfg->act_dtype == SRNL_BF16, gen_bf16 = cfg->gen_dtype == SRNL_BF16;
  const size_t tokens = (size_t)cfg->B * cfg->H * cfg->W;
  const size_t act_bytes = tokens * cfg->C * (act_bf16 ? 2 : 4);
  {
    const uintptr_t xa = reinterpret_cast<uintptr_t>(x), ya = reinterpret_cast<uintptr_t>(y);
    if (xa < ya + act_bytes && ya < xa + act_bytes) {
      srnl::set_thread_error("x and y overlap");
      return SRNL_E_INVAL;
    }
  }
  const size_t n_wq = (size_t)cfg->C * cfg->C;
  const size_t n_g = (size_t)4 * cfg->heads * srnl::kGen * srnl::kD;
  const size_t wq_b = round_up(n_wq * 4), g_b = round_up(n_g * 4);
  const size_t wqb_b = gen_bf16 ? round_up(n_wq * 2) : 0;
  const size_t q_b = round_up(tokens * cfg->C * (gen_bf16 ? 2 : 4));
  const size_t yr_b = round_up(4 * tokens * cfg->C * sizeof(float));
  const size_t err_b = 256;  // device status word of the scan kernel
  const size_t need = err_b + wq_b + wqb_b + g_b + q_b + yr_b;
  if (need > kNoallocScratchBytes) {
    srnl::set_thread_error("workload needs " + std::to_string(need) +
                           " bytes of scratch; the no-allocation forward holds " +
                           std::to_string(kNoallocScratchBytes));
    return SRNL_E_INVAL;
  }
  {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
      srnl::set_thread_error("cudaGetDevice failed");
      return SRNL_E_CUDA;
    }
    const void* ps[9] = {x, y, p->W_q, p->scales, p->M_mem0, p->M_k0, p->M_v0, p->m_eta0, p->m_alpha0};
    const char* names[9] = {"x", "y", "W_q", "scales", "M_mem0", "M_k0", "M_v0", "m_eta0", "m_alpha0"};
    for (int i = 0; i < 9; ++i)
      if (!on_this_device(ps[i], dev)) {
        srnl::set_thread_error(std::string(names[i]) + " is not device (or managed) memory of the current device");
        return SRNL_E_INVAL;
      }
  }
  void* base = nullptr;
  st = scratch_address(&base);
  if (st != SRNL_OK) return st;
  unsigned char* s8 = static_cast<unsigned char*>(base);
  int* dev_err = reinterpret_cast<int*>(s8);
  s8 += err_b;
  float* Wq = reinterpret_cast<float*>(s8);
  __nv_bfloat16* Wqb = gen_bf16 ? reinterpret_cast<__nv_bfloat16*>(s8 + wq_b) : nullptr;
  s8 += wq_b + wqb_b;
  float* G = reinterpret_cast<float*>(s8);
  void* q = s8 + g_b;
  float* yr = reinterpret_cast<float*>(s8 + g_b + q_b);

  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(dev_err, 0, sizeof(int), cs);   // status of this call
  const size_t n_pack = n_wq > n_g ? n_wq : n_g;
  if (e == cudaSuccess) {
    noalloc_pack_kernel<<<(unsigned)((n_pack + 255) / 256), 256, 0, cs>>>(
        p->W_q, Wq, Wqb, (int64_t)n_wq, gen_bf16, p->M_k0, p->M_v0, p->m_eta0, p->m_alpha0, G, (int64_t)n_g);
    e = cudaGetLastError();
  }

  srnl::ScanGeom g{};
  g.B = cfg->B; g.H = cfg->H; g.W = cfg->W; g.C = cfg->C; g.heads = cfg->heads;
  g.Lrow = cfg->chunk_row > 0 ? cfg->chunk_row : cfg->W;
  g.Lcol = cfg->chunk_col > 0 ? cfg->chunk_col : cfg->H;
  g.alpha = cfg->alpha; g.eps = cfg->eps;
  g.act_bf16 = act_bf16; g.gen_bf16 = gen_bf16;
  g.hard_cap = cfg->injection_cap == SRNL_CAP_HARD;
  const srnl::ScanParamsDev dp{Wq, Wqb, G, p->M_mem0, p->scales};
  if (e == cudaSuccess && !srnl::scan_fuses_query(g, dp)) e = srnl::launch_query_projection(g, dp, x, q, dev_err, cs);
  if (e == cudaSuccess) e = srnl::launch_scan(g, dp, x, q, yr, nullptr, dev_err, nullptr, cs);
  if (e == cudaSuccess) e = srnl::launch_fuse(g, yr, y, cs);
  if (e != cudaSuccess) {
    srnl::set_thread_error(std::string("no-allocation forward launch: ") + cudaGetErrorString(e));
    return SRNL_E_CUDA;
  }
  return SRNL_OK;
}

extern "C" srnl_status srnl_scan_noalloc_status(void* stream) {
  srnl::set_thread_error("");
  void* base = nullptr;
  const srnl_status st = scratch_address(&base);
  if (st != SRNL_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_noalloc_scratch, sizeof(int), 0, cudaMemcpyDeviceToHost, cs);
  if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
  if (e != cudaSuccess) {
    srnl::set_thread_error(std::string("no-allocation status read: ") + cudaGetErrorString(e));
    return SRNL_E_CUDA;
  }
  if (v != 0) {
    srnl::set_thread_error("a bounded in-kernel wait of the last no-allocation forward gave up");
    return static_cast<srnl_status>(v);
  }
  return SRNL_OK;
}

extern "C" srnl_status srnl_selftest_noalloc_wait_timeout(int wait_ms, void* stream) {
  srnl::set_thread_error("");
  if (wait_ms < 1 || wait_ms > 5000) {
    srnl::set_thread_error("wait_ms must lie in [1, 5000]");
    return SRNL_E_INVAL;
  }
  void* base = nullptr;
  const srnl_status st = scratch_address(&base);
  if (st != SRNL_OK) return st;
  const cudaError_t e = srnl::launch_wait_probe((unsigned long long)wait_ms * 1000000ull,
                                                static_cast<int*>(base), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    srnl::set_thread_error(std::string("self-test launch: ") + cudaGetErrorString(e));
    return SRNL_E_CUDA;
  }
  return SRNL_OK;
}
