// Device helpers shared by the backward scan kernels (32- and 64-wide heads): accurate scalar
// gate math and its reverse mode.  Sources as in srnl_scan_bwd.cu.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace srnl {
namespace bwd {

__device__ __forceinline__ float load_act(const void* base, int64_t idx, bool bf16) {
  if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[idx]);
  return reinterpret_cast<const float*>(base)[idx];
}

__device__ __forceinline__ float sigmoid_f(float z) {
  const float e = expf(-fabsf(z));
  return z >= 0.f ? 1.f / (1.f + e) : e / (1.f + e);
}

__device__ __forceinline__ float softplus_f(float z) { return fmaxf(z, 0.f) + log1pf(expf(-fabsf(z))); }

// phi(z) = tanh(z) / z, by 1 - z^2/3 below 1e-4.
__device__ __forceinline__ float phi_f(float z) { return z < 1e-4f ? 1.f - z * z * (1.f / 3.f) : tanhf(z) / z; }

// phi'(z) for z >= 0: below 0.25 the Taylor series -2z/3 + 8z^3/15 - 102z^5/315 + 496z^7/2835
// of the derivative of tanh(z)/z (the closed form cancels there in fp32), else
// (z sech^2 z - tanh z) / z^2, with sech^2 z = 4e / (1 + e)^2 and e = exp(-2z) returned in
// sech2 (0 below 0.25, where it is not used).  1 - tanh^2 z would lose the small value once
// tanh z rounds near 1: its relative error reaches 1e-3 around z = 5.
__device__ __forceinline__ float dphi_f(float z, float& sech2) {
  if (z < 0.25f) {
    const float z2 = z * z;
    sech2 = 0.f;
    return z * (-2.f / 3.f + z2 * (8.f / 15.f + z2 * (-102.f / 315.f + z2 * (496.f / 2835.f))));
  }
  const float e = expf(-2.f * z);
  const float inv = 1.f / (1.f + e);
  const float t = (1.f - e) * inv;
  sech2 = 4.f * e * inv * inv;
  return (z * sech2 - t) / (z * z);
}

// Scalar gates of one token from |k|^2, |k - v|^2, a and beta (the forward's clamp decisions):
// alpha_t and eta.
__device__ __forceinline__ void gate_scalars_f(float kn2, float ne2, float a, float beta, float alpha_max, bool hard,
                                               float& al, float& eta) {
  const float gain = sqrtf(ne2) * sqrtf(kn2);
  al = fminf(sigmoid_f(beta), alpha_max);
  const float eta0 = softplus_f(a);
  const float m = 1.f - al;
  float eta1;
  if (hard) eta1 = (eta0 * gain > m) ? m / gain : eta0;
  else eta1 = eta0 * phi_f(eta0 * gain / m);
  eta = (eta1 * kn2 > 2.f) ? 2.f / kn2 : eta1;
}

// Scalar part of the gate backward for one token (one lane per token).  In: sc[0] = dL/dalpha_t
// so far, sc[1] = dL/deta_t, sc[2] = |k|^2, sc[3] = |k - v|^2; the token's alpha_t, a, beta.
// Out: sc[4] = c_e, sc[5] = c_k with dk += c_e (k - v) + c_k k and dv -= c_e (k - v) (the gain
// and spectral-clamp paths), sc[6] = dL/da, sc[7] = dL/dbeta.
__device__ __forceinline__ void gate_backward_scalars_f(float* sc, float al, float a, float beta, float alpha_max,
                                                        bool hard) {
  float dal = sc[0];
  const float deta = sc[1], kn2 = sc[2];
  const float ne = sqrtf(sc[3]), kn = sqrtf(kn2), gain = ne * kn;
  const float sg = sigmoid_f(beta);
  const float eta0 = softplus_f(a);
  const float m = 1.f - al;
  float eta1;
  if (hard) eta1 = (eta0 * gain > m) ? m / gain : eta0;
  else eta1 = eta0 * phi_f(eta0 * gain / m);
  const bool over = eta1 * kn2 > 2.f;                        // spectral clamp eta = 2 / |k|^2
  const float deta1 = over ? 0.f : deta;
  const float dkn2 = over ? -2.f * deta / (kn2 * kn2) : 0.f;
  float deta0, dgain;
  if (hard) {                                                // eta1 = min(eta0, (1 - alpha_t) / g)
    const bool binds = eta0 * gain > m;
    deta0 = binds ? 0.f : deta1;
    dgain = binds ? -deta1 * m / (gain * gain) : 0.f;
    if (binds) dal -= deta1 / gain;
  } else {                                                   // eta1 = eta0 phi(eta0 g / (1 - alpha_t))
    const float z = eta0 * gain / m;
    float sech2;
    const float dph = dphi_f(z, sech2);
    const float dz = deta1 * eta0 * dph;
    // d(eta0 phi(eta0 g / m)) / d eta0 = phi(z) + z phi'(z) = sech^2 z: taken directly above the
    // series range, where the sum of the two would cancel
    deta0 = (z < 0.25f) ? deta1 * phi_f(z) + dz * gain / m : deta1 * sech2;
    dgain = dz * eta0 / m;
    dal += dz * eta0 * gain / (m * m);
  }
  sc[4] = (ne > 0.f) ? dgain * kn / ne : 0.f;                // g = |k - v| |k|
  sc[5] = 2.f * dkn2 + (kn > 0.f ? dgain * ne / kn : 0.f);
  sc[6] = deta0 * sigmoid_f(a);                              // eta0 = softplus(a)
  sc[7] = (sg > alpha_max) ? 0.f : dal * sg * (1.f - sg);    // alpha_t = min(sigmoid(beta), alpha)
}

}  // namespace bwd
}  // namespace srnl
