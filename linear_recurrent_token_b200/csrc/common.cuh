// Shared device helpers of the mLSTM / retention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mlstm {

// Storage types of q, k, v, o, h.
template <typename T> struct io;
template <> struct io<float> {
  static __device__ __forceinline__ float load(const float* p, size_t i) { return p[i]; }
  static __device__ __forceinline__ void store(float* p, size_t i, float x) { p[i] = x; }
};
template <> struct io<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p, size_t i) {
    return __bfloat162float(p[i]);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, size_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
  }
};

// log(sigmoid(x)) in the form that cannot overflow: min(x, 0) - log1p(exp(-|x|)).
__device__ __forceinline__ float log_sigmoid(float x) {
  return fminf(x, 0.f) - log1pf(expf(-fabsf(x)));
}

// log(gamma_h) of retention head h: gamma_h = 1 - 2^(-5-h)  (RetNet "Multi-Scale Retention").
__device__ __forceinline__ float retention_log_gamma(int head) {
  return log1pf(-exp2f(-5.f - (float)head));
}

// One step of the stabiliser recurrence x_t = max(a_t + x_{t-1}, b_t), stored as the affine
// max-plus map x -> max(A + x, Bm).  Composition "first p then q" is
// (p.A + q.A, max(p.Bm + q.A, q.Bm)); identity is (0, -inf).
struct MaxPlus {
  float A, Bm;
};
__device__ __forceinline__ MaxPlus mp_then(MaxPlus p, MaxPlus q) {
  return MaxPlus{p.A + q.A, fmaxf(p.Bm + q.A, q.Bm)};
}
__device__ __forceinline__ float mp_apply(MaxPlus p, float x) { return fmaxf(p.A + x, p.Bm); }

}  // namespace mlstm
