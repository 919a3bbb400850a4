// Helpers of the CUDA-core (SIMT) kernels: input loads, the feature map in
// fp32, complex arithmetic on float2, per-mode constants of the S4D
// recurrence in fp64 and a warp sum.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace ia {
namespace simt {

template <typename T>
__device__ __forceinline__ float ldf(const T* p);
template <>
__device__ __forceinline__ float ldf<float>(const float* p) {
  return *p;
}
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

__device__ __forceinline__ float feat_acc(float x) { return x > 0.f ? x + 1.f : expf(x); }
__device__ __forceinline__ float dfeat_acc(float x) { return x > 0.f ? 1.f : expf(x); }

__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
  return make_float2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}
__device__ __forceinline__ float2 cfma(float2 a, float2 b, float2 c) {  // a*b + c
  return make_float2(fmaf(a.x, b.x, fmaf(-a.y, b.y, c.x)), fmaf(a.x, b.y, fmaf(a.y, b.x, c.y)));
}
__device__ __forceinline__ float re_conj_mul(float2 a, float2 b) {  // Re(conj(a) b)
  return fmaf(a.x, b.x, a.y * b.y);
}

// Mode constants in fp64: A_m (S4D-Lin unless given), lambda = exp(Delta A),
// b = (lambda - 1) / A (zero-order hold).
struct ModeD {
  double ar, ai, lr, li, br, bi;
};
__device__ __forceinline__ ModeD mode_consts(float delta, const float* A, int m) {
  ModeD r;
  r.ar = A ? static_cast<double>(A[2 * m]) : -0.5;
  r.ai = A ? static_cast<double>(A[2 * m + 1]) : 3.14159265358979323846 * m;
  double d = static_cast<double>(delta);
  double e = exp(d * r.ar), s, c;
  sincos(d * r.ai, &s, &c);
  r.lr = e * c;
  r.li = e * s;
  double nr = r.lr - 1.0, ni = r.li, den = r.ar * r.ar + r.ai * r.ai;
  r.br = (nr * r.ar + ni * r.ai) / den;
  r.bi = (ni * r.ar - nr * r.ai) / den;
  return r;
}

// lambda^n = exp(n Delta A) with the phase reduced in fp64.
__device__ __forceinline__ void cpow_d(double re_dA, double im_dA, double n, double* pr, double* pi) {
  double e = exp(n * re_dA);
  double ph = fmod(n * im_dA, 6.283185307179586476925);
  double s, c;
  sincos(ph, &s, &c);
  *pr = e * c;
  *pi = e * s;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}


}  // namespace simt
using namespace simt;
}  // namespace ia
