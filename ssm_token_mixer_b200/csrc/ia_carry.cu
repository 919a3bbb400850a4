// Carry composition across spans of one sequence (summary sec. A.2: parallel
// passes over pieces, sequential state passing between them).  The recurrence
// is linear in its state: after L more tokens, a state S0 has become
// lambda^L S0 plus what those tokens alone would have built from zero.  So a
// span's carry-in is its predecessor's carry-in decayed by lambda^L (L the
// predecessor span's length) plus the predecessor's local end state:
//   out = lambda^L carry_in + local,  per (b,h) and mode, over U, Gamma, eta,
// with lambda = exp(Delta A).  This is what a sequence split across GPUs
// exchanges: one all-gather of the local end states, then this composition.
#include <cmath>

#include "ia_device.cuh"
#include "ia_internal.h"

namespace ia {
namespace {

constexpr int kCarryThreads = 128;

// one block per (b,h,m): lambda^L once in fp64, then every entry of that row
__global__ void __launch_bounds__(kCarryThreads) state_carry_kernel(
    int H, int M, int DX, int DV, const float* __restrict__ delta, int dpm, const float* __restrict__ A,
    double L, const float2* cin, const float2* loc, float2* out, long long BH) {   // out may alias cin or loc
  __shared__ double lam[2];
  const long long row = blockIdx.x;   // bh * M + m
  const long long bh = row / M;
  const int m = static_cast<int>(row - bh * M);
  const int h = static_cast<int>(bh % H);
  if (threadIdx.x == 0) {
    const double ar = A ? A[2 * m] : -0.5;
    const double ai = A ? A[2 * m + 1] : 3.14159265358979323846 * m;
    const double d = delta_hm(delta, dpm, M, h, m);
    const double e = exp(L * d * ar);
    const double ph = fmod(L * d * ai, 6.283185307179586476925);
    double sn, cs;
    sincos(ph, &sn, &cs);
    lam[0] = e * cs;
    lam[1] = e * sn;
  }
  __syncthreads();
  const double lr = lam[0], li = lam[1];
  auto mac = [&](long long i) {
    const float2 x = cin ? cin[i] : make_float2(0.f, 0.f);
    const float2 y = loc[i];
    out[i] = make_float2(static_cast<float>(lr * x.x - li * x.y + y.x),
                         static_cast<float>(lr * x.y + li * x.x + y.y));
  };
  for (int f = threadIdx.x; f < DX; f += kCarryThreads) mac(row * DX + f);
  for (int f = threadIdx.x; f < DV; f += kCarryThreads) mac(BH * M * DX + row * DV + f);
  if (threadIdx.x == 0) mac(BH * M * (DX + DV) + row);
}

}  // namespace

cudaError_t launch_state_carry(const ia_shape_t& s, const float* delta, const float* A, long long L,
                               const void* carry_in, const void* local, void* out, cudaStream_t st) {
  const long long BH = static_cast<long long>(s.B) * s.H;
  const long long rows = BH * s.M;
  state_carry_kernel<<<static_cast<unsigned>(rows), kCarryThreads, 0, st>>>(
      s.H, s.M, s.d_xi, s.d_v, delta, s.delta_per_mode, A, static_cast<double>(L),
      static_cast<const float2*>(carry_in), static_cast<const float2*>(local), static_cast<float2*>(out), BH);
  return cudaGetLastError();
}

}  // namespace ia
