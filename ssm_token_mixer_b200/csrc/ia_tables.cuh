// Per-head constant tables of the chunked IA recurrence (paperlayer.ai
// summary of 'Interdomain Attention', sec. 3.2: complex-diagonal S4D with
// zero-order hold; chunk length 64 per sec. A.2).
//
// With C = 64, centre c = C/2 and positions j in [0, C):
//   E'[j,m]   = b_m lambda_m^(c-j)         (one table serves the within-chunk
//                                            decay, the readout and the carry)
//   lamC[m]   = lambda_m^C                  chunk-to-chunk decay
//   sc[m]     = lambda_m^(C-c-1)            the running state is kept as
//                                            S_hat = S / sc  (sc_inv = 1/sc)
//   esum[m]   = sum_j E'[j,m]               carry of the constant-1 channel
//   r2[m]     = |lambda_m|^2, s0[m] = |lambda_m|^(-2c)   readout row scale
//                                            s[i,m] = s0 r2^i = |lambda|^(2(i-c))
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace ia {

constexpr int kChunk = 64;
constexpr int kModesTC = 64;            // modes on the tensor-core path (2M = 128 MMA rows)

struct alignas(256) HeadTables {
  // E'^T as fp16 rows k = 2m + {0: re, 1: im}, columns j, in the no-swizzle
  // K-major core-matrix layout: byte (k/8)*1024 + (j/8)*128 + (k%8)*16 + (j%8)*2.
  __half E[2 * kModesTC * kChunk];
  float2 lam[kModesTC];
  float2 b[kModesTC];
  float2 lamC[kModesTC];
  float2 sc[kModesTC];
  float2 sc_inv[kModesTC];
  float2 esum[kModesTC];
  float r2[kModesTC];
  float s0[kModesTC];
  double re_dA[kModesTC];   // Delta * Re(A_m)
  double im_dA[kModesTC];   // Delta * Im(A_m)
};

__host__ __device__ constexpr uint32_t etab_offset(int k, int j) {
  return static_cast<uint32_t>((k >> 3) * 1024 + (j >> 3) * 128 + (k & 7) * 16 + (j & 7) * 2);
}

// The complex readout matrix W_h [M x M] as the real [2M x 2M] matrix W' of
// rows k = 2m + {0: re, 1: im} and columns k' = 2m' + {0, 1}
// (W'[2m][2m'] = W'[2m+1][2m'+1] = Re W[m][m'], W'[2m][2m'+1] = -Im W[m][m'],
// W'[2m+1][2m'] = Im W[m][m']), fp16 in the no-swizzle K-major core-matrix
// layout with K = 2M: byte (k/8)*2048 + (k'/8)*128 + (k%8)*16 + (k'%8)*2.
constexpr uint32_t kWprimeBytes = 2 * kModesTC * 2 * kModesTC * 2;
__host__ __device__ constexpr uint32_t wprime_offset(int k, int kp) {
  return static_cast<uint32_t>((k >> 3) * 2048 + (kp >> 3) * 128 + (k & 7) * 16 + (kp & 7) * 2);
}

}  // namespace ia
