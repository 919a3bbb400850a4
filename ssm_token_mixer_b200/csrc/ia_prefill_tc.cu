// Chunked IA prefill on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// What it computes is the causal IA layer (paper 'Interdomain Attention:
// Beyond Token-Level Key-Value Memory'; paperlayer.ai summary sec. 3.1-3.2;
// AI-radio page formula extract "O = Fq U^T Gamma / Fq U^T eta"), run
// chunkwise with chunk length C = 64 and state passing between chunks as the
// summary's sec. A.2 describes.  Per (b,h) and chunk, with positions i, j in
// [0, C), centre c = C/2 and the per-head table E'[j,m] = b_m lambda_m^(c-j):
//
//   S^T   = xi(K) xi(Q)^T                         GEMM1  (masked j <= i)
//   a~^T  = E'^T S^T + R_U xi(Q)^T                GEMM2 + GEMM3   (a_i = lambda^(i-c) a~_i)
//   X     = |lambda|^(2(i-c)) a~                  (rows re/im; = conj(a) lambda^(i-c))
//   P     = X E'^T                                GEMM4  (masked j <= i)
//   num   = P V + X R_Gamma,  den = P 1 + X R_eta GEMM5,5b + GEMM6,6b
//   o     = num / den
//   S_hat <- R + E'^T [xi(K) | V]                 GEMM7  (accumulated onto R in TMEM)
//
// where the running state is kept scaled, S_hat = lambda^-(C-c-1) S, so that
// R = lambda^C S_hat is both the decayed state the chunk adds to and the
// carried state its queries read (lambda^(c+1) S0).  Complex numbers are
// split into real rows k = 2m (re) and 2m+1 (im), so every contraction is a
// real fp16 x fp16 -> fp32 tcgen05 MMA with M = 64 or 128.
//
// Layouts: every shared-memory operand is in the no-swizzle canonical layout
// (core matrices of 8 rows x 16 bytes, 128 contiguous bytes).  A tile with
// rows r and columns x (x contiguous) of width W stores element (r, x) at
//   (r/8)*(W*16) + (x/8)*128 + (r%8)*16 + (x%8)*2,
// which serves as K-major (rows = M/N, lbo 128, sbo W*16) or as MN-major
// (columns = M/N, lbo W*16, sbo 128) depending on the contraction.
//
// TMEM columns: [0,F) scaled state rows k; [F,F+64) a~^T (den aliases its
// first 16 columns later in the chunk); [F+64,F+128) S^T then P (M=64
// layout); [F+128, F+128+DV) num (M=64 layout).  F = d_xi + d_v.
//
// Sequences are split into segments when (b,h) pairs alone cannot fill the
// GPU: a state-only pass produces each segment's local end state, a scan
// combines them (S_in(s+1) = lambda^L S_in(s) + S_local(s)), and the full
// pass recomputes every segment from its carried-in state -- the two
// parallel passes around a sequential carry pass of the summary's sec. A.2.
#include <cmath>
#include <cstdlib>

#include "ia_device.cuh"
#include "ia_internal.h"
#include "ia_tables.cuh"
#include "ia_tc_common.cuh"

namespace ia {
namespace {

using namespace tc;

template <int DX, int DV>
struct Cfg {
  static constexpr int F = DX + DV;
  static constexpr uint32_t RSX = DX * 16;   // row-group stride of an [r][DX] fp16 tile
  static constexpr uint32_t RSV = DV * 16;
  static constexpr uint32_t T_STATE = 0, T_A = F, T_DEN = F, T_SP = F + 64, T_NUM = F + 128;
  static_assert(F + 128 + DV <= 512, "TMEM budget");
  static_assert(DX % 64 == 0 && DV % 64 == 0, "feature widths must be multiples of 64");
  static constexpr uint32_t STG_Q = 0;
  static constexpr uint32_t STG_K = STG_Q + C * DX * 2;
  static constexpr uint32_t STG_V = STG_K + C * DX * 2;
  static constexpr uint32_t S_Q = STG_V + C * DV * 2;
  static constexpr uint32_t S_K = S_Q + C * DX * 2;
  static constexpr uint32_t S_V = S_K + C * DX * 2;
  static constexpr uint32_t S_E = S_V + C * DV * 2;
  static constexpr uint32_t S_SP = S_E + KR * C * 2;
  static constexpr uint32_t S_X = S_SP + C * C * 2;
  static constexpr uint32_t S_RU = S_X + KR * C * 2;
  static constexpr uint32_t S_RG = S_RU + KR * DX * 2;
  static constexpr uint32_t S_RE = S_RG + KR * DV * 2;
  static constexpr uint32_t S_ONES = S_RE + KR * 16 * 2;
  static constexpr uint32_t S_BAR = S_ONES + C * 16 * 2;
  static constexpr uint32_t S_TMEMH = S_BAR + 32;
  static constexpr uint32_t SMEM = S_TMEMH + 16;
};

struct TcArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const HeadTables* tabs;
  const float2* state_in;   // public layout, unscaled; seeds segment 0 of the full pass
  float* seg_state;         // [BH][nseg-1][128][F] scaled: local end states, then carries
  float* seg_eta;           // [BH][nseg-1][128]
  float* o;
  float* num;
  float* den;
  float2* state_out;
  int* err;                 // device error flag
  float* dump_R;            // optional: R = lambda^C S_hat at every chunk start, [BH][nch][128][F]
  float* dump_Re;           // optional: the eta part, [BH][nch][128]
  int H, N, nseg, seg_chunks;
  long long BH;
};

template <int DX, int DV, bool FULL>
__global__ void __launch_bounds__(NTHR, 1) tc_prefill_kernel(const TcArgs a) {
  using K = Cfg<DX, DV>;
  constexpr int F = K::F;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;
  const int nrun = FULL ? a.nseg : a.nseg - 1;
  const long long bh = blockIdx.x / nrun;
  const int seg = static_cast<int>(blockIdx.x % nrun);
  const int h = static_cast<int>(bh % a.H);
  const HeadTables* T = a.tabs + h;
  const int nch_total = (a.N + C - 1) / C;
  const int ch0 = seg * a.seg_chunks;
  const int ch1 = min(ch0 + a.seg_chunks, nch_total);

  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(smem + K::S_BAR);
  uint64_t* bar_mma = bar_tma + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + K::S_TMEMH);
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar_tma, 1);
    mbar_init(bar_mma, 1);
    fence_barrier_init();
  }
  {  // E' table -> shared (already in canonical layout), constant tiles
    const uint4* src = reinterpret_cast<const uint4*>(T->E);
    uint4* dst = reinterpret_cast<uint4*>(smem + K::S_E);
    for (int i = tid; i < KR * C * 2 / 16; i += NTHR) dst[i] = src[i];
    if (FULL) {
      uint4* ones = reinterpret_cast<uint4*>(smem + K::S_ONES);
      const uint32_t one2 = 0x3C003C00u;   // two fp16 ones
      for (int i = tid; i < C * 16 * 2 / 16; i += NTHR) ones[i] = make_uint4(one2, one2, one2, one2);
      uint4* re = reinterpret_cast<uint4*>(smem + K::S_RE);
      for (int i = tid; i < KR * 16 * 2 / 16; i += NTHR) re[i] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // Per-thread row constants: TMEM lane / state row k = 2m + comp.
  const int k = 32 * quad + lane;
  const int m = k >> 1, comp = k & 1;
  const float2 lamC = T->lamC[m];
  const float sgnLi = comp ? lamC.y : -lamC.y;
  const float r2 = T->r2[m];
  const float s_start = static_cast<float>(exp(2.0 * T->re_dA[m] * (32.0 * half - C / 2)));
  const float esum_c = comp ? T->esum[m].y : T->esum[m].x;
  const uint32_t trow = tmem + (static_cast<uint32_t>(32 * quad) << 16);

  // Initial (scaled) state into TMEM rows.
  float eta_c = 0.f;
  {
    const float* carry = nullptr;
    const float* carry_eta = nullptr;
    if (FULL && seg > 0) {
      carry = a.seg_state + ((bh * (a.nseg - 1) + (seg - 1)) * KR + k) * F;
      carry_eta = a.seg_eta + (bh * (a.nseg - 1) + (seg - 1)) * KR + k;
    }
    const bool from_in = FULL && seg == 0 && a.state_in != nullptr;
    const float2 si = T->sc_inv[m];
    for (int cb = 0; cb < F / 2; cb += 16) {
      const int col0 = half * (F / 2) + cb;
      uint32_t r[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        float val = 0.f;
        const int f = col0 + e;
        if (carry) {
          val = carry[f];
        } else if (from_in) {
          float2 x = f < DX ? a.state_in[(bh * 64 + m) * DX + f]
                            : a.state_in[a.BH * 64 * DX + (bh * 64 + m) * DV + (f - DX)];
          val = comp ? fmaf(si.x, x.y, si.y * x.x) : fmaf(si.x, x.x, -si.y * x.y);
        }
        r[e] = __float_as_uint(val);
      }
      tmem_st16(trow + K::T_STATE + col0, r);
    }
    if (carry_eta) {
      eta_c = *carry_eta;
    } else if (from_in) {
      float2 x = a.state_in[a.BH * 64 * F + bh * 64 + m];
      eta_c = comp ? fmaf(si.x, x.y, si.y * x.x) : fmaf(si.x, x.x, -si.y * x.y);
    }
    tmem_st_wait();
  }

  auto issue_load = [&](int ch) {
    const int n0 = ch * C;
    const int nv = min(C, a.N - n0);
    const uint32_t bq = static_cast<uint32_t>(nv * DX * 2), bv = static_cast<uint32_t>(nv * DV * 2);
    mbar_arrive_expect_tx(bar_tma, FULL ? 2 * bq + bv : bq + bv);
    const long long row = bh * a.N + n0;
    if (FULL) bulk_g2s(smem + K::STG_Q, a.q + row * DX, bq, bar_tma);
    bulk_g2s(smem + K::STG_K, a.k + row * DX, bq, bar_tma);
    bulk_g2s(smem + K::STG_V, a.v + row * DV, bv, bar_tma);
  };

  if (tid == 0 && ch0 < ch1) issue_load(ch0);
  bool tma_pending = ch0 < ch1;
  uint32_t ph_tma = 0, ph_mma = 0;
  bool aborted = false;

  auto mma_sync = [&](void) -> bool {   // wait for the last commit; uniform result
    bool ok = mbar_wait(bar_mma, ph_mma, a.err);
    ph_mma ^= 1u;
    tc_fence_after();
    return !__syncthreads_or(!ok);
  };
  auto to_tensor_core = [&]() {   // make thread smem / TMEM writes visible to the MMA issuer
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
  };

  int nv = C;
  for (int ch = ch0; ch < ch1; ++ch) {
    const int n0 = ch * C;
    nv = min(C, a.N - n0);
    {
      bool ok = mbar_wait(bar_tma, ph_tma, a.err);
      ph_tma ^= 1u;
      if (__syncthreads_or(!ok)) { aborted = true; break; }
      tma_pending = false;
    }
    if (FULL) convert_tile<DX, true>(smem + K::STG_Q, smem + K::S_Q, nv, warp, lane);
    convert_tile<DX, true>(smem + K::STG_K, smem + K::S_K, nv, warp, lane);
    convert_tile<DV, false>(smem + K::STG_V, smem + K::S_V, nv, warp, lane);
    __syncthreads();   // staging consumed
    if (tid == 0 && ch + 1 < ch1) issue_load(ch + 1);
    tma_pending = ch + 1 < ch1;

    // ---- state: R = lambda^C S_hat -> TMEM (for GEMM7) and fp16 operands
    for (int cb = 0; cb < F / 2; cb += 16) {
      const int col0 = half * (F / 2) + cb;
      uint32_t r[16];
      tmem_ld16(trow + K::T_STATE + col0, r);
      tmem_ld_wait16(r);
      uint32_t w[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float x = __uint_as_float(r[e]);
        const float y = __shfl_xor_sync(kFull, x, 1);
        w[e] = __float_as_uint(fmaf(lamC.x, x, sgnLi * y));
      }
      tmem_st16(trow + K::T_STATE + col0, w);
      if (FULL && a.dump_R) {
        float4* d4 = reinterpret_cast<float4*>(a.dump_R + ((bh * nch_total + ch) * KR + k) * F + col0);
#pragma unroll
        for (int g = 0; g < 4; ++g)
          d4[g] = make_float4(__uint_as_float(w[4 * g]), __uint_as_float(w[4 * g + 1]),
                              __uint_as_float(w[4 * g + 2]), __uint_as_float(w[4 * g + 3]));
      }
      if (FULL) {
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          uint4 pk;
          pk.x = pack_half2(__uint_as_float(w[8 * g + 0]), __uint_as_float(w[8 * g + 1]));
          pk.y = pack_half2(__uint_as_float(w[8 * g + 2]), __uint_as_float(w[8 * g + 3]));
          pk.z = pack_half2(__uint_as_float(w[8 * g + 4]), __uint_as_float(w[8 * g + 5]));
          pk.w = pack_half2(__uint_as_float(w[8 * g + 6]), __uint_as_float(w[8 * g + 7]));
          const int f = col0 + 8 * g;
          if (f < DX)
            *reinterpret_cast<uint4*>(smem + K::S_RU + tile_off(k, f, K::RSX)) = pk;
          else
            *reinterpret_cast<uint4*>(smem + K::S_RG + tile_off(k, f - DX, K::RSV)) = pk;
        }
      }
    }
    tmem_st_wait();
    {  // eta: R_eta = lambda^C eta_hat;  eta_hat <- R_eta + sum_{j<nv} E'[j]
      const float y = __shfl_xor_sync(kFull, eta_c, 1);
      const float Re = fmaf(lamC.x, eta_c, sgnLi * y);
      if (FULL && half == 0 && a.dump_Re) a.dump_Re[(bh * nch_total + ch) * KR + k] = Re;
      if (FULL && half == 0)
        *reinterpret_cast<uint4*>(smem + K::S_RE + tile_off(k, 0, 256)) =
            make_uint4(pack_half2(Re, 0.f), 0u, 0u, 0u);
      float add = esum_c;
      if (nv < C) {   // ragged last chunk: partial sum of E' over the valid keys
        double pr, pi, sr = 0.0, si = 0.0;
        const double br = T->b[m].x, bi = T->b[m].y;
        for (int j = 0; j < nv; ++j) {
          double e = exp((C / 2 - j) * T->re_dA[m]);
          double ph = fmod((C / 2 - j) * T->im_dA[m], 6.283185307179586476925);
          double s, c;
          sincos(ph, &s, &c);
          pr = e * c;
          pi = e * s;
          sr += br * pr - bi * pi;
          si += br * pi + bi * pr;
        }
        add = static_cast<float>(comp ? si : sr);
      }
      eta_c = Re + add;
    }
    to_tensor_core();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t sE = sbase + K::S_E, sK = sbase + K::S_K, sV = sbase + K::S_V;
      if (FULL) {
        const uint32_t sQ = sbase + K::S_Q;
        gemm(tmem + K::T_SP, sK, 128, K::RSX, 256, sQ, 128, K::RSX, 256, idesc_f16(64, 64, 0, 0),
             DX / 16, false);   // GEMM1: S^T
      }
      gemm(tmem + K::T_STATE, sE, 128, 1024, 256, sK, K::RSX, 128, 2 * K::RSX,
           idesc_f16(128, DX, 0, 1), C / 16, true);   // GEMM7: U carry
      gemm(tmem + K::T_STATE + DX, sE, 128, 1024, 256, sV, K::RSV, 128, 2 * K::RSV,
           idesc_f16(128, DV, 0, 1), C / 16, true);   // GEMM7: Gamma carry
      mma_commit(bar_mma);
    }
    if (!mma_sync()) { aborted = true; break; }
    if (!FULL) continue;

    // ---- E1: S^T (M=64 rows j) -> masked fp16, MN-major B of GEMM2
    {
      const int j = 16 * quad + lane;
#pragma unroll
      for (int cb = 0; cb < 32; cb += 16) {
        const int i0 = 32 * half + cb;
        uint32_t r[16];
        tmem_ld16(trow + K::T_SP + i0, r);
        tmem_ld_wait16(r);
        if (lane < 16) {
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = i0 + 8 * g + 2 * e;
              const bool keep = j < nv;
              float x0 = (keep && i >= j) ? __uint_as_float(r[8 * g + 2 * e]) : 0.f;
              float x1 = (keep && i + 1 >= j) ? __uint_as_float(r[8 * g + 2 * e + 1]) : 0.f;
              w[e] = pack_half2(x0, x1);
            }
            *reinterpret_cast<uint4*>(smem + K::S_SP + tile_off(j, i0 + 8 * g, 1024)) =
                make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
    to_tensor_core();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t sE = sbase + K::S_E, sSP = sbase + K::S_SP, sQ = sbase + K::S_Q,
                     sRU = sbase + K::S_RU;
      gemm(tmem + K::T_A, sE, 128, 1024, 256, sSP, 1024, 128, 2048, idesc_f16(128, 64, 0, 1),
           C / 16, false);   // GEMM2
      gemm(tmem + K::T_A, sRU, 128, K::RSX, 256, sQ, 128, K::RSX, 256, idesc_f16(128, 64, 0, 0),
           DX / 16, true);   // GEMM3
      mma_commit(bar_mma);
    }
    if (!mma_sync()) { aborted = true; break; }

    // ---- E2: X = |lambda|^(2(i-c)) a~  (rows k, columns i) -> MN-major A of GEMM4/6
    {
      float s = s_start;
#pragma unroll
      for (int cb = 0; cb < 32; cb += 16) {
        const int i0 = 32 * half + cb;
        uint32_t r[16];
        tmem_ld16(trow + K::T_A + i0, r);
        tmem_ld_wait16(r);
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = __uint_as_float(r[8 * g + 2 * e]) * s;
            s *= r2;
            const float x1 = __uint_as_float(r[8 * g + 2 * e + 1]) * s;
            s *= r2;
            w[e] = pack_half2(x0, x1);
          }
          *reinterpret_cast<uint4*>(smem + K::S_X + tile_off(k, i0 + 8 * g, 1024)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    to_tensor_core();
    if (tid == 0) {
      tc_fence_after();
      gemm(tmem + K::T_SP, sbase + K::S_X, 1024, 128, 2048, sbase + K::S_E, 1024, 128, 2048,
           idesc_f16(64, 64, 1, 1), KR / 16, false);   // GEMM4: P
      mma_commit(bar_mma);
    }
    if (!mma_sync()) { aborted = true; break; }

    // ---- E3: P (M=64 rows i) -> masked fp16, K-major A of GEMM5
    {
      const int i = 16 * quad + lane;
#pragma unroll
      for (int cb = 0; cb < 32; cb += 16) {
        const int j0 = 32 * half + cb;
        uint32_t r[16];
        tmem_ld16(trow + K::T_SP + j0, r);
        tmem_ld_wait16(r);
        if (lane < 16) {
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = j0 + 8 * g + 2 * e;
              float x0 = j <= i ? __uint_as_float(r[8 * g + 2 * e]) : 0.f;
              float x1 = j + 1 <= i ? __uint_as_float(r[8 * g + 2 * e + 1]) : 0.f;
              w[e] = pack_half2(x0, x1);
            }
            *reinterpret_cast<uint4*>(smem + K::S_SP + tile_off(i, j0 + 8 * g, 1024)) =
                make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
    to_tensor_core();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t sSP = sbase + K::S_SP, sX = sbase + K::S_X;
      gemm(tmem + K::T_NUM, sSP, 128, 1024, 256, sbase + K::S_V, K::RSV, 128, 2 * K::RSV,
           idesc_f16(64, DV, 0, 1), C / 16, false);   // GEMM5: P V
      gemm(tmem + K::T_DEN, sSP, 128, 1024, 256, sbase + K::S_ONES, 256, 128, 512,
           idesc_f16(64, 16, 0, 1), C / 16, false);   // GEMM5b: P 1
      gemm(tmem + K::T_NUM, sX, 1024, 128, 2048, sbase + K::S_RG, K::RSV, 128, 2 * K::RSV,
           idesc_f16(64, DV, 1, 1), KR / 16, true);   // GEMM6: X R_Gamma
      gemm(tmem + K::T_DEN, sX, 1024, 128, 2048, sbase + K::S_RE, 256, 128, 512,
           idesc_f16(64, 16, 1, 1), KR / 16, true);   // GEMM6b: X R_eta
      mma_commit(bar_mma);
    }
    if (!mma_sync()) { aborted = true; break; }

    // ---- E4: o = num / den (M=64 rows i)
    {
      const int i = 16 * quad + lane;
      uint32_t rd[16];
      tmem_ld16(trow + K::T_DEN, rd);
      tmem_ld_wait16(rd);
      const float dn = __uint_as_float(rd[0]);
      const float rdn = 1.0f / dn;
      const long long row = bh * a.N + n0 + i;
      const bool valid = lane < 16 && i < nv;
      if (valid && a.den && half == 0) a.den[row] = dn;
#pragma unroll
      for (int cb = 0; cb < DV / 2; cb += 16) {
        const int f0 = half * (DV / 2) + cb;
        uint32_t r[16];
        tmem_ld16(trow + K::T_NUM + f0, r);
        tmem_ld_wait16(r);
        if (valid) {
          float4* op = reinterpret_cast<float4*>(a.o + row * DV + f0);
#pragma unroll
          for (int g = 0; g < 4; ++g)
            op[g] = make_float4(__uint_as_float(r[4 * g]) * rdn, __uint_as_float(r[4 * g + 1]) * rdn,
                                __uint_as_float(r[4 * g + 2]) * rdn, __uint_as_float(r[4 * g + 3]) * rdn);
          if (a.num) {
            float4* np = reinterpret_cast<float4*>(a.num + row * DV + f0);
#pragma unroll
            for (int g = 0; g < 4; ++g)
              np[g] = make_float4(__uint_as_float(r[4 * g]), __uint_as_float(r[4 * g + 1]),
                                  __uint_as_float(r[4 * g + 2]), __uint_as_float(r[4 * g + 3]));
          }
        }
      }
    }
    tc_fence_before();
    __syncthreads();
  }

  if (!aborted) {
    if (FULL) {
      if (a.state_out && seg == a.nseg - 1) {
        // state after the last token: sc * lambda^(nv - C) * S_hat = lambda^(nv-c-1) S_hat
        double pr, pi, e = exp((nv - C / 2 - 1) * T->re_dA[m]);
        double ph = fmod((nv - C / 2 - 1) * T->im_dA[m], 6.283185307179586476925), s, c;
        sincos(ph, &s, &c);
        pr = e * c;
        pi = e * s;
        const float fr = static_cast<float>(pr), fi = static_cast<float>(pi);
        for (int cb = 0; cb < F / 2; cb += 16) {
          const int col0 = half * (F / 2) + cb;
          uint32_t r[16];
          tmem_ld16(trow + K::T_STATE + col0, r);
          tmem_ld_wait16(r);
#pragma unroll
          for (int e2 = 0; e2 < 16; ++e2) {
            const float x = __uint_as_float(r[e2]);
            const float y = __shfl_xor_sync(kFull, x, 1);
            if (comp == 0) {   // x = re, y = im
              const float2 z = make_float2(fr * x - fi * y, fr * y + fi * x);
              const int f = col0 + e2;
              if (f < DX) a.state_out[(bh * 64 + m) * DX + f] = z;
              else a.state_out[a.BH * 64 * DX + (bh * 64 + m) * DV + (f - DX)] = z;
            }
          }
        }
        const float y = __shfl_xor_sync(kFull, eta_c, 1);
        if (comp == 0 && half == 0)
          a.state_out[a.BH * 64 * F + bh * 64 + m] =
              make_float2(fr * eta_c - fi * y, fr * y + fi * eta_c);
      }
    } else {
      float* dst = a.seg_state + ((bh * (a.nseg - 1) + seg) * KR + k) * F;
      for (int cb = 0; cb < F / 2; cb += 16) {
        const int col0 = half * (F / 2) + cb;
        uint32_t r[16];
        tmem_ld16(trow + K::T_STATE + col0, r);
        tmem_ld_wait16(r);
        float4* d4 = reinterpret_cast<float4*>(dst + col0);
#pragma unroll
        for (int g = 0; g < 4; ++g)
          d4[g] = make_float4(__uint_as_float(r[4 * g]), __uint_as_float(r[4 * g + 1]),
                              __uint_as_float(r[4 * g + 2]), __uint_as_float(r[4 * g + 3]));
      }
      if (half == 0) a.seg_eta[(bh * (a.nseg - 1) + seg) * KR + k] = eta_c;
    }
  } else if (tma_pending) {
    mbar_wait(bar_tma, ph_tma, a.err);   // bounded: let our own copy land before exiting
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int DX, int DV>
cudaError_t launch_impl(const TcArgs& args, const ia_shape_t& s, const TcPlan& p, cudaStream_t st) {
  using K = Cfg<DX, DV>;
  cudaError_t e;
  if (p.nseg > 1) {
    auto k1 = tc_prefill_kernel<DX, DV, false>;
    e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, K::SMEM);
    if (e != cudaSuccess) return e;
    k1<<<static_cast<unsigned>(args.BH * (p.nseg - 1)), NTHR, K::SMEM, st>>>(args);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    e = launch_segment_scan(s.B, s.H, DX, DV, p.nseg, p.seg_chunks * C, args.tabs, args.state_in,
                            args.seg_state, args.seg_eta, st);
    if (e != cudaSuccess) return e;
  }
  auto k3 = tc_prefill_kernel<DX, DV, true>;
  e = cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, K::SMEM);
  if (e != cudaSuccess) return e;
  mark_launch_begin(st);
  k3<<<static_cast<unsigned>(args.BH * p.nseg), NTHR, K::SMEM, st>>>(args);
  e = cudaGetLastError();
  mark_launch_end(st);
  return e;
}

}  // namespace

bool tc_prefill_supported(const ia_shape_t& s) {
  const bool dx = s.d_xi == 64 || s.d_xi == 128;
  const bool dv = s.d_v == 64 || s.d_v == 128;
  return s.in_dtype == IA_BF16 && s.M == kModesTC && dx && dv;
}

TcPlan tc_plan(const ia_shape_t& s, int num_sms) {
  const long long BH = static_cast<long long>(s.B) * s.H;
  const int nch = (s.N + C - 1) / C;
  // Forced segment count (tuning and tests): IA_PREFILL_SEGMENTS=n.
  if (const char* env = std::getenv("IA_PREFILL_SEGMENTS")) {
    const int n = std::atoi(env);
    if (n >= 1 && n <= nch) {
      const int L = (nch + n - 1) / n;
      return TcPlan{(nch + L - 1) / L, L};
    }
  }
  // Cost in units of one full chunk pass: waves x (chunks per CTA + per-CTA
  // prologue/epilogue), a state-only chunk costing alpha, plus the scan.
  const double alpha = 0.35, cta_overhead = 1.0, scan = 1.0;
  const int min_len = 4;   // shorter segments spend more on state round trips than they save
  TcPlan best{1, nch};
  double best_t = 1e300;
  for (int nseg = 1; nseg <= 32 && nseg <= nch; ++nseg) {
    const int L = (nch + nseg - 1) / nseg;
    if ((nch + L - 1) / L != nseg) continue;
    if (nseg > 1 && L < min_len) continue;
    const double w1 = nseg > 1 ? std::ceil(static_cast<double>(BH * (nseg - 1)) / num_sms) : 0.0;
    const double w3 = std::ceil(static_cast<double>(BH * nseg) / num_sms);
    const double t = w1 * (L * alpha + cta_overhead) + w3 * (L + cta_overhead) + (nseg > 1 ? scan : 0.0);
    if (t < best_t - 1e-9) {
      best_t = t;
      best = TcPlan{nseg, L};
    }
  }
  return best;
}

size_t tc_workspace_bytes(const ia_shape_t& s, const TcPlan& p) {
  const size_t BH = static_cast<size_t>(s.B) * s.H;
  size_t bytes = sizeof(HeadTables) * static_cast<size_t>(s.H);
  if (p.nseg > 1) {
    bytes += BH * (p.nseg - 1) * (static_cast<size_t>(KR) * (s.d_xi + s.d_v) + KR) * sizeof(float);
  }
  return bytes + 256;
}

HeadTables* tc_tables(void* ws) {
  return reinterpret_cast<HeadTables*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~static_cast<uintptr_t>(255));
}

cudaError_t launch_tc_prefill(const ia_shape_t& s, const TcPlan& p, const void* q, const void* k,
                              const void* v, const float* delta, const float* A,
                              const void* state_in, float* o, float* num, float* den,
                              void* state_out, void* ws, cudaStream_t st, float* dump_R,
                              float* dump_Re) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  w = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(w) + 255) & ~static_cast<uintptr_t>(255));
  HeadTables* tabs = reinterpret_cast<HeadTables*>(w);
  float* seg_state = reinterpret_cast<float*>(w + sizeof(HeadTables) * s.H);
  const size_t BH = static_cast<size_t>(s.B) * s.H;
  float* seg_eta = seg_state + BH * (p.nseg > 1 ? p.nseg - 1 : 0) * KR * (s.d_xi + s.d_v);
  cudaError_t e = launch_param_tables(s.H, delta, A, tabs, st);
  if (e != cudaSuccess) return e;
  TcArgs args;
  args.q = static_cast<const __nv_bfloat16*>(q);
  args.k = static_cast<const __nv_bfloat16*>(k);
  args.v = static_cast<const __nv_bfloat16*>(v);
  args.tabs = tabs;
  args.state_in = static_cast<const float2*>(state_in);
  args.seg_state = seg_state;
  args.seg_eta = seg_eta;
  args.o = o;
  args.num = num;
  args.den = den;
  args.state_out = static_cast<float2*>(state_out);
  args.err = device_error_ptr();
  args.dump_R = dump_R;
  args.dump_Re = dump_Re;
  if (!args.err) return cudaErrorInvalidSymbol;
  args.H = s.H;
  args.N = s.N;
  args.nseg = p.nseg;
  args.seg_chunks = p.seg_chunks;
  args.BH = static_cast<long long>(BH);
  if (s.d_xi == 64 && s.d_v == 64) return launch_impl<64, 64>(args, s, p, st);
  if (s.d_xi == 128 && s.d_v == 128) return launch_impl<128, 128>(args, s, p, st);
  if (s.d_xi == 64 && s.d_v == 128) return launch_impl<64, 128>(args, s, p, st);
  if (s.d_xi == 128 && s.d_v == 64) return launch_impl<128, 64>(args, s, p, st);
  return cudaErrorInvalidValue;
}

}  // namespace ia
