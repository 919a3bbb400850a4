// Reverse mode of the chunked IA layer on tcgen05 tensor cores (training
// step: dq, dk, dv, dDelta) for bf16 inputs, M = 64 modes, d_xi = d_v = 64.
//
// The layer is the causal IA layer of 'Interdomain Attention: Beyond
// Token-Level Key-Value Memory' (paperlayer.ai summary sec. 3.1-3.2, chunkwise
// execution per sec. A.2; bf16 training per sec. A.3 and App. G).  The
// backward differentiates the same chunk algorithm the forward runs, in the
// real-row form (rows k = 2m re, 2m+1 im; E'' = E' split into rows; x = [xi(K)|V]):
//
//   forward per chunk:  R = lambda^C S_hat0;  a~ = S E'' + xi(Q) R_U^T;  X = s * a~
//                       P = mask(X E''^T);  num = P V + X R_G;  den = P 1 + X R_eta
//                       S_hat1 = R + E''^T x
//   reverse per chunk (from dO and the adjoint dS1 of S_hat1, chunks last to first):
//     dnum = dO/den, dden = -(dO.o)/den           dP = mask(dnum V^T + dden 1^T)
//     dX^T = E''^T dP^T + R_G dnum^T + R_eta dden   da~ = s * dX
//     dS = mask(da~ E''^T)
//     dxi(Q) = dS xi(K) + da~ R_U      dxi(K) = dS^T xi(Q) + E'' dS1_U
//     dV = P^T dnum + E'' dS1_G        dR = dS1 + [da~^T xi(Q) | X^T dnum | X^T dden]
//     dS_hat0 = conj(lambda^C) dR
//   Delta and A enter only through the per-head tables, so their adjoints are
//   gathered over all chunks and contracted once with the tables' derivatives:
//     dE''^T += da~^T S + X^T dP + dS1 x^T    (accumulated in TMEM)
//     ds     += dX * a~,  dlambda^C += sum dR conj(S_hat0)
//     d(b lambda^n)/dDelta = (lambda + n A b) lambda^n,  ds/dDelta = 2 Re(A)(i-c) s,
//     d(lambda^C)/dDelta = C A lambda^C;  along A_m the same with
//     d(b lambda^n)/dA = ((Delta lambda - b)/A + n Delta b) lambda^n,
//     ds/dRe A = 2 Delta (i-c) s,  d(lambda^C)/dA = C Delta lambda^C.
//   Each CTA writes its (b,h)'s per-mode sums of dL/dDelta, dL/dRe A and
//   dL/dIm A; a fixed-order reduction turns them into dDelta and dA.
// A dedicated MMA warp issues the contraction groups (tcgen05.mma blocks its
// issuing thread) on ready barriers from the 8 epilogue warps, in the order
// F1+B1, F2, B2, F4, B3-B5, dQ/dK/dV, so the readout chain (S, a~, P) and the
// adjoint chain (dP, dX) overlap: each epilogue runs while the other chain's
// contraction executes; dP and dS use their own TMEM tile (T_X2).
// The forward pass (the prefill kernel) stores R (fp16 tiles R_U, R_Gamma in
// the 128-byte swizzled operand layout, loaded here with one bulk copy per
// chunk, one chunk ahead), R_eta (fp32) and den for every chunk.
//
// TMEM columns: [0,128) adjoint of the state (dS1, then dR, then dS_hat0);
// [128,192) dE''^T; [192,256) a~^T then dK; [256,320) dX^T then dV;
// [320,384) S^T, then P (M=64 layout); [384,448) dQ; [448,512) dP, then dS.
#include <cmath>

#include "ia_device.cuh"
#include "ia_internal.h"
#include "ia_tables.cuh"
#include "ia_tc_common.cuh"

namespace ia {
namespace {

using namespace tc;

struct B {
  static constexpr int DX = 64, DV = 64, F = 128;
  static constexpr uint32_t T_ADJ = 0, T_EBAR = 128, T_A = 192, T_DK = 192, T_DX = 256,
                            T_DV = 256, T_SP = 320, T_DQ = 384, T_X2 = 448;
  static constexpr uint32_t TILE64 = C * 64 * 2;     // 8 KB: [64 rows][64 cols] fp16
  static constexpr uint32_t TILE128 = KR * 64 * 2;   // 16 KB: [128 rows][64 cols] fp16
  static constexpr uint32_t STG_Q = 0;
  static constexpr uint32_t STG_K = STG_Q + TILE64;
  static constexpr uint32_t STG_V = STG_K + TILE64;
  static constexpr uint32_t STG_G = STG_V + TILE64;
  static constexpr uint32_t S_Q = STG_G + TILE64;
  static constexpr uint32_t S_K = S_Q + TILE64;
  static constexpr uint32_t S_V = S_K + TILE64;
  static constexpr uint32_t S_E = S_V + TILE64;
  static constexpr uint32_t S_S = S_E + TILE128;
  static constexpr uint32_t S_X = S_S + TILE64;
  static constexpr uint32_t S_P = S_X + TILE128;
  static constexpr uint32_t S_DP = S_P + TILE64;
  static constexpr uint32_t S_DA = S_DP + TILE64;
  static constexpr uint32_t S_DS = S_DA + TILE128;
  static constexpr uint32_t S_DN = S_DS + TILE64;
  static constexpr uint32_t S_RU = S_DN + TILE64;
  static constexpr uint32_t S_RG = S_RU + TILE128;
  static constexpr uint32_t S_DS1 = S_RG + TILE128;          // [128][F] fp16
  static constexpr uint32_t S_DD = S_DS1 + KR * F * 2;       // dden [64] fp32
  static constexpr uint32_t S_RED = S_DD + C * 4;            // dR_eta halves [2][128] fp32
  static constexpr uint32_t S_BAR = S_RED + 2 * KR * 4;    // 17 mbarriers (see the kernel)
  static constexpr uint32_t S_FLAG = S_BAR + 17 * 8;       // abort flag
  static constexpr uint32_t S_TMEMH = S_FLAG + 8;
  static constexpr uint32_t S_OST = S_TMEMH + 16;            // o rows of the chunk, fp32 [64][64]
  static constexpr uint32_t RT = KR * 64 * 2;                // one fp16 R tile: 16 KB
  // dq, dk, dv leave by TMA stores from tiles that are free between the
  // gradient contractions and the next chunk's readout (E2, E3, dP, dX):
  // each as two 64-row x 128-byte boxes in the 128-byte swizzled layout
  static constexpr uint32_t O_DQ = S_X, O_DK = S_P, O_DV = S_DA, OBOX = C * 128;
  static_assert(S_DP == S_P + OBOX && O_DQ % 1024 == 0 && O_DK % 1024 == 0 && O_DV % 1024 == 0,
                "output staging: three 16 KB areas on the swizzle period");
  static_assert(S_RG == S_RU + RT && S_RU % 1024 == 0, "R tiles adjacent, on the swizzle period");
  static constexpr uint32_t SMEM = S_OST + C * 64 * 4;
  static_assert(SMEM <= 232448, "fits one CTA's opt-in shared memory");
};

struct BwdArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* dO;
  const float* o;
  const float* den;
  const float* A;
  const float* delta;
  int dpm;
  const HeadTables* tabs;
  const uint8_t* R;  // [BH][nch] x (R_U, R_Gamma) fp16 swizzled tiles of 16 KB
  const float* Re;   // [BH][nch][128]
  const float* dtab; // [3][H][128][64] d(E'')/dDelta, dRe A, dIm A rows, then [3][H][128] row sums
  float* dq;
  float* dk;
  float* dv;
  float* gpart;      // [BH][M][3]: this (b,h)'s dL/dDelta_hm, dL/dRe A_m, dL/dIm A_m
  int* err;
  int H, N;
  long long BH;
};

__device__ __forceinline__ uint4 pack8(const float* x) {
  return make_uint4(pack_half2(x[0], x[1]), pack_half2(x[2], x[3]), pack_half2(x[4], x[5]),
                    pack_half2(x[6], x[7]));
}

constexpr int NEPI = NTHR;        // epilogue threads (warps 0-7)
constexpr int NBWD = NEPI + 32;   // + one MMA warp

__global__ void __launch_bounds__(NBWD, 1)
    tc_bwd_kernel(const __grid_constant__ BwdArgs a, const __grid_constant__ CUtensorMap tm_dq,
                  const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv) {
  constexpr int DX = B::DX, DV = B::DV, F = B::F;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;
  // The M = 64 accumulators fill lanes 0-15 of each quadrant: thread t of an
  // epilogue warp takes row 16 * quad + t % 16 and 16 of the warp's 32 columns.
  const int r16 = 16 * quad + (lane & 15), c16 = 32 * half + 16 * (lane >> 4);
  const long long bh = blockIdx.x;
  const int h = static_cast<int>(bh % a.H);
  const HeadTables* T = a.tabs + h;
  const int nch = (a.N + C - 1) / C;
  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(smem + B::S_BAR);   // q, k, v, dO, o of a chunk
  uint64_t* bar_drain = bar_tma + 1;
  uint64_t* bar_r = bar_tma + 2;   // the R tiles of the next chunk to process
  uint64_t* rdy = bar_tma + 3;     // [6] epilogue -> MMA warp: operands of group i are in place
  uint64_t* dn = bar_tma + 9;      // [7] MMA warp -> epilogue: F1, B1, F2, B2, F4, B3-B5, G done
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + B::S_FLAG);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + B::S_TMEMH);
  float* sDD = reinterpret_cast<float*>(smem + B::S_DD);
  float* sRED = reinterpret_cast<float*>(smem + B::S_RED);
  const uint32_t sb = smem_u32(smem);

  if (warp == 0) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar_tma, 1);
    mbar_init(bar_drain, 1);
    mbar_init(bar_r, 1);
    for (int i = 0; i < 6; ++i) mbar_init(rdy + i, NEPI);
    for (int i = 0; i < 7; ++i) mbar_init(dn + i, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  {
    const uint4* src = reinterpret_cast<const uint4*>(T->E);
    uint4* dst = reinterpret_cast<uint4*>(smem + B::S_E);
    for (int i = tid; i < static_cast<int>(B::TILE128 / 16); i += NBWD) dst[i] = src[i];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int k = 32 * quad + lane;   // state row: mode m, component comp
  const int m = k >> 1, comp = k & 1;
  const uint32_t trow = tmem + (static_cast<uint32_t>(32 * quad) << 16);
  const float2 lamC = T->lamC[m];
  const float ReA = a.A ? a.A[2 * m] : -0.5f;
  const float ImA = a.A ? a.A[2 * m + 1] : static_cast<float>(3.14159265358979323846 * m);
  const float Dm = delta_hm(a.delta, a.dpm, kModesTC, h, m);
  const float r2 = T->r2[m];
  const float s_start = static_cast<float>(exp(2.0 * T->re_dA[m] * (32.0 * half - C / 2)));
  const float sgn = comp ? 1.f : -1.f;
  // this row of the three derivative tables over j (from the table prologue)
  // and their sums: along Delta, Re A and Im A
  const size_t tstride = static_cast<size_t>(a.H) * KR * C;
  const float* dErow = a.dtab + (static_cast<size_t>(h) * KR + k) * C;
  auto dEsum = [&](int w) { return a.dtab[3 * tstride + (static_cast<size_t>(w) * a.H + h) * KR + k]; };

  // zero the state adjoint and the table adjoint
  if (warp < NEPI / 32) {
    uint32_t z[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) z[e] = 0u;
    for (int cb = 0; cb < F / 2; cb += 16) tmem_st16(trow + B::T_ADJ + half * (F / 2) + cb, z);
    for (int cb = 0; cb < 32; cb += 16) tmem_st16(trow + B::T_EBAR + half * 32 + cb, z);
    tmem_st_wait();
  }
  float de_c = 0.f;     // adjoint of the eta channel of the chunk-end state (this row)
  // this thread's shares of dL/dDelta_hm, dL/dRe A_m, dL/dIm A_m, gathered as
  //   gs  = sum dX a~ 2 (i-c) s                     (readout scale: Delta Re A in s)
  //   zr, zn = sum over dR . R components            (Re z and -Im z of z = sum conj(dR) R,
  //                                                    R = lambda^C S_hat0: C A and C Delta)
  //   tD, tR, tI = the derivative-table contractions (E' and its chunk sum)
  float gs = 0.f, zr = 0.f, zn = 0.f, tD = 0.f, tR = 0.f, tI = 0.f;

  auto issue_load = [&](int ch) {
    const int n0 = ch * C;
    const int nv = min(C, a.N - n0);
    const uint32_t bq = static_cast<uint32_t>(nv * DX * 2), bv = static_cast<uint32_t>(nv * DV * 2);
    const uint32_t bo = static_cast<uint32_t>(nv * DV * 4);
    mbar_arrive_expect_tx(bar_tma, 2 * bq + 2 * bv + bo);
    const long long row = bh * a.N + n0;
    bulk_g2s(smem + B::STG_Q, a.q + row * DX, bq, bar_tma);
    bulk_g2s(smem + B::STG_K, a.k + row * DX, bq, bar_tma);
    bulk_g2s(smem + B::STG_V, a.v + row * DV, bv, bar_tma);
    bulk_g2s(smem + B::STG_G, a.dO + row * DV, bv, bar_tma);
    bulk_g2s(smem + B::S_OST, a.o + row * DV, bo, bar_tma);   // row * 256 bytes: 16-byte aligned
  };
  auto issue_r = [&](int ch) {   // both R tiles of chunk ch: 32 KB contiguous
    mbar_arrive_expect_tx(bar_r, 2 * B::RT);
    bulk_g2s(smem + B::S_RU, a.R + (bh * nch + ch) * 2 * B::RT, 2 * B::RT, bar_r);
  };
  if (tid == 0) {
    issue_load(nch - 1);
    issue_r(nch - 1);
  }
  // den of row tid/4 of the next chunk to process, loaded a chunk ahead
  auto load_den = [&](int ch) -> float {
    const int i = tid >> 2;
    return tid < NEPI && i < a.N - ch * C ? a.den[bh * a.N + ch * C + i] : 1.f;
  };
  float den_next = load_den(nch - 1);
  bool tma_pending = true, r_pending = true;
  uint32_t ph_tma = 0, ph_r = 0;
  bool aborted = false;
  if (warp == NEPI / 32) {
    // ------------------------------------------------ MMA warp: the contraction groups, in order
    if (lane == 0) {
      uint32_t pr[6] = {0u, 0u, 0u, 0u, 0u, 0u};
      bool ok = true;
      auto wait_rdy = [&](int i) -> bool {
        const bool r = mbar_wait_or_abort(rdy + i, pr[i], a.err, abort_flag);
        pr[i] ^= 1u;
        tc_fence_after();
        return r;
      };
      for (int ch = nch - 1; ch >= 0; --ch) {
        if (!(ok = wait_rdy(0))) break;   // operands, R, dS1 of the chunk
        // F1: S^T = xi(K) xi(Q)^T
        gemm(tmem + B::T_SP, sb + B::S_K, kmaj_lbo(), kmaj_sbo(DX), kmaj_step(), sb + B::S_Q,
             kmaj_lbo(), kmaj_sbo(DX), kmaj_step(), idesc_f16(64, 64, 0, 0), DX / 16, false);
        mma_commit(dn + 0);
        // B1: dP = dnum V^T
        gemm(tmem + B::T_X2, sb + B::S_DN, kmaj_lbo(), kmaj_sbo(DV), kmaj_step(), sb + B::S_V,
             kmaj_lbo(), kmaj_sbo(DV), kmaj_step(), idesc_f16(64, 64, 0, 0), DV / 16, false);
        mma_commit(dn + 1);
        if (!(ok = wait_rdy(1))) break;   // E1 done
        // F2: a~^T = E''^T S^T + R_U xi(Q)^T
        gemm(tmem + B::T_A, sb + B::S_E, kmaj_lbo(), kmaj_sbo(64), kmaj_step(), sb + B::S_S,
             mn_lbo(64), mn_sbo(), mn_step(64), idesc_f16(128, 64, 0, 1), C / 16, false);
        gemm_dd(tmem + B::T_A, smem_desc_sw128(sb + B::S_RU, 16, 1024), 32,
                smem_desc(sb + B::S_Q, kmaj_lbo(), kmaj_sbo(DX)), kmaj_step(), idesc_f16(128, 64, 0, 0),
                DX / 16, true);
        mma_commit(dn + 2);
        if (!(ok = wait_rdy(2))) break;   // dP done
        // B2: dX^T = E''^T dP^T + R_G dnum^T
        gemm(tmem + B::T_DX, sb + B::S_E, kmaj_lbo(), kmaj_sbo(64), kmaj_step(), sb + B::S_DP,
             kmaj_lbo(), kmaj_sbo(64), kmaj_step(), idesc_f16(128, 64, 0, 0), C / 16, false);
        gemm_dd(tmem + B::T_DX, smem_desc_sw128(sb + B::S_RG, 16, 1024), 32,
                smem_desc(sb + B::S_DN, kmaj_lbo(), kmaj_sbo(DV)), kmaj_step(), idesc_f16(128, 64, 0, 0),
                DV / 16, true);
        mma_commit(dn + 3);
        if (!(ok = wait_rdy(3))) break;   // E2 done
        // F4: P = X E''^T
        gemm(tmem + B::T_SP, sb + B::S_X, mn_lbo(64), mn_sbo(), mn_step(64), sb + B::S_E, mn_lbo(64),
             mn_sbo(), mn_step(64), idesc_f16(64, 64, 1, 1), KR / 16, false);
        mma_commit(dn + 4);
        if (!(ok = wait_rdy(4))) break;   // dX done
        {
        const uint32_t sDA = sb + B::S_DA, sX = sb + B::S_X, sE = sb + B::S_E;
        // B3: dS = da~ E''^T
        gemm(tmem + B::T_X2, sDA, mn_lbo(64), mn_sbo(), mn_step(64), sE, mn_lbo(64), mn_sbo(),
             mn_step(64), idesc_f16(64, 64, 1, 1), KR / 16, false);
        // B4, B5: dR += [da~^T xi(Q) | X^T dnum]
        gemm(tmem + B::T_ADJ, sDA, kmaj_lbo(), kmaj_sbo(64), kmaj_step(), sb + B::S_Q, mn_lbo(DX),
             mn_sbo(), mn_step(DX), idesc_f16(128, DX, 0, 1), C / 16, true);
        gemm(tmem + B::T_ADJ + DX, sX, kmaj_lbo(), kmaj_sbo(64), kmaj_step(), sb + B::S_DN,
             mn_lbo(DV), mn_sbo(), mn_step(DV), idesc_f16(128, DV, 0, 1), C / 16, true);
        // table adjoint: dE''^T += da~^T S + X^T dP + dS1 x^T
        gemm(tmem + B::T_EBAR, sDA, kmaj_lbo(), kmaj_sbo(64), kmaj_step(), sb + B::S_S, kmaj_lbo(),
             kmaj_sbo(64), kmaj_step(), idesc_f16(128, 64, 0, 0), C / 16, true);
        gemm(tmem + B::T_EBAR, sX, kmaj_lbo(), kmaj_sbo(64), kmaj_step(), sb + B::S_DP, mn_lbo(64),
             mn_sbo(), mn_step(64), idesc_f16(128, 64, 0, 1), C / 16, true);
        gemm(tmem + B::T_EBAR, sb + B::S_DS1, kmaj_lbo(), kmaj_sbo(F), kmaj_step(), sb + B::S_K,
             kmaj_lbo(), kmaj_sbo(DX), kmaj_step(), idesc_f16(128, 64, 0, 0), DX / 16, true);
        gemm(tmem + B::T_EBAR, sb + B::S_DS1 + (DX / 8) * 128, kmaj_lbo(), kmaj_sbo(F), kmaj_step(),
             sb + B::S_V, kmaj_lbo(), kmaj_sbo(DV), kmaj_step(), idesc_f16(128, 64, 0, 0), DV / 16,
             true);
        }
        mma_commit(dn + 5);
        if (!(ok = wait_rdy(5))) break;   // E3, carry and dS done
        {
        const uint32_t sDS = sb + B::S_DS, sDA = sb + B::S_DA, sE = sb + B::S_E, sDS1 = sb + B::S_DS1;
        // dQ = dS xi(K) + da~ R_U
        gemm(tmem + B::T_DQ, sDS, kmaj_lbo(), kmaj_sbo(64), kmaj_step(), sb + B::S_K, mn_lbo(DX),
             mn_sbo(), mn_step(DX), idesc_f16(64, DX, 0, 1), C / 16, false);
        gemm_dd(tmem + B::T_DQ, smem_desc(sDA, mn_lbo(64), mn_sbo()), mn_step(64),
                smem_desc_sw128(sb + B::S_RU, 16, 1024), 2048, idesc_f16(64, DX, 1, 1), KR / 16, true);
        // dK = dS^T xi(Q) + E'' dS1_U
        gemm(tmem + B::T_DK, sDS, mn_lbo(64), mn_sbo(), mn_step(64), sb + B::S_Q, mn_lbo(DX),
             mn_sbo(), mn_step(DX), idesc_f16(64, DX, 1, 1), C / 16, false);
        gemm(tmem + B::T_DK, sE, mn_lbo(64), mn_sbo(), mn_step(64), sDS1, mn_lbo(F), mn_sbo(),
             mn_step(F), idesc_f16(64, DX, 1, 1), KR / 16, true);
        // dV = P^T dnum + E'' dS1_G
        gemm(tmem + B::T_DV, sb + B::S_P, mn_lbo(64), mn_sbo(), mn_step(64), sb + B::S_DN, mn_lbo(DV),
             mn_sbo(), mn_step(DV), idesc_f16(64, DV, 1, 1), C / 16, false);
        gemm(tmem + B::T_DV, sE, mn_lbo(64), mn_sbo(), mn_step(64), sDS1 + (DX / 8) * 128, mn_lbo(F),
             mn_sbo(), mn_step(F), idesc_f16(64, DV, 1, 1), KR / 16, true);
        }
        mma_commit(dn + 6);
      }
      if (!ok) {   // drain every group issued so far
        mma_commit(bar_drain);
        mbar_wait(bar_drain, 0u, a.err);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue warps
    uint32_t pd[7] = {0u, 0u, 0u, 0u, 0u, 0u, 0u};
    auto wait_dn = [&](int i) -> bool {   // outcome uniform over the epilogue warps
      const bool r = mbar_wait_or_abort(dn + i, pd[i], a.err, abort_flag);
      pd[i] ^= 1u;
      tc_fence_after();
      return !named_sync_or(1, NEPI, !r);
    };
    auto signal = [&](int i) {   // this thread's shared / TMEM writes are done
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(rdy + i);
    };
  for (int ch = nch - 1; ch >= 0; --ch) {
    const int n0 = ch * C;
    const int nv = min(C, a.N - n0);
    {
      bool ok = mbar_wait_or_abort(bar_tma, ph_tma, a.err, abort_flag);
      ph_tma ^= 1u;
      if (named_sync_or(1, NEPI, !ok)) { aborted = true; break; }
      tma_pending = false;
    }
    // ---- P0: operands of this chunk
    convert_tile<DX, true>(smem + B::STG_Q, smem + B::S_Q, nv, warp, lane);
    convert_tile<DX, true>(smem + B::STG_K, smem + B::S_K, nv, warp, lane);
    convert_tile<DV, false>(smem + B::STG_V, smem + B::S_V, nv, warp, lane);
    {  // dnum = dO / den (fp16 tile [i][f]), dden = -(dO . o) / den
      const int i = tid >> 2, part = tid & 3;
      float g[16];
      float dot = 0.f, rden = 0.f;
      if (i < nv) {
        rden = 1.0f / den_next;
        const __nv_bfloat162* gs =
            reinterpret_cast<const __nv_bfloat162*>(smem + B::STG_G + i * DV * 2 + part * 32);
        const float4* op = reinterpret_cast<const float4*>(smem + B::S_OST + i * DV * 4 + part * 64);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float2 x = __bfloat1622float2(gs[e]);
          g[2 * e] = x.x;
          g[2 * e + 1] = x.y;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float4 ov = op[e];
          dot = fmaf(g[4 * e], ov.x, fmaf(g[4 * e + 1], ov.y, fmaf(g[4 * e + 2], ov.z, fmaf(g[4 * e + 3], ov.w, dot))));
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) g[e] *= rden;
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) g[e] = 0.f;
      }
      dot += __shfl_xor_sync(kFull, dot, 1);
      dot += __shfl_xor_sync(kFull, dot, 2);
      *reinterpret_cast<uint4*>(smem + B::S_DN + tile_off(i, part * 16, DV * 16)) = pack8(g);
      *reinterpret_cast<uint4*>(smem + B::S_DN + tile_off(i, part * 16 + 8, DV * 16)) = pack8(g + 8);
      if (part == 0) sDD[i] = i < nv ? -dot * rden : 0.f;
    }
    if (ch > 0) den_next = load_den(ch - 1);
    named_sync(1, NEPI);   // staging consumed
    if (tid == 0 && ch > 0) issue_load(ch - 1);
    tma_pending = ch > 0;
    const float Reta = a.Re[(bh * nch + ch) * KR + k];
    {  // the R tiles of this chunk have landed; dS1 -> fp16
      bool ok = mbar_wait_or_abort(bar_r, ph_r, a.err, abort_flag);
      ph_r ^= 1u;
      if (named_sync_or(1, NEPI, !ok)) { aborted = true; break; }
      r_pending = false;
      for (int cb = 0; cb < 64; cb += 16) {
        const int col0 = half * 64 + cb;
        uint32_t r[16];
        tmem_ld16(trow + B::T_ADJ + col0, r);
        tmem_ld_wait16(r);
        float xs[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) xs[e] = __uint_as_float(r[e]);
        *reinterpret_cast<uint4*>(smem + B::S_DS1 + tile_off(k, col0, F * 16)) = pack8(xs);
        *reinterpret_cast<uint4*>(smem + B::S_DS1 + tile_off(k, col0 + 8, F * 16)) = pack8(xs + 8);
      }
    }
    signal(0);
    if (!wait_dn(0)) { aborted = true; break; }   // F1
    {  // E1: masked S^T -> [j][i]
      const int j = r16, i0 = c16;
      uint32_t r[16];
      tmem_ld16_halves<16>(trow + B::T_SP + 32 * half, r);
      tmem_ld_wait16(r);
      float xs[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        xs[e] = (j < nv && i0 + e >= j) ? __uint_as_float(r[e]) : 0.f;
      *reinterpret_cast<uint4*>(smem + B::S_S + tile_off(j, i0, 1024)) = pack8(xs);
      *reinterpret_cast<uint4*>(smem + B::S_S + tile_off(j, i0 + 8, 1024)) = pack8(xs + 8);
    }
    signal(1);
    if (tid == 0) bulk_wait_read_0();   // last chunk's dq/dk/dv staging (sX, sP, sDP, sDA) has been read
    if (!wait_dn(1)) { aborted = true; break; }   // B1
    {  // E_dP: + dden_i, mask j <= i -> [i][j]
      const int i = r16, j0 = c16;
      const float ddi = sDD[i];
      uint32_t r[16];
      tmem_ld16_halves<16>(trow + B::T_X2 + 32 * half, r);
      tmem_ld_wait16(r);
      float xs[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) xs[e] = (j0 + e <= i) ? __uint_as_float(r[e]) + ddi : 0.f;
      *reinterpret_cast<uint4*>(smem + B::S_DP + tile_off(i, j0, 1024)) = pack8(xs);
      *reinterpret_cast<uint4*>(smem + B::S_DP + tile_off(i, j0 + 8, 1024)) = pack8(xs + 8);
    }
    signal(2);
    if (!wait_dn(2)) { aborted = true; break; }   // F2
    {  // E2: X = s a~  (rows k), dR_eta partial = sum_i X dden_i
      float s = s_start, acc = 0.f;
#pragma unroll
      for (int cb = 0; cb < 32; cb += 16) {
        const int i0 = 32 * half + cb;
        uint32_t r[16];
        tmem_ld16(trow + B::T_A + i0, r);
        tmem_ld_wait16(r);
        float xs[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          xs[e] = __uint_as_float(r[e]) * s;
          acc = fmaf(xs[e], sDD[i0 + e], acc);
          s *= r2;
        }
        *reinterpret_cast<uint4*>(smem + B::S_X + tile_off(k, i0, 1024)) = pack8(xs);
        *reinterpret_cast<uint4*>(smem + B::S_X + tile_off(k, i0 + 8, 1024)) = pack8(xs + 8);
      }
      sRED[half * KR + k] = acc;
    }
    signal(3);
    if (!wait_dn(3)) { aborted = true; break; }   // B2
    {  // E_dX: dX += R_eta dden; da~ = s dX; dDelta += dX a~ ds/dDelta
      float s = s_start;
#pragma unroll
      for (int cb = 0; cb < 32; cb += 16) {
        const int i0 = 32 * half + cb;
        uint32_t rx[16], ra[16];
        tmem_ld16(trow + B::T_DX + i0, rx);
        tmem_ld_wait16(rx);
        tmem_ld16(trow + B::T_A + i0, ra);
        tmem_ld_wait16(ra);
        float xs[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int i = i0 + e;
          const float dx = fmaf(Reta, sDD[i], __uint_as_float(rx[e]));
          xs[e] = dx * s;
          gs = fmaf(dx * __uint_as_float(ra[e]), 2.f * static_cast<float>(i - C / 2) * s, gs);
          s *= r2;
        }
        *reinterpret_cast<uint4*>(smem + B::S_DA + tile_off(k, i0, 1024)) = pack8(xs);
        *reinterpret_cast<uint4*>(smem + B::S_DA + tile_off(k, i0 + 8, 1024)) = pack8(xs + 8);
      }
    }
    signal(4);
    if (!wait_dn(4)) { aborted = true; break; }   // F4
    {  // E3: masked P -> [i][j]
      const int i = r16, j0 = c16;
      uint32_t r[16];
      tmem_ld16_halves<16>(trow + B::T_SP + 32 * half, r);
      tmem_ld_wait16(r);
      float xs[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) xs[e] = (j0 + e <= i) ? __uint_as_float(r[e]) : 0.f;
      *reinterpret_cast<uint4*>(smem + B::S_P + tile_off(i, j0, 1024)) = pack8(xs);
      *reinterpret_cast<uint4*>(smem + B::S_P + tile_off(i, j0 + 8, 1024)) = pack8(xs + 8);
    }
    if (!wait_dn(5)) { aborted = true; break; }   // B3-B5, table adjoint
    // dR of this chunk is complete: Delta terms, then the carry to the previous chunk
    {  // adjoint carry: dS_hat0 = conj(lambda^C) dR;  dDelta += C Re(conj(sum dR conj(R)) A)
      for (int cb = 0; cb < 64; cb += 16) {
        const int col0 = half * 64 + cb;
        uint32_t r[16];
        tmem_ld16(trow + B::T_ADJ + col0, r);
        tmem_ld_wait16(r);
        // R of this row, columns col0..col0+15, from the fp16 swizzled tile
        const uint8_t* rrow = smem + B::S_RU + half * B::RT + k * 128;
        float rv[16];
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const uint4 x = *reinterpret_cast<const uint4*>(rrow + ((((cb >> 3) + g) ^ (k & 7)) << 4));
          const __half2* h2 = reinterpret_cast<const __half2*>(&x);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(h2[e]);
            rv[8 * g + 2 * e] = f.x;
            rv[8 * g + 2 * e + 1] = f.y;
          }
        }
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float x = __uint_as_float(r[e]);
          const float y = __shfl_xor_sync(kFull, x, 1);
          const float rpart = __shfl_xor_sync(kFull, rv[e], 1);
          zr = fmaf(x, rv[e], zr);
          zn = fmaf(sgn * x, rpart, zn);
          w[e] = __float_as_uint(fmaf(lamC.x, x, -sgn * lamC.y * y));
        }
        tmem_st16(trow + B::T_ADJ + col0, w);
      }
      tmem_st_wait();
      // eta channel (each row once: half 0 counts the Delta terms)
      const float dRe = de_c + sRED[k] + sRED[KR + k];
      const float y = __shfl_xor_sync(kFull, dRe, 1);
      const float Rp = __shfl_xor_sync(kFull, Reta, 1);
      float dEpart[3] = {dEsum(0), dEsum(1), dEsum(2)};
      if (nv < C) {   // ragged chunk: only the valid keys carry the constant channel
        for (int w = 0; w < 3; ++w) {
          float acc = 0.f;
          for (int j = 0; j < nv; ++j) acc += dErow[w * tstride + j];
          dEpart[w] = acc;
        }
      }
      if (half == 0) {
        zr = fmaf(dRe, Reta, zr);
        zn = fmaf(sgn * dRe, Rp, zn);
        tD = fmaf(de_c, dEpart[0], tD);
        tR = fmaf(de_c, dEpart[1], tR);
        tI = fmaf(de_c, dEpart[2], tI);
      }
      de_c = fmaf(lamC.x, dRe, -sgn * lamC.y * y);
    }
    tc_fence_before();
    named_sync(1, NEPI);
    {  // E_dS: mask (j <= i, j < nv) -> [i][j]
      const int i = r16, j0 = c16;
      uint32_t r[16];
      tmem_ld16_halves<16>(trow + B::T_X2 + 32 * half, r);
      tmem_ld_wait16(r);
      float xs[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        xs[e] = (j0 + e <= i && j0 + e < nv) ? __uint_as_float(r[e]) : 0.f;
      *reinterpret_cast<uint4*>(smem + B::S_DS + tile_off(i, j0, 1024)) = pack8(xs);
      *reinterpret_cast<uint4*>(smem + B::S_DS + tile_off(i, j0 + 8, 1024)) = pack8(xs + 8);
    }
    signal(5);
    if (!wait_dn(6)) { aborted = true; break; }   // dQ, dK, dV
    if (tid == 0 && ch > 0) issue_r(ch - 1);   // R tiles are free: every contraction reading them is done
    r_pending = ch > 0;
    {  // outputs: dq = dxi(Q) xi'(q), dk likewise, dv; xi'(x) = min(xi(x), 1).  Staged as
       // swizzled boxes (rows past the sequence are clipped by the tensor maps)
      const int i = r16, f0 = c16, cg = 4 * (lane >> 4);
      uint32_t rq[16], rk[16], rv[16];
      tmem_ld16_halves<16>(trow + B::T_DQ + 32 * half, rq);
      tmem_ld16_halves<16>(trow + B::T_DK + 32 * half, rk);
      tmem_ld16_halves<16>(trow + B::T_DV + 32 * half, rv);
      tmem_ld_wait16(rq);
      tmem_ld_wait16(rk);
      tmem_ld_wait16(rv);
      // xi(q), xi(k) of this row, columns f0..f0+15, from the fp16 operand tiles
      float fq[16], fk[16];
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const uint4 xq = *reinterpret_cast<const uint4*>(smem + B::S_Q + tile_off(i, f0 + 8 * g, DX * 16));
        const uint4 xk = *reinterpret_cast<const uint4*>(smem + B::S_K + tile_off(i, f0 + 8 * g, DX * 16));
        const __half2* hq = reinterpret_cast<const __half2*>(&xq);
        const __half2* hk = reinterpret_cast<const __half2*>(&xk);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 a2 = __half22float2(hq[e]), b2 = __half22float2(hk[e]);
          fq[8 * g + 2 * e] = a2.x; fq[8 * g + 2 * e + 1] = a2.y;
          fk[8 * g + 2 * e] = b2.x; fk[8 * g + 2 * e + 1] = b2.y;
        }
      }
      const uint32_t rowoff = half * B::OBOX + i * 128;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const uint32_t pos = rowoff + (((cg + g) ^ (i & 7)) << 4);
        float4 oq, ok;
        oq.x = __uint_as_float(rq[4 * g]) * fminf(fq[4 * g], 1.f);
        oq.y = __uint_as_float(rq[4 * g + 1]) * fminf(fq[4 * g + 1], 1.f);
        oq.z = __uint_as_float(rq[4 * g + 2]) * fminf(fq[4 * g + 2], 1.f);
        oq.w = __uint_as_float(rq[4 * g + 3]) * fminf(fq[4 * g + 3], 1.f);
        ok.x = __uint_as_float(rk[4 * g]) * fminf(fk[4 * g], 1.f);
        ok.y = __uint_as_float(rk[4 * g + 1]) * fminf(fk[4 * g + 1], 1.f);
        ok.z = __uint_as_float(rk[4 * g + 2]) * fminf(fk[4 * g + 2], 1.f);
        ok.w = __uint_as_float(rk[4 * g + 3]) * fminf(fk[4 * g + 3], 1.f);
        *reinterpret_cast<float4*>(smem + B::O_DQ + pos) = oq;
        *reinterpret_cast<float4*>(smem + B::O_DK + pos) = ok;
        *reinterpret_cast<float4*>(smem + B::O_DV + pos) =
            make_float4(__uint_as_float(rv[4 * g]), __uint_as_float(rv[4 * g + 1]),
                        __uint_as_float(rv[4 * g + 2]), __uint_as_float(rv[4 * g + 3]));
      }
      fence_async_smem();
      named_sync(1, NEPI);
      if (tid == 0) {
        const int y = n0, z = static_cast<int>(bh);
        tma_store_3d(&tm_dq, sb + B::O_DQ, 0, y, z);
        tma_store_3d(&tm_dq, sb + B::O_DQ + B::OBOX, 32, y, z);
        tma_store_3d(&tm_dk, sb + B::O_DK, 0, y, z);
        tma_store_3d(&tm_dk, sb + B::O_DK + B::OBOX, 32, y, z);
        tma_store_3d(&tm_dv, sb + B::O_DV, 0, y, z);
        tma_store_3d(&tm_dv, sb + B::O_DV + B::OBOX, 32, y, z);
        bulk_commit();
      }
    }
    tc_fence_before();
    named_sync(1, NEPI);
  }

  if (!aborted) {
    // contract the table adjoint with the three derivative tables
#pragma unroll
    for (int cb = 0; cb < 32; cb += 16) {
      const int j0 = 32 * half + cb;
      uint32_t r[16];
      tmem_ld16(trow + B::T_EBAR + j0, r);
      tmem_ld_wait16(r);
      float* acc[3] = {&tD, &tR, &tI};
#pragma unroll
      for (int w = 0; w < 3; ++w) {
        const float4* dq4 = reinterpret_cast<const float4*>(dErow + w * tstride + j0);
        float t = *acc[w];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const float4 d = dq4[g];
          t = fmaf(__uint_as_float(r[4 * g]), d.x, t);
          t = fmaf(__uint_as_float(r[4 * g + 1]), d.y, t);
          t = fmaf(__uint_as_float(r[4 * g + 2]), d.z, t);
          t = fmaf(__uint_as_float(r[4 * g + 3]), d.w, t);
        }
        *acc[w] = t;
      }
    }
    // this thread's shares, then the sum over the mode's four threads (two
    // rows re/im in adjacent lanes, two column halves in warps w and w + 4),
    // written for the fixed-order reduction over the batch
    float g3[3];
    g3[0] = fmaf(ReA, gs, fmaf(static_cast<float>(C), fmaf(ReA, zr, ImA * zn), tD));
    g3[1] = fmaf(Dm, gs, fmaf(static_cast<float>(C) * Dm, zr, tR));
    g3[2] = fmaf(static_cast<float>(C) * Dm, zn, tI);
#pragma unroll
    for (int w = 0; w < 3; ++w) g3[w] += __shfl_xor_sync(kFull, g3[w], 1);
    named_sync(1, NEPI);
    if (half == 1 && comp == 0)
      for (int w = 0; w < 3; ++w) sRED[w * KR / 2 + m] = g3[w];
    named_sync(1, NEPI);
    if (half == 0 && comp == 0)
      for (int w = 0; w < 3; ++w) a.gpart[(bh * kModesTC + m) * 3 + w] = g3[w] + sRED[w * KR / 2 + m];
  } else {   // let our own copies land before exiting (bounded)
    if (tid == 0 && tma_pending) mbar_wait(bar_tma, ph_tma, a.err);
    if (tid == 0 && r_pending) mbar_wait(bar_r, ph_r, a.err);
  }
    if (tid == 0) bulk_wait_all();   // dq, dk, dv are in global memory before the block exits
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace

bool tc_bwd_supported(const ia_shape_t& s) {
  return s.in_dtype == IA_BF16 && s.M == kModesTC && s.d_xi == 64 && s.d_v == 64;
}

size_t tc_fwd_bwd_workspace_bytes(const ia_shape_t& s, const TcPlan& p) {
  const size_t BH = static_cast<size_t>(s.B) * s.H;
  const size_t nch = (s.N + C - 1) / C;
  size_t bytes = tc_workspace_bytes(s, p);
  bytes = (bytes + 255) & ~static_cast<size_t>(255);
  bytes += BH * nch * 2 * KR * 64 * 2;                        // R per chunk: two fp16 tiles
  bytes += BH * nch * KR * sizeof(float);                      // R_eta per chunk
  bytes += BH * s.N * sizeof(float) + 256;                     // den
  bytes += dtab_floats(s.H) * sizeof(float) + 256;              // derivative tables
  bytes += grad_partials_bytes(s) + 256;                        // per-(b,h,m) gradient partials
  return bytes + 256;
}

cudaError_t launch_tc_fwd_bwd(const ia_shape_t& s, const TcPlan& p, const void* q, const void* k,
                              const void* v, const float* delta, const float* A, const void* dO,
                              float* o, float* dq, float* dk, float* dv, float* dDelta, float* dA,
                              void* ws, cudaStream_t st) {
  const size_t BH = static_cast<size_t>(s.B) * s.H;
  const size_t nch = (s.N + C - 1) / C;
  uint8_t* base = reinterpret_cast<uint8_t*>(tc_tables(ws));
  size_t off = (tc_workspace_bytes(s, p) + 255) & ~static_cast<size_t>(255);
  uint8_t* dumpR = base + off;   // 32 KB per chunk, 256-byte aligned
  float* dumpRe = reinterpret_cast<float*>(dumpR + BH * nch * 2 * B::RT);
  float* den = dumpRe + BH * nch * KR;
  den = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(den) + 255) & ~static_cast<uintptr_t>(255));
  float* dtab = den + BH * s.N;
  dtab = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(dtab) + 255) & ~static_cast<uintptr_t>(255));
  float* gpart = dtab + dtab_floats(s.H);
  gpart = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(gpart) + 255) & ~static_cast<uintptr_t>(255));
  cudaError_t e = launch_tc_prefill(s, p, q, k, v, delta, A, nullptr, o, nullptr, den, nullptr, ws,
                                    st, dumpR, dumpRe, dtab);
  if (e != cudaSuccess) return e;
  BwdArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.dO = static_cast<const __nv_bfloat16*>(dO);
  a.o = o;
  a.den = den;
  a.A = A;
  a.delta = delta;
  a.dpm = s.delta_per_mode;
  a.tabs = tc_tables(ws);
  a.R = dumpR;
  a.Re = dumpRe;
  a.dtab = dtab;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.gpart = gpart;
  a.err = device_error_ptr();
  if (!a.err) return cudaErrorInvalidSymbol;
  a.H = s.H;
  a.N = s.N;
  a.BH = static_cast<long long>(BH);
  CUtensorMap tm_dq, tm_dk, tm_dv;
  if (!encode_rows64_f32_map(&tm_dq, dq, a.BH, s.N, 64) || !encode_rows64_f32_map(&tm_dk, dk, a.BH, s.N, 64) ||
      !encode_rows64_f32_map(&tm_dv, dv, a.BH, s.N, 64))
    return cudaErrorNotSupported;
  e = cudaFuncSetAttribute(tc_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, B::SMEM);
  if (e != cudaSuccess) return e;
  mark_launch_begin(st);
  tc_bwd_kernel<<<static_cast<unsigned>(BH), NBWD, B::SMEM, st>>>(a, tm_dq, tm_dk, tm_dv);
  e = cudaGetLastError();
  mark_launch_end(st);
  if (e != cudaSuccess) return e;
  return launch_grad_reduce(s, gpart, dDelta, dA, st);
}

}  // namespace ia
