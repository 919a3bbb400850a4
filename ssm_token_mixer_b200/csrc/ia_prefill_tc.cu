// Chunked IA prefill on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// What it computes is the causal IA layer (paper 'Interdomain Attention:
// Beyond Token-Level Key-Value Memory'; paperlayer.ai summary sec. 3.1-3.2;
// AI-radio page formula extract "O = Fq U^T Gamma / Fq U^T eta"), run
// chunkwise with chunk length C = 64 and state passing between chunks as the
// summary's sec. A.2 describes.  Per (b,h) and chunk, with positions i, j in
// [0, C), centre c = C/2 and the per-head table E'[j,m] = b_m lambda_m^(c-j):
//
//   S^T   = xi(K) xi(Q)^T                         G1  (masked j <= i)
//   a~^T  = E'^T S^T + R_U xi(Q)^T                G2 + G3   (a_i = lambda^(i-c) a~_i)
//   X     = |lambda|^(2(i-c)) a~                  (rows re/im; = conj(a) lambda^(i-c))
//   P     = X E'^T                                G4  (masked j <= i)
//   num   = P V + X R_Gamma,  den = P 1 + X R_eta G5 + G6
//   o     = num / den
//   S_hat <- R + E'^T [xi(K) | V]                 G7  (accumulated onto R in TMEM)
//
// where the running state is kept scaled, S_hat = lambda^-(C-c-1) S, so that
// R = lambda^C S_hat is both the decayed state the chunk adds to and the
// carried state its queries read (lambda^(c+1) S0).  Complex numbers are
// split into real rows k = 2m (re) and 2m+1 (im), so every contraction is a
// real fp16 x fp16 -> fp32 tcgen05 MMA with M = 64 or 128.
//
// Work split.  The value columns are cut into blocks of 64 (one per CTA at a
// time), so a "stream" is one (b,h, value block): its CTA carries the whole
// U (M x d_xi) but only its block of Gamma.  The grid is at most one CTA per
// SM, and every CTA takes an equal contiguous range of the flattened
// (stream, chunk) space, so all SMs get the same number of chunks whatever
// the batch.  A range may start or end inside a stream.  The carried state
// at such a boundary comes from the chunk algebra's linearity (the summary's
// sec. A.2: parallel work within pieces, sequential state passing between
// them): a CTA whose range ends inside a stream first runs the state-only
// chain over that last piece from a zero state and publishes the result
// (its local aggregate) to global memory; a CTA whose range starts inside a
// stream composes its carry-in from its predecessors' published states,
// S_in = sum over hops of lambda^(C n) A_p (a decoupled look-back, every
// wait bounded), then runs the full chunk pass over its pieces.
#include <cuda.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>

#include "ia_device.cuh"
#include "ia_internal.h"
#include "ia_tables.cuh"
#include "ia_tc_common.cuh"

namespace ia {

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (the library links no driver stub).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// q, k or v [BH][N][W] bf16 (W a multiple of 64): one box is 64 rows x 64
// columns (128 bytes) of one (b,h), 128-byte swizzled in shared memory.  Rows
// >= N lie outside the map and read as zero.
bool encode_input_map(CUtensorMap* m, const void* x, long long BH, int N, int W, bool fp16) {
  const EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(W), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(W) * 2, static_cast<cuuint64_t>(N) * W * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kChunk), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x),
             dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// An fp32 [BH][N][W] array (o, dq, dk, dv) seen as boxes of 32 columns x 64
// rows of one (b,h), 128-byte swizzled in shared memory; rows >= N lie
// outside the map (TMA stores skip them).
bool encode_rows64_f32_map(CUtensorMap* m, float* o, long long BH, int N, int W) {
  const EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(W), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(W) * sizeof(float),
                                 static_cast<cuuint64_t>(N) * W * sizeof(float)};
  const cuuint32_t box[3] = {32, static_cast<cuuint32_t>(kChunk), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, o, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

using namespace tc;

constexpr int kVB = 64;                  // value columns per stream (one CTA's block of Gamma)
constexpr int kMinPiece = 4;             // fewest chunks per CTA the planner hands out

// Four roles: 8 prepare warps (0-7) convert the inputs and rotate the carried
// state into R; 8 output warps (8-15) run the masks, the readout scale and
// o = num/den, and convert the k and v tiles of the state-only chain that
// precedes their first chunk; warp 16 issues every tensor-core contraction;
// warp 17 brings q, k, v in with TMA tensor loads that land in the operand
// layout.  The inputs are bf16 (q, k through the feature map on the way to
// fp16), or, for the layer's input stabilisation, k and v arrive as ready
// fp16 operands and only their rows past the sequence are cleared.
constexpr int GW = 8;                    // warps per epilogue group
constexpr int GT = GW * 32;              // threads per epilogue group
constexpr int NTH = 2 * GT + 64;         // + the MMA warp and the fetch warp

template <int DX, bool RW>
struct PCfg {
  static constexpr int F = DX + kVB;                // state columns: U | Gamma block
  static constexpr int FH = F / 2;                  // state columns per prepare thread
  static constexpr int WV = 80, NV = 80;            // [V | 1 0..] and [R_Gamma | R_eta 0..] widths
  // q, k, v and R_Gamma buffer sets: two when the readout matrix W' takes
  // its 32 KB of shared memory (d_xi = 64 only)
  static constexpr int NB = DX == 64 && !RW ? 3 : 2;
  static_assert(!RW || DX == 64, "the readout matrix runs at d_xi = 64");
  // d_xi = 128 needs 64 more state columns; S^T, a~ and P then share one tile
  // (each is dead before the next is written within a chunk), at the price
  // of issuing G1 of a chunk only after the previous chunk's P has been read.
  static constexpr bool SHARED_SAP = DX == 128;
  static constexpr uint32_t RSV = WV * 16;
  static constexpr uint32_t T_STATE = 0;
  static constexpr uint32_t T_A = F;
  static constexpr uint32_t T_S = SHARED_SAP ? F : F + 64;
  static constexpr uint32_t T_P = SHARED_SAP ? F : F + 128;
  static constexpr uint32_t T_NUM = SHARED_SAP ? F + 64 : F + 192;
  static constexpr uint32_t T_DEN = T_NUM + 64;
  static constexpr uint32_t RU_COLS = DX / 2;       // R_U as fp16 pairs: columns per buffer
  static constexpr uint32_t T_RU = SHARED_SAP ? 384 : 400;   // [2] x RU_COLS
  static_assert(T_RU >= T_NUM + NV && T_RU + 2 * RU_COLS <= 512, "TMEM budget");
  static constexpr uint32_t BOX = C * 64 * 2;       // one 64 x 64 bf16 box: 8 KB
  static constexpr uint32_t TQ = C * DX * 2;        // q or k tile: DX / 64 boxes
  static constexpr uint32_t TV = C * kVB * 2;
  static constexpr uint32_t TRG = KR * WV * 2;
  static constexpr uint32_t TO = C * kVB * 4;       // o block of one chunk: two 64 x 128-byte boxes
  static constexpr uint32_t SW = 1024;              // one swizzle atom: 8 rows x 128 bytes
  static constexpr uint32_t S_Q = 0;
  static constexpr uint32_t S_K = S_Q + NB * TQ;
  static constexpr uint32_t S_V = S_K + NB * TQ;
  static constexpr uint32_t S_ONES = S_V + NB * TV;   // [V | 1]: MN-block 64..127 of G5's B operand
  static constexpr uint32_t S_E = S_ONES + TV;
  static constexpr uint32_t S_S = S_E + KR * C * 2;
  static constexpr uint32_t S_P = S_S + C * C * 2;
  static constexpr uint32_t S_X = S_P + C * C * 2;
  static constexpr uint32_t S_O = S_X + KR * C * 2;   // [2] o staging, 128-byte swizzled
  static constexpr uint32_t S_RG = S_O + 2 * TO;      // [NB]
  static constexpr uint32_t S_W = S_RG + NB * TRG;    // W' [2M x 2M] fp16, no-swizzle K-major (RW)
  static constexpr uint32_t S_BAR = S_W + (RW ? KR * KR * 2 : 0);   // mbarriers
  static constexpr uint32_t S_FLAG = S_BAR + 256;     // abort flag, look-back exchange
  static constexpr uint32_t S_TMEMH = S_FLAG + 16;
  static constexpr uint32_t SMEM = S_TMEMH + 16;
  static_assert(SMEM <= 232448, "fits one CTA's opt-in shared memory");
  static_assert(S_O % 1024 == 0 && S_K % 1024 == 0 && S_V % 1024 == 0 && S_ONES % 1024 == 0,
                "swizzled tiles start on the 128-byte swizzle period");
  // byte offset of K-step kk (16 features) inside a K-major swizzled q/k tile
  static __device__ __forceinline__ uint32_t kstep(int kk) { return (kk >> 2) * BOX + (kk & 3) * 32; }
};

struct TcArgs {
  const HeadTables* tabs;
  const float2* state_in;   // public layout, unscaled
  float* o;
  float* num;
  float* den;
  float2* state_out;
  int* err;                 // device error flag
  uint8_t* dump_R;          // optional: R = lambda^C S_hat at every chunk start, fp16 tiles (dump_r16)
  float* dump_Re;           // optional: the eta part, [BH][nch][128] fp32
  float* agg;               // [G][128 * F + 128]: local end state of a CTA's last piece
  float* incl;              // [G][128 * F + 128]: inclusive end state of a CTA's last piece
  int* flags;               // [G]: 0 nothing yet, 1 agg published, 2 incl published
  int kv_ready;             // 1: k, v arrive as fp16 operands (k already through the feature map)
  const __half* Wt;         // readout matrix per head as W' tiles (wprime_offset layout), RW only
  int H, N, DV, nch, nvb, G;
  long long BH, total;      // total = BH * nvb * nch chunks
};

__device__ __forceinline__ uint4 pack8f(const uint32_t* r, float scale) {
  return make_uint4(pack_half2(__uint_as_float(r[0]) * scale, __uint_as_float(r[1]) * scale),
                    pack_half2(__uint_as_float(r[2]) * scale, __uint_as_float(r[3]) * scale),
                    pack_half2(__uint_as_float(r[4]) * scale, __uint_as_float(r[5]) * scale),
                    pack_half2(__uint_as_float(r[6]) * scale, __uint_as_float(r[7]) * scale));
}

// R for the reverse pass: per chunk two fp16 tiles, R_U then R_Gamma, each
// 128 rows (k) x 64 columns in the 128-byte swizzled layout (16-byte chunk c
// of row k at byte k * 128 + (c ^ (k % 8)) * 16), 32 KB per chunk, so that a
// plain bulk copy lands them ready to serve as tensor-core operands.  Stores
// columns col0..col0+15 (col0 a multiple of 16) of row k of chunk `chunk`.
constexpr uint32_t kDumpTile = KR * 64 * 2;
__device__ __forceinline__ void dump_r16(uint8_t* base, long long chunk, int k, int col0, const uint32_t* w) {
  uint8_t* row = base + (chunk * 2 + (col0 >= 64 ? 1 : 0)) * kDumpTile + k * 128;
  const int c0 = (col0 & 63) >> 3;
#pragma unroll
  for (int g = 0; g < 2; ++g)
    *reinterpret_cast<uint4*>(row + (((c0 + g) ^ (k & 7)) << 4)) = pack8f(w + 8 * g, 1.f);
}

// The CTA's schedule: its range [g0, g1) of the flattened (stream, chunk)
// space; if the range ends inside a stream, the state-only items [gA, g1)
// come first, then the full items [g0, g1).
struct Sched {
  long long g0, g1, gA;
  int nA, nF, nch;
  __device__ __forceinline__ Sched(long long total, int G, int c, int nch_) : nch(nch_) {
    g0 = total * c / G;
    g1 = total * (c + 1) / G;
    const bool mid_end = g1 % nch != 0;
    gA = mid_end ? max(g0, (g1 - 1) / nch * nch) : g1;
    nA = static_cast<int>(g1 - gA);
    nF = static_cast<int>(g1 - g0);
  }
  __device__ __forceinline__ bool state_only(int i) const { return i < nA; }
  __device__ __forceinline__ int items() const { return nA + nF; }
};

// Walks the items of a schedule in order without a 64-bit division per item:
// (stream, chunk) advance by one chunk at a time, the stream splitting into
// (b,h) and value block (nvb = 1 or 2 blocks, so lgv = nvb - 1) and the head
// following the (b,h).
struct Walker {
  int ch, vb, bh, h;
  __device__ __forceinline__ void seek(long long g, int nch, int nvb, int H) {
    const long long stream = g / nch;
    ch = static_cast<int>(g - stream * nch);
    vb = static_cast<int>(stream & (nvb - 1));
    bh = static_cast<int>(stream >> (nvb - 1));
    h = bh % H;
  }
  __device__ __forceinline__ void step(int nch, int nvb, int H) {
    if (++ch < nch) return;
    ch = 0;
    if (++vb < nvb) return;
    vb = 0;
    ++bh;
    if (++h == H) h = 0;
  }
  // position of item i + 1 of the schedule, after item i
  __device__ __forceinline__ void next(const Sched& sc, int i, int nch, int nvb, int H) {
    if (i + 1 == sc.nA) seek(sc.g0, nch, nvb, H);
    else step(nch, nvb, H);
  }
};

// Range start of CTA c (same arithmetic as Sched).
__device__ __forceinline__ long long range_lo(long long total, int G, int c) { return total * c / G; }

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---------------------------------------------------------------------------
// Cold paths of the prepare warps, kept out of line so that the chunk loop's
// code stays small (the four roles run different code and share the SM's
// instruction cache).  Each prepare thread owns TMEM lane / state row
// k = 2m + comp and one half of the state columns.
struct PrepThread {
  uint32_t trow;   // this warp's TMEM lane quadrant
  int tid, k, m, comp, half;
};

// lambda_m^n in fp64 from the table's Delta A (phase reduced modulo 2 pi)
__device__ __noinline__ void lam_pow(const HeadTables* T, int m, double n, double* pr, double* pi) {
  const double e = exp(n * T->re_dA[m]);
  const double ph = fmod(n * T->im_dA[m], 6.283185307179586476925);
  double sn, cs;
  sincos(ph, &sn, &cs);
  *pr = e * cs;
  *pi = e * sn;
}

// component comp of sum_{j < nv} E'[j, m]: the constant channel's carry of
// a ragged last chunk
__device__ __noinline__ float ragged_esum(const HeadTables* T, int m, int comp, int nv) {
  double sr = 0.0, si = 0.0;
  const double br = T->b[m].x, bi = T->b[m].y;
  for (int j = 0; j < nv; ++j) {
    double pr, pi;
    lam_pow(T, m, C / 2 - j, &pr, &pi);
    sr += br * pr - bi * pi;
    si += br * pi + bi * pr;
  }
  return static_cast<float>(comp ? si : sr);
}

// state column f of row m in the public layout (complex): U for f < DX,
// else column vb * 64 + f - DX of Gamma
template <int DX, bool RW>
__device__ __forceinline__ long long pub_index(const TcArgs& a, long long bh, int m, int vb, int f) {
  return f < DX ? (bh * 64 + m) * DX + f : a.BH * 64 * DX + (bh * 64 + m) * a.DV + vb * kVB + (f - DX);
}

template <int DX, bool RW>
__device__ __noinline__ void prep_zero(const PrepThread& th) {
  constexpr int FH = PCfg<DX, RW>::FH;
  uint32_t z[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) z[e] = 0u;
  for (int cb = 0; cb < FH; cb += 16) tmem_st16(th.trow + PCfg<DX, RW>::T_STATE + th.half * FH + cb, z);
  tmem_st_wait();
}

// initial scaled state of a piece from state_in (zero without it); returns
// this row's eta
template <int DX, bool RW>
__device__ __noinline__ float prep_init_from_input(const TcArgs& a, const HeadTables* T, const PrepThread& th,
                                                  long long bh, int vb) {
  constexpr int FH = PCfg<DX, RW>::FH;
  if (!a.state_in) {
    prep_zero<DX, RW>(th);
    return 0.f;
  }
  const float2 si = T->sc_inv[th.m];
  for (int cb = 0; cb < FH; cb += 16) {
    const int col0 = th.half * FH + cb;
    uint32_t r[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float2 x = a.state_in[pub_index<DX, RW>(a, bh, th.m, vb, col0 + e)];
      r[e] = __float_as_uint(th.comp ? fmaf(si.x, x.y, si.y * x.x) : fmaf(si.x, x.x, -si.y * x.y));
    }
    tmem_st16(th.trow + PCfg<DX, RW>::T_STATE + col0, r);
  }
  tmem_st_wait();
  const float2 x = a.state_in[a.BH * 64 * (DX + a.DV) + bh * 64 + th.m];
  return th.comp ? fmaf(si.x, x.y, si.y * x.x) : fmaf(si.x, x.x, -si.y * x.y);
}

// the state after the last token of a stream: sc lambda^(nv - C) S_hat = lambda^(nv-c-1) S_hat
template <int DX, bool RW>
__device__ __noinline__ void prep_write_state_out(const TcArgs& a, const HeadTables* T, const PrepThread& th,
                                                  long long bh, int vb, int ch, float eta_c) {
  constexpr int FH = PCfg<DX, RW>::FH;
  const int nv = a.N - ch * C;
  double pr, pi;
  lam_pow(T, th.m, nv - C / 2 - 1, &pr, &pi);
  const float fr = static_cast<float>(pr), fi = static_cast<float>(pi);
  for (int cb = 0; cb < FH; cb += 16) {
    const int col0 = th.half * FH + cb;
    uint32_t r[16];
    tmem_ld16(th.trow + PCfg<DX, RW>::T_STATE + col0, r);
    tmem_ld_wait16(r);
#pragma unroll
    for (int e2 = 0; e2 < 16; ++e2) {
      const float x = __uint_as_float(r[e2]);
      const float y = __shfl_xor_sync(kFull, x, 1);
      const int f = col0 + e2;
      if (th.comp == 0 && (f >= DX || vb == 0))   // U is the same in every value block
        a.state_out[pub_index<DX, RW>(a, bh, th.m, vb, f)] = make_float2(fr * x - fi * y, fr * y + fi * x);
    }
  }
  const float y = __shfl_xor_sync(kFull, eta_c, 1);
  if (th.comp == 0 && th.half == 0 && vb == 0)
    a.state_out[a.BH * 64 * (DX + a.DV) + bh * 64 + th.m] = make_float2(fr * eta_c - fi * y, fr * y + fi * eta_c);
}

// A published state (workspace only) holds columns in groups of four, each
// group row after row: float4 (c / 4) * KR + k is row k, columns c .. c + 3,
// so the 32 rows of a warp read or write 512 contiguous bytes per
// instruction; eta follows, one float per row.
__device__ __forceinline__ int pub4(int c, int k) { return (c >> 2) * KR + k; }

// this thread's part of the TMEM state (and eta) -> dst [128 * F + 128]
template <int DX, bool RW>
__device__ __noinline__ void prep_publish(const PrepThread& th, float* dst, float eta_c) {
  constexpr int F = PCfg<DX, RW>::F, FH = PCfg<DX, RW>::FH;
  float4* d4 = reinterpret_cast<float4*>(dst);
  for (int cb = 0; cb < FH; cb += 16) {
    const int col0 = th.half * FH + cb;
    uint32_t r[16];
    tmem_ld16(th.trow + PCfg<DX, RW>::T_STATE + col0, r);
    tmem_ld_wait16(r);
#pragma unroll
    for (int g = 0; g < 4; ++g)
      d4[pub4(col0 + 4 * g, th.k)] = make_float4(__uint_as_float(r[4 * g]), __uint_as_float(r[4 * g + 1]),
                                                 __uint_as_float(r[4 * g + 2]), __uint_as_float(r[4 * g + 3]));
  }
  if (th.half == 0) dst[KR * F + th.k] = eta_c;
}

// every prepare thread's stores are visible GPU-wide before one thread raises
// the flag (release)
__device__ __noinline__ void prep_raise_flag(int* flag, int value, int tid) {
  __threadfence();
  named_sync(4, GT);
  if (tid == 0) st_release(flag, value);
}

// TMEM state (and eta) += (mr + i mi) src, complex per mode (rows 2m, 2m+1).
// src was written by another SM: each load is an L2 round trip, so a
// thread's row segment is fetched in two batches (not one block at a time).
template <int DX, bool RW>
__device__ __noinline__ void prep_accumulate(const PrepThread& th, const float* src, double mr, double mi, float* eta) {
  constexpr int F = PCfg<DX, RW>::F, FH = PCfg<DX, RW>::FH;
  constexpr int HB = FH / 8;   // float4 per batch: half of this thread's segment
  static_assert(HB % 4 == 0, "a batch holds whole 16-column blocks");
  const float fr = static_cast<float>(mr), fs = static_cast<float>(th.comp ? mi : -mi);
  const float4* s4 = reinterpret_cast<const float4*>(src);
  const float xe = __ldcg(src + KR * F + th.k);
#pragma unroll
  for (int hb = 0; hb < 2; ++hb) {
    float4 g[HB];
#pragma unroll
    for (int u = 0; u < HB; ++u) g[u] = __ldcg(s4 + pub4(th.half * FH + 4 * (hb * HB + u), th.k));
#pragma unroll
    for (int blk = 0; blk < HB / 4; ++blk) {
      const int col0 = th.half * FH + (hb * HB + 4 * blk) * 4;
      uint32_t r[16];
      tmem_ld16(th.trow + PCfg<DX, RW>::T_STATE + col0, r);
      tmem_ld_wait16(r);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float4 v4 = g[4 * blk + e / 4];
        const float x = (e & 3) == 0 ? v4.x : ((e & 3) == 1 ? v4.y : ((e & 3) == 2 ? v4.z : v4.w));
        const float y = __shfl_xor_sync(kFull, x, 1);
        r[e] = __float_as_uint(__uint_as_float(r[e]) + fmaf(fr, x, fs * y));
      }
      tmem_st16(th.trow + PCfg<DX, RW>::T_STATE + col0, r);
    }
  }
  tmem_st_wait();
  const float ye = __shfl_xor_sync(kFull, xe, 1);
  *eta += fmaf(fr, xe, fs * ye);
}

// Carry into a first piece that starts inside a stream: the sum over the
// predecessors q = c-1, c-2, ... in the stream of lambda^(C d_q) times their
// published end states, d_q the chunks from q's range end to our start,
// down to the first inclusive state.  The flags of up to kLookBackWindow
// predecessors are awaited together and their states summed in one round,
// so a CTA pays one wait for all of them instead of one per hop.  Leaves the
// carry in the TMEM state and *eta.  Returns false if a wait gave up
// (uniform over the prepare group).
constexpr int kLookBackWindow = 8;

template <int DX, bool RW>
__device__ __noinline__ bool prep_look_back(const TcArgs& a, const HeadTables* T, const PrepThread& th,
                                            volatile int* abort_flag, volatile int* xchg, float* eta) {
  constexpr int STRIDE = KR * PCfg<DX, RW>::F + KR;
  const double re_dA = T->re_dA[th.m], im_dA = T->im_dA[th.m];
  prep_zero<DX, RW>(th);
  *eta = 0.f;
  const long long g0 = range_lo(a.total, a.G, blockIdx.x);
  for (int p = static_cast<int>(blockIdx.x) - 1; p >= 0;) {
    if (th.tid == 0) {   // await p, p-1, ... (bounded): stop at an inclusive state or the window's end
      int lo = -1, incl = 0;
      const unsigned long long t0 = global_ns();
      for (int q = p; q >= 0 && q > p - kLookBackWindow; --q) {
        int f = ld_acquire(a.flags + q);
        while (f == 0 && !*abort_flag) {
          if (global_ns() - t0 > kWaitLimitNs) {
            atomicOr(a.err, kErrTimeout);
            *abort_flag = 1;
            break;
          }
          f = ld_acquire(a.flags + q);
        }
        if (f == 0) {
          lo = -1;
          break;
        }
        lo = q;
        if (f == 2) {
          incl = 1;
          break;
        }
      }
      *xchg = lo < 0 ? 0 : (((lo + 1) << 1) | incl);
    }
    named_sync(4, GT);
    const int v = *xchg;
    named_sync(4, GT);
    if (v == 0) return false;
    const int lo = (v >> 1) - 1;
    const bool incl = (v & 1) != 0;
    __threadfence();
    for (int q = p; q >= lo; --q) {
      const double n = static_cast<double>(C) * static_cast<double>(g0 - range_lo(a.total, a.G, q + 1));
      double lr = 1.0, li = 0.0;
      if (n > 0.0) {
        const double e = exp(n * re_dA);
        double sn, cs;
        sincos(fmod(n * im_dA, 6.283185307179586476925), &sn, &cs);
        lr = e * cs;
        li = e * sn;
      }
      prep_accumulate<DX, RW>(th, (q == lo && incl ? a.incl : a.agg) + static_cast<long long>(q) * STRIDE, lr, li, eta);
    }
    if (incl) return true;
    p = lo - 1;
  }
  return false;   // unreachable: the stream's first piece publishes an inclusive state
}

// A CTA whose one piece lies inside a stream publishes its inclusive end
// state once its carry (in TMEM, eta) is known: local + lambda^(C n) carry.
template <int DX, bool RW>
__device__ __noinline__ void prep_publish_inclusive(const TcArgs& a, const HeadTables* T, const PrepThread& th,
                                                    int n, float eta_c) {
  constexpr int F = PCfg<DX, RW>::F, FH = PCfg<DX, RW>::FH, STRIDE = KR * F + KR;
  double lr, li;
  lam_pow(T, th.m, static_cast<double>(C) * n, &lr, &li);
  const float fr = static_cast<float>(lr), fs = static_cast<float>(th.comp ? li : -li);
  const float* loc = a.agg + static_cast<long long>(blockIdx.x) * STRIDE;
  float* dst = a.incl + static_cast<long long>(blockIdx.x) * STRIDE;
  constexpr int HB = FH / 8;   // float4 per batch (the local state is re-read from L2)
  const float4* l4 = reinterpret_cast<const float4*>(loc);
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int hb = 0; hb < 2; ++hb) {
    float4 g[HB];
#pragma unroll
    for (int u = 0; u < HB; ++u) g[u] = __ldcg(l4 + pub4(th.half * FH + 4 * (hb * HB + u), th.k));
#pragma unroll
    for (int blk = 0; blk < HB / 4; ++blk) {
      const int col0 = th.half * FH + (hb * HB + 4 * blk) * 4;
      uint32_t r[16];
      tmem_ld16(th.trow + PCfg<DX, RW>::T_STATE + col0, r);
      tmem_ld_wait16(r);
      float o[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float x = __uint_as_float(r[e]);
        const float y = __shfl_xor_sync(kFull, x, 1);
        o[e] = fmaf(fr, x, fs * y);
      }
#pragma unroll
      for (int gg = 0; gg < 4; ++gg) {
        const float4 lv = g[4 * blk + gg];
        d4[pub4(th.half * FH + 4 * (hb * HB + 4 * blk + gg), th.k)] =
            make_float4(lv.x + o[4 * gg], lv.y + o[4 * gg + 1], lv.z + o[4 * gg + 2], lv.w + o[4 * gg + 3]);
      }
    }
  }
  const float y = __shfl_xor_sync(kFull, eta_c, 1);
  if (th.half == 0) dst[KR * F + th.k] = loc[KR * F + th.k] + fmaf(fr, eta_c, fs * y);
  prep_raise_flag(a.flags + blockIdx.x, 2, th.tid);
}

// What a piece start hands back to the chunk loop.
struct PieceStart {
  float eta;      // this row's eta of the piece's initial state
  bool ok;        // false if a wait gave up (uniform over the prepare group)
  bool pending;   // the CTA still owes its inclusive state
};

// Everything the prepare warps do at a piece start, between the G7 wait of
// the previous item and the rotation of the piece's first item: publish the
// end of the state-only chain or write state_out of the stream that ended,
// reload E' on a change of head (once every contraction reading the old one
// is done), and set the piece's initial state (zero, state_in, or the carry
// from the look-back).  One call out of the chunk loop, so that the loop keeps
// its registers for the per-chunk work.
template <int DX, bool RW>
__device__ __noinline__ PieceStart prep_piece_start(const TcArgs& a, const PrepThread& th, int i, int nA, long long gA,
                                                    int nF, bool so, int ch, long long bh, int vb, int h,
                                                    int prev_bh, int prev_vb, int prev_ch, int cur_h, float eta_c,
                                                    bool pending, volatile int* abort_flag, volatile int* xchg,
                                                    volatile int* g4_seen, uint8_t* sE, uint8_t* sW) {
  constexpr int STRIDE = KR * PCfg<DX, RW>::F + KR;   // floats per published state
  PieceStart r{eta_c, true, pending};
  const HeadTables* T = a.tabs + cur_h;
  if (i > 0) {
    if (i - 1 < nA) {
      // end of the state-only chain: publish our last piece's state
      const bool inclusive = gA % a.nch == 0;
      prep_publish<DX, RW>(th, (inclusive ? a.incl : a.agg) + static_cast<long long>(blockIdx.x) * STRIDE, eta_c);
      prep_raise_flag(a.flags + blockIdx.x, inclusive ? 2 : 1, th.tid);
      r.pending = !inclusive;
    } else if (prev_ch == a.nch - 1 && a.state_out) {
      prep_write_state_out<DX, RW>(a, T, th, prev_bh, prev_vb, prev_ch, eta_c);
    }
  }
  if (h != cur_h) {
    // A new head: its E' table (and W') replaces the old one once every
    // contraction reading the old one is done.  G7 of the previous item is;
    // every G2, G_W and G4 of the previous full items is once the output warps
    // have seen G4 of the last of them complete.
    const int t = i - nA;
    if (t >= 1) {
      bool ok = true;
      if (th.tid == 0) {
        const unsigned long long t0 = global_ns();
        while (*g4_seen < t) {
          if (*abort_flag) {
            ok = false;
            break;
          }
          if (global_ns() - t0 > kWaitLimitNs) {
            atomicOr(a.err, kErrTimeout);
            *abort_flag = 1;
            ok = false;
            break;
          }
          __nanosleep(64);
        }
        __threadfence_block();
      }
      if (named_sync_or(2, GT, !ok)) {
        r.ok = false;
        return r;
      }
    }
    const uint4* src = reinterpret_cast<const uint4*>(a.tabs[h].E);
    uint4* dst = reinterpret_cast<uint4*>(sE);
    for (int x = th.tid; x < KR * C * 2 / 16; x += GT) dst[x] = src[x];
    if constexpr (RW) {   // the head's readout matrix, read by G_W between G2+G3 and G4
      const uint4* ws = reinterpret_cast<const uint4*>(a.Wt) + static_cast<size_t>(h) * (kWprimeBytes / 16);
      uint4* wd = reinterpret_cast<uint4*>(sW);
      for (int x = th.tid; x < static_cast<int>(kWprimeBytes / 16); x += GT) wd[x] = ws[x];
    }
    T = a.tabs + h;
  }
  if (so && gA % a.nch != 0) {   // a local aggregate starts from zero
    prep_zero<DX, RW>(th);
    r.eta = 0.f;
  } else if (so || ch == 0) {    // a stream's start: state_in or zero
    r.eta = prep_init_from_input<DX, RW>(a, T, th, bh, vb);
  } else {                       // inside a stream: the carry from the predecessors
    float e = 0.f;
    if (!prep_look_back<DX, RW>(a, T, th, abort_flag, xchg, &e)) {
      r.ok = false;
      return r;
    }
    r.eta = e;
    if (r.pending) {
      prep_publish_inclusive<DX, RW>(a, T, th, nF, e);
      r.pending = false;
    }
  }
  fence_async_smem();   // a reloaded E' table is read by the next contractions
  return r;
}

// The prepare warps' chunk loop over the n items of one piece: for each,
// wait for its tiles, convert them (a full item's q, k, v; the output warps
// convert a state-only item's k, v), wait for G7 of the item before (except
// for the piece's first item, whose wait comes before the piece start),
// rotate the carried state into R and signal the MMA warp.  It sits out of
// line, apart from the piece starts and their calls, so that its registers
// hold only what the chunks need.
struct PrepRun {
  float eta;
  uint32_t pd0, pld, pldv;   // parities of the G7 barrier and of the q,k / v loaded barriers (bit per set)
  bool ok;
};

template <int DX, bool RW>
__device__ __noinline__ PrepRun prep_chunks(const TcArgs& a_in, uint8_t* smem, const PrepThread th, const HeadTables* T,
                                            int i, int n, int b, bool so, long long bh, int ch, float eta_c,
                                            uint32_t pd0, uint32_t pld, uint32_t pldv, float esum_tail) {
  const TcArgs a = a_in;
  using K = PCfg<DX, RW>;
  constexpr int FH = K::FH, NB = K::NB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K::S_BAR);
  uint64_t* rdy0 = bars + 0;
  uint64_t* dne0 = bars + 4;
  uint64_t* loadedQK = bars + 16;
  uint64_t* loadedV = bars + 22;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + K::S_FLAG);
  const float2 lamC = T->lamC[th.m];
  const float sgnLi = th.comp ? lamC.y : -lamC.y;
  const uint64_t lamC2 = f2_pack(lamC.x, lamC.x), sgnLi2 = f2_pack(sgnLi, sgnLi);
  const float esum_c = th.comp ? T->esum[th.m].y : T->esum[th.m].x;
  PrepRun r{eta_c, pd0, pld, pldv, true};
  // waits for set b's q, k (QK) or v tiles, uniform over the prepare group
  auto wait_tiles = [&](uint64_t* bar, uint32_t& bits) -> bool {
    const bool ok = mbar_wait_or_abort(bar + b, (bits >> b) & 1u, a.err, abort_flag);
    bits ^= 1u << b;
    tc_fence_after();
    return !named_sync_or(2, GT, !ok);
  };
  for (int j = 0; j < n; ++j, ++i, ++ch, b = b + 1 == NB ? 0 : b + 1) {
    const int p = i & 1;
    const int nv = min(C, a.N - ch * C);
    if (!wait_tiles(loadedQK, r.pld)) {
      r.ok = false;
      return r;
    }
    // bf16 -> fp16 in place (q, k through the feature map); rows past the
    // sequence become 0.  A tile is a sequence of 8 KB boxes of 64 rows x
    // 128 bytes; the map is elementwise, so the swizzle does not matter.
    // q and k land before v (their buffers are released one contraction
    // group earlier), so they are converted first.
    constexpr int PQ = K::TQ / 16 / GT;   // 16-byte pieces of a q or k tile per thread
    constexpr int PV = K::TV / 16 / GT;
    auto convert = [&](const int tsel, const int NPIECE) {
      // every load first (a store may alias a later load, so loads issued in
      // between would queue behind it), then convert and store
      uint4 in[2 * PQ];
      const uint32_t base = tsel == 0 ? K::S_Q + b * K::TQ : (tsel == 1 ? K::S_K + b * K::TQ : K::S_V + b * K::TV);
#pragma unroll
      for (int u = 0; u < 2 * PQ; ++u) {
        if (u >= NPIECE) break;
        const int t = tsel == 0 && u >= PQ ? 1 : tsel;   // tsel 0 converts q then k
        const uint32_t bs = t == 0 ? base : (t == 1 ? K::S_K + b * K::TQ : base);
        const int pc = th.tid + (tsel == 0 ? u % PQ : u) * GT;
        in[u] = *reinterpret_cast<const uint4*>(smem + bs + pc * 16);
      }
#pragma unroll
      for (int u = 0; u < 2 * PQ; ++u) {
        if (u >= NPIECE) break;
        const int t = tsel == 0 && u >= PQ ? 1 : tsel;
        const uint32_t bs = t == 0 ? base : (t == 1 ? K::S_K + b * K::TQ : base);
        const int pc = th.tid + (tsel == 0 ? u % PQ : u) * GT;
        const int row = (pc >> 3) & 63;   // row within its box
        uint4 out = make_uint4(0u, 0u, 0u, 0u);
        if (row < nv && t > 0 && a.kv_ready) {   // k, v already fp16 operands
          out = in[u];
        } else if (row < nv) {
          const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&in[u]);
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(x2[e]);
            w[e] = t < 2 ? feat_h2(f.x, f.y) : pack_half2(f.x, f.y);
          }
          out = make_uint4(w[0], w[1], w[2], w[3]);
        }
        *reinterpret_cast<uint4*>(smem + bs + pc * 16) = out;
      }
    };
    if (!so) convert(0, 2 * PQ);   // the output warps convert a state-only item's k, v
    if (!wait_tiles(loadedV, r.pldv)) {
      r.ok = false;
      return r;
    }
    if (!so) convert(2, PV);
    if (j > 0) {   // G7 of the previous item: the state is current
      const bool ok = mbar_wait_or_abort(dne0, r.pd0, a.err, abort_flag);
      r.pd0 ^= 1u;
      tc_fence_after();
      if (named_sync_or(2, GT, !ok)) {
        r.ok = false;
        return r;
      }
    }
    // R = lambda^C S_hat -> TMEM (the state G7 adds to); for full items also
    // R_U (fp16 pairs in TMEM, A operand of G3) and R_Gamma (shared memory,
    // B operand of G6)
    uint8_t* sRG = smem + K::S_RG + b * K::TRG;
#pragma unroll
    for (int blk = 0; blk < FH / 16; ++blk) {
      const int col0 = th.half * FH + 16 * blk;
      uint32_t w[16];
      tmem_ld16(th.trow + K::T_STATE + col0, w);
      tmem_ld_wait16(w);
#pragma unroll
      for (int e = 0; e < 16; e += 2) {   // in place: Re/Im of lambda^C times the partner row, two columns at once
        const float x0 = __uint_as_float(w[e]), x1 = __uint_as_float(w[e + 1]);
        const uint64_t y = f2_pack(__shfl_xor_sync(kFull, x0, 1), __shfl_xor_sync(kFull, x1, 1));
        float w0, w1;
        f2_unpack(f2_fma(lamC2, f2_pack(x0, x1), f2_mul(sgnLi2, y)), w0, w1);
        w[e] = __float_as_uint(w0);
        w[e + 1] = __float_as_uint(w1);
      }
      tmem_st16(th.trow + K::T_STATE + col0, w);
      if (!so) {
        if (a.dump_R) dump_r16(a.dump_R, bh * a.nch + ch, th.k, col0, w);
        if (col0 < DX) {   // R_U: fp16 pairs into tensor memory, 8 columns per block
          uint32_t ru[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) ru[e] = pack_half2(__uint_as_float(w[2 * e]), __uint_as_float(w[2 * e + 1]));
          tmem_st8(th.trow + K::T_RU + K::RU_COLS * p + col0 / 2, ru);
        } else {           // R_Gamma: shared memory, B operand of G6
#pragma unroll
          for (int g2 = 0; g2 < 2; ++g2)
            *reinterpret_cast<uint4*>(sRG + tile_off(th.k, col0 - DX + 8 * g2, K::RSV)) = pack8f(w + 8 * g2, 1.f);
        }
      }
    }
    tmem_st_wait();
    {
      const float y = __shfl_xor_sync(kFull, r.eta, 1);
      const float Re = fmaf(lamC.x, r.eta, sgnLi * y);
      if (th.half == 0 && !so) {
        if (a.dump_Re) a.dump_Re[(bh * a.nch + ch) * KR + th.k] = Re;
        *reinterpret_cast<uint4*>(sRG + tile_off(th.k, kVB, K::RSV)) = make_uint4(pack_half2(Re, 0.f), 0u, 0u, 0u);
      }
      // ragged last chunk: partial sum of E' over the valid keys
      r.eta = Re + (nv < C ? esum_tail : esum_c);
    }
    fence_async_smem();
    tc_fence_before();
    mbar_arrive(rdy0);
  }
  return r;
}

// bf16 -> fp16 in place over one tile of PIECES 16-byte pieces, by NT
// threads (ct = 0 .. NT-1), through the feature map when FEAT; rows past the
// sequence become 0.  A tile is a sequence of 8 KB boxes of 64 rows x 128
// bytes; the map is elementwise, so the swizzle does not matter.
template <bool FEAT, int PIECES, int NT>
__device__ __forceinline__ void convert_tile(uint8_t* base, int nv, int ct, bool ready = false) {
  constexpr int U = PIECES / NT;
  static_assert(PIECES % NT == 0 && U <= 8, "pieces per thread");
  uint4 in[U];
#pragma unroll
  for (int u = 0; u < U; ++u) in[u] = *reinterpret_cast<const uint4*>(base + (ct + u * NT) * 16);
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int pc = ct + u * NT;
    uint4 out = make_uint4(0u, 0u, 0u, 0u);
    if (((pc >> 3) & 63) < nv) {   // row within its box
      if (ready) {
        out = in[u];
      } else {
        const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&in[u]);
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(x2[e]);
          w[e] = FEAT ? feat_h2(f.x, f.y) : pack_half2(f.x, f.y);
        }
        out = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    *reinterpret_cast<uint4*>(base + pc * 16) = out;
  }
}

// The four roles of the chunk pass, each out of line so that its registers
// are allocated for its own loop alone (the prepare warps' piece starts call
// out of line, and the spills around those calls stay in that role).  Each
// derives its barriers, tiles and schedule from shared memory and the
// arguments; the barriers are described where the kernel initialises them.
template <int DX, bool RW>
__device__ __noinline__ void tc_role_mma(const TcArgs& a, uint8_t* smem, int h_first) {
  using K = PCfg<DX, RW>;
  constexpr int NB = K::NB;
  const int tid = threadIdx.x, lane = tid & 31;
  const Sched sc(a.total, a.G, blockIdx.x, a.nch);
  const int nI = sc.items();
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K::S_BAR);
  uint64_t* rdy = bars + 0;       // [4]: prepare -> G7 (+G1), output -> G2G3, G4, G5G6
  uint64_t* dne = bars + 4;       // [4]: G7 done, G2G3 done, G4 done, G5G6 done
  uint64_t* dneS = bars + 8;      // G1 done
  uint64_t* freeQK = bars + 9;    // [NB]: sQ, sK of that set reusable
  uint64_t* freeVR = bars + 12;   // [NB]: sV, sR_Gamma of that set reusable
  uint64_t* bar_drain = bars + 15;
  uint64_t* rdyKV = bars + 19;    // [NB]: output warps -> G7 of a state-only item (k, v converted)
  uint64_t* rdyW = bars + 25;     // output warps -> G_W (a staged in the X tile)
  uint64_t* dneW = bars + 26;     // G_W done
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + K::S_FLAG);
  const uint32_t sbase = smem_u32(smem);
  auto sQ = [&](int b) { return K::S_Q + b * K::TQ; };
  auto sK = [&](int b) { return K::S_K + b * K::TQ; };
  auto sV = [&](int b) { return K::S_V + b * K::TV; };
  auto sRG = [&](int b) { return K::S_RG + b * K::TRG; };
  const uint32_t tmem = *reinterpret_cast<const uint32_t*>(smem + K::S_TMEMH);
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t pr[4] = {0u, 0u, 0u, 0u}, prW = 0u;
      bool ok = true;
      auto wait_rdy = [&](int i) -> bool {
        const bool r = mbar_wait_or_abort(rdy + i, pr[i], a.err, abort_flag);
        pr[i] ^= 1u;
        tc_fence_after();
        return r;
      };
      auto gemm_d = [&](uint32_t d, uint64_t ad, uint32_t astep, uint64_t bd, uint32_t bstep, uint32_t idesc,
                        int ksteps, bool acc) {
        for (int kk = 0; kk < ksteps; ++kk)
          mma_f16(d, ad + ((kk * astep) >> 4), bd + ((kk * bstep) >> 4), idesc, (kk > 0 || acc) ? 1u : 0u);
      };
      auto g1 = [&](int b) {   // S^T = xi(K) xi(Q)^T, K-major swizzled tiles of DX / 64 boxes
        for (int kk = 0; kk < DX / 16; ++kk)
          mma_f16(tmem + K::T_S, smem_desc_sw128(sbase + sK(b) + K::kstep(kk), 16, K::SW),
                  smem_desc_sw128(sbase + sQ(b) + K::kstep(kk), 16, K::SW), idesc_f16(64, 64, 0, 0),
                  kk > 0 ? 1u : 0u);
      };
      auto g7 = [&](int b) {   // S_hat += E'^T [xi(K) | V]
        gemm_d(tmem + K::T_STATE, smem_desc(sbase + K::S_E, 128, 1024), 256,
               smem_desc_sw128(sbase + sK(b), K::BOX, K::SW), 2 * K::SW, idesc_f16(128, DX, 0, 1), C / 16,
               true);
        gemm_d(tmem + K::T_STATE + DX, smem_desc(sbase + K::S_E, 128, 1024), 256,
               smem_desc_sw128(sbase + sV(b), K::S_ONES - sV(b), K::SW), 2 * K::SW, idesc_f16(128, kVB, 0, 1),
               C / 16, true);
      };
      auto g5g6 = [&](int bb) {
        gemm_d(tmem + K::T_NUM, smem_desc(sbase + K::S_P, 128, 1024), 256,
               smem_desc_sw128(sbase + sV(bb), K::S_ONES - sV(bb), K::SW), 2 * K::SW,
               idesc_f16(64, K::NV, 0, 1), C / 16, false);   // G5: P [V | 1]
        gemm(tmem + K::T_NUM, sbase + K::S_X, 1024, 128, 2048, sbase + sRG(bb), K::RSV, 128, 2 * K::RSV,
             idesc_f16(64, K::NV, 1, 1), KR / 16, true);   // G6: X [R_Gamma | R_eta]
        mma_commit(dne + 3);
        mma_commit(freeVR + bb);
      };
      static_assert(!(RW && K::SHARED_SAP), "G_W is issued by the in-order loop");
      if constexpr (K::SHARED_SAP) {
        // d_xi = 128 (measured on a B200: the 1.3B prefill 11% faster
        // than with the in-order issue below, which is faster at d_xi = 64)
        // Every group is issued as soon as its inputs are ready (the tensor
        // pipe runs groups in issue order), under these orderings, for item i
        // and full item f = i - nA:
        //   G7(i)     after rdy0(i); for a full item, after G2+G3(f-1), whose
        //             G3 reads the R_U buffer the rotation after G7(i) rewrites;
        //   G1(f)     after G7(f) (the prepare warps convert the tiles before
        //             the rotation), after G5+G6(f-1), as S^T shares P's tile,
        //             and after G2+G3(f-1), whose G2 reads the S^T tile that
        //             E1(f) rewrites;
        //   G2G3(f)   after rdy1(f), G7(f) (R_U), G4(f-1) (a~ read by E2(f-1))
        //             and G5+G6(f-1), whose G6 reads the X tile E2(f) rewrites;
        //   G4(f)     after rdy2(f) and G5+G6(f-1), whose G5 reads the P tile
        //             E3(f) rewrites;
        //   G5G6(f)   after rdy3(f).
        // The state chain then waits on the output warps only through E1(f-1).
        const int nA = sc.nA, nF = sc.nF;
        int i7 = 0, f1 = 0, f23 = 0, f4 = 0, f56 = 0;
        uint32_t pKV = 0u;   // bit b: parity of rdyKV[b]
        unsigned long long t_last = global_ns();
        for (unsigned spin = 0; i7 < nI || f56 < nF; ++spin) {
          if (i7 < nI && (i7 < nA || f23 >= i7 - nA) &&
              (i7 >= nA || mbar_probe(rdyKV + i7 % NB, (pKV >> (i7 % NB)) & 1u)) && mbar_probe(rdy + 0, pr[0])) {
            pr[0] ^= 1u;
            const int b = i7 % NB;
            if (i7 < nA) pKV ^= 1u << b;
            tc_fence_after();
            g7(b);
            mma_commit(dne + 0);
            if (i7 < nA) {
              mma_commit(freeQK + b);
              mma_commit(freeVR + b);
            }
            ++i7;
            t_last = global_ns();
            continue;
          }
          if (f56 < f4 && mbar_probe(rdy + 3, pr[3])) {   // E3(f56): P read
            pr[3] ^= 1u;
            tc_fence_after();
            g5g6((nA + f56) % NB);
            ++f56;
            t_last = global_ns();
            continue;
          }
          if (f1 < nF && f23 >= f1 && i7 > nA + f1 && f56 >= f1) {
            g1((nA + f1) % NB);
            mma_commit(dneS);
            ++f1;
            t_last = global_ns();
            continue;
          }
          if (f23 < f1 && i7 > nA + f23 && f4 >= f23 && f56 >= f23 && mbar_probe(rdy + 1, pr[1])) {
            pr[1] ^= 1u;
            tc_fence_after();
            const int i = nA + f23, b = i % NB, p = i & 1;
            gemm(tmem + K::T_A, sbase + K::S_E, 128, 1024, 256, sbase + K::S_S, 1024, 128, 2048,
                 idesc_f16(128, 64, 0, 1), C / 16, false);   // G2
            for (int kk = 0; kk < DX / 16; ++kk)   // G3: A = R_U from tensor memory
              mma_f16_ts(tmem + K::T_A, tmem + K::T_RU + K::RU_COLS * p + 8 * kk,
                         smem_desc_sw128(sbase + sQ(b) + K::kstep(kk), 16, K::SW), idesc_f16(128, 64, 0, 0), 1u);
            mma_commit(dne + 1);
            mma_commit(freeQK + b);
            ++f23;
            t_last = global_ns();
            continue;
          }
          if (f4 < f23 && f56 >= f4 && mbar_probe(rdy + 2, pr[2])) {
            pr[2] ^= 1u;
            tc_fence_after();
            gemm(tmem + K::T_P, sbase + K::S_X, 1024, 128, 2048, sbase + K::S_E, 1024, 128, 2048,
                 idesc_f16(64, 64, 1, 1), KR / 16, false);   // G4: P
            mma_commit(dne + 2);
            ++f4;
            t_last = global_ns();
            continue;
          }
          __nanosleep(32);   // nothing ready: leave the issue slots to the other warps
          if ((spin & 63u) != 63u) continue;
          if (*abort_flag) {
            ok = false;
            break;
          }
          if (global_ns() - t_last > kWaitLimitNs) {
            atomicOr(a.err, kErrTimeout);
            *abort_flag = 1;
            ok = false;
            break;
          }
        }
      } else {
        int t = 0, prev_b = 0;   // full items issued so far; set of the previous full item
        uint32_t pKV = 0u;       // bit b: parity of rdyKV[b]
        for (int i = 0; i < nI; ++i) {
          const int b = i % NB, p = i & 1;
          if (!(ok = wait_rdy(0))) break;
          if (sc.state_only(i)) {
            ok = mbar_wait_or_abort(rdyKV + b, (pKV >> b) & 1u, a.err, abort_flag);   // k, v converted
            pKV ^= 1u << b;
            tc_fence_after();
            if (!ok) break;
            g7(b);
            mma_commit(dne + 0);
            mma_commit(freeQK + b);
            mma_commit(freeVR + b);
            continue;
          }
          if (!K::SHARED_SAP) {
            g1(b);
            mma_commit(dneS);
          }
          g7(b);
          mma_commit(dne + 0);
          if (t > 0) {
            if (!(ok = wait_rdy(3))) break;   // E3 of the previous chunk: P read
            if (K::SHARED_SAP) {
              g1(b);
              mma_commit(dneS);
            }
            g5g6(prev_b);
          } else if (K::SHARED_SAP) {
            g1(b);
            mma_commit(dneS);
          }
          if (!(ok = wait_rdy(1))) break;
          gemm(tmem + K::T_A, sbase + K::S_E, 128, 1024, 256, sbase + K::S_S, 1024, 128, 2048,
               idesc_f16(128, 64, 0, 1), C / 16, false);   // G2
          for (int kk = 0; kk < DX / 16; ++kk)   // G3: A = R_U from tensor memory
            mma_f16_ts(tmem + K::T_A, tmem + K::T_RU + K::RU_COLS * p + 8 * kk,
                       smem_desc_sw128(sbase + sQ(b) + K::kstep(kk), 16, K::SW), idesc_f16(128, 64, 0, 0), 1u);
          mma_commit(dne + 1);
          mma_commit(freeQK + b);
          if constexpr (RW) {   // G_W: a~~ = W' a, over the a~ columns E2 has read
            ok = mbar_wait_or_abort(rdyW, prW, a.err, abort_flag);
            prW ^= 1u;
            tc_fence_after();
            if (!ok) break;
            gemm(tmem + K::T_A, sbase + K::S_W, 128, 2048, 256, sbase + K::S_X, 1024, 128, 2048,
                 idesc_f16(128, 64, 0, 1), KR / 16, false);
            mma_commit(dneW);
          }
          if (!(ok = wait_rdy(2))) break;
          gemm(tmem + K::T_P, sbase + K::S_X, 1024, 128, 2048, sbase + K::S_E, 1024, 128, 2048,
               idesc_f16(64, 64, 1, 1), KR / 16, false);   // G4: P
          mma_commit(dne + 2);
          prev_b = b;
          ++t;
        }
        if (ok && t > 0) {
          if ((ok = wait_rdy(3))) g5g6(prev_b);
        }
      }
      if (!ok) {   // drain every tensor-core group issued so far
        mma_commit(bar_drain);
        mbar_wait(bar_drain, 0u, a.err);
      }
    }
    __syncwarp();
}

template <int DX, bool RW>
__device__ __noinline__ void tc_role_prepare(const TcArgs& a, uint8_t* smem, int h_first) {
  using K = PCfg<DX, RW>;
  constexpr int NB = K::NB;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gw = warp & (GW - 1);          // warp index within its epilogue group
  const int quad = warp & 3, half = gw >> 2;
  const Sched sc(a.total, a.G, blockIdx.x, a.nch);
  const int nI = sc.items();
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K::S_BAR);
  uint64_t* dne = bars + 4;       // [4]: G7 done, G2G3 done, G4 done, G5G6 done
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + K::S_FLAG);
  volatile int* xchg = reinterpret_cast<volatile int*>(smem + K::S_FLAG + 4);   // look-back result
  volatile int* g4_seen = reinterpret_cast<volatile int*>(smem + K::S_FLAG + 8);   // G4 groups seen done
  // stream s = bh * nvb + vb
  auto first_item = [&](Walker& w) { w.seek(sc.nA > 0 ? sc.gA : sc.g0, a.nch, a.nvb, a.H); };
  const uint32_t tmem = *reinterpret_cast<const uint32_t*>(smem + K::S_TMEMH);
    // ------------------------------------------------ prepare warps
    const int k = 32 * quad + lane;
    const int m = k >> 1, comp = k & 1;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * quad) << 16);
    uint32_t pd0 = 0u, pld = 0u, pldv = 0u;   // parities; pld, pldv bit b for buffer set b
    int cur_h = h_first;
    const HeadTables* T = a.tabs + cur_h;
    auto set_head = [&](int h) {
      cur_h = h;
      T = a.tabs + h;
    };
    auto waitA = [&](uint64_t* bar, uint32_t& ph) -> bool {   // uniform over the prepare group
      const bool r = mbar_wait_or_abort(bar, ph, a.err, abort_flag);
      ph ^= 1u;
      tc_fence_after();
      return !named_sync_or(2, GT, !r);
    };
    const PrepThread th{trow, tid, k, m, comp, half};
    float eta_c = 0.f;

    bool ok = true;
    bool single_piece_pending = false;   // publish our inclusive state once the carry is known
    Walker w;
    first_item(w);
    int prev_bh = 0, prev_vb = 0, prev_ch = 0;
    int b = 0;   // buffer set of item i (i % NB)
    // One piece at a time: the state-only chain, then each run of a stream's
    // chunks in the range.  Its start runs after G7 of the item before.
    for (int i = 0; ok && i < nI;) {
      const bool so = sc.state_only(i);
      const int n = so ? sc.nA : min(a.nch - w.ch, nI - i);
      if (i > 0 && !(ok = waitA(dne + 0, pd0))) break;   // G7 of the previous item: the state is current
      const PieceStart ps = prep_piece_start<DX, RW>(a, th, i, sc.nA, sc.gA, sc.nF, so, w.ch, w.bh, w.vb, w.h, prev_bh,
                                                 prev_vb, prev_ch, cur_h, eta_c, single_piece_pending, abort_flag,
                                                 xchg, g4_seen, smem + K::S_E, smem + K::S_W);
      if (!(ok = ps.ok)) break;
      eta_c = ps.eta;
      single_piece_pending = ps.pending;
      if (w.h != cur_h) set_head(w.h);
      const int last_nv = min(C, a.N - (w.ch + n - 1) * C);
      const float esum_tail = last_nv < C ? ragged_esum(T, m, comp, last_nv) : 0.f;
      const PrepRun run = prep_chunks<DX, RW>(a, smem, th, T, i, n, b, so, w.bh, w.ch, eta_c, pd0, pld, pldv, esum_tail);
      eta_c = run.eta;
      pd0 = run.pd0;
      pld = run.pld;
      pldv = run.pldv;
      if (!(ok = run.ok)) break;
      prev_bh = w.bh;
      prev_vb = w.vb;
      prev_ch = w.ch + n - 1;
      i += n;
      b = (b + n) % NB;
      if (i < nI) w.seek(i < sc.nA ? sc.gA + i : sc.g0 + (i - sc.nA), a.nch, a.nvb, a.H);
    }
    if (ok && nI > 0 && a.state_out && sc.g1 % a.nch == 0) {
      ok = waitA(dne + 0, pd0);   // G7 of the last chunk
      if (ok) prep_write_state_out<DX, RW>(a, T, th, prev_bh, prev_vb, prev_ch, eta_c);
    }
}

template <int DX, bool RW>
__device__ __noinline__ void tc_role_output(const TcArgs& a, uint8_t* smem, int h_first,
                                          const CUtensorMap& tm_o) {
  using K = PCfg<DX, RW>;
  constexpr int NB = K::NB;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gw = warp & (GW - 1);          // warp index within its epilogue group
  const int quad = warp & 3, half = gw >> 2;
  const Sched sc(a.total, a.G, blockIdx.x, a.nch);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K::S_BAR);
  uint64_t* rdy = bars + 0;       // [4]: prepare -> G7 (+G1), output -> G2G3, G4, G5G6
  uint64_t* dne = bars + 4;       // [4]: G7 done, G2G3 done, G4 done, G5G6 done
  uint64_t* dneS = bars + 8;      // G1 done
  uint64_t* loadedQK = bars + 16;   // [NB]: that set's q, k rows have landed
  uint64_t* loadedV = bars + 22;    // [NB]: that set's v rows have landed
  uint64_t* rdyKV = bars + 19;    // [NB]: output warps -> G7 of a state-only item (k, v converted)
  uint64_t* rdyW = bars + 25;     // output warps -> G_W (a staged in the X tile)
  uint64_t* dneW = bars + 26;     // G_W done
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + K::S_FLAG);
  volatile int* g4_seen = reinterpret_cast<volatile int*>(smem + K::S_FLAG + 8);   // G4 groups seen done
  const uint32_t sbase = smem_u32(smem);
  auto sK = [&](int b) { return K::S_K + b * K::TQ; };
  auto sV = [&](int b) { return K::S_V + b * K::TV; };
  const uint32_t tmem = *reinterpret_cast<const uint32_t*>(smem + K::S_TMEMH);
    // ------------------------------------------------ output warps
    const int k = 32 * quad + lane;
    const int m = k >> 1;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * quad) << 16);
    const int i0 = 32 * half;     // this thread's 32 columns of the 64-wide tiles
    uint32_t pd[4] = {0u, 0u, 0u, 0u}, pS = 0u, pW = 0u;
    int cur_h = -1;
    float r2 = 0.f, s_start = 0.f;
    float2 p_start = make_float2(0.f, 0.f), lam_m = make_float2(0.f, 0.f);   // RW: lambda_m^(i0 - c), lambda_m
    auto waitB = [&](uint64_t* bar, uint32_t& ph) -> bool {
      const bool r = mbar_wait_or_abort(bar, ph, a.err, abort_flag);
      ph ^= 1u;
      tc_fence_after();
      return !named_sync_or(3, GT, !r);
    };
    auto signalB = [&](int i) {
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(rdy + i);
    };
    // The M = 64 accumulators (S^T, P, num) fill lanes 0-15 of each quadrant:
    // thread t takes row 16 * quad + t % 16 and columns c0 .. c0 + 15 of the
    // warp's 32, the two half-warps splitting them.
    const int r16 = 16 * quad + (lane & 15);
    const int c0 = i0 + 16 * (lane >> 4);
    auto e3 = [&]() {   // masked P -> [i][j]
      uint32_t r[16];
      tmem_ld16_halves<16>(trow + K::T_P + i0, r);
      tmem_ld_wait16(r);
#pragma unroll
      for (int e = 0; e < 16; ++e)
        if (c0 + e > r16) r[e] = 0u;
      *reinterpret_cast<uint4*>(smem + K::S_P + tile_off(r16, c0, 1024)) = pack8f(r, 1.f);
      *reinterpret_cast<uint4*>(smem + K::S_P + tile_off(r16, c0 + 8, 1024)) = pack8f(r + 8, 1.f);
      signalB(3);
    };
    // o = num / den, staged as two boxes of 64 rows x 128 bytes (columns 0-31
    // and 32-63 of the value block) in the 128-byte swizzled layout, which
    // keeps the row-per-lane writes free of bank conflicts, then written by
    // one TMA store per box.  Rows past the sequence lie outside the tensor
    // map and are not written.  Staging alternates between two buffers.
    // Before the barrier that precedes each store, the issuing thread waits
    // until the store before it has finished reading its buffer; every thread
    // passes that barrier before it writes that buffer again one chunk later.
    auto e4 = [&](long long bh, int vb, int ch, int nv, int t) {
      const int i = r16, hb = lane >> 4;
      uint32_t rd, rr[16];
      tmem_ld1(trow + K::T_DEN, rd);   // one column of all 32 lanes: rows in lanes 0-15
      tmem_ld16_halves<16>(trow + K::T_NUM + i0, rr);
      tmem_ld_wait1(rd);
      tmem_ld_wait16(rr);
      const float dn = __shfl_sync(kFull, __uint_as_float(rd), lane & 15);
      const float rdn = 1.0f / dn;
      const uint64_t rdn2 = f2_pack(rdn, rdn);
      const long long row = bh * a.N + ch * C + i;
      const uint32_t stage = K::S_O + (t & 1) * K::TO;
      if (i < nv && a.den && half == 0 && hb == 0 && vb == 0) a.den[row] = dn;
      uint8_t* box = smem + stage + half * (K::TO / 2) + i * 128;
#pragma unroll
      for (int gg = 0; gg < 4; ++gg) {
        const uint32_t* r = rr + 4 * gg;
        float4 q;
        f2_unpack(f2_mul(f2_pack(__uint_as_float(r[0]), __uint_as_float(r[1])), rdn2), q.x, q.y);
        f2_unpack(f2_mul(f2_pack(__uint_as_float(r[2]), __uint_as_float(r[3])), rdn2), q.z, q.w);
        *reinterpret_cast<float4*>(box + (((4 * hb + gg) ^ (i & 7)) << 4)) = q;
      }
      if (i < nv && a.num) {
        float4* np = reinterpret_cast<float4*>(a.num + row * a.DV + vb * kVB + c0);
#pragma unroll
        for (int gg = 0; gg < 4; ++gg)
          np[gg] = make_float4(__uint_as_float(rr[4 * gg]), __uint_as_float(rr[4 * gg + 1]),
                               __uint_as_float(rr[4 * gg + 2]), __uint_as_float(rr[4 * gg + 3]));
      }
      fence_async_smem();
      if (tid == GT) bulk_wait_read_0();
      named_sync(1, GT);
      if (tid == GT) {
        tma_store_3d(&tm_o, sbase + stage, vb * kVB, ch * C, static_cast<int>(bh));
        tma_store_3d(&tm_o, sbase + stage + K::TO / 2, vb * kVB + 32, ch * C, static_cast<int>(bh));
        bulk_commit();
      }
    };
    bool ok = true;
    {
      // The state-only chain of the range's last piece (items 0 .. nA-1)
      // runs before any full chunk, when these warps have no readout to do:
      // they convert its k and v tiles, so that the prepare warps only rotate
      // and the chain is the rotation and G7 alone.
      Walker wa;
      wa.seek(sc.gA, a.nch, a.nvb, a.H);
      for (int i = 0; ok && i < sc.nA; ++i, wa.step(a.nch, a.nvb, a.H)) {
        const int b = i % NB;
        const uint32_t par = static_cast<uint32_t>((i / NB) & 1);
        const int nv = min(C, a.N - wa.ch * C);
        bool r = mbar_wait_or_abort(loadedQK + b, par, a.err, abort_flag);
        if (named_sync_or(3, GT, !r)) {
          ok = false;
          break;
        }
        convert_tile<true, K::TQ / 16, GT>(smem + sK(b), nv, tid - GT, a.kv_ready);
        r = mbar_wait_or_abort(loadedV + b, par, a.err, abort_flag);
        if (named_sync_or(3, GT, !r)) {
          ok = false;
          break;
        }
        convert_tile<false, K::TV / 16, GT>(smem + sV(b), nv, tid - GT, a.kv_ready);
        fence_async_smem();
        mbar_arrive(rdyKV + b);
      }
    }
    bool have_prev = false;
    int prev_bh = 0, prev_vb = 0, prev_ch = 0, prev_nv = C, t = 0;
    Walker w;
    w.seek(sc.g0, a.nch, a.nvb, a.H);
    // E2(t) comes before E4(t-1) so that G4(t) can start while E4 runs;
    // t == nF runs only the tail (E3, E4) of the last chunk
    for (t = 0; ok && t <= sc.nF && sc.nF > 0; ++t) {
      const bool head = t < sc.nF;
      const int nv = head ? min(C, a.N - w.ch * C) : 0;
      if (have_prev) {
        if (!(ok = waitB(dne + 2, pd[2]))) break;   // G4(t-1)
        if (tid == GT) {
          __threadfence_block();
          *g4_seen = t;
        }
        e3();
      }
      if (head) {
        const int h = w.h;
        if (h != cur_h) {
          cur_h = h;
          r2 = a.tabs[h].r2[m];
          s_start = static_cast<float>(exp(2.0 * a.tabs[h].re_dA[m] * (32.0 * half - C / 2)));
          if constexpr (RW) {
            const double n = 32.0 * half - C / 2;
            const double mag = exp(n * a.tabs[h].re_dA[m]);
            double sn, cs;
            sincos(fmod(n * a.tabs[h].im_dA[m], 6.283185307179586476925), &sn, &cs);
            p_start = make_float2(static_cast<float>(mag * cs), static_cast<float>(mag * sn));
            lam_m = a.tabs[h].lam[m];
          }
        }
        if (!(ok = waitB(dneS, pS))) break;   // G1(t)
        {  // E1(t): masked S^T -> [j][i]
          const int j = r16;
          const bool keep = j < nv;
          uint32_t r[16];
          tmem_ld16_halves<16>(trow + K::T_S + i0, r);
          tmem_ld_wait16(r);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (!(keep && c0 + e >= j)) r[e] = 0u;
          *reinterpret_cast<uint4*>(smem + K::S_S + tile_off(j, c0, 1024)) = pack8f(r, 1.f);
          *reinterpret_cast<uint4*>(smem + K::S_S + tile_off(j, c0 + 8, 1024)) = pack8f(r + 8, 1.f);
          signalB(1);
        }
        if (!(ok = waitB(dne + 1, pd[1]))) break;   // G2 + G3(t)
        if constexpr (RW) {
          // E2a(t): a = lambda^(i-c) a~ into the X tile (G_W's B operand);
          // each complex product takes the other part from the partner lane
          // (rows 2m and 2m+1 sit in adjacent lanes)
          const float sg = (k & 1) ? 1.f : -1.f;
          float2 pw = p_start;
#pragma unroll 1
          for (int bb = 0; bb < 2; ++bb) {
            uint32_t r[16];
            tmem_ld16(trow + K::T_A + i0 + 16 * bb, r);
            tmem_ld_wait16(r);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float x = __uint_as_float(r[e]);
              const float y = __shfl_xor_sync(kFull, x, 1);
              r[e] = __float_as_uint(fmaf(pw.x, x, sg * pw.y * y));
              pw = make_float2(fmaf(pw.x, lam_m.x, -pw.y * lam_m.y), fmaf(pw.x, lam_m.y, pw.y * lam_m.x));
            }
            *reinterpret_cast<uint4*>(smem + K::S_X + tile_off(k, i0 + 16 * bb, 1024)) = pack8f(r, 1.f);
            *reinterpret_cast<uint4*>(smem + K::S_X + tile_off(k, i0 + 16 * bb + 8, 1024)) = pack8f(r + 8, 1.f);
          }
          fence_async_smem();
          tc_fence_before();
          mbar_arrive(rdyW);
          if (!(ok = waitB(dneW, pW))) break;   // G_W(t): a~~ = W' a in the a~ columns
          // E2b(t): X = conj(lambda^(i-c)) a~~
          pw = p_start;
#pragma unroll 1
          for (int bb = 0; bb < 2; ++bb) {
            uint32_t r[16];
            tmem_ld16(trow + K::T_A + i0 + 16 * bb, r);
            tmem_ld_wait16(r);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float x = __uint_as_float(r[e]);
              const float y = __shfl_xor_sync(kFull, x, 1);
              r[e] = __float_as_uint(fmaf(pw.x, x, -sg * pw.y * y));
              pw = make_float2(fmaf(pw.x, lam_m.x, -pw.y * lam_m.y), fmaf(pw.x, lam_m.y, pw.y * lam_m.x));
            }
            *reinterpret_cast<uint4*>(smem + K::S_X + tile_off(k, i0 + 16 * bb, 1024)) = pack8f(r, 1.f);
            *reinterpret_cast<uint4*>(smem + K::S_X + tile_off(k, i0 + 16 * bb + 8, 1024)) = pack8f(r + 8, 1.f);
          }
          signalB(2);
        } else {  // E2(t): X = |lambda|^(2(i-c)) a~
          uint64_t s2 = f2_pack(s_start, s_start * r2);   // scales of two adjacent columns
          const uint64_t r4 = f2_pack(r2 * r2, r2 * r2);
#pragma unroll
          for (int bb = 0; bb < 2; ++bb) {
            uint32_t r[16];
            tmem_ld16(trow + K::T_A + i0 + 16 * bb, r);
            tmem_ld_wait16(r);
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              float x0, x1;
              f2_unpack(f2_mul(f2_pack(__uint_as_float(r[e]), __uint_as_float(r[e + 1])), s2), x0, x1);
              r[e] = __float_as_uint(x0);
              r[e + 1] = __float_as_uint(x1);
              s2 = f2_mul(s2, r4);
            }
            *reinterpret_cast<uint4*>(smem + K::S_X + tile_off(k, i0 + 16 * bb, 1024)) = pack8f(r, 1.f);
            *reinterpret_cast<uint4*>(smem + K::S_X + tile_off(k, i0 + 16 * bb + 8, 1024)) = pack8f(r + 8, 1.f);
          }
          signalB(2);
        }
      }
      if (have_prev) {
        if (!(ok = waitB(dne + 3, pd[3]))) break;   // G5 + G6(t-1)
        e4(prev_bh, prev_vb, prev_ch, prev_nv, t - 1);
      }
      have_prev = head;
      prev_bh = w.bh;
      prev_vb = w.vb;
      prev_ch = w.ch;
      prev_nv = nv;
      if (head) w.step(a.nch, a.nvb, a.H);
    }
    if (tid == GT) bulk_wait_all();   // o is in global memory before the block exits
}

template <int DX, bool RW>
__device__ __noinline__ void tc_role_fetch(const TcArgs& a, uint8_t* smem, int h_first, const CUtensorMap& tm_q,
                                         const CUtensorMap& tm_k, const CUtensorMap& tm_v) {
  using K = PCfg<DX, RW>;
  constexpr int NB = K::NB;
  const int tid = threadIdx.x, lane = tid & 31;
  const Sched sc(a.total, a.G, blockIdx.x, a.nch);
  const int nI = sc.items();
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K::S_BAR);
  uint64_t* freeQK = bars + 9;    // [NB]: sQ, sK of that set reusable
  uint64_t* freeVR = bars + 12;   // [NB]: sV, sR_Gamma of that set reusable
  uint64_t* loadedQK = bars + 16;   // [NB]: that set's q, k rows have landed
  uint64_t* loadedV = bars + 22;    // [NB]: that set's v rows have landed
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + K::S_FLAG);
  const uint32_t sbase = smem_u32(smem);
  auto sQ = [&](int b) { return K::S_Q + b * K::TQ; };
  auto sK = [&](int b) { return K::S_K + b * K::TQ; };
  auto sV = [&](int b) { return K::S_V + b * K::TV; };
  // stream s = bh * nvb + vb
  auto first_item = [&](Walker& w) { w.seek(sc.nA > 0 ? sc.gA : sc.g0, a.nch, a.nvb, a.H); };
    // ------------------------------------------------ fetch warp
    if (lane == 0) {
      int issued_qk = 0, issued_v = 0;
      Walker w;
      first_item(w);
      // q, k of an item go as soon as the contractions reading that set's q,
      // k are done (G2+G3 of the item that last held it); v waits for G5+G6
      for (int i = 0, b = 0; i < nI; ++i, w.next(sc, i - 1, a.nch, a.nvb, a.H), b = b + 1 == NB ? 0 : b + 1) {
        const bool so = sc.state_only(i);
        const uint32_t par = static_cast<uint32_t>((i / NB - 1) & 1);   // release phase of the set's last item
        const int y = w.ch * C, z = w.bh;
        if (i >= NB && !mbar_wait_or_abort(freeQK + b, par, a.err, abort_flag)) break;
        mbar_arrive_expect_tx(loadedQK + b, (so ? 1 : 2) * K::TQ);
        for (int x = 0; x < DX / 64; ++x) {
          if (!so) tma_load_3d(sbase + sQ(b) + x * K::BOX, &tm_q, 64 * x, y, z, loadedQK + b);
          tma_load_3d(sbase + sK(b) + x * K::BOX, &tm_k, 64 * x, y, z, loadedQK + b);
        }
        issued_qk = i + 1;
        if (i >= NB && !mbar_wait_or_abort(freeVR + b, par, a.err, abort_flag)) break;
        mbar_arrive_expect_tx(loadedV + b, K::TV);
        tma_load_3d(sbase + sV(b), &tm_v, w.vb * kVB, y, z, loadedV + b);
        issued_v = i + 1;
      }
      // no copy of ours lands after the block exits: the last load into each
      // set b was item i_b, the phase (i_b / NB) of its barrier
      for (int b = 0; b < NB; ++b) {
        if (b < issued_qk) {
          const int i_b = b + (issued_qk - 1 - b) / NB * NB;
          mbar_wait(loadedQK + b, static_cast<uint32_t>((i_b / NB) & 1), a.err);
        }
        if (b < issued_v) {
          const int i_b = b + (issued_v - 1 - b) / NB * NB;
          mbar_wait(loadedV + b, static_cast<uint32_t>((i_b / NB) & 1), a.err);
        }
      }
    }
    __syncwarp();
}


// 576 threads: one SM sub-partition carries five of the 18 warps, so its
// 16 K registers cap a thread at 96.
template <int DX, bool RW>
__global__ void __launch_bounds__(NTH, 1)
    tc_prefill_kernel(const __grid_constant__ TcArgs a, const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_o) {
  using K = PCfg<DX, RW>;
  constexpr int NB = K::NB;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5;
  const int role = warp < 2 * GW ? warp / GW : warp - 2 * GW + 2;   // prepare, output, mma, fetch
  const Sched sc(a.total, a.G, blockIdx.x, a.nch);
  const int nI = sc.items();

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K::S_BAR);
  uint64_t* rdy = bars + 0;       // [4]: prepare -> G7 (+G1), output -> G2G3, G4, G5G6
  uint64_t* dne = bars + 4;       // [4]: G7 done, G2G3 done, G4 done, G5G6 done
  uint64_t* dneS = bars + 8;      // G1 done
  uint64_t* freeQK = bars + 9;    // [NB]: sQ, sK of that set reusable
  uint64_t* freeVR = bars + 12;   // [NB]: sV, sR_Gamma of that set reusable
  uint64_t* bar_drain = bars + 15;
  uint64_t* loadedQK = bars + 16;   // [NB]: that set's q, k rows have landed
  uint64_t* loadedV = bars + 22;    // [NB]: that set's v rows have landed
  // [NB]: output warps -> G7 of a state-only item, that set's k and v are
  // fp16 operands.  A set is refilled only after that G7, so no barrier runs
  // a phase ahead of the MMA warp's wait.
  uint64_t* rdyKV = bars + 19;
  uint64_t* rdyW = bars + 25;     // output warps -> G_W (the readout's input a staged), RW only
  uint64_t* dneW = bars + 26;     // G_W done
  static_assert(NB <= 3 && 27 * 8 <= K::S_FLAG - K::S_BAR, "the mbarriers fit their slot");
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + K::S_FLAG);
  volatile int* xchg = reinterpret_cast<volatile int*>(smem + K::S_FLAG + 4);   // look-back result
  // G4 groups known done: the output warps see each G4 complete, in order,
  // before E3 of its chunk, and count them here for the prepare warps
  volatile int* g4_seen = reinterpret_cast<volatile int*>(smem + K::S_FLAG + 8);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + K::S_TMEMH);
  const uint32_t sbase = smem_u32(smem);
  auto sQ = [&](int b) { return K::S_Q + b * K::TQ; };
  auto sK = [&](int b) { return K::S_K + b * K::TQ; };
  auto sV = [&](int b) { return K::S_V + b * K::TV; };
  auto sRG = [&](int b) { return K::S_RG + b * K::TRG; };
  // stream s = bh * nvb + vb
  auto first_item = [&](Walker& w) { w.seek(sc.nA > 0 ? sc.gA : sc.g0, a.nch, a.nvb, a.H); };

  if (warp == 0) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(rdy + i, i == 0 ? GT : GT);
      mbar_init(dne + i, 1);
    }
    mbar_init(dneS, 1);
    for (int i = 0; i < NB; ++i) {
      mbar_init(freeQK + i, 1);
      mbar_init(freeVR + i, 1);
      mbar_init(loadedQK + i, 1);
      mbar_init(loadedV + i, 1);
    }
    mbar_init(bar_drain, 1);
    for (int i = 0; i < NB; ++i) mbar_init(rdyKV + i, GT);
    mbar_init(rdyW, GT);
    mbar_init(dneW, 1);
    *abort_flag = 0;
    *g4_seen = 0;
    fence_barrier_init();
  }
  {
    // the ones block after V: MN element 64 (first of the second 64-block)
    // is 1 in every row, the rest 0, in the swizzled layout
    for (int i = tid; i < C * 8; i += NTH) {
      const int r = i >> 3, c = i & 7;
      *reinterpret_cast<uint4*>(smem + K::S_ONES + r * 128 + c * 16) =
          make_uint4((c == (r & 7)) ? 0x00003C00u : 0u, 0u, 0u, 0u);
    }
    // R_Gamma's extra columns start at zero (column 64 receives R_eta every chunk)
    for (int r = tid; r < KR; r += NTH) {
      for (int b = 0; b < NB; ++b) {
        *reinterpret_cast<uint4*>(smem + sRG(b) + tile_off(r, kVB, K::RSV)) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(smem + sRG(b) + tile_off(r, kVB + 8, K::RSV)) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    // Everything above touches only this CTA's own resources.  The kernel may
    // have been launched while the table kernel before it still runs: every
    // global read (tables, inputs, look-back flags, which the table kernel
    // clears) comes after this wait, and nothing global is written before it.
    griddep_wait();
  }
  // The E' table depends on the head; a CTA may span heads, so it is copied
  // per piece by the prepare warps (see load_table) -- except that the first
  // item's head is loaded here by everyone.
  int h_first = 0;
  {
    Walker w;
    first_item(w);
    h_first = w.h;
  }
  {
    const uint4* src = reinterpret_cast<const uint4*>(a.tabs[h_first].E);
    uint4* dst = reinterpret_cast<uint4*>(smem + K::S_E);
    for (int i = tid; i < KR * C * 2 / 16; i += NTH) dst[i] = src[i];
    if constexpr (RW) {
      const uint4* ws = reinterpret_cast<const uint4*>(a.Wt) + static_cast<size_t>(h_first) * (kWprimeBytes / 16);
      uint4* wd = reinterpret_cast<uint4*>(smem + K::S_W);
      for (int i = tid; i < static_cast<int>(kWprimeBytes / 16); i += NTH) wd[i] = ws[i];
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (role == 2) tc_role_mma<DX, RW>(a, smem, h_first);
  else if (role == 0) tc_role_prepare<DX, RW>(a, smem, h_first);
  else if (role == 1) tc_role_output<DX, RW>(a, smem, h_first, tm_o);
  else tc_role_fetch<DX, RW>(a, smem, h_first, tm_q, tm_k, tm_v);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// Chunks a CTA carries under grid G: the largest range, plus the state-only
// chain of a last piece that ends inside a stream, plus the hops of the
// look-back.  A state-only chunk costs nearly as much as a full one (on a
// B200, 96 whole 32-chunk streams of d = 64 take 115 us, the same work as 144
// ranges with their state-only chains 155 us): the chain of conversion,
// rotation and G7 that it runs is the latency-bound part of a full chunk.
double plan_cost(long long total, int nch, int G) {
  constexpr double kStateOnly = 0.9, kHop = 0.5;
  double worst = 0.0;
  for (int c = 0; c < G; ++c) {
    const long long g0 = total * c / G, g1 = total * (c + 1) / G;
    double t = static_cast<double>(g1 - g0);
    if (g1 % nch != 0) t += kStateOnly * static_cast<double>(g1 - std::max(g0, (g1 - 1) / nch * nch));
    if (g0 % nch != 0) {   // hops back to the stream's first piece, roughly
      const long long start = g0 / nch * nch;
      t += kHop * std::ceil(static_cast<double>(g0 - start) * G / static_cast<double>(total));
    }
    worst = std::max(worst, t);
  }
  return worst;
}

template <int DX, bool RW>
cudaError_t launch_impl(const TcArgs& args, const void* q, const void* k, const void* v, int DV,
                        cudaStream_t st) {
  using K = PCfg<DX, RW>;
  CUtensorMap tm_q, tm_k, tm_v, tm_o;
  const bool f16 = args.kv_ready != 0;
  if (!encode_input_map(&tm_q, q, args.BH, args.N, DX) || !encode_input_map(&tm_k, k, args.BH, args.N, DX, f16) ||
      !encode_input_map(&tm_v, v, args.BH, args.N, DV, f16) ||
      !encode_rows64_f32_map(&tm_o, args.o, args.BH, args.N, DV))
    return cudaErrorNotSupported;
  auto kern = tc_prefill_kernel<DX, RW>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, K::SMEM);
  if (e != cudaSuccess) return e;
  // Programmatic dependent launch: the CTAs set up barriers, TMEM and
  // constant tiles while the table kernel finishes (see griddep_wait).
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(args.G));
  cfg.blockDim = dim3(NTH);
  cfg.dynamicSmemBytes = K::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, args, tm_q, tm_k, tm_v, tm_o);
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
  const long long nch = (s.N + C - 1) / C;
  const long long streams = static_cast<long long>(s.B) * s.H * (s.d_v / kVB);
  const long long total = streams * nch;
  // Forced grid (tuning and tests): IA_PREFILL_GRID=n.
  if (const char* env = std::getenv("IA_PREFILL_GRID")) {
    const long long n = std::atoll(env);
    if (n >= 1) return TcPlan{static_cast<int>(std::min<long long>({n, total, static_cast<long long>(num_sms)}))};
  }
  // The search below is O(num_sms^2); remember the last few answers.
  struct Entry {
    long long total, nch;
    int num_sms, grid;
  };
  static thread_local Entry cache[4] = {};
  static thread_local int next = 0;
  for (const Entry& e : cache)
    if (e.grid > 0 && e.total == total && e.nch == nch && e.num_sms == num_sms) return TcPlan{e.grid};
  const int gmax = static_cast<int>(std::min<long long>(num_sms, (total + kMinPiece - 1) / kMinPiece));
  // the largest grid first, so that ties keep every SM busy
  TcPlan best{std::max(1, gmax)};
  double best_t = plan_cost(total, static_cast<int>(nch), best.grid);
  for (int G = gmax - 1; G >= 1; --G) {
    const double t = plan_cost(total, static_cast<int>(nch), G);
    if (t < best_t - 1e-9) {
      best_t = t;
      best.grid = G;
    }
  }
  cache[next] = Entry{total, nch, num_sms, best.grid};
  next = (next + 1) % 4;
  return best;
}

bool tc_plan_splits(const ia_shape_t& s, const TcPlan& p) {
  const long long nch = (s.N + C - 1) / C;
  const long long total = static_cast<long long>(s.B) * s.H * (s.d_v / kVB) * nch;
  for (int c = 1; c < p.grid; ++c)
    if ((total * c / p.grid) % nch != 0) return true;
  return false;
}

size_t tc_workspace_bytes(const ia_shape_t& s, const TcPlan& p) {
  size_t bytes = sizeof(HeadTables) * static_cast<size_t>(s.H);
  if (tc_plan_splits(s, p)) {
    const size_t F = static_cast<size_t>(s.d_xi) + kVB;
    bytes += 2 * static_cast<size_t>(p.grid) * (KR * F + KR) * sizeof(float);   // agg, incl
    bytes += static_cast<size_t>(p.grid) * sizeof(int) + 256;                    // flags
  }
  return bytes + 256;
}

HeadTables* tc_tables(void* ws) {
  return reinterpret_cast<HeadTables*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~static_cast<uintptr_t>(255));
}

cudaError_t launch_tc_prefill(const ia_shape_t& s, const TcPlan& p, const void* q, const void* k,
                              const void* v, const float* delta, const float* A,
                              const void* state_in, float* o, float* num, float* den,
                              void* state_out, void* ws, cudaStream_t st, void* dump_R,
                              float* dump_Re, float* dtab, bool kv_ready, const void* Wt) {
  uint8_t* w = reinterpret_cast<uint8_t*>(tc_tables(ws));
  HeadTables* tabs = reinterpret_cast<HeadTables*>(w);
  TcArgs args;
  args.agg = args.incl = nullptr;
  args.flags = nullptr;
  args.kv_ready = kv_ready ? 1 : 0;
  args.Wt = static_cast<const __half*>(Wt);
  const size_t F = static_cast<size_t>(s.d_xi) + kVB;
  if (tc_plan_splits(s, p)) {
    float* agg = reinterpret_cast<float*>(w + sizeof(HeadTables) * s.H);
    args.agg = agg;
    args.incl = agg + static_cast<size_t>(p.grid) * (KR * F + KR);
    uint8_t* fl = reinterpret_cast<uint8_t*>(args.incl + static_cast<size_t>(p.grid) * (KR * F + KR));
    args.flags = reinterpret_cast<int*>((reinterpret_cast<uintptr_t>(fl) + 255) & ~static_cast<uintptr_t>(255));
  }
  // the chunk pass starts under the table kernel, so its timing mark goes
  // before the table kernel
  mark_launch_begin(st);
  cudaError_t e = launch_param_tables(s.H, delta, s.delta_per_mode, A, tabs, st, dtab, args.flags,
                                      args.flags ? p.grid : 0);
  if (e != cudaSuccess) return e;
  args.tabs = tabs;
  args.state_in = static_cast<const float2*>(state_in);
  args.o = o;
  args.num = num;
  args.den = den;
  args.state_out = static_cast<float2*>(state_out);
  args.err = device_error_ptr();
  args.dump_R = static_cast<uint8_t*>(dump_R);
  args.dump_Re = dump_Re;
  if (!args.err) return cudaErrorInvalidSymbol;
  args.H = s.H;
  args.N = s.N;
  args.DV = s.d_v;
  args.nch = (s.N + C - 1) / C;
  args.nvb = s.d_v / kVB;
  args.G = p.grid;
  args.BH = static_cast<long long>(s.B) * s.H;
  args.total = args.BH * args.nvb * args.nch;
  if (Wt) {   // the readout matrix: d_xi = 64, no saved states
    if (s.d_xi != 64 || dump_R) return cudaErrorInvalidValue;
    return launch_impl<64, true>(args, q, k, v, s.d_v, st);
  }
  if (s.d_xi == 64) return launch_impl<64, false>(args, q, k, v, s.d_v, st);
  if (s.d_xi == 128) return launch_impl<128, false>(args, q, k, v, s.d_v, st);
  return cudaErrorInvalidValue;
}

}  // namespace ia
