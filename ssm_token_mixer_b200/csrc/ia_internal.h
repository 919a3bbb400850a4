// Internal launch interface between the C-ABI layer (ia_api.cu) and the
// kernel translation units.  Not part of the public header.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/ia.h"

namespace ia {

struct HeadTables;

// Per-head tables of the tensor-core path (and, with dtab, the Delta
// derivative table of the reverse pass); also clears nflags look-back flags
// of the chunk pass that follows.
cudaError_t launch_param_tables(int H, const float* delta, int dpm, const float* A, HeadTables* tabs,
                                cudaStream_t st, float* dtab = nullptr, int* flags = nullptr,
                                int nflags = 0);
// Floats of the three derivative tables of the reverse pass plus their row sums.
inline size_t dtab_floats(int H) { return 3 * static_cast<size_t>(H) * 128 * (64 + 1); }

// Reverse passes leave per-(b,h,m) partials of dL/dDelta_hm, dL/dRe A_m and
// dL/dIm A_m ([B,H,M][3] fp32); this reduces them in a fixed order into
// dDelta ([H] or [H,M]) and, if dA is not null, dA ([M] complex).
size_t grad_partials_bytes(const ia_shape_t& s);
cudaError_t launch_grad_reduce(const ia_shape_t& s, const float* gpart, float* dDelta, float* dA,
                               cudaStream_t st);

size_t seq_fwd_smem(int DX, int DV, int M);
cudaError_t launch_seq_fwd(const ia_shape_t& s, const void* q, const void* k, const void* v,
                           const float* delta, const float* A, const void* state_in, float* o,
                           float* num, float* den, void* state_out, cudaStream_t st);

size_t seq_bwd_smem(int DX, int DV, int M);
size_t seq_bwd_ws_per_bh(int N, int DX, int DV, int M);   // in float2 units
size_t seq_bwd_workspace_bytes(const ia_shape_t& s);
cudaError_t launch_seq_bwd(const ia_shape_t& s, const void* q, const void* k, const void* v,
                           const float* delta, const float* A, const void* dO, float* o, float* dq,
                           float* dk, float* dv, float* dDelta, float* dA, void* ws, cudaStream_t st);

// Tensor-core chunked prefill (bf16 inputs, M = 64).
bool tc_prefill_supported(const ia_shape_t& s);
struct TcPlan {
  int grid;   // CTAs of the chunk pass, each an equal range of the (stream, chunk) space
};
TcPlan tc_plan(const ia_shape_t& s, int num_sms);
// One CTA per stream (whole value-block sequences, no look-back): the plan
// of the no-allocation entry point.
inline TcPlan tc_plan_whole_streams(const ia_shape_t& s) {
  return TcPlan{static_cast<int>(static_cast<long long>(s.B) * s.H * (s.d_v / 64))};
}
// True if some CTA range of the plan starts inside a stream (the pass then
// needs the look-back buffers of the workspace).
bool tc_plan_splits(const ia_shape_t& s, const TcPlan& p);
size_t tc_workspace_bytes(const ia_shape_t& s, const TcPlan& p);
cudaError_t launch_tc_prefill(const ia_shape_t& s, const TcPlan& p, const void* q, const void* k,
                              const void* v, const float* delta, const float* A,
                              const void* state_in, float* o, float* num, float* den,
                              void* state_out, void* ws, cudaStream_t st,
                              void* dump_R = nullptr, float* dump_Re = nullptr,
                              float* dtab = nullptr, bool kv_ready = false, const void* Wt = nullptr);
// Byte offset of the per-head tables inside a tensor-core workspace (256-aligned start).
HeadTables* tc_tables(void* ws);

// TMA tensor maps (ia_prefill_tc.cu): an fp32 [BH][N][W] array as
// 32-column x 64-row boxes, 128-byte swizzled; q/k/v bf16 [BH][N][W] as
// 64 x 64 boxes, 128-byte swizzled.  False if the driver refuses the map.
bool encode_rows64_f32_map(CUtensorMap* m, float* x, long long BH, int N, int W);
bool encode_input_map(CUtensorMap* m, const void* x, long long BH, int N, int W, bool fp16 = false);

// Tensor-core training step (bf16, M = 64, d_xi = d_v = 64).
bool tc_bwd_supported(const ia_shape_t& s);
size_t tc_fwd_bwd_workspace_bytes(const ia_shape_t& s, const TcPlan& p);
cudaError_t launch_tc_fwd_bwd(const ia_shape_t& s, const TcPlan& p, const void* q, const void* k,
                              const void* v, const float* delta, const float* A, const void* dO,
                              float* o, float* dq, float* dk, float* dv, float* dDelta, float* dA,
                              void* ws, cudaStream_t st);

// Decode step.
// out = lambda^L carry_in + local over a whole state (ia_carry.cu).
cudaError_t launch_state_carry(const ia_shape_t& s, const float* delta, const float* A, long long L,
                               const void* carry_in, const void* local, void* out, cudaStream_t st);

// Shared memory of the decode kernel with a one-row ring: the least it needs.
size_t decode_smem_bytes(const ia_shape_t& s);
cudaError_t launch_decode(const ia_shape_t& s, const void* q, const void* k, const void* v,
                          const float* delta, const float* A, void* state, float* o, float* num,
                          float* den, cudaStream_t st);

// IA_OK for cudaSuccess, else IA_ERR_CUDA after recording the error as this
// thread's last CUDA error (ia_last_cuda_error).
ia_status_t map_cuda(cudaError_t e);

// Failure injection for host tests: with IA_INJECT_LAUNCH_FAILURE set (and
// not "0"), every entry point returns IA_ERR_CUDA after its argument checks,
// launching nothing.
bool inject_launch_failure();

// Caller-registered events bracketing the dominant kernel launch (profiling).
void mark_launch_begin(cudaStream_t st);
void mark_launch_end(cudaStream_t st);
// While held, mark_launch_begin/end do nothing: an entry point that runs
// several passes marks its whole sequence once.
void hold_launch_marks(bool hold);

// The optional parts on the tensor-core chunk pass (ia_layer_tc.cu): input
// stabilisation and the bidirectional layer, for the shapes the chunk pass
// runs; no per-token step and no readout matrix.
bool ex_tc_supported(const ia_shape_t& s, const ia_options_t* opt);
size_t ex_tc_workspace_bytes(const ia_shape_t& s, const ia_options_t* opt, const TcPlan& p);
cudaError_t launch_ex_tc(const ia_shape_t& s, const ia_options_t* opt, const TcPlan& p, const void* q,
                         const void* k, const void* v, const float* delta, const float* A,
                         const void* state_in, float* o, float* num, float* den, void* state_out, void* ws,
                         cudaStream_t st);
int num_sms();

// Shape check shared by every entry point: positive dims (N only when
// need_n), a known dtype, and B*H within int range.
bool valid_dims(const ia_shape_t* s, bool need_n);

// Device address of a __device__ variable of this library on the current
// device.  In host code the variable's name is only a host-side stand-in, so
// the address is looked up with the device current and cached per device,
// keyed on the device's current context: a context created after
// cudaDeviceReset triggers a fresh lookup.
struct SymbolCache {
  static constexpr int kMaxDevices = 64;
  void* addr[kMaxDevices] = {};
  void* ctx_of[kMaxDevices] = {};
  void* get(const void* symbol, cudaError_t* err);
};

// Device address of the library's error flag on the current device, or
// nullptr if the lookup fails.
int* device_error_ptr();
int read_and_clear_device_error(cudaStream_t st, cudaError_t* err);

}  // namespace ia
