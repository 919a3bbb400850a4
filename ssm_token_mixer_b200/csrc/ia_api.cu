// C-ABI of libia: argument validation on the host (before any launch),
// workspace sizing and dispatch to the kernels.  See include/ia.h for the
// contract of every entry point.
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "ia_device.cuh"
#include "ia_internal.h"
#include "ia_tables.cuh"

namespace ia {

// Raised by device-side bounded waits that expire (bit 0); read and cleared
// by ia_check_device_errors().
__device__ int g_device_error = 0;

namespace {

constexpr size_t kMaxSmem = 232448;   // 227 KB opt-in shared memory per block on sm_100

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool env_set(const char* name) {
  const char* s = std::getenv(name);
  return s && s[0] && std::strcmp(s, "0") != 0;
}


bool use_tc(const ia_shape_t& s) {
  if (env_set("IA_PREFILL_SIMT")) return false;   // debug switch: force the CUDA-core path
  return tc_prefill_supported(s);
}

bool use_tc_bwd(const ia_shape_t& s) {
  if (env_set("IA_BWD_SIMT")) return false;       // debug switch: force the CUDA-core adjoint
  return tc_bwd_supported(s);
}

cudaEvent_t g_ev_begin = nullptr, g_ev_end = nullptr;

}  // namespace

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();   // clear a sticky "no device" error; plan for a B200
    return 148;
  }
  return n;
}

bool valid_dims(const ia_shape_t* s, bool need_n) {
  if (!s) return false;
  if (s->B <= 0 || s->H <= 0 || s->d_xi <= 0 || s->d_v <= 0 || s->M <= 0) return false;
  if (need_n && s->N <= 0) return false;
  if (s->in_dtype != IA_F32 && s->in_dtype != IA_BF16) return false;
  if (s->delta_per_mode != 0 && s->delta_per_mode != 1) return false;
  // element counts must stay addressable with 64-bit indices and int grid sizes
  const long long BH = static_cast<long long>(s->B) * s->H;
  if (BH > (1LL << 31) - 1) return false;
  return true;
}

// The CUDA error behind this thread's last IA_ERR_CUDA (see ia_last_cuda_error).
thread_local int g_last_cuda_error = 0;

ia_status_t map_cuda(cudaError_t e) {
  if (e == cudaSuccess) return IA_OK;
  g_last_cuda_error = static_cast<int>(e);
  return IA_ERR_CUDA;
}

bool inject_launch_failure() { return env_set("IA_INJECT_LAUNCH_FAILURE"); }

// The current context, through the driver entry point (the library links no
// driver stub); nullptr if there is none or the lookup fails.
void* current_context() {
  using GetCtxFn = int (*)(void**);   // CUresult cuCtxGetCurrent(CUcontext*)
  static const GetCtxFn fn = []() -> GetCtxFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<GetCtxFn>(f);
  }();
  void* ctx = nullptr;
  if (!fn || fn(&ctx) != 0) return nullptr;
  return ctx;
}

void* SymbolCache::get(const void* symbol, cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  void* ctx = current_context();
  if (addr[dev] && ctx && ctx == ctx_of[dev]) {
    *err = cudaSuccess;
    return addr[dev];
  }
  // First use on this device, or its context was replaced (cudaDeviceReset
  // unloads the module): look the address up again.  The lookup creates the
  // primary context if there is none yet, so the key is read after it.
  void* p = nullptr;
  *err = cudaGetSymbolAddress(&p, symbol);
  if (*err != cudaSuccess) return nullptr;
  addr[dev] = p;
  ctx_of[dev] = current_context();
  return p;
}

thread_local bool g_marks_held = false;
void hold_launch_marks(bool hold) { g_marks_held = hold; }
void mark_launch_begin(cudaStream_t st) {
  if (g_ev_begin && !g_marks_held) cudaEventRecord(g_ev_begin, st);
}
void mark_launch_end(cudaStream_t st) {
  if (g_ev_end && !g_marks_held) cudaEventRecord(g_ev_end, st);
}

int* device_error_ptr() {
  static SymbolCache cache;
  cudaError_t e;
  return static_cast<int*>(cache.get(&g_device_error, &e));
}

int read_and_clear_device_error(cudaStream_t st, cudaError_t* err) {
  int flag = 0;
  *err = cudaStreamSynchronize(st);
  if (*err != cudaSuccess) return 0;
  *err = cudaMemcpyFromSymbol(&flag, g_device_error, sizeof(int));
  if (*err != cudaSuccess) return 0;
  if (flag) {
    int zero = 0;
    *err = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
  }
  return flag;
}

}  // namespace ia

using namespace ia;

extern "C" {

size_t ia_state_bytes(const ia_shape_t* s) {
  if (!valid_dims(s, false)) return 0;
  return sizeof(float) * 2 * static_cast<size_t>(s->B) * s->H * s->M *
         (static_cast<size_t>(s->d_xi) + s->d_v + 1);
}

size_t ia_prefill_workspace_bytes(const ia_shape_t* s) {
  if (!valid_dims(s, true)) return 0;
  if (!use_tc(*s)) return 0;
  return tc_workspace_bytes(*s, tc_plan(*s, num_sms()));
}

int ia_prefill_grid(const ia_shape_t* s) {
  if (!valid_dims(s, true) || !use_tc(*s)) return 0;
  return tc_plan(*s, num_sms()).grid;
}

int ia_prefill_launches(const ia_shape_t* s) {
  if (!valid_dims(s, true)) return 0;
  if (!use_tc(*s)) return 1;
  return 2;   // the table kernel and the chunk pass
}

size_t ia_fwd_bwd_workspace_bytes(const ia_shape_t* s) {
  if (!valid_dims(s, true)) return 0;
  if (use_tc_bwd(*s)) return tc_fwd_bwd_workspace_bytes(*s, tc_plan(*s, num_sms()));
  return seq_bwd_workspace_bytes(*s);
}

ia_status_t ia_prefill_fwd(const ia_shape_t* s, const void* q, const void* k, const void* v,
                           const float* delta, const float* A, const void* state_in, float* o,
                           float* num, float* den, void* state_out, void* workspace,
                           size_t workspace_bytes, void* stream) {
  if (!valid_dims(s, true)) return IA_ERR_INVALID_ARG;
  if (!q || !k || !v || !delta || !o) return IA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, delta, A, state_in, o, num, den, state_out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return IA_ERR_INVALID_ARG;
  if (state_in && state_in == state_out) return IA_ERR_INVALID_ARG;
  const bool tc = use_tc(*s);
  size_t need = 0;
  TcPlan plan{1};
  if (tc) {
    plan = tc_plan(*s, num_sms());
    need = tc_workspace_bytes(*s, plan);
  } else if (seq_fwd_smem(s->d_xi, s->d_v, s->M) > kMaxSmem) {
    return IA_ERR_UNSUPPORTED;
  }
  if (need > 0 && (!workspace || workspace_bytes < need)) return IA_ERR_WORKSPACE;
  if (inject_launch_failure()) return IA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc)
    return map_cuda(launch_tc_prefill(*s, plan, q, k, v, delta, A, state_in, o, num, den,
                                      state_out, workspace, st));
  return map_cuda(launch_seq_fwd(*s, q, k, v, delta, A, state_in, o, num, den, state_out, st));
}

ia_status_t ia_fwd_bwd(const ia_shape_t* s, const void* q, const void* k, const void* v,
                       const float* delta, const float* A, const void* dO, float* o, float* dq,
                       float* dk, float* dv, float* dDelta, float* dA, void* workspace,
                       size_t workspace_bytes, void* stream) {
  if (!valid_dims(s, true)) return IA_ERR_INVALID_ARG;
  if (!q || !k || !v || !delta || !dO || !o || !dq || !dk || !dv || !dDelta)
    return IA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, delta, A, dO, o, dq, dk, dv, dDelta, dA, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return IA_ERR_INVALID_ARG;
  const bool tc = use_tc_bwd(*s);
  if (!tc && seq_bwd_smem(s->d_xi, s->d_v, s->M) > kMaxSmem) return IA_ERR_UNSUPPORTED;
  const size_t need = ia_fwd_bwd_workspace_bytes(s);
  if (!workspace || workspace_bytes < need) return IA_ERR_WORKSPACE;
  if (inject_launch_failure()) return IA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc)
    return map_cuda(launch_tc_fwd_bwd(*s, tc_plan(*s, num_sms()), q, k, v, delta, A, dO, o, dq, dk,
                                      dv, dDelta, dA, workspace, st));
  return map_cuda(launch_seq_bwd(*s, q, k, v, delta, A, dO, o, dq, dk, dv, dDelta, dA, workspace, st));
}

ia_status_t ia_decode_step(const ia_shape_t* s, const void* q, const void* k, const void* v,
                           const float* delta, const float* A, void* state, float* o, float* num,
                           float* den, void* stream) {
  if (!valid_dims(s, false)) return IA_ERR_INVALID_ARG;
  if (!q || !k || !v || !delta || !state || !o) return IA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, delta, A, state, o, num, den};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return IA_ERR_INVALID_ARG;
  if ((s->d_xi & 1) || (s->d_v & 1)) return IA_ERR_UNSUPPORTED;   // 16-byte state vectors
  if (s->d_xi > 256 || s->d_v > 256) return IA_ERR_UNSUPPORTED;     // one register pass per row
  if (decode_smem_bytes(*s) > kMaxSmem) return IA_ERR_UNSUPPORTED;
  if (inject_launch_failure()) return IA_ERR_CUDA;
  return map_cuda(launch_decode(*s, q, k, v, delta, A, state, o, num, den,
                                static_cast<cudaStream_t>(stream)));
}

ia_status_t ia_state_carry(const ia_shape_t* s, const float* delta, const float* A, long long L,
                           const void* carry_in, const void* local, void* out, void* stream) {
  if (!valid_dims(s, false)) return IA_ERR_INVALID_ARG;
  if (!delta || !local || !out || L < 0) return IA_ERR_INVALID_ARG;
  const void* ptrs[] = {delta, A, carry_in, local, out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return IA_ERR_INVALID_ARG;
  if (static_cast<long long>(s->B) * s->H * s->M > (1LL << 31) - 1) return IA_ERR_UNSUPPORTED;   // one block per row
  if (inject_launch_failure()) return IA_ERR_CUDA;
  return map_cuda(launch_state_carry(*s, delta, A, L, carry_in, local, out, static_cast<cudaStream_t>(stream)));
}

ia_status_t ia_set_launch_events(void* begin, void* end) {
  if ((begin == nullptr) != (end == nullptr)) return IA_ERR_INVALID_ARG;
  g_ev_begin = static_cast<cudaEvent_t>(begin);
  g_ev_end = static_cast<cudaEvent_t>(end);
  return IA_OK;
}

ia_status_t ia_check_device_errors(void* stream) {
  cudaError_t e;
  int flag = read_and_clear_device_error(static_cast<cudaStream_t>(stream), &e);
  if (e != cudaSuccess) return map_cuda(e);
  if (flag & kErrTimeout) return IA_ERR_TIMEOUT;
  if (flag & kErrParamRange) return IA_ERR_PARAM_RANGE;
  return IA_OK;
}

ia_path_t ia_prefill_path(const ia_shape_t* s) {
  if (!valid_dims(s, true)) return IA_PATH_NONE;
  return use_tc(*s) ? IA_PATH_TENSOR_CORE : IA_PATH_SEQUENTIAL;
}

ia_path_t ia_fwd_bwd_path(const ia_shape_t* s) {
  if (!valid_dims(s, true)) return IA_PATH_NONE;
  return use_tc_bwd(*s) ? IA_PATH_TENSOR_CORE : IA_PATH_SEQUENTIAL;
}

int ia_last_cuda_error(void) { return g_last_cuda_error; }

const char* ia_last_cuda_error_string(void) {
  return g_last_cuda_error ? cudaGetErrorString(static_cast<cudaError_t>(g_last_cuda_error)) : "no error";
}

const char* ia_status_string(ia_status_t st) {
  switch (st) {
    case IA_OK: return "IA_OK: success";
    case IA_ERR_INVALID_ARG: return "IA_ERR_INVALID_ARG: null, misaligned or inconsistent argument";
    case IA_ERR_UNSUPPORTED: return "IA_ERR_UNSUPPORTED: shape or dtype not implemented";
    case IA_ERR_WORKSPACE: return "IA_ERR_WORKSPACE: workspace missing or too small";
    case IA_ERR_CUDA: return "IA_ERR_CUDA: CUDA runtime or launch failure";
    case IA_ERR_TIMEOUT: return "IA_ERR_TIMEOUT: a device-side bounded wait expired";
    case IA_ERR_PARAM_RANGE:
      return "IA_ERR_PARAM_RANGE: Delta or A outside the range the tensor-core path holds in fp16";
  }
  return "unknown ia_status_t";
}

}  // extern "C"
