// ia_prefill_fwd_static: the tensor-core prefill for callers that cannot
// allocate device memory.
//
// ia_prefill_fwd needs a small device workspace (per-head decay tables, and
// segment carries when it splits long sequences).  Some callers cannot hand
// one over: a plugin running inside another framework whose memory pool owns
// the whole device and forbids raw allocations, or a latency-critical serving
// loop that must never reach cudaMalloc/cudaFree, because those calls can
// synchronise the device and stall every other stream.  This entry point takes
// the same inputs and outputs but keeps its scratch in a fixed array compiled
// into the library (kStaticScratchBytes per GPU, held by every GPU that loads
// the library until the process exits).  It never allocates.
//
// It always runs the sequences unsplit (one CTA per (b,h)), so the scratch
// only holds the per-head tables: 21.5 KB per head, up to 97 heads.
#include <cstdint>

#include "ia_internal.h"
#include "ia_tables.cuh"

namespace ia {
namespace {

constexpr size_t kStaticScratchBytes = size_t(2) << 20;   // 2 MiB per GPU
constexpr int kMaxDevices = 64;

// Shared by every call on a device; it keeps the last call's contents.  The
// tables are rewritten at the start of every call, so nothing in it has to
// start at zero.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
void* static_scratch_on_current_device(cudaError_t* err) {
  static void* cache[kMaxDevices] = {};
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  if (!cache[dev]) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_static_scratch);
    if (*err != cudaSuccess) return nullptr;
    cache[dev] = p;
  }
  *err = cudaSuccess;
  return cache[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace ia

using namespace ia;

extern "C" IA_API ia_status_t ia_prefill_fwd_static(const ia_shape_t* s, const void* q,
                                                    const void* k, const void* v,
                                                    const float* delta, const float* A,
                                                    const void* state_in, float* o, float* num,
                                                    float* den, void* state_out, void* stream) {
  if (!s || s->B <= 0 || s->H <= 0 || s->N <= 0 || s->d_xi <= 0 || s->d_v <= 0 || s->M <= 0)
    return IA_ERR_INVALID_ARG;
  if (s->in_dtype != IA_F32 && s->in_dtype != IA_BF16) return IA_ERR_INVALID_ARG;
  if (!q || !k || !v || !delta || !o) return IA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, delta, A, state_in, o, num, den, state_out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return IA_ERR_INVALID_ARG;
  if (state_in && state_in == state_out) return IA_ERR_INVALID_ARG;
  if (!tc_prefill_supported(*s)) return IA_ERR_UNSUPPORTED;
  const int nch = (s->N + kChunk - 1) / kChunk;
  const TcPlan plan{1, nch};
  if (tc_workspace_bytes(*s, plan) > kStaticScratchBytes) return IA_ERR_WORKSPACE;
  if (inject_launch_failure()) return IA_ERR_CUDA;
  cudaError_t e;
  void* scratch = static_scratch_on_current_device(&e);
  if (!scratch) return IA_ERR_CUDA;
  e = launch_tc_prefill(*s, plan, q, k, v, delta, A, state_in, o, num, den, state_out, scratch,
                        static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? IA_OK : IA_ERR_CUDA;
}
