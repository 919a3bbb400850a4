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
// only holds the per-head tables: sizeof(HeadTables) per head plus 256 bytes
// of alignment slack, kStaticMaxHeads heads at most.
#include <cstdint>

#include "ia_internal.h"
#include "ia_tables.cuh"

namespace ia {
namespace {

constexpr size_t kStaticScratchBytes = size_t(2) << 20;   // 2 MiB per GPU
// The per-head tables of an unsplit prefill take sizeof(HeadTables) per head
// after a 256-byte alignment allowance (tc_workspace_bytes with one segment).
constexpr int kStaticMaxHeads = static_cast<int>((kStaticScratchBytes - 256) / sizeof(HeadTables));
static_assert(sizeof(HeadTables) == 20992 && kStaticMaxHeads == 99,
              "the head limit stated in include/ia.h follows the table size");

// Shared by every call on a device; it keeps the last call's contents.  The
// tables are rewritten at the start of every call, so nothing in it has to
// start at zero.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace ia

using namespace ia;

extern "C" IA_API int ia_prefill_static_max_heads(void) { return kStaticMaxHeads; }

extern "C" IA_API ia_status_t ia_prefill_fwd_static(const ia_shape_t* s, const void* q,
                                                    const void* k, const void* v,
                                                    const float* delta, const float* A,
                                                    const void* state_in, float* o, float* num,
                                                    float* den, void* state_out, void* stream) {
  if (!valid_dims(s, true)) return IA_ERR_INVALID_ARG;
  if (!q || !k || !v || !delta || !o) return IA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, delta, A, state_in, o, num, den, state_out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return IA_ERR_INVALID_ARG;
  if (state_in && state_in == state_out) return IA_ERR_INVALID_ARG;
  if (!tc_prefill_supported(*s)) return IA_ERR_UNSUPPORTED;
  const TcPlan plan = tc_plan_whole_streams(*s);   // one CTA per stream: tables only
  if (tc_workspace_bytes(*s, plan) > kStaticScratchBytes) return IA_ERR_WORKSPACE;
  if (inject_launch_failure()) return IA_ERR_CUDA;
  // Device address of the scratch array: in host code its name is only a
  // host-side stand-in, so it is looked up with the device current, once per
  // device (again after a device reset), and cached.
  static SymbolCache scratch_cache;
  cudaError_t e;
  void* scratch = scratch_cache.get(&g_static_scratch, &e);
  if (!scratch) return map_cuda(e);
  return map_cuda(launch_tc_prefill(*s, plan, q, k, v, delta, A, state_in, o, num, den, state_out,
                                    scratch, static_cast<cudaStream_t>(stream)));
}
