/*
 * libia -- Interdomain Attention (IA) layer hot path on NVIDIA B200 (sm_100a).
 *
 * The layer (paper "Interdomain Attention: Beyond Token-Level Key-Value
 * Memory", Kiyohara et al.; paperlayer.ai summary sec. 3.1-3.2, sec. A.2,
 * sec. D.2 and sec. F.2; AI-radio page formula extract "O = Fq U^T Gamma /
 * Fq U^T eta") feeds positive key features xi(k_t) = elu(k_t) + 1, values v_t
 * and the constant 1 through one complex-diagonal S4D recurrence with M modes:
 *
 *   lambda_m = exp(Delta_h A_m),   b_m = (lambda_m - 1) / A_m     (zero-order hold)
 *   U_t     = lambda U_{t-1}     + b xi(k_t)^T     M x d_xi complex
 *   Gamma_t = lambda Gamma_{t-1} + b v_t^T         M x d_v  complex
 *   eta_t   = lambda eta_{t-1}   + b               M        complex
 *   a_t = U_t xi(q_t),  num_t = Re(a_t^H Gamma_t),  den_t = Re(a_t^H eta_t),
 *   o_t = num_t / den_t            (no epsilon; den may change sign)
 *
 * A_m defaults to S4D-Lin, A_m = -1/2 + i pi m.  The state is updated with
 * token t before query t reads it.  Delta is one scalar per head.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers, row-major and contiguous, owned
 *     by the caller.  The library never allocates device memory; scratch
 *     comes from a caller-provided workspace sized by the *_workspace_bytes
 *     queries.  Tensor pointers must be 16-byte aligned.
 *   - q, k: [B,H,N,d_xi]; v: [B,H,N,d_v]; o, num: [B,H,N,d_v] fp32;
 *     den: [B,H,N] fp32; delta: [H] fp32 (> 0); A: [M] complex fp32 stored as
 *     (re, im) pairs, or NULL for S4D-Lin.  The input dtype (IA_F32 or
 *     IA_BF16) applies to q, k, v and dO; all outputs are fp32.
 *   - State: one buffer of ia_state_bytes() bytes, complex fp32 stored as
 *     (re, im): U [B,H,M,d_xi] | Gamma [B,H,M,d_v] | eta [B,H,M].
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and never synchronise the host.
 *   - Arguments are validated on the host before any launch; a bad argument
 *     returns a status and launches nothing.  Nothing throws across the ABI.
 *   - A launch failure returns IA_ERR_CUDA.  Device-side bounded waits that
 *     expire set a device flag, reported as IA_ERR_TIMEOUT by
 *     ia_check_device_errors().
 */
#ifndef IA_H
#define IA_H

#include <stddef.h>

#if defined(__GNUC__)
#define IA_API __attribute__((visibility("default")))
#else
#define IA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  IA_OK = 0,
  IA_ERR_INVALID_ARG = 1,   /* null pointer, non-positive or inconsistent dims, misalignment */
  IA_ERR_UNSUPPORTED = 2,   /* shape or dtype outside what the kernels implement */
  IA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than the query says */
  IA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
  IA_ERR_TIMEOUT = 5        /* a device-side bounded wait expired (see ia_check_device_errors) */
} ia_status_t;

typedef enum { IA_F32 = 0, IA_BF16 = 1 } ia_dtype_t;

typedef struct {
  int B, H, N;       /* batch, heads, sequence length (N >= 1; ignored by decode) */
  int d_xi, d_v;     /* feature width of q/k, value width */
  int M;             /* complex S4D modes */
  ia_dtype_t in_dtype;
} ia_shape_t;

/* Bytes of one state buffer: 8 * B * H * M * (d_xi + d_v + 1). */
IA_API size_t ia_state_bytes(const ia_shape_t* shape);

/* Workspace bytes ia_prefill_fwd needs for this shape (may be 0). */
IA_API size_t ia_prefill_workspace_bytes(const ia_shape_t* shape);

/* Workspace bytes ia_fwd_bwd needs for this shape. */
IA_API size_t ia_fwd_bwd_workspace_bytes(const ia_shape_t* shape);

/* Number of kernel launches one ia_prefill_fwd call makes for this shape
 * (the tensor-core path adds a state-only pass and a carry scan when it
 * splits sequences into segments); 0 for an invalid shape. */
IA_API int ia_prefill_launches(const ia_shape_t* shape);

/*
 * Causal prefill over N tokens (paperlayer.ai summary sec. 3.2 and sec. A.2:
 * chunkwise execution, chunk 64, with state passing; sec. F.2: chunked
 * prefill that builds the decoding state).
 *   state_in  : NULL = zero state, else the state before token 0.
 *   o         : required output.  num, den: optional (NULL to skip).
 *   state_out : optional; the state after token N-1 (may not alias state_in).
 * bf16 inputs run on the tcgen05 tensor-core path (fp16 operands, fp32
 * accumulation and fp32 state); fp32 inputs run on the fp32 CUDA-core path.
 */
IA_API ia_status_t ia_prefill_fwd(const ia_shape_t* shape, const void* q, const void* k,
                           const void* v, const float* delta, const float* A,
                           const void* state_in, float* o, float* num, float* den,
                           void* state_out, void* workspace, size_t workspace_bytes,
                           void* stream);

/*
 * ia_prefill_fwd for callers that cannot allocate device memory, for example
 * a plugin inside another framework whose memory pool owns the device, or a
 * serving loop that must never reach cudaMalloc/cudaFree because those calls
 * can synchronise the device.  No counterpart in the paper: same arguments
 * and results as ia_prefill_fwd, minus the workspace.
 *   - Scratch lives in a fixed 2 MiB array compiled into the library, held by
 *     every GPU that loads the library until the process exits.  It holds
 *     the per-head tables of unsplit sequences: up to 97 heads.  More heads
 *     return IA_ERR_WORKSPACE and launch nothing.
 *   - Only the tensor-core shapes run here (bf16 inputs, M = 64, d_xi and d_v
 *     in {64, 128}); other shapes return IA_ERR_UNSUPPORTED.
 *   - The first call on each device looks up the array's device address;
 *     make that first call before any stream capture.
 *   - Every call shares the array and it keeps the last call's contents.
 *     Calls that overlap on the GPU (different streams, unordered host
 *     threads) race on it; the caller must serialise them.
 *   - Never calls cudaMalloc, cudaFree or any other allocating routine.
 */
IA_API ia_status_t ia_prefill_fwd_static(const ia_shape_t* shape, const void* q, const void* k,
                                         const void* v, const float* delta, const float* A,
                                         const void* state_in, float* o, float* num, float* den,
                                         void* state_out, void* stream);

/*
 * Training step of the layer from a zero state (paperlayer.ai summary
 * sec. A.3 and App. G: bf16 mixed-precision training).  Given the upstream
 * gradient dO [B,H,N,d_v] (input dtype), writes o, and the gradients
 * dq, dk [B,H,N,d_xi], dv [B,H,N,d_v] (fp32) and dDelta [H] (fp32, summed
 * over batch and time; overwritten).
 */
IA_API ia_status_t ia_fwd_bwd(const ia_shape_t* shape, const void* q, const void* k, const void* v,
                       const float* delta, const float* A, const void* dO, float* o,
                       float* dq, float* dk, float* dv, float* dDelta, void* workspace,
                       size_t workspace_bytes, void* stream);

/*
 * One recurrent decode step (paperlayer.ai summary sec. 3.2: fixed state of
 * size O(M(R + d)), constant work per token; sec. F.3: graphed decode).
 * q, k [B,H,d_xi], v [B,H,d_v] (input dtype); state updated in place;
 * o [B,H,d_v] fp32; num [B,H,d_v] and den [B,H] optional.  shape->N is
 * ignored.  Needs no workspace and does not allocate, so it can be captured
 * in a CUDA graph.
 */
IA_API ia_status_t ia_decode_step(const ia_shape_t* shape, const void* q, const void* k,
                           const void* v, const float* delta, const float* A, void* state,
                           float* o, float* num, float* den, void* stream);

/*
 * Profiling aid (no counterpart in the paper): registers two caller-owned
 * CUDA events (cudaEvent_t handles).  While set, every later entry-point call
 * records `begin` on its stream immediately before launching its dominant
 * kernel (the full chunk pass of the prefill, the reverse-mode kernel of the
 * training step, the decode kernel) and `end` immediately after it, so the
 * caller can time that kernel alone.  One exception: the unsplit d = 64
 * chunk pass starts while the per-head table kernel before it still runs
 * (programmatic dependent launch), so there `begin` precedes the table
 * kernel and the interval covers both.  Pass NULL, NULL to stop.  The events
 * are not owned or destroyed by the library.
 */
IA_API ia_status_t ia_set_launch_events(void* begin, void* end);

/* Synchronises `stream`, then reports (and clears) the device error flag
 * that bounded waits set when they expire: IA_OK or IA_ERR_TIMEOUT. */
IA_API ia_status_t ia_check_device_errors(void* stream);

/* Static description of a status code. */
IA_API const char* ia_status_string(ia_status_t status);

#ifdef __cplusplus
}
#endif
#endif /* IA_H */
