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
 *     den: [B,H,N] fp32; delta: [H] fp32 (> 0), or [H,M] when
 *     shape->delta_per_mode = 1 (lambda_hm = exp(Delta_hm A_m)); A: [M]
 *     complex fp32 stored as (re, im) pairs, shared by all heads, or NULL
 *     for S4D-Lin.  The input dtype (IA_F32 or IA_BF16) applies to q, k, v
 *     and dO; all outputs are fp32.
 *   - State: one buffer of ia_state_bytes() bytes, complex fp32 stored as
 *     (re, im): U [B,H,M,d_xi] | Gamma [B,H,M,d_v] | eta [B,H,M].
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and never synchronise the host.
 *   - Arguments are validated on the host before any launch; a bad argument
 *     returns a status and launches nothing.  Nothing throws across the ABI.
 *   - A launch failure returns IA_ERR_CUDA.  Device-side bounded waits that
 *     expire set a device flag, reported as IA_ERR_TIMEOUT by
 *     ia_check_device_errors().
 *   - The tensor-core path holds the per-mode decay over half a chunk,
 *     |lambda_m|^(-32) = exp(32 Delta_h |Re A_m|), in fp16 operands.  A head
 *     whose factor exceeds 64 (Delta > 0.26 for S4D-Lin, whose
 *     initialisation range [1e-3, 1e-1] gives at most 5), or whose Delta is
 *     not positive, sets the device flag reported as IA_ERR_PARAM_RANGE by
 *     ia_check_device_errors(); its outputs are then not to be used.  The
 *     CUDA-core paths compute in fp32 and have no such limit.
 *   - The library caches the device addresses of its own __device__
 *     variables per device, keyed on the current context, so a context that
 *     cudaDeviceReset replaced is looked up again.
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
  IA_ERR_TIMEOUT = 5,       /* a device-side bounded wait expired (see ia_check_device_errors) */
  IA_ERR_PARAM_RANGE = 6    /* Delta or A outside what the tensor-core path holds (see above) */
} ia_status_t;

/* Which kernels a shape runs on (see ia_prefill_path, ia_fwd_bwd_path). */
typedef enum {
  IA_PATH_NONE = 0,          /* invalid shape */
  IA_PATH_TENSOR_CORE = 1,   /* chunked tcgen05 kernels, chunk length 64 */
  IA_PATH_SEQUENTIAL = 2     /* token-serial fp32 CUDA-core kernel, one CTA per (b,h) */
} ia_path_t;

typedef enum { IA_F32 = 0, IA_BF16 = 1 } ia_dtype_t;

typedef struct {
  int B, H, N;       /* batch, heads, sequence length (N >= 1; ignored by decode) */
  int d_xi, d_v;     /* feature width of q/k, value width */
  int M;             /* complex S4D modes */
  ia_dtype_t in_dtype;
  int delta_per_mode;   /* 0: delta [H], one step per head (S4D-Lin init, paper's
                           default); 1: delta [H,M], one step per head and mode.
                           Zero when the struct is aggregate-initialised without it. */
} ia_shape_t;

/* Bytes of one state buffer: 8 * B * H * M * (d_xi + d_v + 1). */
IA_API size_t ia_state_bytes(const ia_shape_t* shape);

/* Workspace bytes ia_prefill_fwd needs for this shape (may be 0). */
IA_API size_t ia_prefill_workspace_bytes(const ia_shape_t* shape);

/* Workspace bytes ia_fwd_bwd needs for this shape. */
IA_API size_t ia_fwd_bwd_workspace_bytes(const ia_shape_t* shape);

/* Path of ia_prefill_fwd for this shape.  The tensor-core path takes bf16
 * inputs with M = 64 and d_xi, d_v in {64, 128}; every other shape (and fp32
 * input) runs the token-serial CUDA-core kernel, which is correct for any
 * shape whose state fits in shared memory but one to two orders of
 * magnitude slower on long sequences. */
IA_API ia_path_t ia_prefill_path(const ia_shape_t* shape);

/* Path of ia_fwd_bwd for this shape.  The tensor-core reverse pass takes
 * bf16 inputs with M = 64 and d_xi = d_v = 64; every other shape, d = 128
 * included, runs the token-serial CUDA-core adjoint. */
IA_API ia_path_t ia_fwd_bwd_path(const ia_shape_t* shape);

/* Number of kernel launches one ia_prefill_fwd call makes for this shape:
 * 2 on the tensor-core path (per-head tables, then the chunk pass), 1 on
 * the sequential path; 0 for an invalid shape. */
IA_API int ia_prefill_launches(const ia_shape_t* shape);

/* CTAs of the tensor-core chunk pass for this shape (0 off that path).  The
 * pass cuts the value columns into blocks of 64 (a "stream" is one (b,h) and
 * value block) and gives every CTA an equal contiguous range of the
 * (stream, chunk) space, at most one CTA per SM.  A range that starts inside
 * a stream takes its carried state from its predecessors (see
 * ia_prefill_fwd); the workspace then also holds two states per CTA.
 * IA_PREFILL_GRID=n forces n CTAs (tuning and tests). */
IA_API int ia_prefill_grid(const ia_shape_t* shape);

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
 *     the per-head tables of unsplit sequences (20,992 bytes per head): up
 *     to ia_prefill_static_max_heads() = 99 heads.  More heads return
 *     IA_ERR_WORKSPACE and launch nothing.
 *   - Only the tensor-core shapes run here (bf16 inputs, M = 64, d_xi and d_v
 *     in {64, 128}); other shapes return IA_ERR_UNSUPPORTED.
 *   - The first call on each device looks up the array's device address;
 *     make that first call before any stream capture.
 *   - Every call shares the array and it keeps the last call's contents.
 *     Calls that overlap on the GPU (different streams, unordered host
 *     threads) race on it; the caller must serialise them.
 *   - Never calls cudaMalloc, cudaFree or any other allocating routine.
 */
/* Largest H that ia_prefill_fwd_static accepts (99). */
IA_API int ia_prefill_static_max_heads(void);

IA_API ia_status_t ia_prefill_fwd_static(const ia_shape_t* shape, const void* q, const void* k,
                                         const void* v, const float* delta, const float* A,
                                         const void* state_in, float* o, float* num, float* den,
                                         void* state_out, void* stream);

/*
 * Training step of the layer from a zero state (paperlayer.ai summary
 * sec. A.3 and App. G: bf16 mixed-precision training; sec. 3.2: the S4D
 * recurrence, whose A and step Delta train with the model).  Given the
 * upstream gradient dO [B,H,N,d_v] (input dtype), writes o, the gradients
 * dq, dk [B,H,N,d_xi], dv [B,H,N,d_v] (fp32), dDelta (fp32, delta's shape:
 * [H] or [H,M]; summed over batch and time) and, when dA is not NULL, dA [M]
 * complex as (dL/dRe A_m, dL/dIm A_m) fp32 pairs, summed over batch, heads
 * and time (A itself may still be NULL = S4D-Lin).  dDelta and dA are
 * overwritten, reduced in a fixed order (bitwise reproducible run to run).
 */
IA_API ia_status_t ia_fwd_bwd(const ia_shape_t* shape, const void* q, const void* k, const void* v,
                       const float* delta, const float* A, const void* dO, float* o,
                       float* dq, float* dk, float* dv, float* dDelta, float* dA, void* workspace,
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
 * Carry composition for one sequence split into consecutive spans (summary
 * sec. A.2: parallel passes over pieces with sequential state passing
 * between them; across GPUs, the spans' local end states are exchanged once
 * and each span's carry-in is composed from them).  The recurrence is linear
 * in its state, so
 *     out = lambda^L * carry_in + local
 * per (b,h) and mode over U, Gamma and eta, with lambda = exp(Delta A) as in
 * ia_prefill_fwd (A NULL = S4D-Lin).  L >= 0 is the length in tokens of the
 * span whose end state from a zero start is `local` (an ia_prefill_fwd
 * state_out); carry_in is the state before that span (NULL = zero).  All
 * three are states in the ia_state_bytes layout, device memory, 16-byte
 * aligned; out may alias carry_in or local.  shape: B, H, d_xi, d_v, M,
 * delta_per_mode (N ignored).  Errors as for the other entry points.
 */
IA_API ia_status_t ia_state_carry(const ia_shape_t* shape, const float* delta, const float* A, long long L,
                                  const void* carry_in, const void* local, void* out, void* stream);

/*
 * Optional parts of the layer that the pages name beside the plain readout.
 * Every pointer is a caller-owned device array; NULL (or 0) leaves that part
 * out, so an all-zero ia_options_t is the plain layer.
 *   delta_t [B,H,N] fp32 (> 0): selective writing and memory decay
 *       (paperlayer.ai summary sec. 3.3 and sec. 5.3): token t uses its own
 *       step, lambda_t = exp(delta_t A), b_t = (lambda_t - 1)/A, for every
 *       mode; a small step writes little and forgets little.  `delta` is then
 *       not read (it may be NULL).  For a decode step: [B,H].
 *   gain, bias [H, d_xi + d_v] fp32: input stabilisation (AI-radio page,
 *       "Implementation Details"): the SSM input z_t = (xi(k_t), v_t) passes
 *       an RMSNorm over its d_xi + d_v entries with a per-head gain and bias,
 *       z <- z / sqrt(mean(z^2) + eps) * gain_h + bias_h, before the
 *       recurrence (NULL gain = 1, NULL bias = 0; the norm is on when either
 *       is given).  The query features are not normalised.
 *   eps: the RMSNorm epsilon (>= 0).
 *   W [H,M,M] complex fp32 ((re, im) pairs; W[h][m][m'] row m, column m'):
 *       the full complex readout matrix (summary sec. A.3; the M^2 term of
 *       the decode cost, sec. 3.2): a~_t = W_h a_t replaces a_t in
 *       num = Re(a~^H Gamma) and den = Re(a~^H eta).
 *   bidirectional: 1 for the bidirectional layer of the genomics models
 *       (summary sec. 5.2: Caduceus-IA keeps Caduceus' bidirectional
 *       handling): o = f(x) + flip(f(flip x)), f the causal layer, flip the
 *       time reversal.  Prefill only, with no state_in, state_out, num, den.
 */
typedef struct {
  const float* delta_t;
  const float* gain;
  const float* bias;
  float eps;
  const float* W;
  int bidirectional;
} ia_options_t;

/*
 * ia_prefill_fwd with the optional parts (NULL opt = the plain layer).
 * Two forms, chosen per call (ia_prefill_ex_path tells which):
 *   - bf16 inputs on a shape of the tensor-core chunk pass (M = 64, d_xi and
 *     d_v in {64, 128}) with no delta_t, and W only at d_xi = 64, run on
 *     tensor cores: a prologue kernel writes the stabilised SSM input z (when
 *     gain or bias is given) as fp16 k and v operands, and the time-reversed
 *     q and z (for the bidirectional layer); a second kernel writes W as the
 *     real fp16 matrix [[Re W, -Im W], [Im W, Re W]] (rows and columns
 *     interleaved by mode), and the chunk pass then runs one more contraction
 *     per chunk, W times the readout vectors of its 64 tokens; the chunk pass
 *     runs once, or twice for the bidirectional layer, whose second output an
 *     epilogue kernel adds back in forward order.  z, and with W the readout
 *     vectors and W, are rounded to fp16 once more than in the token-serial
 *     form.  Needs ia_prefill_ex_workspace_bytes of workspace.
 *   - everything else runs the token-serial fp32 CUDA-core kernel (any
 *     input dtype), correct for every shape whose state fits in shared memory
 *     but much slower.  With ia_prefill_ex_workspace_bytes of workspace it
 *     cuts each sequence into segments of at least 64 tokens, one CTA each,
 *     enough to fill the GPU's resident CTA slots: a first pass runs every
 *     segment but the last from a zero state (the first from state_in) for
 *     its end state, a carry kernel composes those into the state entering
 *     each segment (the decay over a segment is exp(A times its summed
 *     steps)), and a second pass runs every segment from its entering state
 *     with the readout (paper summary sec. A.2: parallel passes over pieces
 *     of the sequence, the state passed between them).  A smaller workspace,
 *     or NULL, gives fewer segments, down to one CTA per (b,h) token after
 *     token; results differ from one segment count to another only by fp32
 *     rounding.
 * workspace: device scratch of at least ia_prefill_ex_workspace_bytes bytes,
 * any alignment; for the tensor-core form too small gives IA_ERR_WORKSPACE
 * before anything is launched.
 */
IA_API size_t ia_prefill_ex_workspace_bytes(const ia_shape_t* shape, const ia_options_t* opt);
IA_API int ia_prefill_ex_path(const ia_shape_t* shape, const ia_options_t* opt);
/*
 * Segments per sequence that ia_prefill_fwd_ex runs with this workspace
 * (pointer and size as the call would get them; only the pointer's being
 * non-NULL matters): 1 for the tensor-core form and for a single token-serial
 * pass, else the count of the two-pass form, whose call then launches pass 1,
 * the carry kernel (when more than two segments) and pass 2 per direction.
 * 0 for an invalid shape or options.  Asks the device for the kernel's
 * resident CTAs per SM (1 when no device answers).
 */
IA_API int ia_prefill_ex_segments(const ia_shape_t* shape, const ia_options_t* opt, const void* workspace,
                                  size_t workspace_bytes);
IA_API ia_status_t ia_prefill_fwd_ex(const ia_shape_t* shape, const ia_options_t* opt, const void* q,
                                     const void* k, const void* v, const float* delta, const float* A,
                                     const void* state_in, float* o, float* num, float* den,
                                     void* state_out, void* workspace, size_t workspace_bytes,
                                     void* stream);

/*
 * ia_decode_step with the optional parts (bidirectional excluded: that layer
 * is not causal).  delta_t, if given, is [B,H]: this token's step.
 */
IA_API ia_status_t ia_decode_step_ex(const ia_shape_t* shape, const ia_options_t* opt, const void* q,
                                     const void* k, const void* v, const float* delta, const float* A,
                                     void* state, float* o, float* num, float* den, void* stream);

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

/* Synchronises `stream`, then reports (and clears) the device error flag:
 * IA_ERR_TIMEOUT if a bounded wait expired, else IA_ERR_PARAM_RANGE if a
 * tensor-core call met an out-of-range Delta, else IA_OK. */
IA_API ia_status_t ia_check_device_errors(void* stream);

/*
 * Self-test of the bounded waits (a diagnostic with no counterpart in the
 * paper).  Launches one small kernel on `stream` that waits on shared-memory
 * barriers nobody completes, with nothing else in flight: one plain bounded
 * wait and one abortable wait that expire after limit_ns (1e3 .. 1e9 ns),
 * and one abortable wait with the full one-second limit that must give up as
 * soon as the other raises the CTA's abort flag.  out (device, 6 x u64):
 * per waiter, 1 if its barrier completed (it never does) and the ns its wait
 * took.  After the kernel, ia_check_device_errors() returns IA_ERR_TIMEOUT
 * once and clears the flag.  Faults, traps and hangs nothing.
 */
IA_API ia_status_t ia_selftest_wait_expiry(unsigned long long limit_ns, unsigned long long* out,
                                           void* stream);

/* The CUDA error (a cudaError_t value; 0 if none) behind the last
 * IA_ERR_CUDA that an entry point returned on the calling thread, and its
 * description.  A diagnostic with no counterpart in the paper. */
IA_API int ia_last_cuda_error(void);
IA_API const char* ia_last_cuda_error_string(void);

/* Static description of a status code. */
IA_API const char* ia_status_string(ia_status_t status);

#ifdef __cplusplus
}
#endif
#endif /* IA_H */
