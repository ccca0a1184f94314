/*
 * dr.h -- C ABI of the chunkwise gated delta-rule linear-attention library
 * (libdr.so, CUDA, sm_100a).
 *
 * Operation (per batch b and head h; S is d_v x d_k):
 *
 *   S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *   o_t = S_t q_t                       (the state is read after the write)
 *
 * This is the real, phase-free form of the delta-rule update in the SFDA
 * explainer ("Semidirect Fourier Delta Attention", gist.science, section
 * "Kernarchitektur"; zero phase recovers KDA), transposed so that S maps keys
 * to values.  alpha_t = exp(g_t) with g the log-gate: absent (DeltaNet), one
 * scalar per head and token (GDN) or one per key channel (KDA), as named in
 * the ReWY abstract (paperdot listing).  In Kaczmarz mode (KLA abstract,
 * thelatestinai.com) beta_t = eta_t / (||k_t||^2 + eps) and the beta argument
 * carries eta.
 *
 * dr_chunk_fwd evaluates the recurrence chunkwise (chunk = 64 tokens): an
 * intra-chunk UT transform (I + A) [U' | W] = diag(beta) [V | K e^gamma] with
 * A the beta- and gate-scaled strictly-lower key Gram, an inter-chunk state
 * scan S <- S Diag(e^{gamma_C}) + U^T K~ ("exact affine chunk transfer", SFDA
 * explainer, "Zentrale Beiträge"), and the output q S^T plus the causal
 * intra-chunk term.  dr_chunk_bwd returns the exact gradients of the same
 * function; the chunk correction is differentiated as one triangular residual
 * system (ReWY abstract), so no adjoint of the inverse is formed.
 *
 * Conventions for every entry point:
 *  - Tensor pointers are DEVICE pointers, 16-byte aligned, row-major and
 *    contiguous, owned by the caller; the library never allocates device
 *    memory and keeps no pointer after a call returns.
 *  - Layouts: q, k [B, T, H, dk]; v, o, dO [B, T, H, dv] (storage dtype
 *    dr_problem.dtype); beta [B, T, H] fp32; g [B, T, H] fp32 (scalar gate)
 *    or [B, T, H, dk] fp32 (per-channel and phase gates), NULL for gate NONE;
 *    S0, ST, dST, dS0 [B, H, dv, dk] fp32.
 *  - Phase gate (DR_GATE_PHASE, SFDA: the explainer's complex diagonal
 *    Lambda_t = diag(alpha_t e^{i theta_t}), section "Kernarchitektur", in
 *    real coordinates): key channels pair up as (2j, 2j+1); g[..., 2j] is
 *    log alpha_j and g[..., 2j+1] the phase theta_j (radians), and the decay
 *    maps each state row's pair (x, y) to
 *    alpha_j (cos theta_j x - sin theta_j y, sin theta_j x + cos theta_j y)
 *    before the erase-and-write (zero phase: KDA with each pair's channels
 *    sharing one decay).  Supported by dr_chunk_fwd and dr_chunk_bwd (bf16,
 *    dk = dv = 128; other shapes give DR_ERR_UNSUPPORTED) and by
 *    dr_decode_step; dg[..., 2j] is then d/d log alpha_j and dg[..., 2j+1]
 *    d/d theta_j.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  Arguments are validated on the host before any launch; a
 *    non-DR_OK status means nothing was launched, except DR_ERR_CUDA, which
 *    reports a launch failure.  Device-side conditions (a bounded wait that
 *    timed out) are recorded in a device flag and reported by
 *    dr_last_device_error.
 *  - Calls on different streams must not share a workspace or saved buffer.
 */
#ifndef DR_H
#define DR_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DR_OK = 0,
  DR_ERR_INVALID_ARG = 1,  /* null required pointer, bad size, misaligned pointer */
  DR_ERR_UNSUPPORTED = 2,  /* valid but not implemented (chunk != 64, head dim) */
  DR_ERR_WORKSPACE = 3,    /* workspace or saved buffer missing or too small */
  DR_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed */
  DR_ERR_TIMEOUT = 5       /* a bounded device-side wait gave up */
} dr_status;

typedef enum { DR_F32 = 0, DR_BF16 = 1 } dr_dtype;
typedef enum {
  DR_GATE_NONE = 0,     /* alpha = 1 (DeltaNet) */
  DR_GATE_SCALAR = 1,   /* one log-gate per head and token (GDN) */
  DR_GATE_CHANNEL = 2,  /* one log-gate per key channel (KDA) */
  DR_GATE_PHASE = 3     /* SFDA rotation-decay per key pair (see above) */
} dr_gate;
typedef enum { DR_BETA_DIRECT = 0, DR_BETA_KACZMARZ = 1 } dr_beta_mode;

/* Problem description.  Supported: B, H, T >= 1; chunk == 64;
   dk, dv multiples of 16 in [16, 128]; dtype DR_F32 or DR_BF16.
   eps is used only in Kaczmarz mode (must be >= 0). */
typedef struct {
  int B, H, T, dk, dv, chunk;
  int dtype;      /* dr_dtype */
  int gate;       /* dr_gate */
  int beta_mode;  /* dr_beta_mode */
  float eps;
} dr_problem;

/* Bytes of scratch ("workspace") that dr_chunk_fwd (pass 0) or dr_chunk_bwd
   (pass 1) needs for problem *p.  Writes *bytes; host only, no CUDA call. */
dr_status dr_workspace_size(const dr_problem* p, int pass, size_t* bytes);

/* Bytes of the forward-to-backward "saved" buffer (per-chunk start states,
   internal layout).  Host only. */
dr_status dr_saved_size(const dr_problem* p, size_t* bytes);

/* Chunkwise forward.
   In:  q, k, v, beta (eta in Kaczmarz mode), g (NULL iff gate NONE),
        S0 (NULL = zero initial state).
   The phase gate needs dtype DR_BF16 and dk = dv = 128 (else
   DR_ERR_UNSUPPORTED); its chunk decay is the per-pair rotation-decay
   product, the rest of the chunk form is unchanged.
   Out: o (storage dtype), ST (final state, fp32; NULL = not wanted),
        saved (NULL = not wanted; else dr_saved_size bytes, which dr_chunk_bwd
        may then read instead of recomputing the states).
   ws:  at least dr_workspace_size(p, 0) bytes of device scratch, 256-byte
        aligned; its contents are undefined after the call. */
dr_status dr_chunk_fwd(const dr_problem* p, const void* q, const void* k, const void* v,
                       const float* beta, const float* g, const float* S0, void* o,
                       float* ST, void* saved, void* ws, size_t ws_bytes, void* stream);

/* Chunkwise backward of the same call.
   In:  the forward inputs, dO (storage dtype), dST (upstream gradient of the
        final state, fp32; NULL = zero), saved (the buffer a previous
        dr_chunk_fwd filled for the same inputs, or NULL to recompute).
   Out: dq, dk, dv (storage dtype), dbeta (fp32; d/deta in Kaczmarz mode),
        dg (fp32, shaped like g; ignored and may be NULL for gate NONE),
        dS0 (fp32; NULL = not wanted).
   The phase gate needs dtype DR_BF16 and dk = dv = 128 (else
   DR_ERR_UNSUPPORTED, nothing launched).
   ws:  at least dr_workspace_size(p, 1) bytes, 256-byte aligned. */
dr_status dr_chunk_bwd(const dr_problem* p, const void* q, const void* k, const void* v,
                       const float* beta, const float* g, const float* S0, const void* dO,
                       const float* dST, const void* saved, void* dq, void* dk, void* dv,
                       float* dbeta, float* dg, float* dS0, void* ws, size_t ws_bytes,
                       void* stream);

/* Single-token recurrent step (decode), the update itself applied to one
   token per head: with alpha = exp(g) (1 for gate NONE),
     P = S Diag(alpha),  e = v - P k,  S <- P + beta e k^T,  o = S q
   ("Semidirect Fourier Delta Attention" explainer, gist.science, section
   Kernarchitektur, with zero phase; the KLA abstract, "How AI settled the
   complexity of the oldest SGD algorithm", reports the decode throughput of
   this step).  In Kaczmarz mode beta carries eta and beta = eta / (||k||^2 +
   eps).
   p:   as for the chunkwise calls with T == 1 (chunk is not used but must be
        64); any other T gives DR_ERR_INVALID_ARG.
   In:  q, k [B,1,H,dk] and v [B,1,H,dv] in the storage dtype, beta [B,1,H]
        fp32, g [B,1,H] (scalar gate) or [B,1,H,dk] (per-channel or phase
        gate) fp32, NULL iff gate NONE.  With the phase gate, P is the
        rotation-decay of each key pair instead of S Diag(alpha).
   In/out: S [B,H,dv,dk] fp32, the state before the token on entry and after
        it on return (the caller owns it; it is updated in place).
   Out: o [B,1,H,dv] in the storage dtype.
   All pointers 16-byte aligned device memory; no workspace; asynchronous on
   `stream`.  Host-side argument errors return before any launch. */
dr_status dr_decode_step(const dr_problem* p, const void* q, const void* k, const void* v,
                         const float* beta, const float* g, float* S, void* o, void* stream);

/* Size of the library's built-in forward scratch (64 MiB), held on every GPU
   that loads the library, until the process exits. */
#define DR_STATIC_SCRATCH_BYTES (64u << 20)

/* Chunkwise forward that allocates nothing and takes no workspace, for
   callers that cannot call cudaMalloc (for example a plugin inside a host
   framework that owns all device memory through its own pool, or a
   latency-critical path that cannot afford cudaMalloc's implicit device
   synchronisation).  It has no counterpart in the paper.
   Same arguments and results as dr_chunk_fwd without saved and workspace:
   the scratch is a static device array of DR_STATIC_SCRATCH_BYTES shared by
   every call in the process.
   - Returns DR_ERR_WORKSPACE, launching nothing, when the problem's forward
     scratch exceeds DR_STATIC_SCRATCH_BYTES: the exact test is
     dr_workspace_size(p, 0) <= DR_STATIC_SCRATCH_BYTES.  With dk = dv = 128
     the forward keeps about 129 KiB per (batch x head x 64-token chunk)
     block, so about 500 blocks fit; a long sequence with few heads (which
     takes the chunk-parallel affine scan) also keeps 192 KiB per segment of
     each head.
   - Uses the device current at the call, which must own `stream` and every
     pointer.  The first call on a device looks up the scratch's device
     address (cudaGetSymbolAddress) with that device current; make that first
     call before any stream capture.
   - Calls that overlap on the GPU (for example on concurrent streams, or from
     several host threads using one device) race on the shared scratch:
     serialise them.  The
     scratch keeps the last call's contents; nothing in it needs clearing,
     because each call writes every scratch region before reading it. */
dr_status dr_chunk_fwd_static(const dr_problem* p, const void* q, const void* k,
                              const void* v, const float* beta, const float* g,
                              const float* S0, void* o, float* ST, void* stream);

/* Static, NUL-terminated description of a status code. */
const char* dr_status_string(dr_status s);

/* Synchronises `stream`, then reports and clears the device error flag:
   DR_ERR_TIMEOUT if a bounded device wait gave up since the last check,
   DR_ERR_CUDA if the stream reported an error, else DR_OK. */
dr_status dr_last_device_error(void* stream);

/* Fault injection, for testing the timeout path without faulting a GPU.
   Every wait of the library's tensor-core kernels on an mbarrier is bounded:
   when one gives up, the kernel records DR_ERR_TIMEOUT in the device flag
   that dr_last_device_error reports, lets its copies in flight land, frees
   its tensor memory and returns, leaving the context usable; its outputs are
   then undefined.  After dr_inject_timeout(n), each of the next n launches
   of the chunk backward kernel (inside dr_chunk_bwd) first waits, with a
   limit of a few hundred polls, on an mbarrier that nothing arrives on, once
   all its inputs have landed and before its first tensor-core instruction,
   and so takes that path.  n = 0 cancels pending injections; n < 0 gives
   DR_ERR_INVALID_ARG.  Process-wide, host only. */
dr_status dr_inject_timeout(int launches);

/* Opt-in per-kernel timing, for benchmarking.  While enabled (on != 0),
   every kernel the library launches is bracketed by two CUDA events recorded
   on the launch stream.  The first enable creates the events (no device
   memory is allocated); enabling or disabling discards pending records. */
dr_status dr_profile_enable(int on);

/* Per-kernel summary of the launches recorded since the last read or enable:
   name, launch count, summed event time, and the kernel's work model, the
   mean over its launches: bytes_per_launch counts the operator's own inputs
   and outputs that the launch reads or writes (q, k, v, g, beta, dO, o, the
   gradients and the states, each once: the algorithmic bytes);
   design_bytes_per_launch adds everything else the launch moves by this
   library's design (the per-chunk tiles and states kept between kernels);
   flops_per_launch is its arithmetic. */
typedef struct {
  char name[32];
  int launches;
  double ms_total;
  double bytes_per_launch;
  double flops_per_launch;
  double design_bytes_per_launch;
} dr_kernel_time;

/* Waits for the recorded events, writes up to max_out entries to out and
   returns their number (-1 on a CUDA error); clears the records. */
int dr_profile_read(dr_kernel_time* out, int max_out);

/* Library ABI version (major * 100 + minor): 200. */
int dr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DR_H */
