// dr_common.cuh -- shared definitions of the CUDA library (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace dr {

constexpr int kC = 64;         // chunk length (tokens); the only supported value
constexpr int kThreads = 256;  // threads per CTA of the generic kernels

enum { kGateNone = 0, kGateScalar = 1, kGateChannel = 2, kGatePhase = 3 };
enum { kBetaDirect = 0, kBetaKaczmarz = 1 };

struct Problem {
  int B, H, T, dk, dv;
  int NC;         // number of chunks, ceil(T / 64)
  int gate;       // kGate* (kGatePhase: SFDA pairs, log alpha at 2j, theta at 2j + 1)
  int beta_mode;  // kBeta*
  int gk;         // columns of the cumulative gate per row: dk (per-channel) or 1
  float eps;
};

// Scratch regions carved out of the caller's workspace.  All fp32; per
// (b, h, chunk) block `cb = (b*H + h)*NC + n`:
//   gam [cb][C][gk]  inclusive within-chunk cumulative log-gate
//   beff[cb][C]      effective beta (Kaczmarz step applied), kn[cb][C] = ||k||^2
//   Tm  [cb][C][C]   (I + A)^{-1}, unit lower triangular
//   Mm  [cb][C][C]   inclusive-causal q-k gate-scaled Gram (output mask applied)
//   W   [cb][C][dk]  T diag(beta) K e^{gamma};  Up [cb][C][dv] = T diag(beta) V
//   U   [cb][C][dv]  Up - W S^T  (pseudo-values)
//   h   [cb][dv][dk] chunk start states;  dh [cb][dv][dk] = dL/d(chunk end state)
//   dU  [cb][C][dv]; dQs, dWs, dKt, dk_acc, dg_acc [cb][C][dk]; dgC [cb][dk]
struct Ws {
  float *gam, *beff, *kn, *Tm, *Mm, *W, *Up, *U, *h;
  float *dh, *dU, *dQs, *dWs, *dKt, *dgC, *dk_acc, *dg_acc;
};

__host__ __device__ inline size_t chunk_id(const Problem& p, int b, int h, int n) {
  return ((size_t)b * p.H + h) * p.NC + n;
}
__host__ __device__ inline size_t row_id(const Problem& p, int b, int t, int h) {
  return ((size_t)b * p.T + t) * p.H + h;
}

template <typename T>
__device__ __forceinline__ float load_f(const T* p);
template <>
__device__ __forceinline__ float load_f<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float load_f<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

template <typename T>
__device__ __forceinline__ void store_f(T* p, float x);
template <>
__device__ __forceinline__ void store_f<float>(float* p, float x) { *p = x; }
template <>
__device__ __forceinline__ void store_f<__nv_bfloat16>(__nv_bfloat16* p, float x) {
  *p = __float2bfloat16_rn(x);
}

// Kernel ids for the opt-in per-kernel timing (profile.cu).
enum {
  kKIntraFwd = 0, kKScanFwd, kKScanBwd, kKStateGrads, kKIntraBwd,
  kKTcIntraFwd, kKTcScanFwd, kKTcScanBwd, kKTcChunkBwd, kKDecode, kKAffine
};
const char* kernel_name(int id);
// Bracket one launch with events on its stream when profiling is enabled.
// io_bytes: the operator's own inputs and outputs that the launch reads or
// writes (q, k, v, g, beta, dO, o, the gradients, the states), each once: the
// algorithmic bytes.  bytes: everything the launch moves by this library's
// design, including the chunk tiles and states kept between kernels.
// flops: its arithmetic.
void prof_begin(int kernel, double io_bytes, double bytes, double flops, cudaStream_t st);
void prof_end(cudaStream_t st);

// Reads the device-side error word (bounded waits that gave up record a
// nonzero code there) into *flag and clears it.
cudaError_t read_and_clear_device_error(int* flag);
// Device address of that error word on the current device (nullptr on failure).
int* device_error_word();
// Streaming multiprocessors of the current device (cached per device; 148 on B200).
int sm_count();
// Fault injection (dr_inject_timeout): true, and one fewer pending, if the
// next chunk-backward launch is to take its bounded-wait timeout path.
bool take_injected_timeout();

// Launchers of the generic (fp32 SIMT) kernels; TIn is float or __nv_bfloat16.
template <typename TIn>
cudaError_t launch_generic_fwd(const Problem& p, const TIn* q, const TIn* k, const TIn* v,
                               const float* beta, const float* g, const float* S0, TIn* o,
                               float* ST, float* hsave, const Ws& ws, cudaStream_t st);

template <typename TIn>
cudaError_t launch_generic_bwd(const Problem& p, const TIn* q, const TIn* k, const TIn* v,
                               const float* beta, const float* g, const float* S0,
                               const TIn* dO, const float* dST, const float* hsaved,
                               TIn* dq, TIn* dk, TIn* dv, float* dbeta, float* dg,
                               float* dS0, const Ws& ws, cudaStream_t st);

// The single-token recurrent step (decode.cu); bf16 != 0 for bf16 q, k, v, o.
cudaError_t launch_decode_step(const Problem& p, int bf16, const void* q, const void* k,
                               const void* v, const float* beta, const float* g, float* S, void* o,
                               cudaStream_t st);

}  // namespace dr
