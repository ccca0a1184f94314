// fast.cuh -- launchers of the tensor-core path (bf16 storage, d_k = d_v = 128).
#pragma once

#include "dr_common.cuh"

namespace dr {
namespace fast {

// True when the problem runs on the tensor-core path.
inline bool eligible(const Problem& p, int dtype_bf16) {
  return dtype_bf16 && p.dk == 128 && p.dv == 128;
}

// Per-chunk byte sizes of the tensors the fast path keeps between kernels.
constexpr size_t kTBytes = 64 * 64 * 2;        // (I + A)^{-1}, bf16
constexpr size_t kBetaBytes = 64 * 4;          // effective beta, fp32
constexpr size_t kStateBytes = 128 * 128 * 2;  // chunk start state / state gradient, bf16
constexpr size_t kUBytes = 64 * 128 * 2;       // pseudo-values U / dU, bf16

// Views of the forward-to-backward buffer (saved) or of scratch holding the
// same tensors: per chunk T, beta, start state h and U.
struct Saved {
  __nv_bfloat16* T;
  float* beta;
  __nv_bfloat16* h;
  __nv_bfloat16* U;
};
inline size_t saved_bytes(const Problem& p) {
  const size_t nb = (size_t)p.B * p.H * p.NC;
  return nb * (kTBytes + kBetaBytes + kStateBytes + kUBytes);
}
inline Saved carve_saved(const Problem& p, void* base) {
  const size_t nb = (size_t)p.B * p.H * p.NC;
  char* c = (char*)base;
  Saved s;
  s.T = (__nv_bfloat16*)c;
  s.beta = (float*)(c + nb * kTBytes);
  s.h = (__nv_bfloat16*)(c + nb * (kTBytes + kBetaBytes));
  s.U = (__nv_bfloat16*)(c + nb * (kTBytes + kBetaBytes + kStateBytes));
  return s;
}

cudaError_t launch_prep(const Problem& p, const __nv_bfloat16* k, const float* beta,
                        const float* g, __nv_bfloat16* T, float* beta_eff, cudaStream_t st);
cudaError_t launch_fwd_scan(const Problem& p, const __nv_bfloat16* q, const __nv_bfloat16* k,
                            const __nv_bfloat16* v, const float* g, const __nv_bfloat16* T,
                            const float* beta_eff, const float* S0, __nv_bfloat16* o,
                            float* ST, __nv_bfloat16* hsave, __nv_bfloat16* Usave,
                            cudaStream_t st);

cudaError_t launch_bwd_scan(const Problem& p, const __nv_bfloat16* q, const __nv_bfloat16* k,
                            const __nv_bfloat16* dO, const float* g, const __nv_bfloat16* T,
                            const float* beta_eff, const float* dST, float* dS0,
                            __nv_bfloat16* dU, __nv_bfloat16* dh, cudaStream_t st);
cudaError_t launch_bwd_chunk(const Problem& p, const __nv_bfloat16* q, const __nv_bfloat16* k,
                             const __nv_bfloat16* v, const __nv_bfloat16* dO, const float* g,
                             const __nv_bfloat16* T, const float* beta_eff,
                             const __nv_bfloat16* h, const __nv_bfloat16* dh,
                             const __nv_bfloat16* U, const __nv_bfloat16* dU,
                             __nv_bfloat16* dq, __nv_bfloat16* dk, __nv_bfloat16* dv,
                             float* dbeta, float* dg, cudaStream_t st);

// Backward scratch beyond the saved tensors: per chunk dU (bf16) and dh (bf16).
inline size_t bwd_extra_bytes(const Problem& p) {
  return (size_t)p.B * p.H * p.NC * (kUBytes + kStateBytes);
}

}  // namespace fast
}  // namespace dr
