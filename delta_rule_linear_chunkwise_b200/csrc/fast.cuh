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
constexpr size_t kDecBytes = 128 * 4;          // chunk decay e^{gamma_C}, fp32
constexpr size_t kTileBytes = 64 * 128 * 2;    // a 64 x 128 bf16 chunk tile
constexpr size_t kMBytes = 64 * 64 * 2;        // M = tril(Q^c Kb^c^T), bf16
constexpr size_t kStateBytes = 128 * 128 * 2;  // chunk start state / state gradient, bf16
constexpr size_t kUBytes = kTileBytes;         // pseudo-values U / dU, bf16

// The per-chunk tensors of the forward that the backward reuses ("saved"):
// the state-independent chunk tiles written by tc_prep and the chunk start
// states and pseudo-values written by the forward scan.  All row-major.
struct Saved {
  __nv_bfloat16* T;    // [nb][64][64]    (I + A)^{-1}
  float* beta;         // [nb][64]        beta (Kaczmarz step applied)
  float* dec;          // [nb][128]       e^{gamma_C}
  __nv_bfloat16* W;    // [nb][64][128]   T diag(beta) k e^gamma
  __nv_bfloat16* Up;   // [nb][64][128]   T diag(beta) v
  __nv_bfloat16* M;    // [nb][64][64]    tril(Q^c Kb^c^T)
  __nv_bfloat16* Qh;   // [nb][64][128]   q e^gamma
  __nv_bfloat16* Kt;   // [nb][64][128]   k e^{gamma_C - gamma}
  __nv_bfloat16* h;    // [nb][128][128]  chunk start state S (value-major)
  __nv_bfloat16* U;    // [nb][64][128]   U = U' - W S^T
  float* knorm;        // [nb][64]        ||k||^2 of each row
};
inline size_t saved_bytes(const Problem& p) {
  const size_t nb = (size_t)p.B * p.H * p.NC;
  return nb * (kTBytes + 2 * kBetaBytes + kDecBytes + 4 * kTileBytes + kMBytes + kStateBytes +
               kUBytes);
}
inline Saved carve_saved(const Problem& p, void* base) {
  const size_t nb = (size_t)p.B * p.H * p.NC;
  char* c = (char*)base;
  Saved s;
  s.T = (__nv_bfloat16*)c;            c += nb * kTBytes;
  s.beta = (float*)c;                 c += nb * kBetaBytes;
  s.dec = (float*)c;                  c += nb * kDecBytes;
  s.W = (__nv_bfloat16*)c;            c += nb * kTileBytes;
  s.Up = (__nv_bfloat16*)c;           c += nb * kTileBytes;
  s.M = (__nv_bfloat16*)c;            c += nb * kMBytes;
  s.Qh = (__nv_bfloat16*)c;           c += nb * kTileBytes;
  s.Kt = (__nv_bfloat16*)c;           c += nb * kTileBytes;
  s.h = (__nv_bfloat16*)c;            c += nb * kStateBytes;
  s.U = (__nv_bfloat16*)c;             c += nb * kUBytes;
  s.knorm = (float*)c;
  return s;
}

// tc_prep: all state-independent per-chunk tensors (T, beta, dec, W, U', M, Qh, Kt).
cudaError_t launch_prep(const Problem& p, const __nv_bfloat16* q, const __nv_bfloat16* k,
                        const __nv_bfloat16* v, const float* beta, const float* g,
                        const Saved& sv, cudaStream_t st);
// tc_fwd_scan: state chain, output and (when sv.h / sv.U are non-null) the
// chunk start states and pseudo-values.
cudaError_t launch_fwd_scan(const Problem& p, const Saved& sv, const float* S0,
                            __nv_bfloat16* o, float* ST, bool save, cudaStream_t st);
cudaError_t launch_bwd_scan(const Problem& p, const Saved& sv, const __nv_bfloat16* dO,
                            const float* dST, float* dS0, __nv_bfloat16* dU,
                            __nv_bfloat16* dh, cudaStream_t st);
cudaError_t launch_bwd_chunk(const Problem& p, const __nv_bfloat16* q, const __nv_bfloat16* k,
                             const __nv_bfloat16* v, const __nv_bfloat16* dO, const float* g,
                             const Saved& sv, const __nv_bfloat16* dh,
                             const __nv_bfloat16* dU, __nv_bfloat16* dq, __nv_bfloat16* dk,
                             __nv_bfloat16* dv, float* dbeta, float* dg, cudaStream_t st);

cudaError_t launch_bwd_chunk_tc(const Problem& p, const __nv_bfloat16* q,
                                const __nv_bfloat16* k, const __nv_bfloat16* v,
                                const __nv_bfloat16* dO, const float* g, const Saved& sv,
                                const __nv_bfloat16* dh, const __nv_bfloat16* dU,
                                __nv_bfloat16* dq, __nv_bfloat16* dk, __nv_bfloat16* dv,
                                float* dbeta, float* dg, cudaStream_t st);

// Backward scratch beyond the saved tensors: per chunk dU (bf16) and dh (bf16).
inline size_t bwd_extra_bytes(const Problem& p) {
  return (size_t)p.B * p.H * p.NC * (kUBytes + kStateBytes);
}

}  // namespace fast
}  // namespace dr
