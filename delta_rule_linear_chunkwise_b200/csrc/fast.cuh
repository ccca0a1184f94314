// fast.cuh -- launchers of the tensor-core path (bf16 storage, d_k = d_v = 128).
#pragma once

#include "dr_common.cuh"
#include "frag.cuh"

namespace dr {
namespace fast {

// True when the problem runs on the tensor-core path.
inline bool eligible(const Problem& p, int dtype_bf16) {
  return dtype_bf16 && p.dk == 128 && p.dv == 128;
}

// Segmented scans (the chunk-parallel affine scan for long sequences with few
// heads): the chunks of a head are split into G segments of L chunks and one
// CTA runs one segment (blockIdx.z = b * G + segment).
//   forward  mode 0: the output scan from the given segment start states;
//            mode 1: the segment's transfer matrix P (start I, U' = 0);
//            mode 2: its offset B (start 0), so that S_end = S_start P + B.
//   backward mode 0: the gradient scan from the given segment end gradients;
//            mode 1: the segment's offset C (end gradient 0), so that
//            dS_start = dS_end P^T + C.
//   forward  mode 3: modes 1 and 2 in one launch (blockIdx.x selects), the
//            transfer matrices to ST and the offsets to ST2.
struct ScanSeg {
  int G, L, mode;
  const float* S0;  // [B][G][H][128][128] start states (forward) / end gradients (backward)
  float* ST;        // [B][G][H][128][128] end states (forward) / start gradients (backward)
  float* ST2;       // mode 3: the offsets
};

// Number of sequence segments for the affine scan (1 = plain sequential scans):
// used when the plain scans would occupy at most half of the 148 SMs and the
// sequence is long, with as many segments as fill one wave.
inline int affine_segments(const Problem& p) {
  const long ctas = (long)p.B * p.H * 2;  // plain scans: two 64-row value tiles per head
  if (ctas > 74 || p.NC < 64) return 1;
  int G = (int)(148 / ctas);
  if (G > 16) G = 16;
  const int L = (p.NC + G - 1) / G;
  return (p.NC + L - 1) / L;
}
inline int affine_seg_len(const Problem& p, int G) { return (p.NC + G - 1) / G; }
// Bytes of one [B][G][H][128][128] fp32 buffer of segment maps or states.
inline size_t affine_map_bytes(const Problem& p, int G) {
  return G > 1 ? (size_t)p.B * G * p.H * 128 * 128 * 4 : 0;
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
// states and pseudo-values written by the forward scan, all core-tiled (see
// ct_off); the backward scan's dU and dh use the same layout.
struct Saved {
  __nv_bfloat16* T;    // [nb][64][64]    (I + A)^{-1}                         [ct]
  float* beta;         // [nb][64]        beta (Kaczmarz step applied)
  float* dec;          // [nb][128]       e^{gamma_C}
  __nv_bfloat16* W;    // [nb][64][128]   T diag(beta) k e^gamma               [ct]
  __nv_bfloat16* Up;   // [nb][64][128]   T diag(beta) v                       [ct]
  __nv_bfloat16* M;    // [nb][64][64]    tril(Q^c Kb^c^T)                     [ct]
  __nv_bfloat16* Qh;   // [nb][64][128]   q e^gamma                            [ct]
  __nv_bfloat16* Kt;   // [nb][64][128]   k e^{gamma_C - gamma}                [ct]
  __nv_bfloat16* h;    // [nb][128][128]  chunk start state S [c][a]             [ct]
  __nv_bfloat16* U;    // [nb][64][128]   U = U' - W S^T                       [ct]
  float* knorm;        // [nb][64]        ||k||^2 of each row
  float* Pseg;         // [B][G][H][128][128] segment transfer matrices (affine scan; else null)
};

// Core-tiled storage of an [R][ncol] bf16 tile: 8 x 8 blocks of 128
// contiguous bytes in row-block-major order, element (r, c) at ct_off.  It is
// the tcgen05 no-swizzle operand layout, so such a tile moves between HBM and
// shared memory as one contiguous block; 16-byte chunk idx holds row
// ct_row(idx), columns ct_col(idx) .. + 7.
__host__ __device__ __forceinline__ size_t ct_off(int r, int c, int ncol) {
  return ((size_t)(r >> 3) * (ncol >> 3) + (c >> 3)) * 64 + (r & 7) * 8 + (c & 7);
}
__host__ __device__ __forceinline__ int ct_row(int idx, int ncol) {
  return ((idx >> 3) / (ncol >> 3)) * 8 + (idx & 7);
}
__host__ __device__ __forceinline__ int ct_col(int idx, int ncol) {
  return ((idx >> 3) % (ncol >> 3)) * 8;
}

// Columns c0 .. c0 + w - 1 of a core-tiled [R][128] tile into a core-tiled
// [R][w] shared tile.
template <int NTHREADS>
__device__ __forceinline__ void cp_ct_cols(__nv_bfloat16* smem, const __nv_bfloat16* g, int R,
                                           int c0, int w, int tid) {
  for (int idx = tid; idx < R * w / 8; idx += NTHREADS) {
    const int grp = idx / w, k = idx % w;
    frag::cp16(smem + (size_t)grp * w * 8 + 8 * k, g + ((size_t)grp * 16 + (c0 >> 3)) * 64 + 8 * k,
               true);
  }
}
// A contiguous copy of `elems` bf16 (a multiple of 8).
template <int NTHREADS>
__device__ __forceinline__ void cp_linear(__nv_bfloat16* smem, const __nv_bfloat16* g, int elems,
                                          int tid) {
  for (int idx = tid; idx < elems / 8; idx += NTHREADS) frag::cp16(smem + 8 * idx, g + 8 * idx, true);
}
inline size_t saved_bytes(const Problem& p) {
  const size_t nb = (size_t)p.B * p.H * p.NC;
  return nb * (kTBytes + 2 * kBetaBytes + kDecBytes + 4 * kTileBytes + kMBytes + kStateBytes +
               kUBytes) +
         affine_map_bytes(p, affine_segments(p));
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
  s.knorm = (float*)c;                c += nb * kBetaBytes;
  s.Pseg = affine_segments(p) > 1 ? (float*)c : nullptr;
  return s;
}

// tc_prep (fast_prep.cu): all state-independent per-chunk tensors (T, beta,
// dec, W, U', M, Qh, Kt, ||k||^2), on tcgen05 with TMA loads.
cudaError_t launch_prep(const Problem& p, const __nv_bfloat16* q, const __nv_bfloat16* k,
                        const __nv_bfloat16* v, const float* beta, const float* g,
                        const Saved& sv, cudaStream_t st);
cudaError_t launch_fwd_scan_tc(const Problem& p, const Saved& sv, const float* S0,
                               __nv_bfloat16* o, float* ST, bool save, cudaStream_t st);
// Segmented forms (see ScanSeg); bv = 64 or 128 value rows per CTA.
cudaError_t launch_fwd_scan_tc_seg(const Problem& p, const Saved& sv, const ScanSeg& sg,
                                   __nv_bfloat16* o, bool save, int bv, cudaStream_t st);
cudaError_t launch_bwd_scan_tc_seg(const Problem& p, const Saved& sv, const __nv_bfloat16* dO,
                                   const ScanSeg& sg, __nv_bfloat16* dU, __nv_bfloat16* dh,
                                   int bv, cudaStream_t st);
// Composition of the segment maps (fast_affine.cu).
//   forward:  Sst[0] = S0 (or 0); Sst[g+1] = Sst[g] P[g] + Bm[g]; ST = Sst[G-1] P + Bm
//   backward: dSe[G-1] = dST (or 0); dSe[g-1] = dSe[g] P[g]^T + Cm[g];
//             dS0 = dSe[0] P[0]^T + Cm[0]
cudaError_t launch_affine_compose_fwd(const Problem& p, int G, const float* S0, const float* P,
                                      const float* Bm, float* Sst, float* ST, cudaStream_t st);
cudaError_t launch_affine_compose_bwd(const Problem& p, int G, const float* dST, const float* P,
                                      const float* Cm, float* dSe, float* dS0, cudaStream_t st);
cudaError_t launch_bwd_scan_tc(const Problem& p, const Saved& sv, const __nv_bfloat16* dO,
                               const float* dST, float* dS0, __nv_bfloat16* dU,
                               __nv_bfloat16* dh, cudaStream_t st);
// The chunk-parallel backward: products on tcgen05, element-wise work on 16 warps.
cudaError_t launch_bwd_chunk_hy(const Problem& p, const __nv_bfloat16* q,
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
