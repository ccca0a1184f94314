// fast_affine.cu -- composition of the per-segment affine maps of the
// chunk-parallel state scan (long sequences with few heads).
//
// The chunkwise forward transfers the state affinely chunk by chunk,
//   S_{n+1} = S_n P_n + B_n,   P_n = Diag(e^{gamma_C}) - W^T K~,   B_n = U'^T K~,
// (the exact affine chunk transfer of the chunkwise WY form), so a segment of
// chunks maps its start state to its end state by S_end = S_start P + B with
// P the product of its P_n and B the end state from a zero start.  The
// segmented scan computes (P, B) for every segment in parallel; these kernels
// chain them across the segments of each head:
//   Sst[0] = S0,  Sst[g + 1] = Sst[g] P_g + B_g,  S_T = Sst[G-1] P_{G-1} + B_{G-1}.
// The state gradient is transferred by the transposed maps,
//   dS_start = dS_end P^T + C   (C: the segment's gradient from a zero end gradient),
// so dSe[G-1] = dS_T, dSe[g-1] = dSe[g] P_g^T + C_g and dS0 = dSe[0] P_0^T + C_0.
// Rows of the state are independent: one CTA owns 16 rows of one head, fp32.

#include "dr_common.cuh"
#include "fast.cuh"

namespace dr {
namespace fast {
namespace {

constexpr int D = 128, RB = 16, NTA = 256;

__device__ __forceinline__ size_t map_off(const Problem& p, int G, int b, int g, int h) {
  return (((size_t)b * G + g) * p.H + h) * D * D;
}

__global__ void __launch_bounds__(NTA)
    k_affine_fwd(Problem p, int G, const float* __restrict__ S0, const float* __restrict__ P,
                 const float* __restrict__ Bm, float* __restrict__ Sst, float* __restrict__ ST) {
  __shared__ float rows[RB][D];
  const int r0 = blockIdx.x * RB, h = blockIdx.y, b = blockIdx.z;
  const int c = threadIdx.x & (D - 1), rh = threadIdx.x >> 7;  // column, which 8 rows
  const size_t head = ((size_t)b * p.H + h) * D * D;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int a = r0 + 8 * rh + r;
    const float x = S0 ? S0[head + (size_t)a * D + c] : 0.f;
    rows[8 * rh + r][c] = x;
    Sst[map_off(p, G, b, 0, h) + (size_t)a * D + c] = x;
  }
  __syncthreads();
  for (int g = 0; g < G; ++g) {
    const float* Pg = P + map_off(p, G, b, g, h);
    const float* Bg = Bm + map_off(p, G, b, g, h);
    float acc[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) acc[r] = Bg[(size_t)(r0 + 8 * rh + r) * D + c];
#pragma unroll 4
    for (int k = 0; k < D; ++k) {
      const float pk = Pg[(size_t)k * D + c];
#pragma unroll
      for (int r = 0; r < 8; ++r) acc[r] = fmaf(rows[8 * rh + r][k], pk, acc[r]);
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 8; ++r) rows[8 * rh + r][c] = acc[r];
    __syncthreads();
    float* dst = g + 1 < G ? Sst + map_off(p, G, b, g + 1, h) : (ST ? ST + head : nullptr);
    if (dst) {
#pragma unroll
      for (int r = 0; r < 8; ++r) dst[(size_t)(r0 + 8 * rh + r) * D + c] = acc[r];
    }
  }
}

// P_g^T is staged in shared memory (row stride D + 1) so that a thread's
// column of P is read without bank conflicts.
__global__ void __launch_bounds__(NTA)
    k_affine_bwd(Problem p, int G, const float* __restrict__ dST, const float* __restrict__ P,
                 const float* __restrict__ Cm, float* __restrict__ dSe, float* __restrict__ dS0) {
  extern __shared__ float sm[];
  float* Pt = sm;                       // [D][D + 1]: Pt[c][c'] = P[c'][c]
  float* rows = sm + D * (D + 1);       // [RB][D]
  const int r0 = blockIdx.x * RB, h = blockIdx.y, b = blockIdx.z;
  const int c = threadIdx.x & (D - 1), rh = threadIdx.x >> 7;
  const size_t head = ((size_t)b * p.H + h) * D * D;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int a = r0 + 8 * rh + r;
    const float x = dST ? dST[head + (size_t)a * D + c] : 0.f;
    rows[(8 * rh + r) * D + c] = x;
    dSe[map_off(p, G, b, G - 1, h) + (size_t)a * D + c] = x;
  }
  for (int g = G - 1; g >= 0; --g) {
    const float* Pg = P + map_off(p, G, b, g, h);
    for (int idx = threadIdx.x; idx < D * D; idx += NTA) {
      const int r = idx >> 7, cc = idx & (D - 1);
      Pt[cc * (D + 1) + r] = Pg[idx];
    }
    __syncthreads();
    const float* Cg = Cm + map_off(p, G, b, g, h);
    float acc[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) acc[r] = Cg[(size_t)(r0 + 8 * rh + r) * D + c];
#pragma unroll 4
    for (int k = 0; k < D; ++k) {
      const float pk = Pt[k * (D + 1) + c];  // P[c][k]
#pragma unroll
      for (int r = 0; r < 8; ++r) acc[r] = fmaf(rows[(8 * rh + r) * D + k], pk, acc[r]);
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 8; ++r) rows[(8 * rh + r) * D + c] = acc[r];
    float* dst = g > 0 ? dSe + map_off(p, G, b, g - 1, h) : (dS0 ? dS0 + head : nullptr);
    if (dst) {
#pragma unroll
      for (int r = 0; r < 8; ++r) dst[(size_t)(r0 + 8 * rh + r) * D + c] = acc[r];
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_affine_compose_fwd(const Problem& p, int G, const float* S0, const float* P,
                                      const float* Bm, float* Sst, float* ST, cudaStream_t st) {
  const double heads = (double)p.B * p.H;
  // reads S0, every P_g (once per 16-row block, mostly from L2) and B_g; writes Sst, ST
  const double bytes = heads * D * D * 4.0 * (1 + 2.0 * G + G + 1);
  const double io = heads * D * D * 4.0 * ((S0 ? 1 : 0) + (ST ? 1 : 0));
  prof_begin(kKAffine, io, bytes, heads * G * 2.0 * D * D * D, st);
  k_affine_fwd<<<dim3(D / RB, p.H, p.B), NTA, 0, st>>>(p, G, S0, P, Bm, Sst, ST);
  const cudaError_t e = cudaGetLastError();
  prof_end(st);
  return e;
}

cudaError_t launch_affine_compose_bwd(const Problem& p, int G, const float* dST, const float* P,
                                      const float* Cm, float* dSe, float* dS0, cudaStream_t st) {
  const size_t sm = sizeof(float) * (D * (D + 1) + RB * D);
  cudaError_t e =
      cudaFuncSetAttribute(k_affine_bwd, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const double heads = (double)p.B * p.H;
  const double bytes = heads * D * D * 4.0 * (1 + 2.0 * G + G + 1);
  const double io = heads * D * D * 4.0 * ((dST ? 1 : 0) + (dS0 ? 1 : 0));
  prof_begin(kKAffine, io, bytes, heads * G * 2.0 * D * D * D, st);
  k_affine_bwd<<<dim3(D / RB, p.H, p.B), NTA, sm, st>>>(p, G, dST, P, Cm, dSe, dS0);
  e = cudaGetLastError();
  prof_end(st);
  return e;
}

}  // namespace fast
}  // namespace dr
