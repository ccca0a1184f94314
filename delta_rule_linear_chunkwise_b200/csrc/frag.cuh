// frag.cuh -- warp-level bf16 tensor-core tiles (mma.sync m16n8k16) for the
// latency-bound chains of the fast path, plus cp.async staging.
//
// Shared-memory tiles are row-major bf16 with a padded row stride (row length
// + 8 elements) so that the eight 16-byte rows an ldmatrix phase touches fall
// in distinct banks.  Fragment conventions (PTX ISA, m16n8k16 .bf16):
//   A (16x16): a0 (r, c..c+1) a1 (r+8, c..) a2 (r, c+8..) a3 (r+8, c+8..)
//   B (16x8):  b0 (k..k+1, n) b1 (k+8.., n)
//   C (16x8):  c0,c1 (r, c..c+1) c2,c3 (r+8, c..c+1)
// with r = lane/4, c = 2*(lane%4), k = 2*(lane%4), n = lane/4.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "tc.cuh"

namespace dr {
namespace frag {

using bf16 = __nv_bfloat16;

__device__ __forceinline__ uint32_t pack(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack(uint32_t x) {
  __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&x);
  return __bfloat1622float2(v);
}

__device__ __forceinline__ void ldsm_x4(uint32_t* r, const bf16* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(tc::smem_u32(p))
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t* r, const bf16* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(tc::smem_u32(p))
               : "memory");
}

// Element (r, c) of a shared tile with leading dimension ld: row-major with
// row stride ld when ld > 0; when ld < 0, core-tiled with -ld columns (8 x 8
// blocks of 128 contiguous bytes, row-block-major), the layout the tcgen05
// operands and the saved chunk tiles use.  ldmatrix reads one such block per
// 8 x 8 matrix, so the core-tiled form needs no padding against bank
// conflicts.  c is a multiple of 8 wherever 16 contiguous bytes are addressed.
__device__ __forceinline__ int toff(int r, int c, int ld) {
  return ld > 0 ? r * ld + c : (((r >> 3) * ((-ld) >> 3) + (c >> 3)) * 64 + (r & 7) * 8 + (c & 7));
}

// A fragment of rows r0..r0+15, cols k0..k0+15 of a row-major tile.
__device__ __forceinline__ void ld_a(uint32_t* a, const bf16* t, int ld, int r0, int k0) {
  const int l = threadIdx.x & 31;
  ldsm_x4(a, t + toff(r0 + (l & 7) + ((l >> 3) & 1) * 8, k0 + (l >> 4) * 8, ld));
}
// A fragment of X^T (rows m0.., cols k0..) where X is stored row-major [k][m].
__device__ __forceinline__ void ld_at(uint32_t* a, const bf16* x, int ld, int m0, int k0) {
  const int l = threadIdx.x & 31;
  ldsm_x4_t(a, x + toff(k0 + (l & 7) + (l >> 4) * 8, m0 + ((l >> 3) & 1) * 8, ld));
}
// B fragments of two n-tiles (n0, n0+8), k0..k0+15, B stored as [n][k].
// b[0..1] -> n-tile n0, b[2..3] -> n-tile n0+8.
__device__ __forceinline__ void ld_b_nk(uint32_t* b, const bf16* t, int ld, int n0, int k0) {
  const int l = threadIdx.x & 31;
  ldsm_x4(b, t + toff(n0 + (l & 7) + (l >> 4) * 8, k0 + ((l >> 3) & 1) * 8, ld));
}
// B fragments of two n-tiles, B stored as [k][n] (n contiguous).
__device__ __forceinline__ void ld_b_kn(uint32_t* b, const bf16* t, int ld, int k0, int n0) {
  const int l = threadIdx.x & 31;
  ldsm_x4_t(b, t + toff(k0 + (l & 7) + ((l >> 3) & 1) * 8, n0 + (l >> 4) * 8, ld));
}

// A fragment for k-step ks from accumulators of n-tiles 2ks, 2ks+1.
template <int NT>
__device__ __forceinline__ void c_to_a(const float (&c)[NT][4], int ks, uint32_t* a) {
  a[0] = pack(c[2 * ks][0], c[2 * ks][1]);
  a[1] = pack(c[2 * ks][2], c[2 * ks][3]);
  a[2] = pack(c[2 * ks + 1][0], c[2 * ks + 1][1]);
  a[3] = pack(c[2 * ks + 1][2], c[2 * ks + 1][3]);
}

template <int NT>
__device__ __forceinline__ void zero(float (&c)[NT][4]) {
#pragma unroll
  for (int j = 0; j < NT; ++j) c[j][0] = c[j][1] = c[j][2] = c[j][3] = 0.f;
}

// acc[16 x 8NT] += A[16 x 16KS] * B, A rows r0.. of a row-major tile.
template <int NT, int KS, bool B_KN>
__device__ __forceinline__ void mm_rows(float (&acc)[NT][4], const bf16* A, int lda, int r0,
                                        const bf16* B, int ldb, int n0 = 0, int k0 = 0) {
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    uint32_t a[4];
    ld_a(a, A, lda, r0, k0 + ks * 16);
#pragma unroll
    for (int j = 0; j < NT; j += 2) {
      uint32_t b[4];
      if (B_KN)
        ld_b_kn(b, B, ldb, k0 + ks * 16, n0 + j * 8);
      else
        ld_b_nk(b, B, ldb, n0 + j * 8, k0 + ks * 16);
      tc::mma16816(acc[j], a, b);
      tc::mma16816(acc[j + 1], a, b + 2);
    }
  }
}
// Two products sharing the B operand: acc1 += A1 B, acc2 += A2 B (rows r0..).
template <int NT, int KS, bool B_KN>
__device__ __forceinline__ void mm_rows2(float (&acc1)[NT][4], float (&acc2)[NT][4],
                                         const bf16* A1, const bf16* A2, int lda, int r0,
                                         const bf16* B, int ldb, int n0 = 0, int k0 = 0) {
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    uint32_t a1[4], a2[4];
    ld_a(a1, A1, lda, r0, k0 + ks * 16);
    ld_a(a2, A2, lda, r0, k0 + ks * 16);
#pragma unroll
    for (int j = 0; j < NT; j += 2) {
      uint32_t b[4];
      if (B_KN)
        ld_b_kn(b, B, ldb, k0 + ks * 16, n0 + j * 8);
      else
        ld_b_nk(b, B, ldb, n0 + j * 8, k0 + ks * 16);
      tc::mma16816(acc1[j], a1, b);
      tc::mma16816(acc1[j + 1], a1, b + 2);
      tc::mma16816(acc2[j], a2, b);
      tc::mma16816(acc2[j + 1], a2, b + 2);
    }
  }
}
// Same with A = X^T, X stored row-major [k][m].
template <int NT, int KS, bool B_KN>
__device__ __forceinline__ void mm_rows_at(float (&acc)[NT][4], const bf16* X, int ldx, int m0,
                                           const bf16* B, int ldb, int n0 = 0, int k0 = 0) {
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    uint32_t a[4];
    ld_at(a, X, ldx, m0, k0 + ks * 16);
#pragma unroll
    for (int j = 0; j < NT; j += 2) {
      uint32_t b[4];
      if (B_KN)
        ld_b_kn(b, B, ldb, k0 + ks * 16, n0 + j * 8);
      else
        ld_b_nk(b, B, ldb, n0 + j * 8, k0 + ks * 16);
      tc::mma16816(acc[j], a, b);
      tc::mma16816(acc[j + 1], a, b + 2);
    }
  }
}
// Same with A given as register fragments (KS k-steps of 4 registers).
template <int NT, int KS, bool B_KN>
__device__ __forceinline__ void mm_regs(float (&acc)[NT][4], const uint32_t (&a)[KS][4],
                                        const bf16* B, int ldb, int n0 = 0, int k0 = 0) {
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
    for (int j = 0; j < NT; j += 2) {
      uint32_t b[4];
      if (B_KN)
        ld_b_kn(b, B, ldb, k0 + ks * 16, n0 + j * 8);
      else
        ld_b_nk(b, B, ldb, n0 + j * 8, k0 + ks * 16);
      tc::mma16816(acc[j], a[ks], b);
      tc::mma16816(acc[j + 1], a[ks], b + 2);
    }
  }
}

// Store accumulators (rows r0.., cols n0..) as bf16 into a row-major tile.
template <int NT>
__device__ __forceinline__ void st_c(const float (&c)[NT][4], bf16* t, int ld, int r0, int n0 = 0) {
  const int l = threadIdx.x & 31;
  const int r = r0 + (l >> 2), cc = n0 + 2 * (l & 3);
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    *reinterpret_cast<uint32_t*>(t + toff(r, cc + j * 8, ld)) = pack(c[j][0], c[j][1]);
    *reinterpret_cast<uint32_t*>(t + toff(r + 8, cc + j * 8, ld)) = pack(c[j][2], c[j][3]);
  }
}

// tf32 m16n8k8 (fp32 accumulate) for the fp32 block products of the solve.
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void mma1688_tf32(float* d, const uint32_t* a, const uint32_t* b) {
  asm(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// acc[16 x 16] += A[r0.., k0..k0+K) * B[k0.., n0..n0+16) with fp32 row-major
// shared tiles (A stride lda, B stride ldb), K a multiple of 8.
__device__ __forceinline__ void mm16x16_tf32(float (&acc)[2][4], const float* A, int lda, int r0,
                                             const float* B, int ldb, int n0, int k0, int K) {
  const int l = threadIdx.x & 31, g = l >> 2, t = l & 3;
  for (int k = k0; k < k0 + K; k += 8) {
    uint32_t a[4] = {to_tf32(A[(r0 + g) * lda + k + t]), to_tf32(A[(r0 + g + 8) * lda + k + t]),
                     to_tf32(A[(r0 + g) * lda + k + t + 4]),
                     to_tf32(A[(r0 + g + 8) * lda + k + t + 4])};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      uint32_t b[2] = {to_tf32(B[(k + t) * ldb + n0 + nt * 8 + g]),
                       to_tf32(B[(k + t + 4) * ldb + n0 + nt * 8 + g])};
      mma1688_tf32(acc[nt], a, b);
    }
  }
}

// cp.async 16-byte copy (zero-filled when !valid).
__device__ __forceinline__ void cp16(void* smem, const void* gmem, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(tc::smem_u32(smem)),
               "l"(gmem), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

}  // namespace frag
}  // namespace dr
