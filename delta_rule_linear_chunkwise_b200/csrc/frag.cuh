// frag.cuh -- bf16 packing, the warp-level accumulator fragment store,
// cp.async staging and small element-wise helpers shared by the tensor-core
// kernels.
//
// Accumulator fragments (the register layout tcgen05.ld.16x256b returns for an
// M = 64 accumulator, the same as a warp-level m16n8 product's C):
//   c0,c1 (r, c..c+1) c2,c3 (r+8, c..c+1), with r = lane/4, c = 2*(lane%4).
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

// Element (r, c) of a shared tile with leading dimension ld: row-major with
// row stride ld when ld > 0; when ld < 0, core-tiled with -ld columns (8 x 8
// blocks of 128 contiguous bytes, row-block-major), the layout the tcgen05
// operands and the saved chunk tiles use.
__device__ __forceinline__ int toff(int r, int c, int ld) {
  return ld > 0 ? r * ld + c : (((r >> 3) * ((-ld) >> 3) + (c >> 3)) * 64 + (r & 7) * 8 + (c & 7));
}

// stmatrix / ldmatrix of four 8 x 8 bf16 matrices: lanes 8 m .. 8 m + 7 give the
// row addresses (16 bytes each) of matrix m; register m of thread t holds the
// pair (row t / 4, columns 2 (t % 4), + 1) of matrix m -- the accumulator
// fragment layout above.
__device__ __forceinline__ void stm_x4(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2,
                                       uint32_t r3) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr),
               "r"(r0), "r"(r1), "r"(r2), "r"(r3)
               : "memory");
}
__device__ __forceinline__ void ldm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}

// Store accumulators (rows r0 .. r0 + 15, cols n0 .. n0 + 8 NT - 1) as bf16 into
// a tile (toff layout); a core-tiled tile takes whole 8 x 8 matrices by
// stmatrix (each is one 128-byte core matrix).
template <int NT>
__device__ __forceinline__ void st_c(const float (&c)[NT][4], bf16* t, int ld, int r0, int n0 = 0) {
  const int l = threadIdx.x & 31;
  if (ld < 0 && NT % 2 == 0) {
    // matrices of one stmatrix: (r0, j), (r0 + 8, j), (r0, j + 1), (r0 + 8, j + 1)
    const int m = l >> 3, rr = r0 + (l & 7) + ((m & 1) ? 8 : 0);
#pragma unroll
    for (int j = 0; j < NT; j += 2)
      stm_x4(tc::smem_u32(t + toff(rr, n0 + 8 * (j + (m >> 1)), ld)), pack(c[j][0], c[j][1]),
             pack(c[j][2], c[j][3]), pack(c[j + 1][0], c[j + 1][1]), pack(c[j + 1][2], c[j + 1][3]));
    return;
  }
  const int r = r0 + (l >> 2), cc = n0 + 2 * (l & 3);
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    *reinterpret_cast<uint32_t*>(t + toff(r, cc + j * 8, ld)) = pack(c[j][0], c[j][1]);
    *reinterpret_cast<uint32_t*>(t + toff(r + 8, cc + j * 8, ld)) = pack(c[j][2], c[j][3]);
  }
}

// 2^x (the ex2.approx.ftz instruction: relative error about 2^-22, flushes
// results below the normal range to zero)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
constexpr float kLog2e = 1.4426950408889634f;

// Eight consecutive floats of a 16-byte aligned shared-memory array.
__device__ __forceinline__ void load8(const float* p, float* f) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x, f[1] = a.y, f[2] = a.z, f[3] = a.w, f[4] = b.x, f[5] = b.y, f[6] = b.z, f[7] = b.w;
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

// 4 x 4 transpose of 32-bit words across the four lanes of a quad (lq = lane % 4):
// on entry lane lq holds a[j] = element (lq, j), on exit a[j] = element (j, lq).
// Two exchange rounds (lane masks 1 and 2), two shuffles each; every lane of the
// warp takes part.
__device__ __forceinline__ void quad_transpose(uint32_t (&a)[4], int lq) {
#pragma unroll
  for (int m = 1; m <= 2; m <<= 1)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (j & m) continue;
      const uint32_t send = (lq & m) ? a[j] : a[j | m];
      const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, m);
      if (lq & m)
        a[j] = recv;
      else
        a[j | m] = recv;
    }
}

}  // namespace frag
}  // namespace dr
