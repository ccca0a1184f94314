// tc.cuh -- sm_100a tensor-core helpers: tcgen05 MMA with shared-memory
// operands and tensor-memory (TMEM) accumulators, mbarriers with bounded
// waits, bulk copies.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace dr {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// --- canonical no-swizzle shared-memory layouts for UMMA operands ----------
// A "core matrix" is 8 rows x 16 bytes (8 bf16) stored as 128 contiguous
// bytes.  K-major tile [R x K] (K contiguous in the logical matrix): core
// (r/8, k/8) at ((r/8) * (K/8) + k/8) * 128 bytes, element at (r%8)*16 +
// (k%8)*2 inside it.  LBO = 128 (next core along K), SBO = (K/8) * 128 (next
// 8-row group).  MN-major tile [K x N] (N contiguous): core (k/8, n/8) at
// ((k/8) * (N/8) + n/8) * 128 bytes, element at (k%8)*16 + (n%8)*2; SBO = 128
// (next 8-column group along N), LBO = (N/8) * 128 (next 8-row group along K).
__device__ __forceinline__ int kmaj_off(int r, int k, int K) {
  return ((r >> 3) * (K >> 3) + (k >> 3)) * 64 + (r & 7) * 8 + (k & 7);  // in bf16 elements
}
__device__ __forceinline__ int mnmaj_off(int k, int n, int N) {
  return ((k >> 3) * (N >> 3) + (n >> 3)) * 64 + (k & 7) * 8 + (n & 7);  // in bf16 elements
}

// cp.async of a row-major [R][NCOL] bf16 global tile (row stride ld elements)
// into the core-matrix layout above (K-major [R x K=NCOL], or MN-major
// [K=R x N=NCOL]: both place element (r, c) at ((r/8)*(NCOL/8) + c/8)*64 +
// (r%8)*8 + c%8).  16-byte chunk idx goes to shared offset 16*idx, so eight
// consecutive lanes fill one core matrix (128 contiguous bytes, no bank
// conflicts) while a warp reads 8 rows x 64 contiguous bytes of the source.
// Rows at or beyond valid_rows are zero-filled.
template <int NTHREADS>
__device__ __forceinline__ void cp_core_tile(__nv_bfloat16* tile, const __nv_bfloat16* g,
                                             size_t ld, int R, int NCOL, int valid_rows,
                                             int tid) {
  const int cpr = NCOL >> 3;  // core matrices per row group
  for (int idx = tid; idx < R * cpr; idx += NTHREADS) {
    const int core = idx >> 3, rr = idx & 7;
    const int r = (core / cpr) * 8 + rr, c = (core % cpr) * 8;
    const bool ok = r < valid_rows;
    const __nv_bfloat16* src = g + (size_t)(ok ? r : 0) * ld + c;
    const uint32_t dst = smem_u32(tile + 8 * idx);
    const int n = ok ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n)
                 : "memory");
  }
}

// Shared-memory matrix descriptor (sm100 format, no swizzle).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm100
  return d;
}
// Descriptor of the K-step `ks` (16 elements) of a K-major tile with K columns.
__device__ __forceinline__ uint64_t sdesc_kmaj(const __nv_bfloat16* tile, int K, int ks) {
  return sdesc(smem_u32(tile) + ks * 256, 128, (K >> 3) * 128);
}
// Descriptor of the K-step `ks` (16 rows) of an MN-major tile with N columns.
__device__ __forceinline__ uint64_t sdesc_mnmaj(const __nv_bfloat16* tile, int N, int ks) {
  return sdesc(smem_u32(tile) + ks * 2 * (N >> 3) * 128, (N >> 3) * 128, 128);
}

// Instruction descriptor, kind::f16 with bf16 A/B and an fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
         ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]; issued by one thread.
__device__ __forceinline__ void mma(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                    uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}
// Arrive on the mbarrier once every MMA this thread issued so far completes.
__device__ __forceinline__ void commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Make generic-proxy shared-memory writes visible to the tensor core.
__device__ __forceinline__ void fence_smem_to_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
// Makes mbarrier initialisation visible to the async proxy (bulk copies,
// tcgen05.commit) before the barrier that follows it.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Bounded wait on phase `parity`; returns false if it gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t max_iters) {
  for (uint32_t it = 0; it < max_iters; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}

// Arrive on the mbarrier (the phase's single arrival) and add `bytes` to the
// transaction count the bulk copies below must deliver before the phase ends.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// Bulk copy (TMA engine, no tensor map, this CTA as the only destination) of
// `bytes` contiguous bytes global -> shared memory, completing on `bar`.  Both
// addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Prefetch `bytes` contiguous bytes of global memory into L2 (no shared-memory
// destination, no completion to wait for).  16-byte aligned, a multiple of 16.
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// TMEM allocation (one warp); the base address is written to *dst in smem.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// 16 consecutive fp32 columns of this thread's TMEM lane (warp w reads lanes
// 32*(w%4) .. 32*(w%4)+31; taddr carries the lane in bits 31:16).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// The same without the wait: issue several, then tmem_wait_ld() once before
// the registers are read.
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

}  // namespace tc
}  // namespace dr
