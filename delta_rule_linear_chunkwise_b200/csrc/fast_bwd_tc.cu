// fast_bwd_tc.cu -- chunk-parallel backward on tcgen05 tensor cores (bf16
// storage, d_k = d_v = 128, C = 64): one CTA per (b, h, chunk), 256 threads.
//
// Every product is a tcgen05.mma (M = 64, bf16 operands in shared memory in the
// canonical no-swizzle core-matrix layouts, fp32 accumulators in tensor memory)
// issued by one thread; the other threads stage operands and run the
// element-wise epilogues from tensor memory.  With S_e = S Diag(e^{gamma_r})
// (gamma_r: gate of the chunk's centre row) the gradients of the chunk are
//   L0:  Z   = dO S_e           (= e^{gamma_r} (dO S))
//        dWe = -dU S_e          (= e^{gamma_r} dW,  dW = -dU S)
//        dKt = U dS'            dM = tril(dO U^T)
//   L1:  Lambda_U = T^T dU      G1 = T^T dWe        (= e^{gamma_r} Lambda_W)
//   L2:  dA = -strict_tril(Lambda_U U'^T + Lambda_W W^T)
//   L3:  Gq = Z + dM Kb^c,  G1 += dA Kb^c,  Y = dM^T Q^c + dA^T diag(beta) K^c
// and, with e_p = e^{gamma - gamma_r}, e_m = 1/e_p, e_t = e^{gamma_C - gamma},
//   dq = e_p Gq,  dv = beta Lambda_U,
//   dk = beta e_p G1 + e_m Y + e_t dKt   (+ Kaczmarz chain rule),
//   dgamma = Q^c Gq + beta K^c G1 - Kb^c Y - Kt dKt  (+ chunk-decay terms on
//   the last row), then a reverse cumulative sum down the chunk.
// The residual system (I + A)[U' | W] = diag(beta)[V | K e^gamma] is
// differentiated in one transposed solve (Lambda = T^T [dU | dW]); no adjoint
// of the inverse is formed.

#include "dr_common.cuh"
#include "fast.cuh"
#include "frag.cuh"
#include "tc.cuh"

namespace dr {
namespace fast {

using frag::bf16;

namespace {

constexpr int C = 64, D = 128;
constexpr int NTT = 256;            // threads
constexpr int LDG = D + 4;          // fp32 stride of the gate tile (conflict-free row access)
constexpr int LDK = D + 8;          // bf16 stride of the raw key tile
constexpr uint32_t kSpin = 1u << 22;  // bounded mbarrier wait (iterations)

// Arena slots (bytes).  L0: dO | dU | U | S_e | dS'.  After L0: T^T | dU (MN) |
// dWe | dM | dM^T | U' | W | q.  After L1: Lambda_U | Lambda_W.  After L2:
// dA | dA^T | Kb^c | Q^c | beta K^c.  At the end: the fp32 dgamma tile.
constexpr int A_DO = 0, A_DU = 16, A_U = 32, A_SE = 48, A_DS = 80;         // in KB
constexpr int A_TT = 0, A_DUM = 8, A_DWE = 24, A_DM = 40, A_DMT = 48, A_UP = 56, A_W = 72,
              A_Q = 88;
constexpr int A_LU = 0, A_LW = 16;
constexpr int A_DA = 0, A_DAT = 8, A_KB = 16, A_QC = 56, A_BKC = 72;
constexpr int ARENA_KB = 112;

struct TcSmem {
  unsigned char arena[ARENA_KB * 1024];
  float gam[C * LDG];   // cumulative gate, then e^{gamma - gamma_r} (scalar gate: column 0)
  bf16 k[C * LDK];      // raw keys
  float beta[C];
  float knorm[C];
  float er[D];          // e^{gamma_r}
  float erc[D];         // e^{gamma_C - gamma_r}
  float ec[D];          // e^{gamma_C}
  float ier[D];         // e^{-gamma_r}
  float dgc[16 * D];    // colsum(dS' .* S) partials per group of 8 value rows
  float ktk[4 * D];     // colsum(Kt .* dKt) per row quarter
  float dbp[C * 4];     // dbeta partials
  uint64_t bar;
  uint32_t tmem;
  int fail;
};

__device__ __forceinline__ bf16* slot(TcSmem& s, int kb) {
  return reinterpret_cast<bf16*>(s.arena + kb * 1024);
}

// cp.async of a row-major bf16 global tile into a K-major canonical tile
// [R x Ncol] (rows = M/N, columns = K).
__device__ __forceinline__ void ld_kmaj(bf16* t, const bf16* g, size_t ld, int R, int Ncol,
                                        int valid_rows = 1 << 30) {
  tc::cp_core_tile<NTT>(t, g, ld, R, Ncol, valid_rows, threadIdx.x);
}

__device__ __forceinline__ uint32_t tmem_lane_addr(uint32_t base, int warp, int col) {
  return base + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)col;
}

// Issue KS k-steps of D[tm] (+)= A * B (M = 64).
__device__ __forceinline__ void issue(uint32_t tm, const bf16* A, bool a_mn, int a_dim,
                                      const bf16* B, bool b_mn, int b_dim, int N, int KS,
                                      bool acc_first) {
  const uint32_t id = tc::idesc_bf16(64, N, a_mn, b_mn);
  for (int ks = 0; ks < KS; ++ks) {
    const uint64_t a = a_mn ? tc::sdesc_mnmaj(A, a_dim, ks) : tc::sdesc_kmaj(A, a_dim, ks);
    const uint64_t b = b_mn ? tc::sdesc_mnmaj(B, b_dim, ks) : tc::sdesc_kmaj(B, b_dim, ks);
    tc::mma(tm, a, b, id, (ks > 0 || acc_first) ? 1u : 0u);
  }
}

// Wait for the commit of level `phase` (parity phase & 1); CTA-uniform result.
__device__ __forceinline__ bool level_wait(TcSmem& s, int phase) {
  const bool ok = tc::mbar_wait(&s.bar, (uint32_t)(phase & 1), kSpin);
  const int bad = __syncthreads_or(ok ? 0 : 1);
  tc::fence_after_sync();
  return bad == 0;
}

// Store 8 fp32 values as bf16 (16 bytes).
__device__ __forceinline__ void st8(bf16* p, const float* f) {
  *reinterpret_cast<uint4*>(p) = make_uint4(frag::pack(f[0], f[1]), frag::pack(f[2], f[3]),
                                            frag::pack(f[4], f[5]), frag::pack(f[6], f[7]));
}

// TMEM columns: T0 = Z -> Gq, T1 = dWe -> Lambda_U -> Y, T2 = dKt -> G1, T3 = dM -> dA.
constexpr int T0 = 0, T1 = 128, T2 = 256, T3 = 384;

__global__ void __launch_bounds__(NTT, 1)
    k_bwd_chunk_tc(Problem p, const bf16* __restrict__ q, const bf16* __restrict__ k,
                   const bf16* __restrict__ v, const bf16* __restrict__ dO,
                   const float* __restrict__ g, Saved sv, const bf16* __restrict__ dhst,
                   const bf16* __restrict__ dUg, bf16* __restrict__ dq, bf16* __restrict__ dk,
                   bf16* __restrict__ dv, float* __restrict__ dbeta, float* __restrict__ dg,
                   int* __restrict__ err) {
  extern __shared__ __align__(1024) unsigned char smraw[];
  TcSmem& s = *reinterpret_cast<TcSmem*>(smraw);
  const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, gk = p.gk;
  const int t0 = n * C, nvalid = min(C, p.T - t0);
  const size_t cb = chunk_id(p, b, h, n);
  const int r = (nvalid - 1) / 2;
  // epilogue ownership: row i = 16 (warp % 4) + lane (lane < 16), columns 64 hh ..
  const bool act = lane < 16;
  const int ri = 16 * (warp & 3) + (lane & 15), hh = warp >> 2;
  float dkacc[64], dgacc[64];  // K-side gradient accumulators of row ri, columns 64 hh ..
  float dbv = 0.f;             // dbeta partial of row ri (V side)

  if (warp == 0) tc::tmem_alloc(&s.tmem, 512);
  if (tid == 0) {
    tc::mbar_init(&s.bar, 1);
    s.fail = 0;
  }
  // ---- loads: L0 operands, gate, raw keys
  const size_t tokrow = row_id(p, b, t0, h) * D;  // row stride H * D
  const size_t tstride = (size_t)p.H * D;
  ld_kmaj(slot(s, A_DO), dO + tokrow, tstride, C, D, nvalid);
  cp_linear<NTT>(slot(s, A_DU), dUg + cb * C * D, C * D, tid);
  cp_linear<NTT>(slot(s, A_U), sv.U + cb * C * D, C * D, tid);
  cp_linear<NTT>(slot(s, A_SE), sv.h + cb * D * D, D * D, tid);
  cp_linear<NTT>(slot(s, A_DS), dhst + cb * D * D, D * D, tid);
  for (int idx = tid; idx < C * (D / 8); idx += NTT) {
    const int i = idx >> 4, j = idx & 15;
    const bool ok = i < nvalid;
    frag::cp16(s.k + i * LDK + 8 * j, k + tokrow + (size_t)(ok ? i : 0) * tstride + 8 * j, ok);
  }
  if (gk == D) {
    for (int idx = tid; idx < C * (D / 4); idx += NTT) {
      const int i = idx >> 5, j = idx & 31;
      const bool ok = i < nvalid && p.gate != kGateNone;
      frag::cp16(s.gam + i * LDG + 4 * j, g + row_id(p, b, t0 + (ok ? i : 0), h) * D + 4 * j, ok);
    }
  } else if (tid < C) {
    s.gam[tid * LDG] = (tid < nvalid && p.gate != kGateNone) ? g[row_id(p, b, t0 + tid, h)] : 0.f;
  }
  if (tid < C) {
    s.beta[tid] = sv.beta[cb * C + tid];
    s.knorm[tid] = sv.knorm[cb * C + tid];
  }
  frag::cp_commit();
  frag::cp_wait<0>();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = s.tmem;
  // cumulative gate
  if (tid < gk) {
    float vv[C];
#pragma unroll
    for (int i = 0; i < C; ++i) vv[i] = s.gam[i * LDG + tid];
#pragma unroll
    for (int i = 1; i < C; ++i) vv[i] += vv[i - 1];
#pragma unroll
    for (int i = 0; i < C; ++i) s.gam[i * LDG + tid] = vv[i];
  }
  // colsum(dS' .* S) (before S is scaled): thread -> 8 columns x 8 value rows
  {
    const int j = tid & 15, ag = tid >> 4;
    const bf16* Sm = slot(s, A_SE);
    const bf16* dSm = slot(s, A_DS);
    float acc[8] = {};
#pragma unroll
    for (int a = 8 * ag; a < 8 * ag + 8; ++a) {
      const int o = tc::mnmaj_off(a, 8 * j, D);
      const uint4 x = *reinterpret_cast<const uint4*>(Sm + o);
      const uint4 y = *reinterpret_cast<const uint4*>(dSm + o);
      const uint32_t* wx = reinterpret_cast<const uint32_t*>(&x);
      const uint32_t* wy = reinterpret_cast<const uint32_t*>(&y);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fx = frag::unpack(wx[e]), fy = frag::unpack(wy[e]);
        acc[2 * e] += fx.x * fy.x;
        acc[2 * e + 1] += fx.y * fy.y;
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) s.dgc[ag * D + 8 * j + e] = acc[e];
  }
  __syncthreads();
  auto gamv = [&](int i, int c) -> float { return s.gam[i * LDG + (gk == D ? c : 0)]; };
  if (tid < D) {
    const float gr = gamv(r, tid), gC = gamv(C - 1, tid);
    s.er[tid] = __expf(gr);
    s.ier[tid] = __expf(-gr);
    s.erc[tid] = __expf(gC - gr);
    s.ec[tid] = __expf(gC);
    float t = 0.f;
#pragma unroll
    for (int a = 0; a < 16; ++a) t += s.dgc[a * D + tid];
    s.dgc[tid] = t;
  }
  __syncthreads();
  // gate tile -> e^{gamma - gamma_r} in place (all reads of the centre row happen first)
  if (gk == D) {
    float tmp[32];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int idx = tid + u * NTT, i = idx >> 5, c4 = (idx & 31) * 4;
      const float4 x = *reinterpret_cast<const float4*>(s.gam + i * LDG + c4);
      const float4 y = *reinterpret_cast<const float4*>(s.gam + r * LDG + c4);
      tmp[4 * u] = __expf(x.x - y.x);
      tmp[4 * u + 1] = __expf(x.y - y.y);
      tmp[4 * u + 2] = __expf(x.z - y.z);
      tmp[4 * u + 3] = __expf(x.w - y.w);
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int idx = tid + u * NTT, i = idx >> 5, c4 = (idx & 31) * 4;
      *reinterpret_cast<float4*>(s.gam + i * LDG + c4) =
          make_float4(tmp[4 * u], tmp[4 * u + 1], tmp[4 * u + 2], tmp[4 * u + 3]);
    }
  } else {
    float t = 0.f;
    if (tid < C) t = __expf(s.gam[tid * LDG] - s.gam[r * LDG]);
    __syncthreads();
    if (tid < C) s.gam[tid * LDG] = t;
  }
  __syncthreads();
  // e^{gamma - gamma_r} of row i, columns c0 .. c0+15
  auto ep16 = [&](int i, int c0, float* o) {
    if (gk == D) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 x = *reinterpret_cast<const float4*>(s.gam + i * LDG + c0 + 4 * u);
        o[4 * u] = x.x; o[4 * u + 1] = x.y; o[4 * u + 2] = x.z; o[4 * u + 3] = x.w;
      }
    } else {
      const float x = s.gam[i * LDG];
#pragma unroll
      for (int e = 0; e < 16; ++e) o[e] = x;
    }
  };
  // e^{gamma - gamma_r} of row i, columns c0 .. c0+7
  auto ep8 = [&](int i, int c0, float* o) {
    if (gk == D) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const float4 x = *reinterpret_cast<const float4*>(s.gam + i * LDG + c0 + 4 * u);
        o[4 * u] = x.x; o[4 * u + 1] = x.y; o[4 * u + 2] = x.z; o[4 * u + 3] = x.w;
      }
    } else {
      const float x = s.gam[i * LDG];
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = x;
    }
  };
  // 16 bf16 of a row-major padded tile, as fp32
  auto ld16 = [&](const bf16* base, float* o) {
    const uint4 x0 = *reinterpret_cast<const uint4*>(base);
    const uint4 x1 = *reinterpret_cast<const uint4*>(base + 8);
    const uint32_t* w0 = reinterpret_cast<const uint32_t*>(&x0);
    const uint32_t* w1 = reinterpret_cast<const uint32_t*>(&x1);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 a = frag::unpack(w0[e]), b2 = frag::unpack(w1[e]);
      o[2 * e] = a.x; o[2 * e + 1] = a.y; o[8 + 2 * e] = b2.x; o[8 + 2 * e + 1] = b2.y;
    }
  };
  // S_e = S Diag(e^{gamma_r}) in place (MN-major [a][c]: 8 consecutive c per 16 bytes)
  {
    bf16* Sm = slot(s, A_SE);
    for (int idx = tid; idx < D * (D / 8); idx += NTT) {
      const int a = idx >> 4, j = idx & 15;
      bf16* ptr = Sm + tc::mnmaj_off(a, 8 * j, D);
      uint4 raw = *reinterpret_cast<uint4*>(ptr);
      uint32_t* w = reinterpret_cast<uint32_t*>(&raw);
      float f[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 x = frag::unpack(w[e]);
        f[2 * e] = x.x * s.er[8 * j + 2 * e];
        f[2 * e + 1] = x.y * s.er[8 * j + 2 * e + 1];
      }
      st8(ptr, f);
    }
  }
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();

  // ---- L0
  if (tid == 0) {
    issue(tbase + T0, slot(s, A_DO), false, D, slot(s, A_SE), true, D, 128, 8, false);
    issue(tbase + T1, slot(s, A_DU), false, D, slot(s, A_SE), true, D, 128, 8, false);
    issue(tbase + T2, slot(s, A_U), false, D, slot(s, A_DS), true, D, 128, 8, false);
    issue(tbase + T3, slot(s, A_DO), false, D, slot(s, A_U), false, D, 64, 8, false);
    tc::commit(&s.bar);
  }
  bool ok = level_wait(s, 0);
  if (!ok) goto fail;
  // L1/L2 operands and raw q into the freed arena (overlaps the L0 epilogue)
  cp_linear<NTT>(slot(s, A_TT), sv.T + cb * C * C, C * C, tid);
  cp_linear<NTT>(slot(s, A_DUM), dUg + cb * C * D, C * D, tid);
  cp_linear<NTT>(slot(s, A_UP), sv.Up + cb * C * D, C * D, tid);
  cp_linear<NTT>(slot(s, A_W), sv.W + cb * C * D, C * D, tid);
  {
    bf16* qraw = slot(s, A_Q);  // row-major [64][LDK]
    for (int idx = tid; idx < C * (D / 8); idx += NTT) {
      const int i = idx >> 4, j = idx & 15;
      const bool okr = i < nvalid;
      frag::cp16(qraw + i * LDK + 8 * j, q + tokrow + (size_t)(okr ? i : 0) * tstride + 8 * j, okr);
    }
  }
  frag::cp_commit();
  // L0 epilogue: dKt into the accumulators; dWe and dM to shared memory.
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    const int c0 = 64 * hh + 16 * cc;
    float x[16], ep[16], kv[16];
    tc::tmem_ld16(tmem_lane_addr(tbase + T2, warp, c0), x);
    ep16(ri, c0, ep);
    ld16(s.k + ri * LDK + c0, kv);
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int c = c0 + e;
      const float et = s.erc[c] * __fdividef(1.f, ep[e]);
      const float kt = kv[e] * et;
      dkacc[16 * cc + e] = act ? et * x[e] : 0.f;
      dgacc[16 * cc + e] = act ? -kt * x[e] : 0.f;
      // column sum of Kt .* dKt over the 16 active lanes of this warp
      float z = act ? kt * x[e] : 0.f;
      z += __shfl_xor_sync(0xffffffffu, z, 8);
      z += __shfl_xor_sync(0xffffffffu, z, 4);
      z += __shfl_xor_sync(0xffffffffu, z, 2);
      z += __shfl_xor_sync(0xffffffffu, z, 1);
      if (lane == 0) s.ktk[(warp & 3) * D + c] = z;
    }
  }
  frag::cp_wait<0>();
  {
    // dWe = -(dU S_e): rows i, MN-major [K = i][N = c] for Lambda_W's B operand
    bf16* dWe = slot(s, A_DWE);
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int c0 = 64 * hh + 16 * cc;
      float x[16];
      tc::tmem_ld16(tmem_lane_addr(tbase + T1, warp, c0), x);
#pragma unroll
      for (int e = 0; e < 16; ++e) x[e] = -x[e];
      if (act) {
        st8(dWe + tc::mnmaj_off(ri, c0, D), x);
        st8(dWe + tc::mnmaj_off(ri, c0 + 8, D), x + 8);
      }
    }
    // dM = tril(dO U^T): this thread's 32 columns j = 32 hh ..
    bf16* dM = slot(s, A_DM);
    bf16* dMt = slot(s, A_DMT);
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const int j0 = 32 * hh + 16 * cc;
      float x[16];
      tc::tmem_ld16(tmem_lane_addr(tbase + T3, warp, j0), x);
#pragma unroll
      for (int e = 0; e < 16; ++e)
        if (j0 + e > ri) x[e] = 0.f;
      if (act) {
        st8(dM + tc::kmaj_off(ri, j0, C), x);
        st8(dM + tc::kmaj_off(ri, j0 + 8, C), x + 8);
        st8(dMt + tc::mnmaj_off(ri, j0, C), x);
        st8(dMt + tc::mnmaj_off(ri, j0 + 8, C), x + 8);
      }
    }
  }
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();

  // ---- L1: Lambda_U = T^T dU (T1), G1 = T^T dWe (T2)
  if (tid == 0) {
    issue(tbase + T1, slot(s, A_TT), true, C, slot(s, A_DUM), true, D, 128, 4, false);
    issue(tbase + T2, slot(s, A_TT), true, C, slot(s, A_DWE), true, D, 128, 4, false);
    tc::commit(&s.bar);
  }
  ok = level_wait(s, 1);
  if (!ok) goto fail;
  {
    // Lambda_U: dv, dbeta (V side), A operand of dA; G1 = e^{gamma_r} Lambda_W: A operand of dA
    bf16* LU = slot(s, A_LU);
    bf16* LW = slot(s, A_LW);
    const float bi = s.beta[ri];
    const size_t vrow = tokrow + (size_t)ri * tstride;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int c0 = 64 * hh + 16 * cc;
      float lu[16], lw[16];
      tc::tmem_ld16(tmem_lane_addr(tbase + T1, warp, c0), lu);
      tc::tmem_ld16(tmem_lane_addr(tbase + T2, warp, c0), lw);
      if (act) {
      if (ri < nvalid) {
        const uint4* vp = reinterpret_cast<const uint4*>(v + vrow + c0);
        const uint4 v0 = vp[0], v1 = vp[1];
        const uint32_t* w0 = reinterpret_cast<const uint32_t*>(&v0);
        const uint32_t* w1 = reinterpret_cast<const uint32_t*>(&v1);
        float vv[16], dvv[16];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 a0 = frag::unpack(w0[e]), a1 = frag::unpack(w1[e]);
          vv[2 * e] = a0.x;
          vv[2 * e + 1] = a0.y;
          vv[8 + 2 * e] = a1.x;
          vv[8 + 2 * e + 1] = a1.y;
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          dvv[e] = bi * lu[e];
          dbv += lu[e] * vv[e];
        }
        st8(dv + vrow + c0, dvv);
        st8(dv + vrow + c0 + 8, dvv + 8);
      }
      st8(LU + tc::kmaj_off(ri, c0, D), lu);
      st8(LU + tc::kmaj_off(ri, c0 + 8, D), lu + 8);
#pragma unroll
      for (int e = 0; e < 16; ++e) lw[e] = lw[e] * s.ier[c0 + e];
      st8(LW + tc::kmaj_off(ri, c0, D), lw);
      st8(LW + tc::kmaj_off(ri, c0 + 8, D), lw + 8);
      }
    }
  }
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();

  // ---- L2: dA_raw = Lambda_U U'^T + Lambda_W W^T (T3)
  if (tid == 0) {
    issue(tbase + T3, slot(s, A_LU), false, D, slot(s, A_UP), false, D, 64, 8, false);
    issue(tbase + T3, slot(s, A_LW), false, D, slot(s, A_W), false, D, 64, 8, true);
    tc::commit(&s.bar);
  }
  ok = level_wait(s, 2);
  if (!ok) goto fail;
  {
    float da[2][16];
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const int j0 = 32 * hh + 16 * cc;
      tc::tmem_ld16(tmem_lane_addr(tbase + T3, warp, j0), da[cc]);
#pragma unroll
      for (int e = 0; e < 16; ++e) da[cc][e] = (j0 + e < ri) ? -da[cc][e] : 0.f;
    }
    bf16* dA = slot(s, A_DA);
    bf16* dAt = slot(s, A_DAT);
    if (act) {
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int j0 = 32 * hh + 16 * cc;
        st8(dA + tc::kmaj_off(ri, j0, C), da[cc]);
        st8(dA + tc::kmaj_off(ri, j0 + 8, C), da[cc] + 8);
        st8(dAt + tc::mnmaj_off(ri, j0, C), da[cc]);
        st8(dAt + tc::mnmaj_off(ri, j0 + 8, C), da[cc] + 8);
      }
    }
    // Kb^c, Q^c, beta K^c as MN-major [K = i][N = c] tiles
    bf16* Kb = slot(s, A_KB);
    bf16* Qc = slot(s, A_QC);
    bf16* BKc = slot(s, A_BKC);
    const bf16* qraw = slot(s, A_Q);
    for (int idx = tid; idx < C * (D / 8); idx += NTT) {
      const int i = idx >> 4, j = idx & 15;
      float kb[8], qc[8], bkc[8], ep[8], kv[16], qv[16];
      ep8(i, 8 * j, ep);
      ld16(s.k + i * LDK + 8 * j, kv);
      ld16(qraw + i * LDK + 8 * j, qv);
      const float bi = s.beta[i];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        kb[e] = kv[e] * __fdividef(1.f, ep[e]);
        bkc[e] = bi * kv[e] * ep[e];
        qc[e] = qv[e] * ep[e];
      }
      st8(Kb + tc::mnmaj_off(i, 8 * j, D), kb);
      st8(Qc + tc::mnmaj_off(i, 8 * j, D), qc);
      st8(BKc + tc::mnmaj_off(i, 8 * j, D), bkc);
    }
  }
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();

  // ---- L3: Gq = Z + dM Kb (T0), G1 += dA Kb (T2), Y = dM^T Q^c + dA^T beta K^c (T1)
  if (tid == 0) {
    issue(tbase + T0, slot(s, A_DM), false, C, slot(s, A_KB), true, D, 128, 4, true);
    issue(tbase + T2, slot(s, A_DA), false, C, slot(s, A_KB), true, D, 128, 4, true);
    issue(tbase + T1, slot(s, A_DMT), true, C, slot(s, A_QC), true, D, 128, 4, false);
    issue(tbase + T1, slot(s, A_DAT), true, C, slot(s, A_BKC), true, D, 128, 4, true);
    tc::commit(&s.bar);
  }
  ok = level_wait(s, 3);
  if (!ok) goto fail;
  {
    const float bi = s.beta[ri];
    const size_t qrow = tokrow + (size_t)ri * tstride;
    const bf16* qraw = slot(s, A_Q);
    float dbk = 0.f;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int c0 = 64 * hh + 16 * cc;
      float gq[16], g1[16], y[16], epv[16], kvv[16], qvv[16];
      tc::tmem_ld16(tmem_lane_addr(tbase + T0, warp, c0), gq);
      tc::tmem_ld16(tmem_lane_addr(tbase + T2, warp, c0), g1);
      tc::tmem_ld16(tmem_lane_addr(tbase + T1, warp, c0), y);
      ep16(ri, c0, epv);
      ld16(s.k + ri * LDK + c0, kvv);
      ld16(qraw + ri * LDK + c0, qvv);
      float dqv[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float ep = epv[e];
        const float em = __fdividef(1.f, ep);
        const float kv = kvv[e];
        const float qc = qvv[e] * ep;
        const float kc = kv * ep, kb = kv * em;
        dqv[e] = ep * gq[e];
        dkacc[16 * cc + e] += bi * ep * g1[e] + em * y[e];
        dgacc[16 * cc + e] += qc * gq[e] + bi * kc * g1[e] - kb * y[e];
        dbk += kc * g1[e];
      }
      if (act && ri < nvalid) {
        st8(dq + qrow + c0, dqv);
        st8(dq + qrow + c0 + 8, dqv + 8);
      }
    }
    if (act) s.dbp[ri * 4 + hh] = dbv + dbk;
  }
  tc::fence_before_sync();
  __syncthreads();  // every MMA operand slot is dead: the arena becomes the fp32 dgamma tile
  {
    float* sdg = reinterpret_cast<float*>(s.arena);
    if (act) {
#pragma unroll
      for (int e = 0; e < 64; ++e) sdg[ri * LDG + 64 * hh + e] = dgacc[e];
    }
    if (tid < C) s.dbp[tid * 4] = s.dbp[tid * 4] + s.dbp[tid * 4 + 1];
  }
  __syncthreads();
  {
    // dk with the Kaczmarz chain rule, dbeta
    if (act && ri < nvalid) {
      const float bi = s.beta[ri], db = s.dbp[ri * 4];
      const size_t krow = tokrow + (size_t)ri * tstride;
      const float kla = (p.beta_mode == kBetaKaczmarz) ? -2.f * bi * db / (s.knorm[ri] + p.eps) : 0.f;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        float o8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          o8[e] = dkacc[8 * cc + e] + kla * __bfloat162float(s.k[ri * LDK + 64 * hh + 8 * cc + e]);
        st8(dk + krow + 64 * hh + 8 * cc, o8);
      }
    }
    if (tid < nvalid) {
      float db = s.dbp[tid * 4];
      if (p.beta_mode == kBetaKaczmarz) db /= (s.knorm[tid] + p.eps);
      dbeta[row_id(p, b, t0 + tid, h)] = db;
    }
    // dgamma: chunk-decay terms on the last row, reverse cumulative sum per channel
    float* sdg = reinterpret_cast<float*>(s.arena);
    if (tid < D) {
      const int c = tid;
      const float extra = s.ktk[c] + s.ktk[D + c] + s.ktk[2 * D + c] + s.ktk[3 * D + c] +
                          s.ec[c] * s.dgc[c];
      sdg[(C - 1) * LDG + c] += extra;
      float run = 0.f;
      for (int i = C - 1; i >= 0; --i) {
        run += sdg[i * LDG + c];
        sdg[i * LDG + c] = run;
        if (gk == D && i < nvalid) dg[row_id(p, b, t0 + i, h) * D + c] = run;
      }
    }
    if (gk == 1 && p.gate != kGateNone) {
      __syncthreads();
      if (tid < nvalid) {
        float sum = 0.f;
        for (int c = 0; c < D; ++c) sum += sdg[tid * LDG + c];
        dg[row_id(p, b, t0 + tid, h)] = sum;
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, 512);
  return;
fail:
  // a bounded wait gave up: record it, release tensor memory and leave
  if (tid == 0 && err) atomicExch(err, 1);
  frag::cp_wait<0>();
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, 512);
}

}  // namespace

cudaError_t launch_bwd_chunk_tc(const Problem& p, const bf16* q, const bf16* k, const bf16* v,
                                const bf16* dO, const float* g, const Saved& sv,
                                const bf16* dh, const bf16* dU, bf16* dq, bf16* dk, bf16* dv,
                                float* dbeta, float* dg, cudaStream_t st) {
  const size_t sm = sizeof(TcSmem) + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(k_bwd_chunk_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const double nb = (double)p.B * p.H * p.NC, ntok = nb * C;
  // reads q, k, v, dO, g, beta, T, h, dh, U, dU, W, U'; writes dq, dk, dv, dbeta, dg
  const double bytes = ntok * (4 * D * 2 + p.gk * 4 + 4) + nb * C * C * 2 + nb * 2.0 * D * D * 2 +
                       ntok * 4 * D * 2 + ntok * (3 * D * 2 + p.gk * 4 + 4);
  const double mac = (double)C * D * D * 3 + (double)C * C * D + (double)C * D * C * 2 +
                     (double)C * C * D * 2 + (double)C * D * C * 4;
  prof_begin(kKTcChunkBwd, bytes, nb * 2.0 * mac, st);
  k_bwd_chunk_tc<<<dim3(p.NC, p.H, p.B), NTT, sm, st>>>(p, q, k, v, dO, g, sv, dh, dU, dq, dk,
                                                        dv, dbeta, dg, device_error_word());
  e = cudaGetLastError();
  prof_end(st);
  return e;
}

}  // namespace fast
}  // namespace dr
