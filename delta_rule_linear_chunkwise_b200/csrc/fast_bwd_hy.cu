// fast_bwd_hy.cu -- chunk-parallel backward with the products on tcgen05 and
// the element-wise work on all 16 warps (bf16 storage, d_k = d_v = 128, C = 64).
//
// One CTA per (b, h, chunk).  With ep = e^{gamma - gamma_r} (gamma_r: the cumulative
// gate at the chunk's centre row) and the chunk's saved tiles:
//   level 1  dQs = dO S, dW' = dU S, dKt = U dS', dM = tril(dO U^T)
//   level 2  Lambda = T^T [dU | dW]             (dv = diag(beta) Lambda_U)
//   level 3  dA = -strict_tril(Lambda_U U'^T + Lambda_W W^T)
//   level 4  dM Kb^c, dA Kb^c, dM^T Q^c + dA^T diag(beta) K^c
// and the register epilogue over Z = e^{gamma_r} dQs + dM Kb^c,
// P = e^{gamma_C - gamma_r} dKt + dM^T Q^c + dA^T beta K^c, Q = e^{gamma_r} Lambda_W + dA Kb^c:
// dq = ep Z, dk = P / ep + beta ep Q, dgamma = k (beta ep Q - P / ep) + Q^c Z, then the
// gate reverse cumulative sum and the Kaczmarz chain rule.
//
// Each level is a set of tcgen05.mma (M = 64, operands in shared memory in the
// canonical core-matrix layout, fp32 accumulators in tensor memory) issued by
// one thread, independent accumulation chains interleaved (long chains split
// into partial sums).  An M = 64 accumulator occupies lanes 16 q .. 16 q + 15 of each
// 32-lane quadrant q, and tcgen05.ld.16x256b returns it to the warps of that
// quadrant in exactly the register fragment of a warp-level m16n8 product
// (thread t: row t / 4 and t / 4 + 8, columns 2 (t % 4), + 1 of each 8-column
// group), so warp w = 4 qt + rb owns rows 16 rb .., columns 32 qt ...

#include "dr_common.cuh"
#include "fast.cuh"
#include "frag.cuh"
#include "tc.cuh"

namespace dr {
namespace fast {

using frag::bf16;

namespace {

constexpr int C = 64, D = 128;
constexpr int LDD = D + 8;
constexpr int NTB = 512;
constexpr int LDG = D + 4;  // fp32 row stride of the dgamma tile (fragment stores conflict-free)
constexpr uint32_t kSpinHy = 1u << 22;
// Polls of the injected wait (dr_inject_timeout): short, so the test that
// drives the timeout path ends within milliseconds.
constexpr uint32_t kSpinInjected = 256;

__device__ __forceinline__ int centre_row(int nvalid) { return (nvalid - 1) / 2; }
// Gate tile element (i, c): 8-column groups XOR-swizzled by row.
__device__ __forceinline__ int gsw(int i, int c) { return i * D + (c ^ ((i & 7) << 3)); }

// Tensor memory columns (512 allocated): level 1 uses all four ranges, the
// later levels reuse them once the earlier accumulators are in registers.
constexpr uint32_t T_ZQ = 0, T_ADW = 128, T_AKT = 256, T_ADM = 384;
constexpr uint32_t T_LU = 0, T_LW = 128;
constexpr uint32_t T_DA = 256;  // four 64-column partial sums of dA
constexpr uint32_t T_Z2 = 0, T_X = 128, T_Y = 256, T_Y2 = 384;

struct HySmem {
  bf16 SS[D * D];   // S = h_n [a][c], core-tiled (MN-major B);  then Lambda_U | Lambda_W;
                    // at the end the fp32 dgamma tile
  bf16 SD[D * D];   // dS' [a][c];  then W | U' (level 3);  then Kb^c | beta K^c (level 4)
  bf16 DO[C * D];   // dO [i][a] (K-major A);  then dW [j][c]
  bf16 DU[C * D];   // dU [j][a]
  bf16 UU[C * D];   // U [j][a];  then dM [i][j] | dA [i][j]
  bf16 QC[C * D];   // Q^c [j][c], core-tiled
  bf16 QR[C * LDD]; // raw q, row-major padded
  bf16 k[C * LDD];  // raw k, row-major padded
  bf16 TT[C * C];   // T [j][i], core-tiled (MN-major A of T^T)
  float G[C * D];   // cumulative gate (gsw), then e^{gamma - gamma_r}
  float beta[C];
  float knorm[C];
  float dbp[C * 4];
  float dgc[4 * D];
  float ktk[4 * D];
  float er[D];
  float erc[D];
  uint64_t bar;
  uint64_t never;   // fault injection: a barrier that nothing ever arrives on
  uint32_t tmem;
};

static_assert(offsetof(HySmem, SD) == offsetof(HySmem, SS) + sizeof(bf16) * D * D &&
                  sizeof(float) * C * LDG <= sizeof(bf16) * 2 * D * D,
              "the padded dgamma tile spans the adjacent S and dS' tiles");

// One product chain D[tm] (+)= A B (M = 64) over k-steps ks0, ks0 + kstride, ...
// (count of them); A: K-major [64][K] (a_dim = K) or MN-major [K][64], B: K-major
// [N][K] (b_dim = K) or MN-major [K][N] (b_dim = N).  The first step overwrites
// the accumulator.
struct Chain {
  uint32_t tm;
  uint64_t a0, b0;     // descriptors of k-step 0
  uint32_t da, db;     // descriptor start-address advance per k-step (16-byte units)
  uint32_t id;
  int ks0, kstride, count;
};
__device__ __forceinline__ Chain chain(uint32_t tm, const bf16* A, bool a_mn, int a_dim,
                                       const bf16* B, bool b_mn, int b_dim, int N, int ks0,
                                       int kstride, int count) {
  Chain c;
  c.tm = tm;
  c.a0 = a_mn ? tc::sdesc_mnmaj(A, 64, 0) : tc::sdesc_kmaj(A, a_dim, 0);
  c.b0 = b_mn ? tc::sdesc_mnmaj(B, b_dim, 0) : tc::sdesc_kmaj(B, b_dim, 0);
  c.da = a_mn ? 2 * (64 / 8) * 128 / 16 : 256 / 16;
  c.db = b_mn ? 2 * (b_dim / 8) * 128 / 16 : 256 / 16;
  c.id = tc::idesc_bf16(64, N, a_mn, b_mn);
  c.ks0 = ks0;
  c.kstride = kstride;
  c.count = count;
  return c;
}
// Issue the chains round-robin by step (consecutive instructions go to
// independent accumulators).  Measured on B200: with the descriptors built
// before the loop, one thread issues a tcgen05.mma of M = 64 or 128, N <= 128
// every 55-70 cycles and the tensor core keeps pace, so a level costs about
// its instruction count times that.
template <int NC>
__device__ __forceinline__ void issue_chains(const Chain (&cs)[NC]) {
  int steps = 0;
#pragma unroll
  for (int i = 0; i < NC; ++i) steps = max(steps, cs[i].count);
  for (int j = 0; j < steps; ++j) {
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      if (j < cs[i].count) {
        const uint32_t ks = (uint32_t)(cs[i].ks0 + j * cs[i].kstride);
        tc::mma(cs[i].tm, cs[i].a0 + ks * cs[i].da, cs[i].b0 + ks * cs[i].db, cs[i].id,
                j > 0 ? 1u : 0u);
      }
    }
  }
}

// Fragments of 32 (ld4) or 16 (ld2) accumulator columns from column `col`,
// rows of this warp's quadrant.
__device__ __forceinline__ void frag_ld4(uint32_t col, int warp, float (&f)[4][4]) {
  uint32_t r[16];
  const uint32_t ta = col + ((uint32_t)(32 * (warp & 3)) << 16);
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(ta));
  tc::tmem_wait_ld();
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) f[j][e] = __uint_as_float(r[4 * j + e]);
}
__device__ __forceinline__ void frag_ld2(uint32_t col, int warp, float (&f)[2][4]) {
  uint32_t r[8];
  const uint32_t ta = col + ((uint32_t)(32 * (warp & 3)) << 16);
  asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(ta));
  tc::tmem_wait_ld();
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) f[j][e] = __uint_as_float(r[4 * j + e]);
}

// Bounded wait for the commit of level `phase`; CTA-uniform result.
__device__ __forceinline__ bool hy_wait(uint64_t* bar, int phase,
                                        uint32_t limit = kSpinHy) {
  const bool ok = tc::mbar_wait(bar, (uint32_t)(phase & 1), limit);
  const int bad = __syncthreads_or(ok ? 0 : 1);
  tc::fence_after_sync();
  return bad == 0;
}

__global__ void __launch_bounds__(NTB, 1)
    k_bwd_chunk_hy(Problem p, const bf16* __restrict__ q, const bf16* __restrict__ k,
                const bf16* __restrict__ v, const bf16* __restrict__ dO,
                const float* __restrict__ g, const bf16* __restrict__ Tg,
                const float* __restrict__ beta, const bf16* __restrict__ hst,
                const bf16* __restrict__ dhst, const bf16* __restrict__ Ug,
                const bf16* __restrict__ dUg, const bf16* __restrict__ Wg,
                const bf16* __restrict__ Upg, const float* __restrict__ knorm_g,
                bf16* __restrict__ dq, bf16* __restrict__ dk,
                bf16* __restrict__ dv, float* __restrict__ dbeta, float* __restrict__ dg,
                int* __restrict__ err, int inject_timeout) {
  extern __shared__ __align__(1024) unsigned char smraw[];
  HySmem& s = *reinterpret_cast<HySmem*>(smraw);
  const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, gk = p.gk;
  const int rb = warp & 3, qt = warp >> 2;
  const int lr = lane >> 2, lc = 2 * (lane & 3);
  const int t0 = n * C, nvalid = min(C, p.T - t0);
  const size_t cb = chunk_id(p, b, h, n);
  bf16* const sLU = s.SS;          // Lambda_U, after the first level
  bf16* const sLW = s.SS + C * D;  // Lambda_W
  bf16* const sW = s.SD;           // W, U' for the third level
  bf16* const sUp = s.SD + C * D;
  bf16* const sKb = s.DU;          // Kb^c, beta K^c for the fourth level (built under level 3)
  bf16* const sBk = s.DO;
  bf16* const sdW = s.DO;          // dW, after the first level (then beta K^c)
  bf16* const sdM = s.UU;          // dM, dA [i][j], after the first level
  bf16* const sdA = s.UU + C * C;

  // Loads in three cp.async groups, in the order of first use:
  //   1: gate, q, k   2: dO, dU, U, S, dS', T (first level)   3: W, U' (third level)
  for (int idx = tid; idx < C * (D / 8); idx += NTB) {
    const int i = idx >> 4, j = idx & 15;
    const bool ok = i < nvalid;
    const size_t rr = row_id(p, b, t0 + (ok ? i : 0), h) * D + j * 8;
    frag::cp16(s.QR + i * LDD + j * 8, q + rr, ok);
    frag::cp16(s.k + i * LDD + j * 8, k + rr, ok);
  }
  if (gk == D) {
    for (int idx = tid; idx < C * (D / 4); idx += NTB) {
      const int i = idx >> 5, j = idx & 31;
      const bool ok = i < nvalid && p.gate != kGateNone;
      frag::cp16(s.G + gsw(i, j * 4), g + row_id(p, b, t0 + (ok ? i : 0), h) * D + j * 4, ok);
    }
  } else if (tid < C) {
    s.G[tid] = (tid < nvalid && p.gate != kGateNone) ? g[row_id(p, b, t0 + tid, h)] : 0.f;
  }
  if (tid < C) {
    s.beta[tid] = beta[cb * C + tid];
    s.knorm[tid] = knorm_g[cb * C + tid];
  }
  frag::cp_commit();
  tc::cp_core_tile<NTB>(s.DO, dO + row_id(p, b, t0, h) * D, (size_t)p.H * D, C, D, nvalid, tid);
  cp_linear<NTB>(s.DU, dUg + cb * C * D, C * D, tid);
  cp_linear<NTB>(s.UU, Ug + cb * C * D, C * D, tid);
  cp_linear<NTB>(s.SS, hst + cb * D * D, D * D, tid);
  cp_linear<NTB>(s.SD, dhst + cb * D * D, D * D, tid);
  cp_linear<NTB>(s.TT, Tg + cb * C * C, C * C, tid);
  frag::cp_commit();
  if (warp == 0) tc::tmem_alloc(&s.tmem, 512);
  if (tid == 0) {
    tc::mbar_init(&s.bar, 1);
    tc::mbar_init(&s.never, 1);
  }
  frag::cp_wait<1>();
  __syncthreads();
  // element (i, c) of the gate tile
  auto gat = [&](int i, int c) -> float& { return gk == D ? s.G[gsw(i, c)] : s.G[i]; };
  // cumulative gate down the chunk's rows
  if (gk == D) {
    // thread (column c, row quarter q): scan of 16 rows, then the quarter offsets
    // (the key-column partials of the consume phase hold the quarter totals)
    const int c = tid & 127, q = tid >> 7;
    float run = 0.f;
#pragma unroll
    for (int i = 16 * q; i < 16 * q + 16; ++i) {
      run += gat(i, c);
      gat(i, c) = run;
    }
    s.ktk[q * D + c] = run;
    __syncthreads();
    float off = 0.f;
    for (int q2 = 0; q2 < q; ++q2) off += s.ktk[q2 * D + c];
    if (q > 0) {
#pragma unroll
      for (int i = 16 * q; i < 16 * q + 16; ++i) gat(i, c) += off;
    }
  } else if (warp == 0) {
    // rows 2 lane, 2 lane + 1: an inclusive scan across the warp
    const float a0v = s.G[2 * lane], a1v = s.G[2 * lane + 1];
    float x = a0v + a1v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    s.G[2 * lane + 1] = x;
    s.G[2 * lane] = x - a1v;
  }
  __syncthreads();

  const int r = centre_row(nvalid);
  if (tid < D) {
    const int cg = (gk == D) ? tid : 0;
    const float gr = gat(r, cg), gC = gat(C - 1, cg);
    s.er[tid] = __expf(gr);
    s.erc[tid] = __expf(gC - gr);
  }
  // gate tile -> e^{gamma - gamma_r} in place (every thread reads the centre row first)
  {
    float tmp[C * D / NTB];
    const int cnt = (gk == D) ? C * D / NTB : (tid < C ? 1 : 0);
#pragma unroll
    for (int u = 0; u < C * D / NTB; ++u) {
      if (u < cnt) {
        const int idx = tid + u * NTB;
        const int i = (gk == D) ? idx >> 7 : idx, c = (gk == D) ? idx & 127 : 0;
        tmp[u] = __expf(gat(i, c) - gat(r, c));
      }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < C * D / NTB; ++u) {
      if (u < cnt) {
        const int idx = tid + u * NTB;
        const int i = (gk == D) ? idx >> 7 : idx, c = (gk == D) ? idx & 127 : 0;
        gat(i, c) = tmp[u];
      }
    }
  }
  __syncthreads();
  // e^{gamma - gamma_r} at (i, c), (i, c + 1), c even
  auto ep2 = [&](int i, int c) -> float2 {
    if (gk == D) return *reinterpret_cast<const float2*>(s.G + gsw(i, c));
    const float x = s.G[i];
    return make_float2(x, x);
  };
  // e^{gamma - gamma_r} at (i, c .. c + 3), c a multiple of 4
  auto ep4 = [&](int i, int c) -> float4 {
    if (gk == D) return *reinterpret_cast<const float4*>(s.G + gsw(i, c));
    const float x = s.G[i];
    return make_float4(x, x, x, x);
  };
  // raw keys (i, c), (i, c + 1)
  auto k2 = [&](int i, int c) -> float2 {
    return frag::unpack(*reinterpret_cast<const uint32_t*>(s.k + i * LDD + c));
  };

  // ---- build: Q^c = q e^{gamma - gamma_r} into the core-tiled operand tile
  for (int idx = tid; idx < C * (D / 8); idx += NTB) {
    const int i = ct_row(idx, D), c = ct_col(idx, D);
    const uint4 rq = *reinterpret_cast<const uint4*>(s.QR + i * LDD + c);
    const float4 f0 = ep4(i, c), f1 = ep4(i, c + 4);
    const float2 q0 = frag::unpack(rq.x), q1 = frag::unpack(rq.y);
    const float2 q2 = frag::unpack(rq.z), q3 = frag::unpack(rq.w);
    *reinterpret_cast<uint4*>(s.QC + 8 * idx) =
        make_uint4(frag::pack(q0.x * f0.x, q0.y * f0.y), frag::pack(q1.x * f0.z, q1.y * f0.w),
                   frag::pack(q2.x * f1.x, q2.y * f1.y), frag::pack(q3.x * f1.z, q3.y * f1.w));
  }
  frag::cp_wait<0>();
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tb = s.tmem;
  bool ok = true;
  do {  // leaves early (break) only when a bounded wait gives up

  // Fault injection (dr_inject_timeout): wait, with a short limit, on a barrier
  // that nothing arrives on.  Every copy has landed and no MMA has been issued,
  // so the timeout path below leaves nothing in flight.
  if (inject_timeout) {
    ok = hy_wait(&s.never, 0, kSpinInjected);
    if (!ok) break;
  }

  // ---- level 1 (tensor memory): dQs = dO S, dW' = dU S, dKt = U dS', dM = dO U^T
  if (tid == 0) {
    const Chain cs[4] = {chain(tb + T_ZQ, s.DO, false, D, s.SS, true, D, 128, 0, 1, D / 16),
                         chain(tb + T_ADW, s.DU, false, D, s.SS, true, D, 128, 0, 1, D / 16),
                         chain(tb + T_AKT, s.UU, false, D, s.SD, true, D, 128, 0, 1, D / 16),
                         chain(tb + T_ADM, s.DO, false, D, s.UU, false, D, 64, 0, 1, D / 16)};
    issue_chains(cs);
    tc::commit(&s.bar);
  }
  // colsum(dS' .* S) while they run: thread -> 8 columns (16-byte core rows),
  // 4 rows (one per row group of its quarter); eight lanes read the eight rows
  // of one core matrix (128 contiguous bytes, no bank conflicts)
  {
    const int alo = tid & 7, cg = (tid >> 3) & 15, ag = tid >> 7;
    float acc[8] = {};
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int o = ct_off((ag * 4 + r) * 8 + alo, 8 * cg, D);
      const uint4 x = *reinterpret_cast<const uint4*>(s.SS + o);
      const uint4 y = *reinterpret_cast<const uint4*>(s.SD + o);
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
    for (int e = 0; e < 8; ++e) {
      float x = acc[e];
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      x += __shfl_xor_sync(0xffffffffu, x, 2);
      x += __shfl_xor_sync(0xffffffffu, x, 4);
      acc[e] = x;
    }
    if (alo == 0) {
#pragma unroll
      for (int e = 0; e < 8; ++e) s.dgc[ag * D + 8 * cg + e] = acc[e];
    }
  }
  ok = hy_wait(&s.bar, 0);
  if (!ok) break;
  // W and U' into the dS' tile (its level-1 reads are complete)
  cp_linear<NTB>(sW, Wg + cb * C * D, C * D, tid);
  cp_linear<NTB>(sUp, Upg + cb * C * D, C * D, tid);
  frag::cp_commit();
  float zq[4][4], adw[4][4], akt[4][4], adm[2][4];
  frag_ld4(tb + T_ZQ + 32 * qt, warp, zq);
  frag_ld4(tb + T_ADW + 32 * qt, warp, adw);
  frag_ld4(tb + T_AKT + 32 * qt, warp, akt);
  frag_ld2(tb + T_ADM + 16 * qt, warp, adm);
  // dW = -dW', dM masked (inclusive lower), stored for the later phases
  {
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) adw[j][e] = -adw[j][e];
    frag::st_c(adw, sdW, -D, rb * 16, qt * 32);
#pragma unroll
    for (int jt = 0; jt < 2; ++jt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = rb * 16 + lr + (e >> 1) * 8, jj = qt * 16 + jt * 8 + lc + (e & 1);
        if (jj > i) adm[jt][e] = 0.f;
      }
    frag::st_c(adm, sdM, -C, rb * 16, qt * 16);
  }
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  // ---- level 2: Lambda = T^T [dU | dW]; dv = diag(beta) Lambda_U (runs under the dKt pass)
  if (tid == 0) {
    const Chain cs[2] = {chain(tb + T_LU, s.TT, true, C, s.DU, true, D, 128, 0, 1, C / 16),
                         chain(tb + T_LW, s.TT, true, C, sdW, true, D, 128, 0, 1, C / 16)};
    issue_chains(cs);
    tc::commit(&s.bar);
  }

  // The per-element epilogue works on three accumulators at this thread's
  // fragment positions (rows i0, i0 + 8; key columns c), with ep = e^{gamma - gamma_r}:
  //   Z = e^{gamma_r} dQs + dM Kb^c                               -> dq = ep Z
  //   P = e^{gamma_C - gamma_r} dKt + dM^T Q^c + dA^T diag(beta) K^c
  //   Q = e^{gamma_r} Lambda_W + dA Kb^c
  // so that dk = P / ep + beta ep Q,  dgamma = k (beta ep Q - P / ep) + Q^c Z
  // and d(beta_eff) = Lambda_U . v + k . (ep Q) summed over the row.
  const int i0 = rb * 16 + lr;
  const size_t rowg[2] = {row_id(p, b, t0 + min(i0, nvalid - 1), h) * D,
                          row_id(p, b, t0 + min(i0 + 8, nvalid - 1), h) * D};
  float(&Z)[4][4] = zq;
  float(&P)[4][4] = akt;
  // colsum(Kt .* dKt) for the chunk-end gate term, then the column scalings
  {
    float cs[4][2] = {};
#pragma unroll
    for (int jt = 0; jt < 4; ++jt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int i = i0 + hh * 8, c = qt * 32 + jt * 8 + lc;
        const float2 kk = k2(i, c), f = ep2(i, c);
        cs[jt][0] += kk.x * __fdividef(akt[jt][2 * hh], f.x);
        cs[jt][1] += kk.y * __fdividef(akt[jt][2 * hh + 1], f.y);
      }
#pragma unroll
    for (int jt = 0; jt < 4; ++jt)
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int c = qt * 32 + jt * 8 + lc + u;
        const float fr = s.er[c], frc = s.erc[c];
        float x = cs[jt][u] * frc;
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        x += __shfl_xor_sync(0xffffffffu, x, 8);
        x += __shfl_xor_sync(0xffffffffu, x, 16);
        if (lr == 0) s.ktk[rb * D + c] = x;
        Z[jt][u] *= fr;
        Z[jt][2 + u] *= fr;
        P[jt][u] *= frc;
        P[jt][2 + u] *= frc;
      }
  }
  float dbrow[2] = {0.f, 0.f};  // this thread's d(beta_eff) partials for rows i0, i0 + 8
  float Q[4][4];
  {
    uint32_t vv[4][2];
#pragma unroll
    for (int jt = 0; jt < 4; ++jt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
        vv[jt][hh] = *reinterpret_cast<const uint32_t*>(v + rowg[hh] + qt * 32 + jt * 8 + lc);
    ok = hy_wait(&s.bar, 1);
    if (!ok) break;
    float lu[4][4];
    frag_ld4(tb + T_LU + 32 * qt, warp, lu);
#pragma unroll
    for (int jt = 0; jt < 4; ++jt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int i = i0 + hh * 8, a = qt * 32 + jt * 8 + lc;
        const float bi = s.beta[i];
        if (i < nvalid)
          *reinterpret_cast<uint32_t*>(dv + rowg[hh] + a) =
              frag::pack(bi * lu[jt][2 * hh], bi * lu[jt][2 * hh + 1]);
        const float2 vf = frag::unpack(vv[jt][hh]);
        dbrow[hh] += lu[jt][2 * hh] * vf.x + lu[jt][2 * hh + 1] * vf.y;
      }
    frag::st_c(lu, sLU, -D, rb * 16, qt * 32);
    frag_ld4(tb + T_LW + 32 * qt, warp, Q);
    frag::st_c(Q, sLW, -D, rb * 16, qt * 32);
#pragma unroll
    for (int jt = 0; jt < 4; ++jt)
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const float fr = s.er[qt * 32 + jt * 8 + lc + u];
        Q[jt][u] *= fr;
        Q[jt][2 + u] *= fr;
      }
  }
  __syncthreads();

  frag::cp_wait<0>();  // W, U'
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();

  // ---- level 3: dA = -strict_tril(Lambda_U U'^T + Lambda_W W^T), rows 16rb.., cols 16qt..
  if (tid == 0) {
    const Chain cs[4] = {chain(tb + T_DA, sLU, false, D, sUp, false, D, 64, 0, 2, D / 32),
                         chain(tb + T_DA + 64, sLU, false, D, sUp, false, D, 64, 1, 2, D / 32),
                         chain(tb + T_DA + 128, sLW, false, D, sW, false, D, 64, 0, 2, D / 32),
                         chain(tb + T_DA + 192, sLW, false, D, sW, false, D, 64, 1, 2, D / 32)};
    issue_chains(cs);
    tc::commit(&s.bar);
  }
  // ---- under level 3: Kb^c and beta K^c into the core-tiled operand tiles (dU, dW slots)
  for (int idx = tid; idx < C * (D / 8); idx += NTB) {
    const int i = ct_row(idx, D), c = ct_col(idx, D);
    const uint4 rk = *reinterpret_cast<const uint4*>(s.k + i * LDD + c);
    const float bi = s.beta[i];
    const float4 f0 = ep4(i, c), f1 = ep4(i, c + 4);
    const float f[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
    const uint32_t* wk = reinterpret_cast<const uint32_t*>(&rk);
    uint32_t okb[4], obc[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 kk = frag::unpack(wk[e]);
      okb[e] = frag::pack(__fdividef(kk.x, f[2 * e]), __fdividef(kk.y, f[2 * e + 1]));
      obc[e] = frag::pack(bi * kk.x * f[2 * e], bi * kk.y * f[2 * e + 1]);
    }
    *reinterpret_cast<uint4*>(sKb + 8 * idx) = make_uint4(okb[0], okb[1], okb[2], okb[3]);
    *reinterpret_cast<uint4*>(sBk + 8 * idx) = make_uint4(obc[0], obc[1], obc[2], obc[3]);
  }
  ok = hy_wait(&s.bar, 2);
  if (!ok) break;
  {
    float da[2][4], dp[2][4];
    frag_ld2(tb + T_DA + 16 * qt, warp, da);
#pragma unroll
    for (int part = 1; part < 4; ++part) {
      frag_ld2(tb + T_DA + 64 * part + 16 * qt, warp, dp);
#pragma unroll
      for (int jt = 0; jt < 2; ++jt)
#pragma unroll
        for (int e = 0; e < 4; ++e) da[jt][e] += dp[jt][e];
    }
#pragma unroll
    for (int jt = 0; jt < 2; ++jt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = rb * 16 + lr + (e >> 1) * 8, jj = qt * 16 + jt * 8 + lc + (e & 1);
        da[jt][e] = (jj < i) ? -da[jt][e] : 0.f;
      }
    frag::st_c(da, sdA, -C, rb * 16, qt * 16);
  }

  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  // ---- level 4: dM Kb^c, dA Kb^c, dM^T Q^c + dA^T beta K^c
  if (tid == 0) {
    const Chain cs[4] = {chain(tb + T_Z2, sdM, false, C, sKb, true, D, 128, 0, 1, C / 16),
                         chain(tb + T_X, sdA, false, C, sKb, true, D, 128, 0, 1, C / 16),
                         chain(tb + T_Y, sdM, true, C, s.QC, true, D, 128, 0, 1, C / 16),
                         chain(tb + T_Y2, sdA, true, C, sBk, true, D, 128, 0, 1, C / 16)};
    issue_chains(cs);
    tc::commit(&s.bar);
  }
  ok = hy_wait(&s.bar, 3);
  if (!ok) break;
  {
    float t4[4][4];
    frag_ld4(tb + T_Z2 + 32 * qt, warp, t4);
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) Z[j][e] += t4[j][e];
    frag_ld4(tb + T_X + 32 * qt, warp, t4);
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) Q[j][e] += t4[j][e];
    frag_ld4(tb + T_Y + 32 * qt, warp, t4);
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) P[j][e] += t4[j][e];
    frag_ld4(tb + T_Y2 + 32 * qt, warp, t4);
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) P[j][e] += t4[j][e];
  }

  // ---- per-element epilogue: dq out; P <- dk (before the Kaczmarz term), Q <- dgamma
#pragma unroll
  for (int jt = 0; jt < 4; ++jt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int i = i0 + hh * 8, c = qt * 32 + jt * 8 + lc;
      const float bi = s.beta[i];
      const float2 kk = k2(i, c);
      const float2 qc = frag::unpack(*reinterpret_cast<const uint32_t*>(s.QC + ct_off(i, c, D)));
      const float2 f = ep2(i, c);
      float outq[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int e = 2 * hh + u;
        const float ep = u ? f.y : f.x;
        const float t1 = ep * Q[jt][e], t2 = __fdividef(P[jt][e], ep);
        const float kv = u ? kk.y : kk.x, qv = u ? qc.y : qc.x;
        float dgv = kv * (bi * t1 - t2) + qv * Z[jt][e];
        if (i == C - 1) {  // chunk-end gate term: colsum(Kt .* dKt) + e^{gamma_C} colsum(dS' .* S)
          const int cc = c + u;
          const float eC = s.er[cc] * s.erc[cc];
          dgv += s.ktk[cc] + s.ktk[D + cc] + s.ktk[2 * D + cc] + s.ktk[3 * D + cc] +
                 eC * (s.dgc[cc] + s.dgc[D + cc] + s.dgc[2 * D + cc] + s.dgc[3 * D + cc]);
        }
        dbrow[hh] += kv * t1;
        outq[u] = ep * Z[jt][e];
        P[jt][e] = bi * t1 + t2;
        Q[jt][e] = dgv;
      }
      if (i < nvalid)
        *reinterpret_cast<uint32_t*>(dq + rowg[hh] + c) = frag::pack(outq[0], outq[1]);
    }
  // d(beta_eff) partials: reduce the 4 lanes that share a row, one slot per column quarter
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    float xx = dbrow[hh];
    xx += __shfl_xor_sync(0xffffffffu, xx, 1);
    xx += __shfl_xor_sync(0xffffffffu, xx, 2);
    if ((lane & 3) == 0) s.dbp[(i0 + hh * 8) * 4 + qt] = xx;
  }
  __syncthreads();  // the S and dS' tile regions are free: the dgamma tile (row stride LDG)
  float* sdg = reinterpret_cast<float*>(s.SS);
  if (gk == D) {
#pragma unroll
    for (int jt = 0; jt < 4; ++jt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        sdg[(i0 + (e >> 1) * 8) * LDG + qt * 32 + jt * 8 + lc + (e & 1)] = Q[jt][e];
  } else {
    // scalar gate: the row sums of dgamma, one slot per column quarter
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float xx = 0.f;
#pragma unroll
      for (int jt = 0; jt < 4; ++jt) xx += Q[jt][2 * hh] + Q[jt][2 * hh + 1];
      xx += __shfl_xor_sync(0xffffffffu, xx, 1);
      xx += __shfl_xor_sync(0xffffffffu, xx, 2);
      if ((lane & 3) == 0) sdg[(i0 + hh * 8) * 4 + qt] = xx;
    }
  }
  __syncthreads();
  float dbt = 0.f;
  if (tid < C) dbt = s.dbp[tid * 4] + s.dbp[tid * 4 + 1] + s.dbp[tid * 4 + 2] + s.dbp[tid * 4 + 3];
  const int gc = tid & 127, grq = tid >> 7;  // dgamma reverse scan: channel, row quarter
  if (gk == D) {
    float part = 0.f;
#pragma unroll 4
    for (int i = grq * 16; i < grq * 16 + 16; ++i) part += sdg[i * LDG + gc];
    s.dgc[grq * D + gc] = part;  // the chunk-end term read dgc before the last two barriers
  }
  if (tid < C) s.dbp[tid * 4] = dbt;  // total d(beta_eff) of row tid
  __syncthreads();
  // dk (with the Kaczmarz chain rule) and dbeta
#pragma unroll
  for (int jt = 0; jt < 4; ++jt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int i = i0 + hh * 8, c = qt * 32 + jt * 8 + lc;
      float o0 = P[jt][2 * hh], o1 = P[jt][2 * hh + 1];
      if (p.beta_mode == kBetaKaczmarz) {
        const float f = -2.f * s.beta[i] * s.dbp[i * 4] / (s.knorm[i] + p.eps);
        const float2 kk = k2(i, c);
        o0 += f * kk.x;
        o1 += f * kk.y;
      }
      if (i < nvalid) *reinterpret_cast<uint32_t*>(dk + rowg[hh] + c) = frag::pack(o0, o1);
    }
  if (tid < nvalid) {
    if (p.beta_mode == kBetaKaczmarz) dbt /= (s.knorm[tid] + p.eps);
    dbeta[row_id(p, b, t0 + tid, h)] = dbt;
  }
  // dgamma: reverse cumulative sum over the chunk's rows
  if (gk == D) {
    float run = 0.f;
    for (int q2 = grq + 1; q2 < 4; ++q2) run += s.dgc[q2 * D + gc];
#pragma unroll 4
    for (int i = grq * 16 + 15; i >= grq * 16; --i) {
      run += sdg[i * LDG + gc];
      if (i < nvalid) dg[row_id(p, b, t0 + i, h) * D + gc] = run;
    }
  } else if (p.gate != kGateNone && warp == 0) {
    // rows 2 lane, 2 lane + 1: suffix sums across the warp
    const int ia = 2 * lane, ib = ia + 1;
    const float a0 = sdg[ia * 4] + sdg[ia * 4 + 1] + sdg[ia * 4 + 2] + sdg[ia * 4 + 3];
    const float a1 = sdg[ib * 4] + sdg[ib * 4 + 1] + sdg[ib * 4 + 2] + sdg[ib * 4 + 3];
    float x = a0 + a1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_down_sync(0xffffffffu, x, o);
      if (lane + o < 32) x += y;
    }
    if (ia < nvalid) dg[row_id(p, b, t0 + ia, h)] = x;
    if (ib < nvalid) dg[row_id(p, b, t0 + ib, h)] = x - a0;
  }
  } while (0);
  if (!ok) {
    // a bounded wait gave up: record it and drain the copies in flight
    if (tid == 0 && err) atomicExch(err, 1);
    frag::cp_wait<0>();
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tb, 512);
}

}  // namespace

cudaError_t launch_bwd_chunk_hy(const Problem& p, const bf16* q, const bf16* k, const bf16* v,
                                const bf16* dO, const float* g, const Saved& sv, const bf16* dh,
                                const bf16* dU, bf16* dq, bf16* dk, bf16* dv, float* dbeta,
                                float* dg, cudaStream_t st) {
  const size_t sm = sizeof(HySmem) + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(k_bwd_chunk_hy, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const double nb = (double)p.B * p.H * p.NC, ntok = nb * C;
  // operator I/O: reads q, k, v, dO, g, beta; writes dq, dk, dv, dbeta, dg
  const double io = ntok * (4 * D * 2 + p.gk * 4 + 4) + ntok * (3 * D * 2 + p.gk * 4 + 4);
  // and by design the chunk tiles T, h, dh, U, dU, W, U' (and beta, ||k||^2 from the saved set)
  const double bytes = io + nb * C * C * 2 + nb * 2.0 * D * D * 2 + ntok * 4 * D * 2 + ntok * 4;
  const double mac = (double)C * D * D * 3 + (double)C * C * D + (double)C * D * C * 2 +
                     (double)C * C * D * 2 + (double)C * D * C * 4;
  prof_begin(kKTcChunkBwd, io, bytes, nb * 2.0 * mac, st);
  k_bwd_chunk_hy<<<dim3(p.NC, p.H, p.B), NTB, sm, st>>>(
      p, q, k, v, dO, g, sv.T, sv.beta, sv.h, dh, sv.U, dU, sv.W, sv.Up, sv.knorm, dq, dk, dv,
      dbeta, dg, device_error_word(), take_injected_timeout() ? 1 : 0);
  e = cudaGetLastError();
  prof_end(st);
  return e;
}

}  // namespace fast
}  // namespace dr
