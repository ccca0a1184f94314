// fast_prep.cu -- the intra-chunk forward (WY / UT transform) on tcgen05 tensor
// cores, fed by TMA (bf16 storage, d_k = d_v = 128, C = 64).
//
// One CTA per (b, h, chunk), 256 threads, two CTAs per SM.  Every quantity of
// the chunk that does not depend on the state, computed once:
//   g     inclusive within-chunk cumulative log-gate (per key channel; scalar
//         gates broadcast; zero without a gate)
//   beta  the write strength (Kaczmarz step beta = eta / (||k||^2 + eps) applied)
//   A     = diag(beta) strict_tril(G),  M = tril(Gq)  with the gate-scaled Grams
//         G_ij = sum_c k_ic k_jc e^{g_ic - g_jc},  Gq_ij = sum_c q_ic k_jc e^{g_ic - g_jc}
//   T     = (I + A)^{-1}, in fp32 by column-parallel forward substitution
//   W     = T diag(beta) (k e^g),  U' = T diag(beta) v   (T split into two bf16 terms)
//   Qh    = q e^g,  Kt = k e^{g_C - g},  dec = e^{g_C}
// and writes them to the saved buffer, core-tiled (8 x 8 blocks of 128
// contiguous bytes), for the state scans and the backward.  This is the
// chunk's triangular residual system (I + A)[U' | W] = diag(beta)[V | k e^g]
// (ReWY abstract; the SFDA explainer's constructive chunk-WY theorem).
//
// Grams with per-half reference rows.  Row i of the Grams uses the reference
// row rho of its own 32-row half (rows 15 and 47):
//   G_ij = sum_c (k_ic e^{g_ic - g_rho,c}) (k_jc e^{g_rho,c - g_jc}),
// where the first factor spans at most 16 rows of decay, and the second too for
// j in the same half, while for j in the earlier half it is at most 1.  So no
// operand overflows unless the gates decay by more than about 5.5 nats per
// token over 16 tokens ("centered matrix contractions", ReWY abstract); the
// first half's rows and the second half's are two tcgen05 products
// ([K; Q] of the half, M = 64) against their own reference's write keys.
//
// PHASE: the SFDA rotation-decay gate ("Semidirect Fourier Delta Attention"
// explainer, Kernarchitektur).  Key channels pair up as complex numbers; with
// zeta_i = e^{g_i - i Theta_i} per pair (g, Theta: the cumulative sums at the
// pair's even and odd channels) the chunk is a plain delta rule with read keys
// zeta_i k_i, write keys k_i / conj(zeta_i), queries zeta_i q_i and end keys
// conj(zeta_C / zeta_i) k_i (the explainer's constructive chunk-WY theorem),
// so every real factor above becomes a per-pair complex one; dec holds
// conj(zeta_C) per pair.
//
// Data movement: q, k, v and a per-channel gate arrive by TMA
// (cp.async.bulk.tensor, 128-byte swizzled boxes of 64 tokens x 128 bytes, the
// ragged tail zero-filled as out of bounds); the tcgen05 operands are written
// core-tiled in place of the tiles they are computed from.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <string.h>

#include <mutex>

#include "dr_common.cuh"
#include "fast.cuh"
#include "frag.cuh"
#include "tc.cuh"

namespace dr {
namespace fast {

using frag::bf16;

namespace {

constexpr int C = 64, D = 128;
constexpr int NTP = 256;
constexpr int kRho0 = 15, kRho1 = 47;  // reference rows of the two halves
constexpr uint32_t kSpinPrep = 1u << 22;
constexpr uint32_t kBox = 8192;        // one TMA box: 64 rows x 128 bytes

struct PrepSmem {
  // TMA destinations (1 KB aligned), reused in place for the tcgen05 operands
  alignas(1024) unsigned char Q[2 * kBox];  // q; then [K; Q] of the first half (Gram A, K-major)
  alignas(1024) unsigned char K[2 * kBox];  // k; then [K; Q] of the second half
  alignas(1024) unsigned char V[2 * kBox];  // v; then beta v (MN-major B of U')
  alignas(1024) unsigned char G[4 * kBox];  // per-channel gate (fp32, four boxes) -> cumulative;
                                            // then A^T (fp32 [j][i]) and T hi | lo (bf16)
  alignas(1024) unsigned char KB[3 * kBox]; // write keys: rho0 rows 0..31 | rho1 rows 0..63;
                                            // then beta k e^g (MN-major B of W)
  // per key channel (phase gate: per pair, complex, at the pair's two channels),
  // for the two halves' reference rows rho0 = 15, rho1 = 47:
  alignas(16) float ref[2][D];   // cumulative gate at rho
  float rot[2][D];   // phase gate: (cos, sin) of the cumulative phase at rho
  alignas(16) float zr[2][D];    // zeta_rho                     (real gates: e^{g_rho})
  alignas(16) float ec[2][D];    // conj(zeta_C / zeta_rho)      (real gates: e^{g_C - g_rho})
  // write keys of the first half against the second reference, in two steps
  // through the half boundary: conj(zeta_31 / zeta_rho0), conj(zeta_rho1 / zeta_31)
  alignas(16) float xk[2][D];
  float gs[C];       // scalar gate: cumulative per row
  float eta[C];      // input beta (eta in Kaczmarz mode)
  float beta[C];     // effective beta
  uint64_t bar_tma, bar_mma;
  uint32_t tmem;
};

static_assert(sizeof(float) * (64 * (64 + 4) + 32 * (32 + 4)) <= 4 * kBox &&
                  offsetof(PrepSmem, K) == offsetof(PrepSmem, Q) + 2 * kBox,
              "the fp32 solve tiles fit the adjacent q and k regions");

// Byte offset of 16-byte chunk ch (0..7) of row r in a 128-byte-swizzled TMA
// box (chunk index XOR row mod 8 within each 1 KB block).
__device__ __forceinline__ uint32_t swz(int r, int ch) {
  return (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4));
}
// Byte offset of 16-byte chunk j of row r in a core-tiled [rows][128] bf16 tile.
__device__ __forceinline__ uint32_t ct16(int r, int j) {
  return (uint32_t)((((r >> 3) * 16 + j) << 7) + ((r & 7) << 4));
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, int c3, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(tc::smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(tc::smem_u32(bar))
      : "memory");
}

// L2 prefetch of one TMA box (no shared-memory destination).
__device__ __forceinline__ void tma_prefetch_4d(const CUtensorMap* map, int c0, int c1, int c2,
                                                int c3) {
  asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}

// 32 consecutive fp32 TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
  tc::tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void unpack8(const uint4& r, float* f) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(&r);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 x = frag::unpack(w[e]);
    f[2 * e] = x.x;
    f[2 * e + 1] = x.y;
  }
}
__device__ __forceinline__ uint4 pack8(const float* f) {
  return make_uint4(frag::pack(f[0], f[1]), frag::pack(f[2], f[3]), frag::pack(f[4], f[5]),
                    frag::pack(f[6], f[7]));
}


template <bool PHASE>
__global__ void __launch_bounds__(NTP, 2)
    k_prep_tc(Problem p, const __grid_constant__ CUtensorMap tq,
              const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
              const __grid_constant__ CUtensorMap tg, const float* __restrict__ g_scalar,
              const float* __restrict__ beta_in, Saved sv, int* __restrict__ err,
              int pf_ahead) {
  extern __shared__ __align__(1024) unsigned char smraw[];
  PrepSmem& s = *reinterpret_cast<PrepSmem*>(
      (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int t0 = n * C, nvalid = min(C, p.T - t0);
  const size_t cb = chunk_id(p, b, h, n);
  const bool chan = p.gk == D;  // per-channel (or phase) gate in the G tile

  if (warp == 0) tc::tmem_alloc(&s.tmem, 256);
  if (tid == 0) {
    tc::mbar_init(&s.bar_tma, 1);
    tc::mbar_init(&s.bar_mma, 1);
    tc::fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    tc::mbar_arrive_expect_tx(&s.bar_tma, 6 * kBox + (chan ? 4 * kBox : 0));
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      tma_load_4d(s.Q + x * kBox, &tq, 64 * x, h, t0, b, &s.bar_tma);
      tma_load_4d(s.K + x * kBox, &tk, 64 * x, h, t0, b, &s.bar_tma);
      tma_load_4d(s.V + x * kBox, &tv, 64 * x, h, t0, b, &s.bar_tma);
    }
    if (chan) {
#pragma unroll
      for (int x = 0; x < 4; ++x) tma_load_4d(s.G + x * kBox, &tg, 32 * x, h, t0, b, &s.bar_tma);
    }
  }
  // L2 prefetch of the tiles of the CTA pf_ahead places further in launch order
  // (about one wave ahead), so that its TMA loads are served from L2 (measured:
  // 478 against 493 us when issued after this CTA's own loads have landed)
  if (tid == 32 && pf_ahead > 0) {
    const long L = n + (long)p.NC * (h + (long)p.H * b) + pf_ahead;
    if (L < (long)p.NC * p.H * p.B) {
      const int n2 = (int)(L % p.NC), h2 = (int)((L / p.NC) % p.H), b2 = (int)(L / ((long)p.NC * p.H));
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        tma_prefetch_4d(&tq, 64 * x, h2, n2 * C, b2);
        tma_prefetch_4d(&tk, 64 * x, h2, n2 * C, b2);
        tma_prefetch_4d(&tv, 64 * x, h2, n2 * C, b2);
      }
      if (chan) {
#pragma unroll
        for (int x = 0; x < 4; ++x) tma_prefetch_4d(&tg, 32 * x, h2, n2 * C, b2);
      }
    }
  }

  if (!chan && tid < C)
    s.gs[tid] = (tid < nvalid && p.gate != kGateNone) ? g_scalar[row_id(p, b, t0 + tid, h)] : 0.f;
  const float eta = (tid < C && tid < nvalid) ? beta_in[row_id(p, b, t0 + tid, h)] : 0.f;
  // each thread waits for the TMA tiles itself; a failed wait is settled at the
  // barrier after the gate scan (and the MMA waits below at the next barrier)
  bool bad = !tc::mbar_wait(&s.bar_tma, 0u, kSpinPrep);
  tc::fence_after_sync();
  bool ok = true;
  const uint32_t tb = s.tmem;
  do {  // leaves early (break) only when a bounded wait gives up
  // ---- cumulative gate down the rows (padded rows carry a zero gate)
  // per-channel element (r, c) of the gate tile: box c / 32, chunk (c % 32) / 4
  auto gp = [&](int r, int c) -> float* {
    return reinterpret_cast<float*>(s.G + (c >> 5) * kBox + swz(r, (c & 31) >> 2) + (c & 3) * 4);
  };
  // a scalar gate arrives by plain loads of threads 0..63: visible to warp 0's scan
  // only after a barrier (the per-channel gate came by TMA, which each thread waited for)
  if (!chan) __syncthreads();
  if (chan) {
    // thread: channels 4 qd .. 4 qd + 3 (one 16-byte chunk of a swizzled box), rows
    // 8 sg .. 8 sg + 7, scanned in registers; then the totals of the earlier row
    // segments, through the write-key tile (not yet written)
    const int qd = tid & 31, sg = tid >> 5, c4 = 4 * qd;
    float4* segtot = reinterpret_cast<float4*>(s.KB);  // [8 segments][32 channel quads]
    float4 x[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) x[r] = *reinterpret_cast<const float4*>(gp(8 * sg + r, c4));
#pragma unroll
    for (int r = 1; r < 8; ++r) {
      x[r].x += x[r - 1].x;
      x[r].y += x[r - 1].y;
      x[r].z += x[r - 1].z;
      x[r].w += x[r - 1].w;
    }
    segtot[sg * 32 + qd] = x[7];
    __syncthreads();
    float4 off = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s2 = 0; s2 < sg; ++s2) {
      const float4 t = segtot[s2 * 32 + qd];
      off.x += t.x, off.y += t.y, off.z += t.z, off.w += t.w;
    }
#pragma unroll
    for (int r = 0; r < 8; ++r)
      *reinterpret_cast<float4*>(gp(8 * sg + r, c4)) =
          make_float4(x[r].x + off.x, x[r].y + off.y, x[r].z + off.z, x[r].w + off.w);
  } else if (warp == 0) {
    const float a0 = s.gs[2 * lane], a1 = s.gs[2 * lane + 1];
    float x = a0 + a1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    s.gs[2 * lane + 1] = x;
    s.gs[2 * lane] = x - a1;
  }
  ok = __syncthreads_or(bad ? 1 : 0) == 0;
  if (!ok) break;
  auto gam = [&](int r, int c) -> float { return chan ? *gp(r, c) : s.gs[r]; };
  // per-channel reference factors and the chunk decay
  if (PHASE) {
    if (tid < D / 2) {
      const int c = 2 * tid;
      const float gC = gam(C - 1, c), tC = gam(C - 1, c + 1);
      const float g31 = gam(31, c), t31 = gam(31, c + 1);
      float gr[2], tr[2], sn, cs;
      gr[0] = gam(kRho0, c), tr[0] = gam(kRho0, c + 1);
      gr[1] = gam(kRho1, c), tr[1] = gam(kRho1, c + 1);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        s.ref[hh][c] = gr[hh];
        sincosf(tr[hh], &sn, &cs);
        s.rot[hh][c] = cs, s.rot[hh][c + 1] = sn;
        const float m = __expf(gr[hh]);
        s.zr[hh][c] = m * cs, s.zr[hh][c + 1] = -m * sn;          // zeta_rho
        sincosf(tC - tr[hh], &sn, &cs);
        const float mc = __expf(gC - gr[hh]);
        s.ec[hh][c] = mc * cs, s.ec[hh][c + 1] = mc * sn;         // conj(zeta_C / zeta_rho)
      }
      sincosf(t31 - tr[0], &sn, &cs);
      float m = __expf(g31 - gr[0]);
      s.xk[0][c] = m * cs, s.xk[0][c + 1] = m * sn;
      sincosf(tr[1] - t31, &sn, &cs);
      m = __expf(gr[1] - g31);
      s.xk[1][c] = m * cs, s.xk[1][c + 1] = m * sn;
      // the chunk decay conj(zeta_C) = e^{g_C} e^{+i Theta_C}
      sincosf(tC, &sn, &cs);
      const float a = __expf(gC);
      sv.dec[cb * D + c] = a * cs;
      sv.dec[cb * D + c + 1] = a * sn;
    }
  } else if (tid < D) {
    const int c = tid;
    const float g0 = gam(kRho0, c), g1 = gam(kRho1, c), gC = gam(C - 1, c), g31 = gam(31, c);
    s.ref[0][c] = g0, s.ref[1][c] = g1;
    s.zr[0][c] = __expf(g0), s.zr[1][c] = __expf(g1);
    s.ec[0][c] = __expf(gC - g0), s.ec[1][c] = __expf(gC - g1);
    s.xk[0][c] = __expf(g31 - g0), s.xk[1][c] = __expf(g1 - g31);
    sv.dec[cb * D + c] = __expf(gC);
  }

  // ---- factor pass.  Warp w: rows 8w .. 8w + 7; lane: row 8w + lane % 8 and the
  // 16-byte chunks j = lane / 8 + 4 it (it = 0..3) of its 128 channels, so that
  // the swizzled TMA tiles are read and the core-tiled operands written without
  // bank conflicts.  Per element two exponentials, e^{+-(g - g_rho)}; the other
  // factors are those times per-channel reference factors (a product that
  // underflows there is below e^{-37} of the row's leading terms).
  const int r = 8 * warp + (lane & 7), jq = lane >> 3, hr = r >> 5;
  uint4 qr[4], kr[4], vr[4];
  float nn = 0.f;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int j = jq + 4 * it;
    qr[it] = *reinterpret_cast<const uint4*>(s.Q + (j >> 3) * kBox + swz(r, j & 7));
    kr[it] = *reinterpret_cast<const uint4*>(s.K + (j >> 3) * kBox + swz(r, j & 7));
    vr[it] = *reinterpret_cast<const uint4*>(s.V + (j >> 3) * kBox + swz(r, j & 7));
    float kv[8];
    unpack8(kr[it], kv);
#pragma unroll
    for (int e = 0; e < 8; ++e) nn += kv[e] * kv[e];
  }
  nn += __shfl_xor_sync(0xffffffffu, nn, 8);
  nn += __shfl_xor_sync(0xffffffffu, nn, 16);
  if (tid < C) s.eta[tid] = eta;
  __syncthreads();  // every thread holds its q, k, v: the tiles may be rewritten
  const float br = (r < nvalid)
                       ? ((p.beta_mode == kBetaKaczmarz) ? s.eta[r] / (nn + p.eps) : s.eta[r])
                       : 0.f;
  if (jq == 0) {
    sv.beta[cb * C + r] = br;
    sv.knorm[cb * C + r] = nn;
  }
  uint4 bkr[4];  // beta k e^g, held until the write-key tiles are free
  {
    unsigned char* GAh = hr ? s.K : s.Q;      // [K; Q] of this row's half
    const int R = r & 31;                     // row within the half
    const float sg = chan ? 0.f : s.gs[r];
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int j = jq + 4 * it, c0 = 8 * j;
      float kv[8], qv[8], vv[8], gg[8];
      unpack8(kr[it], kv);
      unpack8(qr[it], qv);
      unpack8(vr[it], vv);
      if (chan) {
        const float4 a = *reinterpret_cast<const float4*>(s.G + (j >> 2) * kBox + swz(r, 2 * (j & 3)));
        const float4 c4 = *reinterpret_cast<const float4*>(s.G + (j >> 2) * kBox + swz(r, 2 * (j & 3) + 1));
        gg[0] = a.x, gg[1] = a.y, gg[2] = a.z, gg[3] = a.w;
        gg[4] = c4.x, gg[5] = c4.y, gg[6] = c4.z, gg[7] = c4.w;
      }
      float kc[8], qc[8], kb[8], kb1[8], qh[8], kt[8], bk[8], bv[8];
      if (PHASE) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int e = 2 * m, cc = c0 + e;
          float sn, cs;
          sincosf(gg[e + 1], &sn, &cs);                  // e^{-i Theta} = cs - i sn
          const float rhc = s.rot[hr][cc], rhs = s.rot[hr][cc + 1];   // e^{i Theta_rho}
          // e^{-i (Theta - Theta_rho)}
          const float wr = cs * rhc + sn * rhs, wi = cs * rhs - sn * rhc;
          const float d = gg[e] - s.ref[hr][cc];
          const float ep = __expf(d), em = __expf(-d);
          const float kx = kv[e], ky = kv[e + 1], qx = qv[e], qy = qv[e + 1];
          const float kwx = wr * kx - wi * ky, kwy = wi * kx + wr * ky;
          const float qwx = wr * qx - wi * qy, qwy = wi * qx + wr * qy;
          kc[e] = ep * kwx, kc[e + 1] = ep * kwy;        // u k
          qc[e] = ep * qwx, qc[e + 1] = ep * qwy;        // u q
          kb[e] = em * kwx, kb[e + 1] = em * kwy;        // k / conj(u)
          const float zx = s.zr[hr][cc], zy = s.zr[hr][cc + 1];
          qh[e] = zx * qc[e] - zy * qc[e + 1], qh[e + 1] = zx * qc[e + 1] + zy * qc[e];  // zeta q
          bk[e] = br * (zx * kc[e] - zy * kc[e + 1]), bk[e + 1] = br * (zx * kc[e + 1] + zy * kc[e]);
          const float ex = s.ec[hr][cc], ey = s.ec[hr][cc + 1];
          kt[e] = ex * kb[e] - ey * kb[e + 1], kt[e + 1] = ex * kb[e + 1] + ey * kb[e];
          if (hr == 0) {
            const float ax = s.xk[0][cc], ay = s.xk[0][cc + 1];
            const float bx = s.xk[1][cc], by = s.xk[1][cc + 1];
            const float tx = ax * kb[e] - ay * kb[e + 1], ty = ax * kb[e + 1] + ay * kb[e];
            kb1[e] = bx * tx - by * ty, kb1[e + 1] = bx * ty + by * tx;
          }
        }
      } else {
        float eps_ = 1.f, ems_ = 1.f;
        if (!chan) {  // one factor per row
          eps_ = __expf(sg - s.ref[hr][0]);
          ems_ = __expf(s.ref[hr][0] - sg);
        }
        // the per-channel reference factors of these 8 channels (vector loads)
        float r8[8], z8[8], e8[8], x0[8], x1[8];
        frag::load8(s.ref[hr] + c0, r8);
        frag::load8(s.zr[hr] + c0, z8);
        frag::load8(s.ec[hr] + c0, e8);
        if (hr == 0) {
          frag::load8(s.xk[0] + c0, x0);
          frag::load8(s.xk[1] + c0, x1);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float ep = eps_, em = ems_;
          if (chan) {  // e^{+-(g - g_rho)} as 2^{+-(g - g_rho) log2 e}
            const float d2 = (gg[e] - r8[e]) * frag::kLog2e;
            ep = frag::ex2_approx(d2), em = frag::ex2_approx(-d2);
          }
          kc[e] = kv[e] * ep;
          qc[e] = qv[e] * ep;
          kb[e] = kv[e] * em;
          qh[e] = qc[e] * z8[e];
          bk[e] = br * kc[e] * z8[e];
          kt[e] = kb[e] * e8[e];
          if (hr == 0) kb1[e] = kb[e] * x0[e] * x1[e];
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) bv[e] = br * vv[e];
      *reinterpret_cast<uint4*>(GAh + ct16(R, j)) = pack8(kc);
      *reinterpret_cast<uint4*>(GAh + ct16(32 + R, j)) = pack8(qc);
      if (hr == 0) {
        *reinterpret_cast<uint4*>(s.KB + ct16(r, j)) = pack8(kb);
        *reinterpret_cast<uint4*>(s.KB + 4 * 2048 + ct16(r, j)) = pack8(kb1);
      } else {
        *reinterpret_cast<uint4*>(s.KB + 4 * 2048 + ct16(r, j)) = pack8(kb);
      }
      *reinterpret_cast<uint4*>(s.V + ct16(r, j)) = pack8(bv);
      *reinterpret_cast<uint4*>(sv.Qh + cb * C * D + ct_off(r, c0, D)) = pack8(qh);
      *reinterpret_cast<uint4*>(sv.Kt + cb * C * D + ct_off(r, c0, D)) = pack8(kt);
      bkr[it] = pack8(bk);
    }
  }
  if (jq == 0) s.beta[r] = br;
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();

  // ---- Grams on tcgen05, one M = 128 product:
  //   rows [K; Q] of the first half (0..63) and of the second half (64..127),
  //   columns: the first reference's write keys of rows 0..31 (0..31) and the
  //   second reference's of rows 0..63 (32..95).  Each half reads only the
  //   columns of its own reference.
  if (tid == 0) {
    const uint32_t id = tc::idesc_bf16(128, 96, false, false);
    const uint64_t a = tc::sdesc_kmaj(reinterpret_cast<const bf16*>(s.Q), D, 0);
    const uint64_t bb = tc::sdesc_kmaj(reinterpret_cast<const bf16*>(s.KB), D, 0);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) tc::mma(tb, a + 16u * ks, bb + 16u * ks, id, ks > 0 ? 1u : 0u);
    tc::commit(&s.bar_mma);
  }
  bad = !tc::mbar_wait(&s.bar_mma, 0u, kSpinPrep);
  tc::fence_after_sync();
  // ---- A^T (fp32, [j][i]) into the gate tile's first half; M (bf16) to global.
  // Accumulator row = lane: quadrant 0 A rows of the first half, 1 its M rows,
  // 2 and 3 those of the second half; warps w and w + 4 split the columns.
  float* At = reinterpret_cast<float*>(s.G);
  {
    const int qd = warp & 3, side = warp >> 2, hq = qd >> 1;
    const int i = 32 * hq + lane;                       // chunk row of A or M
    const bool isA = (qd & 1) == 0;
    const int w = hq ? 32 : 16;                         // columns this warp reads
    float d[32];
    const uint32_t ta = tb + ((uint32_t)(32 * qd) << 16) + (hq ? 32u : 0u) + (uint32_t)(side * w);
    if (hq) {
      tmem_ld32(ta, d);
    } else {
      float t16[32];
      tmem_ld32(ta, t16);  // 32 columns from the warp's start; the first 16 are its own
#pragma unroll
      for (int e = 0; e < 16; ++e) d[e] = t16[e];
    }
    const int j0 = side * w;                            // first column (row j of the chunk)
    if (isA) {
      const float bi = s.beta[i];
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (e < w) At[(j0 + e) * C + i] = (j0 + e < i) ? bi * d[e] : 0.f;
      if (hq == 0 && side == 1) {
#pragma unroll 8
        for (int j = 32; j < C; ++j) At[j * C + i] = 0.f;
      }
    } else {
      bf16* Mg = sv.M + cb * C * C;
#pragma unroll
      for (int j8 = 0; j8 < 4; ++j8) {
        if (8 * j8 < w) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = (j0 + 8 * j8 + e <= i) ? d[8 * j8 + e] : 0.f;
          *reinterpret_cast<uint4*>(Mg + ct_off(i, j0 + 8 * j8, C)) = pack8(f);
        }
      }
      if (hq == 0 && side == 1) {
        const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j8 = 4; j8 < 8; ++j8) *reinterpret_cast<uint4*>(Mg + ct_off(i, 8 * j8, C)) = pack8(z);
      }
    }
  }
  // beta k e^g into the write-key tile (the Grams have read it)
  {
#pragma unroll
    for (int it = 0; it < 4; ++it)
      *reinterpret_cast<uint4*>(s.KB + ct16(r, jq + 4 * it)) = bkr[it];
  }
  tc::fence_before_sync();
  ok = __syncthreads_or(bad ? 1 : 0) == 0;
  if (!ok) break;
  // ---- T = (I + A)^{-1} in fp32, by blocks of 32:
  //   T11 = (I + A11)^{-1}, T22 = (I + A22)^{-1} (thread j < 64 forward-substitutes
  //   one column of one of them, all its rows in registers), then
  //   T21 = -T22 (A21 T11) by two 32 x 32 products on all threads;
  //   finally T = T_hi + T_lo in bf16, the tcgen05 operand.
  // fp32 T, row stride TLD (16-byte rows of 8 consecutive rows in distinct banks),
  // over the Gram operands (read); Y = A21 T11, row stride YLD
  constexpr int TLD = C + 4, YLD = 32 + 4;
  unsigned char* const qk = reinterpret_cast<unsigned char*>(&s) + offsetof(PrepSmem, Q);
  float* Tf = reinterpret_cast<float*>(qk);
  float* Yb = reinterpret_cast<float*>(qk + C * TLD * 4);
  if (tid < C) {
    const int blk = tid >> 5, j = tid & 31, o = 32 * blk;
    float acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = (i == j) ? 1.f : 0.f;
#pragma unroll
    for (int m = 0; m < 31; ++m) {
      const float tm = acc[m];
      const float* arow = At + (o + m) * C + o;  // A[o + .][o + m]
#pragma unroll
      for (int i4 = (m + 1) & ~3; i4 < 32; i4 += 4) {
        const float4 a = *reinterpret_cast<const float4*>(arow + i4);
        if (i4 + 0 > m) acc[i4 + 0] -= a.x * tm;
        if (i4 + 1 > m) acc[i4 + 1] -= a.y * tm;
        if (i4 + 2 > m) acc[i4 + 2] -= a.z * tm;
        if (i4 + 3 > m) acc[i4 + 3] -= a.w * tm;
      }
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) Tf[(o + i) * TLD + o + j] = acc[i];
    if (blk == 0) {
#pragma unroll
      for (int i = 0; i < 32; ++i) Tf[i * TLD + 32 + j] = 0.f;
    }
  }
  __syncthreads();
  // the two 32 x 32 products: thread -> row ti = tid / 8 (of the second half),
  // columns tj .. tj + 3, tj = 4 (tid % 8) (per k-step one scalar and one
  // 16-byte shared load for four FMAs)
  const int ti = tid >> 3, tj = 4 * (tid & 7);
  {
    // Y = A21 T11
    float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
    for (int m = 0; m < 32; ++m) {
      const float a = At[m * C + 32 + ti];
      const float4 t = *reinterpret_cast<const float4*>(Tf + m * TLD + tj);
      y[0] += a * t.x;
      y[1] += a * t.y;
      y[2] += a * t.z;
      y[3] += a * t.w;
    }
    *reinterpret_cast<float4*>(Yb + ti * YLD + tj) = make_float4(y[0], y[1], y[2], y[3]);
  }
  __syncthreads();
  {
    // T21 = -T22 Y
    float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
    for (int m = 0; m < 32; ++m) {
      const float a = Tf[(32 + ti) * TLD + 32 + m];
      const float4 t = *reinterpret_cast<const float4*>(Yb + m * YLD + tj);
      y[0] += a * t.x;
      y[1] += a * t.y;
      y[2] += a * t.z;
      y[3] += a * t.w;
    }
    *reinterpret_cast<float4*>(Tf + (32 + ti) * TLD + tj) = make_float4(-y[0], -y[1], -y[2], -y[3]);
  }
  __syncthreads();
  bf16* Thi = reinterpret_cast<bf16*>(s.G + 2 * kBox);
  bf16* Tlo = reinterpret_cast<bf16*>(s.G + 3 * kBox);
  for (int idx = tid; idx < C * C / 8; idx += NTP) {  // core-tiled [i][j], 16 bytes per thread
    const int i = ct_row(idx, C), j8 = ct_col(idx, C);
    float hi[8], lo[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float t = Tf[i * TLD + j8 + e];
      hi[e] = __bfloat162float(__float2bfloat16_rn(t));
      lo[e] = t - hi[e];
    }
    const uint4 vh = pack8(hi);
    *reinterpret_cast<uint4*>(Thi + 8 * idx) = vh;
    *reinterpret_cast<uint4*>(Tlo + 8 * idx) = pack8(lo);
    *reinterpret_cast<uint4*>(sv.T + cb * C * C + 8 * idx) = vh;
  }
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  // ---- W = T (beta k e^g), U' = T (beta v): T_hi and T_lo terms, M = 64, N = 128
  if (tid == 0) {
    const uint32_t id = tc::idesc_bf16(64, 128, false, true);
    const uint64_t ah = tc::sdesc_kmaj(Thi, C, 0), al = tc::sdesc_kmaj(Tlo, C, 0);
    const uint64_t bk = tc::sdesc_mnmaj(reinterpret_cast<const bf16*>(s.KB), D, 0);
    const uint64_t bw = tc::sdesc_mnmaj(reinterpret_cast<const bf16*>(s.V), D, 0);
#pragma unroll
    for (int ks = 0; ks < C / 16; ++ks) {
      const uint32_t acc = ks > 0 ? 1u : 0u;
      tc::mma(tb + 0, ah + 16u * ks, bk + 256u * ks, id, acc);
      tc::mma(tb + 128, ah + 16u * ks, bw + 256u * ks, id, acc);
      tc::mma(tb + 0, al + 16u * ks, bk + 256u * ks, id, 1u);
      tc::mma(tb + 128, al + 16u * ks, bw + 256u * ks, id, 1u);
    }
    tc::commit(&s.bar_mma);
  }
  // each warp waits for W, U' itself (the TMEM reads below are warp-wide); a
  // warp whose wait gives up records it and skips its stores
  if (!__all_sync(0xffffffffu, tc::mbar_wait(&s.bar_mma, 1u, kSpinPrep))) {
    if (lane == 0 && err) atomicExch(err, 1);
    break;
  }
  tc::fence_after_sync();
  // ---- W (warps 0-3) and U' (warps 4-7), rows 16 (warp % 4) + lane, lanes 0..15
  {
    const int qd = warp & 3, row = 16 * qd + (lane & 15);
    const uint32_t base = tb + ((uint32_t)(32 * qd) << 16) + (warp < 4 ? 0u : 128u);
    bf16* out = (warp < 4 ? sv.W : sv.Up) + cb * C * D;
#pragma unroll
    for (int q32 = 0; q32 < 4; ++q32) {
      float d[32];
      tmem_ld32(base + 32 * q32, d);
      if (lane < 16) {
#pragma unroll
        for (int e8 = 0; e8 < 4; ++e8)
          *reinterpret_cast<uint4*>(out + ct_off(row, 32 * q32 + 8 * e8, D)) = pack8(d + 8 * e8);
      }
    }
  }
  } while (0);
  if (!ok) {
    // a bounded wait gave up: record it, and give the TMA loads in flight a
    // bounded chance to land before the shared memory is released
    if (tid == 0 && err) atomicExch(err, 1);
    if (tid == 0) tc::mbar_wait(&s.bar_tma, 0u, kSpinPrep);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tb, 256);
}

// --- tensor maps (host) ------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// [B, T, H, 128] row-major, elements of `bytes` bytes; box: 128 bytes of
// channels x 64 tokens of one head, 128-byte swizzle, out-of-range tokens zero.
bool encode_btdh(CUtensorMap* m, const void* base, const Problem& p, int bytes) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)p.H, (cuuint64_t)p.T, (cuuint64_t)p.B};
  const cuuint64_t row = (cuuint64_t)D * bytes;
  const cuuint64_t strides[3] = {row, row * p.H, row * p.H * p.T};
  const cuuint32_t box[4] = {(cuuint32_t)(128 / bytes), 1, (cuuint32_t)C, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
             const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_prep(const Problem& p, const bf16* q, const bf16* k, const bf16* v,
                        const float* beta, const float* g, const Saved& sv, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mg;
  memset(&mg, 0, sizeof(mg));
  const bool chan = p.gk == D;
  if (!encode_btdh(&mq, q, p, 2) || !encode_btdh(&mk, k, p, 2) || !encode_btdh(&mv, v, p, 2) ||
      (chan && !encode_btdh(&mg, g, p, 4)))
    return cudaErrorInvalidValue;
  const size_t sm = sizeof(PrepSmem) + 1024;
  const bool phase = p.gate == kGatePhase;
  auto kern = phase ? k_prep_tc<true> : k_prep_tc<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const double nb = (double)p.B * p.H * p.NC, ntok = nb * C;
  // reads q, k, v, g, beta (the operator's inputs); writes T, beta, dec, W, U', M, Qh, Kt, ||k||^2
  const double io = ntok * (3 * D * 2 + p.gk * 4 + 4);
  const double bytes =
      io + nb * ((double)kTBytes + 2 * kBetaBytes + kDecBytes + 4.0 * kTileBytes + kMBytes);
  // Grams (32 + 64 columns of M = 64, K = 128), the solve (C^3 / 3), W and U' (two T terms)
  const double flops = nb * (2.0 * C * 96 * D + C * C * C / 3.0 + 2.0 * 2 * 2 * C * C * D);
  prof_begin(kKTcIntraFwd, io, bytes, flops, st);
  kern<<<dim3(p.NC, p.H, p.B), NTP, sm, st>>>(p, mq, mk, mv, mg, chan ? nullptr : g, beta, sv,
                                             device_error_word(), 2 * sm_count());
  e = cudaGetLastError();
  prof_end(st);
  return e;
}

}  // namespace fast
}  // namespace dr
