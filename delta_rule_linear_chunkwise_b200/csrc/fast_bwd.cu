// fast_bwd.cu -- tensor-core backward for bf16 storage, d_k = d_v = 128, C = 64.
//
// tc_bwd_scan (sequential in reverse over chunks, one CTA per (b, h, 64-wide
// value tile)): with the fp32 gradient dS of the chunk's end state held in
// registers,
//   dU = M^T dO + Kt dS^T                      (M = tril(Q^c Kb^c^T), Kt = k e^{gamma_C - gamma})
//   dS <- dS Diag(e^{gamma_C}) + dO^T (q e^gamma) - dU^T W
// recomputing M and W = T diag(beta) (k e^gamma) per chunk from q, k, g, T.
// Emits dU (bf16) and dh_n = dS at the end of chunk n (bf16) for the
// chunk-parallel kernel, and dS0.
// tc_bwd_chunk (chunk-parallel): everything else, through the triangular
// residual system (I + A)[U' | W] = diag(beta)[V | K e^gamma]:
//   W, U' = T diag(beta) [K e^gamma | V];  dQs = dO S;  dW = -dU S;  dKt = U dS';
//   dM = tril(dO U^T);  Lambda = T^T [dU | dW];  dA = -strict_tril(Lambda [U' | W]^T);
//   dQ^c = dM Kb^c;  x = dA Kb^c;  dKb^c = dM^T Q^c + dA^T diag(beta) K^c
// and the gate chain rule (reverse cumulative sum of the per-row log-gate
// gradient), dbeta and the Kaczmarz chain rule.

#include "dr_common.cuh"
#include "fast.cuh"
#include "frag.cuh"

namespace dr {
namespace fast {

using frag::bf16;

namespace {

constexpr int C = 64, D = 128;
constexpr int LDD = D + 8;
constexpr int LDC = C + 8;
constexpr int CTD = -D, CTC = -C;  // leading dimensions of core-tiled [.][D] / [.][C] tiles
constexpr int BV = 64;
constexpr int NTS = 256;

__device__ __forceinline__ int centre_row(int nvalid) { return (nvalid - 1) / 2; }

// Position of gate element (i, c) in a [C][D] fp32 tile whose 8-column groups
// are XOR-swizzled by row (i mod 8), so that the column pairs an mma fragment
// holds in its 8 rows hit distinct banks without padding the row; groups of 4
// consecutive columns stay contiguous and 16-byte aligned.
__device__ __forceinline__ int gsw(int i, int c) { return i * D + (c ^ ((i & 7) << 3)); }

// ---------------------------------------------------------------------------
// tc_bwd_scan (thin): streams W, Qh, Kt, M, dec and the dO slice of each chunk
// through a two-stage cp.async pipeline; only the state-gradient chain runs here.
struct BscanStage {  // W, Qh, Kt, M core-tiled, as saved
  bf16 W[C * D];
  bf16 Qh[C * D];
  bf16 Kt[C * D];
  bf16 M[C * C];
  bf16 dO[C * LDC];   // dO[:, a0 .. a0+63]
  float dec[D];
};
struct BscanSmem {
  BscanStage st[2];
  bf16 dS[BV * LDD];  // bf16 copy of the state gradient [a][c]
  bf16 dU[C * LDC];
};

__device__ void bscan_issue(const Problem& p, BscanStage& s, const Saved& sv, const bf16* dO,
                            int b, int h, int n, int a0) {
  const int tid = threadIdx.x, t0 = n * C, nvalid = min(C, p.T - t0);
  const size_t cb = chunk_id(p, b, h, n);
  cp_linear<NTS>(s.W, sv.W + cb * C * D, C * D, tid);
  cp_linear<NTS>(s.Qh, sv.Qh + cb * C * D, C * D, tid);
  cp_linear<NTS>(s.Kt, sv.Kt + cb * C * D, C * D, tid);
  cp_linear<NTS>(s.M, sv.M + cb * C * C, C * C, tid);
  for (int idx = tid; idx < C * (C / 8); idx += NTS) {
    const int i = idx >> 3, j = idx & 7;
    const bool ok = i < nvalid;
    frag::cp16(s.dO + i * LDC + j * 8, dO + row_id(p, b, t0 + (ok ? i : 0), h) * D + a0 + j * 8, ok);
  }
  if (tid < D / 4) frag::cp16(s.dec + tid * 4, sv.dec + cb * D + tid * 4, true);
}

__global__ void __launch_bounds__(NTS, 1)
    k_bwd_scan(Problem p, Saved sv, const bf16* __restrict__ dO, const float* __restrict__ dST,
               float* __restrict__ dS0, bf16* __restrict__ dUout, bf16* __restrict__ dhout) {
  extern __shared__ __align__(16) unsigned char smraw[];
  BscanSmem& s = *reinterpret_cast<BscanSmem*>(smraw);
  const int h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int rb = warp & 3, hf = warp >> 2;
  const int a0 = blockIdx.x * BV;
  const int lr = lane >> 2, lc = 2 * (lane & 3);
  const size_t sbase = ((size_t)b * p.H + h) * D * D;

  float dS[8][4];  // rows a0 + 16rb.., key columns 64hf..
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int a = rb * 16 + lr + (e >> 1) * 8, c = hf * 64 + j * 8 + lc + (e & 1);
      dS[j][e] = dST ? dST[sbase + (size_t)(a0 + a) * D + c] : 0.f;
    }
  frag::st_c(dS, s.dS, LDD, rb * 16, hf * 64);

  bscan_issue(p, s.st[0], sv, dO, b, h, p.NC - 1, a0);
  frag::cp_commit();
  if (p.NC > 1) bscan_issue(p, s.st[1], sv, dO, b, h, p.NC - 2, a0);
  frag::cp_commit();
  for (int n = p.NC - 1, it = 0; n >= 0; --n, ++it) {
    const size_t cb = chunk_id(p, b, h, n);
    BscanStage& st = s.st[it & 1];
    frag::cp_wait<1>();
    __syncthreads();
    // dh_n: gradient of this chunk's end state
    for (int idx = tid; idx < BV * (D / 8); idx += NTS)  // core-tiled rows a0 ..
      *reinterpret_cast<uint4*>(dhout + cb * D * D + ct_off(a0, 0, D) + 8 * idx) =
          *reinterpret_cast<const uint4*>(s.dS + ct_row(idx, D) * LDD + ct_col(idx, D));
    // dU = M^T dO + Kt dS^T, rows i = 16rb.., values 32hf..
    {
      float du[4][4];
      frag::zero(du);
      frag::mm_rows_at<4, 4, true>(du, st.M, CTC, rb * 16, st.dO, LDC, hf * 32);
      frag::mm_rows<4, 8, false>(du, st.Kt, CTD, rb * 16, s.dS, LDD, hf * 32);
      frag::st_c(du, s.dU, LDC, rb * 16, hf * 32);
    }
    __syncthreads();
    for (int idx = tid; idx < C * (BV / 8); idx += NTS) {
      const int grp = idx / BV, k = idx % BV, i = grp * 8 + (k & 7), j = k >> 3;
      *reinterpret_cast<uint4*>(dUout + cb * C * D + ct_off(i, a0 + j * 8, D)) =
          *reinterpret_cast<const uint4*>(s.dU + i * LDC + j * 8);
    }
    // dS <- dS Diag(dec) + dO^T Qh - dU^T W, rows a = 16rb.., keys 64hf..
    {
      float pa[8][4], pb[8][4];
      frag::zero(pa);
      frag::mm_rows_at<8, 4, true>(pa, st.dO, LDC, rb * 16, st.Qh, CTD, hf * 64);
      frag::zero(pb);
      frag::mm_rows_at<8, 4, true>(pb, s.dU, LDC, rb * 16, st.W, CTD, hf * 64);
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          dS[j][e] = dS[j][e] * st.dec[hf * 64 + j * 8 + lc + (e & 1)] + pa[j][e] - pb[j][e];
    }
    __syncthreads();
    if (n >= 2) bscan_issue(p, st, sv, dO, b, h, n - 2, a0);
    frag::cp_commit();
    frag::st_c(dS, s.dS, LDD, rb * 16, hf * 64);
  }
  if (dS0) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int a = rb * 16 + lr + (e >> 1) * 8, c = hf * 64 + j * 8 + lc + (e & 1);
        dS0[sbase + (size_t)(a0 + a) * D + c] = dS[j][e];
      }
  }
}

// ---------------------------------------------------------------------------
// tc_bwd_chunk: 16 warps = 4 row blocks (16 chunk rows) x 4 column quarters.
constexpr int NTB = 512;

struct BchunkSmem {
  bf16 Qc[C * LDD];     // q e^{gamma - gamma_r}
  bf16 k[C * LDD];      // raw k
  bf16 W[C * D];        // T diag(beta) k e^gamma      [j][c]  core-tiled
  bf16 Up[C * D];       // T diag(beta) v              [j][a]  core-tiled
  bf16 dO[C * LDD];
  bf16 dU[C * D];       // core-tiled
  bf16 U[C * D];        // core-tiled; then dA [i][j] (stride LDC)
  bf16 dW[C * LDD];
  bf16 dM[C * LDC];     // tril(dO U^T)               [i][j]
  bf16 T[C * LDC];      // core-tiled [j][i]
  bf16 R[2 * C * LDD];  // S half | dS' half  ->  Lambda_U | Lambda_W
                        // -> Kb^c | beta K^c  ->  dgamma (fp32 [C][D])
  float beta[C];
  float knorm[C];
  float dbp[C * 4];     // dbeta partial sums per column quarter
  float dgc[4 * D];     // colsum(dS' .* S) partials per row quarter
  float ktk[4 * D];     // colsum(Kt .* dKt) partials per row block
  float er[D];          // e^{gamma_r}
  float erc[D];         // e^{gamma_C - gamma_r}
  float G[1];           // [C][D] swizzled (gsw) cumulative gate, then e^{gamma - gamma_r}
};

__global__ void __launch_bounds__(NTB, 1)
    k_bwd_chunk(Problem p, const bf16* __restrict__ q, const bf16* __restrict__ k,
                const bf16* __restrict__ v, const bf16* __restrict__ dO,
                const float* __restrict__ g, const bf16* __restrict__ Tg,
                const float* __restrict__ beta, const bf16* __restrict__ hst,
                const bf16* __restrict__ dhst, const bf16* __restrict__ Ug,
                const bf16* __restrict__ dUg, const bf16* __restrict__ Wg,
                const bf16* __restrict__ Upg, const float* __restrict__ knorm_g,
                bf16* __restrict__ dq, bf16* __restrict__ dk,
                bf16* __restrict__ dv, float* __restrict__ dbeta, float* __restrict__ dg) {
  extern __shared__ __align__(16) unsigned char smraw[];
  BchunkSmem& s = *reinterpret_cast<BchunkSmem*>(smraw);
  const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, gk = p.gk;
  const int rb = warp & 3, qt = warp >> 2;
  const int lr = lane >> 2, lc = 2 * (lane & 3);
  const int t0 = n * C, nvalid = min(C, p.T - t0);
  const size_t cb = chunk_id(p, b, h, n);
  bf16* R0 = s.R;            // first half of the shared region
  bf16* R1 = s.R + C * LDD;  // second half
  bf16* sdA = s.U;

  // ---- loads: q (into Qc), k, dO, W, U', dU, U, T, gate, beta
  // Loads in three cp.async groups, in the order of first use:
  //   1: gate, q, k (gate scan, factor tile, Q^c)   2: dO, dU, U, first half of S and dS'
  //   3 (issued after the first phase-1 half): second half of S and dS'; 4: W, U', T
  for (int idx = tid; idx < C * (D / 8); idx += NTB) {
    const int i = idx >> 4, j = idx & 15;
    const bool ok = i < nvalid;
    const size_t rr = row_id(p, b, t0 + (ok ? i : 0), h) * D + j * 8;
    frag::cp16(s.Qc + i * LDD + j * 8, q + rr, ok);
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
  for (int idx = tid; idx < C * (D / 8); idx += NTB) {
    const int i = idx >> 4, j = idx & 15;
    const bool ok = i < nvalid;
    frag::cp16(s.dO + i * LDD + j * 8, dO + row_id(p, b, t0 + (ok ? i : 0), h) * D + j * 8, ok);
  }
  cp_linear<NTB>(s.dU, dUg + cb * C * D, C * D, tid);
  cp_linear<NTB>(s.U, Ug + cb * C * D, C * D, tid);
  cp_linear<NTB>(R0, hst + cb * D * D, C * D, tid);  // state rows 0 .. 63, core-tiled
  cp_linear<NTB>(R1, dhst + cb * D * D, C * D, tid);
  frag::cp_commit();
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

  // ---- build: Q^c in place (4 columns per thread, one row per warp)
  for (int idx = tid; idx < C * (D / 4); idx += NTB) {
    const int i = idx >> 5, c = (idx & 31) * 4;
    uint2 rq = *reinterpret_cast<const uint2*>(s.Qc + i * LDD + c);
    const float4 f = ep4(i, c);
    const float2 q0 = frag::unpack(rq.x), q1 = frag::unpack(rq.y);
    rq.x = frag::pack(q0.x * f.x, q0.y * f.y);
    rq.y = frag::pack(q1.x * f.z, q1.y * f.w);
    *reinterpret_cast<uint2*>(s.Qc + i * LDD + c) = rq;
  }
  __syncthreads();

  // ---- phase 1b/1c over two halves of the value dimension a
  float zq[4][4], adw[4][4], akt[4][4], adm[2][4];
  frag::zero(zq);
  frag::zero(adw);
  frag::zero(akt);
  frag::zero(adm);
  for (int ah = 0; ah < 2; ++ah) {
    if (ah == 1) {
      cp_linear<NTB>(R0, hst + cb * D * D + C * D, C * D, tid);  // rows 64 .. 127
      cp_linear<NTB>(R1, dhst + cb * D * D + C * D, C * D, tid);
      frag::cp_commit();
      // W, U' (phase 3) and T (phase 2) behind it
      cp_linear<NTB>(s.W, Wg + cb * C * D, C * D, tid);
      cp_linear<NTB>(s.Up, Upg + cb * C * D, C * D, tid);
      cp_linear<NTB>(s.T, Tg + cb * C * C, C * C, tid);
      frag::cp_commit();
      frag::cp_wait<1>();
    } else {
      frag::cp_wait<0>();
    }
    __syncthreads();
    // dQs += dO S ; dW' += dU S ; dKt += U dS'   (contraction over this half of a)
    // The half tiles hold local rows 0..63 (core-tiled); mm_rows indexes B rows
    // from k0 = 64ah.
    const bf16* Sh = R0 - ah * 64 * D;
    const bf16* dSh = R1 - ah * 64 * D;
    frag::mm_rows<4, 4, true>(zq, s.dO, LDD, rb * 16, Sh, CTD, qt * 32, ah * 64);
    frag::mm_rows<4, 4, true>(adw, s.dU, CTD, rb * 16, Sh, CTD, qt * 32, ah * 64);
    frag::mm_rows<4, 4, true>(akt, s.U, CTD, rb * 16, dSh, CTD, qt * 32, ah * 64);
    // dM += dO U^T  (U stored [j][a] = [n][k])
    frag::mm_rows<2, 4, false>(adm, s.dO, LDD, rb * 16, s.U, CTD, qt * 16, ah * 64);
    // colsum(dS' .* S) over this half: thread -> column c, row quarter rq
    {
      const int c = tid & 127, rq = tid >> 7;
      float acc = 0.f;
#pragma unroll 4
      for (int a = rq * 16; a < rq * 16 + 16; ++a)
        acc += __bfloat162float(R0[ct_off(a, c, D)]) * __bfloat162float(R1[ct_off(a, c, D)]);
      s.dgc[rq * D + c] = (ah == 0 ? 0.f : s.dgc[rq * D + c]) + acc;
    }
    __syncthreads();
  }
  // dW = -dW', dM masked (inclusive lower), stored for the later phases
  {
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) adw[j][e] = -adw[j][e];
    frag::st_c(adw, s.dW, LDD, rb * 16, qt * 32);
#pragma unroll
    for (int jt = 0; jt < 2; ++jt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = rb * 16 + lr + (e >> 1) * 8, jj = qt * 16 + jt * 8 + lc + (e & 1);
        if (jj > i) adm[jt][e] = 0.f;
      }
    frag::st_c(adm, s.dM, LDC, rb * 16, qt * 16);
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
  frag::cp_wait<0>();  // W, U', T
  __syncthreads();

  // ---- phase 2: Lambda = T^T [dU | dW]; dv = diag(beta) Lambda_U
  float dbrow[2] = {0.f, 0.f};  // this thread's d(beta_eff) partials for rows i0, i0 + 8
  float Q[4][4];
  {
    uint32_t vv[4][2];
#pragma unroll
    for (int jt = 0; jt < 4; ++jt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
        vv[jt][hh] = *reinterpret_cast<const uint32_t*>(v + rowg[hh] + qt * 32 + jt * 8 + lc);
    float lu[4][4];
    frag::zero(lu);
    frag::mm_rows_at<4, 4, true>(lu, s.T, CTC, rb * 16, s.dU, CTD, qt * 32);
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
    frag::st_c(lu, R0, LDD, rb * 16, qt * 32);
    frag::zero(Q);
    frag::mm_rows_at<4, 4, true>(Q, s.T, CTC, rb * 16, s.dW, LDD, qt * 32);
    frag::st_c(Q, R1, LDD, rb * 16, qt * 32);
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

  // ---- phase 3: dA = -strict_tril(Lambda_U U'^T + Lambda_W W^T), rows 16rb.., cols 16qt..
  {
    float da[2][4];
    frag::zero(da);
    frag::mm_rows<2, 8, false>(da, R0, LDD, rb * 16, s.Up, CTD, qt * 16);
    frag::mm_rows<2, 8, false>(da, R1, LDD, rb * 16, s.W, CTD, qt * 16);
#pragma unroll
    for (int jt = 0; jt < 2; ++jt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = rb * 16 + lr + (e >> 1) * 8, jj = qt * 16 + jt * 8 + lc + (e & 1);
        da[jt][e] = (jj < i) ? -da[jt][e] : 0.f;
      }
    frag::st_c(da, sdA, LDC, rb * 16, qt * 16);
  }
  __syncthreads();

  // ---- phase 4: Kb^c into R0, beta K^c into R1 (4 columns per thread, one row per warp)
  for (int idx = tid; idx < C * (D / 4); idx += NTB) {
    const int i = idx >> 5, c = (idx & 31) * 4;
    const uint2 rk = *reinterpret_cast<const uint2*>(s.k + i * LDD + c);
    const float bi = s.beta[i];
    const float4 f = ep4(i, c);
    const float2 k0 = frag::unpack(rk.x), k1 = frag::unpack(rk.y);
    *reinterpret_cast<uint2*>(R0 + i * LDD + c) =
        make_uint2(frag::pack(__fdividef(k0.x, f.x), __fdividef(k0.y, f.y)),
                   frag::pack(__fdividef(k1.x, f.z), __fdividef(k1.y, f.w)));
    *reinterpret_cast<uint2*>(R1 + i * LDD + c) =
        make_uint2(frag::pack(bi * k0.x * f.x, bi * k0.y * f.y),
                   frag::pack(bi * k1.x * f.z, bi * k1.y * f.w));
  }
  __syncthreads();
  frag::mm_rows<4, 4, true>(Z, s.dM, LDC, rb * 16, R0, LDD, qt * 32);     // Z += dM Kb^c
  frag::mm_rows<4, 4, true>(Q, sdA, LDC, rb * 16, R0, LDD, qt * 32);      // Q += dA Kb^c
  frag::mm_rows_at<4, 4, true>(P, s.dM, LDC, rb * 16, s.Qc, LDD, qt * 32); // P += dM^T Q^c
  frag::mm_rows_at<4, 4, true>(P, sdA, LDC, rb * 16, R1, LDD, qt * 32);   // P += dA^T beta K^c

  // ---- per-element epilogue: dq out; P <- dk (before the Kaczmarz term), Q <- dgamma
#pragma unroll
  for (int jt = 0; jt < 4; ++jt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int i = i0 + hh * 8, c = qt * 32 + jt * 8 + lc;
      const float bi = s.beta[i];
      const float2 kk = k2(i, c);
      const float2 qc = frag::unpack(*reinterpret_cast<const uint32_t*>(s.Qc + i * LDD + c));
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
  __syncthreads();  // R0/R1 free: reuse for the dgamma reduction
  float* sdg = reinterpret_cast<float*>(s.R);
  if (gk == D) {
#pragma unroll
    for (int jt = 0; jt < 4; ++jt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        sdg[(i0 + (e >> 1) * 8) * D + qt * 32 + jt * 8 + lc + (e & 1)] = Q[jt][e];
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
    for (int i = grq * 16; i < grq * 16 + 16; ++i) part += sdg[i * D + gc];
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
      run += sdg[i * D + gc];
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
}

}  // namespace

cudaError_t launch_bwd_scan(const Problem& p, const Saved& sv, const bf16* dO, const float* dST,
                            float* dS0, bf16* dU, bf16* dh, cudaStream_t st) {
  const size_t sm = sizeof(BscanSmem);
  cudaError_t e =
      cudaFuncSetAttribute(k_bwd_scan, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const double nb = (double)p.B * p.H * p.NC, ntok = nb * C, heads = (double)p.B * p.H;
  // reads W, Qh, Kt, M, dec, dO; writes dU, dh
  const double bytes = nb * (3.0 * kTileBytes + kMBytes + kDecBytes) + ntok * D * 2 +
                       nb * ((double)kUBytes + kStateBytes) +
                       heads * D * D * 4 * ((dST ? 1 : 0) + (dS0 ? 1 : 0));
  const double flops = nb * (D / BV) * (2.0 * C * C * BV + 2.0 * C * BV * D * 3);
  prof_begin(kKTcScanBwd, bytes, flops, st);
  k_bwd_scan<<<dim3(D / BV, p.H, p.B), NTS, sm, st>>>(p, sv, dO, dST, dS0, dU, dh);
  e = cudaGetLastError();
  prof_end(st);
  return e;
}

static_assert(sizeof(BchunkSmem) + sizeof(float) * C * D <= 232448,
              "chunk backward shared memory exceeds the 227 KB per-block limit");

size_t bwd_chunk_smem(const Problem& p) {
  return sizeof(BchunkSmem) + sizeof(float) * (C * p.gk);
}

cudaError_t launch_bwd_chunk(const Problem& p, const bf16* q, const bf16* k, const bf16* v,
                             const bf16* dO, const float* g, const Saved& sv, const bf16* dh,
                             const bf16* dU, bf16* dq, bf16* dk, bf16* dv, float* dbeta,
                             float* dg, cudaStream_t st) {
  const size_t sm = bwd_chunk_smem(p);
  cudaError_t e =
      cudaFuncSetAttribute(k_bwd_chunk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const double nb = (double)p.B * p.H * p.NC, ntok = nb * C;
  // reads q, k, v, dO, g, beta, T, h, dh, U, dU, W, U'; writes dq, dk, dv, dbeta, dg
  const double bytes = ntok * (4 * D * 2 + p.gk * 4 + 4) + nb * C * C * 2 + nb * 2.0 * D * D * 2 +
                       ntok * 4 * D * 2 + ntok * (3 * D * 2 + p.gk * 4 + 4);
  const double mac = (double)C * D * D * 3      // dO S, dU S, U dS'
                     + (double)C * C * D        // dO U^T
                     + (double)C * D * C * 2    // Lambda
                     + (double)C * C * D * 2    // dA
                     + (double)C * D * C * 4;   // dM Kb, dA Kb, dM^T Q^c, dA^T K^c
  prof_begin(kKTcChunkBwd, bytes, nb * 2.0 * mac, st);
  k_bwd_chunk<<<dim3(p.NC, p.H, p.B), NTB, sm, st>>>(p, q, k, v, dO, g, sv.T, sv.beta, sv.h, dh,
                                                     sv.U, dU, sv.W, sv.Up, sv.knorm, dq, dk, dv,
                                                     dbeta, dg);
  e = cudaGetLastError();
  prof_end(st);
  return e;
}

}  // namespace fast
}  // namespace dr
