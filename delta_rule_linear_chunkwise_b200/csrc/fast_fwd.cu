// fast_fwd.cu -- tensor-core forward for bf16 storage, d_k = d_v = 128, C = 64.
//
// tc_prep (chunk-parallel, one CTA per (b, h, chunk); every state-independent
// quantity of the chunk, computed once):
//   gamma = inclusive cumulative log-gate; beta (Kaczmarz step applied);
//   centred factors K^c = k e^{gamma - gamma_r}, Kb^c = k e^{gamma_r - gamma},
//   Q^c = q e^{gamma - gamma_r} (gamma_r: gate of the chunk's centre row);
//   [A ; M] = [K^c ; Q^c] Kb^c^T on tensor cores, A = diag(beta) strict_tril(.),
//   M = tril(.);  T = (I + A)^{-1} by blocked forward substitution in fp32
//   (16 x 16 diagonal blocks per warp, off-diagonal block products in tf32);
//   W = T diag(beta) (k e^gamma),  U' = T diag(beta) V  on tensor cores;
//   Qh = q e^gamma,  Kt = k e^{gamma_C - gamma},  dec = e^{gamma_C}.

#include "dr_common.cuh"
#include "fast.cuh"
#include "frag.cuh"

namespace dr {
namespace fast {

using frag::bf16;

namespace {

constexpr int C = 64, D = 128;
constexpr int LDD = D + 8;   // bf16 stride of 128-wide tiles
constexpr int LDC = C + 8;   // bf16 stride of 64-wide tiles
constexpr int LDA = C + 1;   // fp32 stride of the 64 x 64 solve tiles
constexpr int NT = 256;      // threads per CTA (8 warps)

__device__ __forceinline__ int centre_row(int nvalid) { return (nvalid - 1) / 2; }

// In-place inclusive cumulative sum down the 64 rows of column `col`.
__device__ __forceinline__ void cumsum_col(float* G, int ld, int col) {
  float v[C];
#pragma unroll
  for (int i = 0; i < C; ++i) v[i] = G[i * ld + col];
#pragma unroll
  for (int i = 1; i < C; ++i) v[i] += v[i - 1];
#pragma unroll
  for (int i = 0; i < C; ++i) G[i * ld + col] = v[i];
}

// Eight consecutive gate values of row i from channel c (scalar gate: broadcast).
__device__ __forceinline__ void gate8(const float* G, int gk, int i, int c, float* out) {
  if (gk == 1) {
    const float x = G[i];
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = x;
  } else {
    const float4 a = *reinterpret_cast<const float4*>(G + i * gk + c);
    const float4 b = *reinterpret_cast<const float4*>(G + i * gk + c + 4);
    out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
    out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
  }
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

// bf16 store of accumulators (rows r0.., cols n0..) into a core-tiled global
// tile with ncol columns, 4-byte pairs: each warp store fills one 8 x 8 block
// (128 contiguous bytes).
template <int NTL>
__device__ __forceinline__ void st_c_global(const float (&c)[NTL][4], bf16* g, int ncol, int r0,
                                            int n0) {
  const int l = threadIdx.x & 31;
  const int r = r0 + (l >> 2), cc = n0 + 2 * (l & 3);
#pragma unroll
  for (int j = 0; j < NTL; ++j) {
    *reinterpret_cast<uint32_t*>(g + ct_off(r, cc + j * 8, ncol)) = frag::pack(c[j][0], c[j][1]);
    *reinterpret_cast<uint32_t*>(g + ct_off(r + 8, cc + j * 8, ncol)) =
        frag::pack(c[j][2], c[j][3]);
  }
}

// ---------------------------------------------------------------------------
// tc_prep
struct PrepSmem {
  bf16 R1[C * LDD];            // K^c, then beta k e^gamma
  bf16 R2[C * LDD];            // Kb^c, then A (fp32 [C][LDA]), then T (bf16 [C][LDC])
  bf16 R3[C * LDD];            // Q^c, then T (fp32 [C][LDA])
  float RG[C * D + 512];       // cumulative gate [C][gk], then beta v (bf16 [C][LDD])
  float X[16 * 48];
  float beta[C];
};

// PHASE: the SFDA rotation-decay gate.  Its per-channel cumulative sums hold,
// for key pair m, gamma (cumulative log alpha) at channel 2m and the cumulative
// phase Theta at 2m + 1; the chunk's decay from its start to row i is then
// Gamma_i ~ e^{gamma_i} e^{-i Theta_i} on each pair read as a complex number
// (x + i y), and the factors below are those of the gate-free chunk form with
// read keys Gamma_i k_i, write keys Gamma_i^{-T} k_i, queries Gamma_i q_i and
// end-of-chunk keys Gamma_C^T Gamma_i^{-T} k_i ("Konstruktives Chunk-WY-
// Theorem", SFDA explainer): per pair, a rotation and a scale.  The decay row
// holds (e^{gamma_C} cos Theta_C, e^{gamma_C} sin Theta_C) per pair.
template <bool PHASE>
__global__ void __launch_bounds__(NT, 2)
    k_prep(Problem p, const bf16* __restrict__ q, const bf16* __restrict__ k,
           const bf16* __restrict__ v, const float* __restrict__ beta_in,
           const float* __restrict__ g, Saved sv) {
  extern __shared__ __align__(16) unsigned char smraw[];
  PrepSmem& s = *reinterpret_cast<PrepSmem*>(smraw);
  const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, gk = p.gk;
  const int lr = lane >> 2, lc = 2 * (lane & 3);
  const int t0 = n * C, nvalid = min(C, p.T - t0);
  const size_t cb = chunk_id(p, b, h, n);
  float* G = s.RG;
  float* sA = reinterpret_cast<float*>(s.R2);
  float* sT = reinterpret_cast<float*>(s.R3);
  bf16* sTb = s.R2;
  bf16* sBV = reinterpret_cast<bf16*>(s.RG);

  if (gk == D) {
    for (int idx = tid; idx < C * (D / 4); idx += NT) {
      const int i = idx >> 5, j = idx & 31;
      const bool ok = i < nvalid && p.gate != kGateNone;
      frag::cp16(G + i * D + j * 4, g + row_id(p, b, t0 + (ok ? i : 0), h) * D + j * 4, ok);
    }
    frag::cp_commit();
  }
  // q into R3 (the factor pass rewrites it in place) and k into registers, in
  // flight while the gate is summed; v follows after the factor pass.  Each
  // thread owns the 16-byte column segment j = tid % 16 of ITEMS rows.
  constexpr int ITEMS = C * (D / 8) / NT;
  uint4 kr[ITEMS], vr[ITEMS];
#pragma unroll
  for (int it = 0; it < ITEMS; ++it) {
    const int idx = tid + it * NT, i = idx >> 4, j = idx & 15;
    const bool ok = i < nvalid;
    const size_t rr = row_id(p, b, t0 + (ok ? i : 0), h) * D + j * 8;
    frag::cp16(s.R3 + i * LDD + j * 8, q + rr, ok);
    kr[it] = ok ? *reinterpret_cast<const uint4*>(k + rr) : make_uint4(0, 0, 0, 0);
  }
  frag::cp_commit();
  frag::cp_wait<0>();
  if (gk != D && tid < C) {
    G[tid] = (tid < nvalid && p.gate != kGateNone) ? g[row_id(p, b, t0 + tid, h)] : 0.f;
  }
  __syncthreads();
  if (tid < gk) cumsum_col(G, gk, tid);
  __syncthreads();

  // Factors: K^c, Kb^c, Q^c to shared memory; Qh, Kt, beta, dec to global.
  const int r = centre_row(nvalid);
  // This thread's segment of the centre row's and the last row's cumulative gate
  // (phase gate: log-decays at the even channels, e^{i Theta_r}, e^{i Theta_C} per pair).
  // Every factor below is the exponential of a difference of cumulative gates:
  // the centred ones stay within half the chunk's decay, and none is formed as a
  // quotient of two exponentials that may underflow.
  float r8[8], c8[8];
  float rc4[4], rs4[4], cc4[4], cs4[4];
  gate8(G, gk, r, (tid & 15) * 8, r8);
  gate8(G, gk, C - 1, (tid & 15) * 8, c8);
  if (PHASE) {
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      sincosf(r8[2 * m + 1], &rs4[m], &rc4[m]);
      sincosf(c8[2 * m + 1], &cs4[m], &cc4[m]);
    }
  }
#pragma unroll
  for (int it = 0; it < ITEMS; ++it) {
    const int idx = tid + it * NT, i = idx >> 4, j = idx & 15;
    const bool valid = i < nvalid;
    const uint4 rq = *reinterpret_cast<const uint4*>(s.R3 + i * LDD + j * 8);
    float kv[8], qv[8], g8[8];
    unpack8(kr[it], kv);
    unpack8(rq, qv);
    gate8(G, gk, i, j * 8, g8);
    float kc[8], kb[8], qc[8], qh[8], kt[8], nn = 0.f;
    if (PHASE) {
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int e = 2 * m;
        float sn, cs;
        sincosf(g8[e + 1], &sn, &cs);                              // e^{-i Theta} = cs - i sn
        const float eg = __expf(g8[e]);                            // e^gamma
        // e^{+-(gamma - gamma_r)} from the centred exponent itself: within half
        // a chunk's decay of 1, so it stays finite where e^gamma underflows
        const float ep = __expf(g8[e] - r8[e]), em = __expf(r8[e] - g8[e]);
        // e^{-i (Theta - Theta_r)} and e^{i (Theta_C - Theta)}
        const float wr = cs * rc4[m] + sn * rs4[m], wi = cs * rs4[m] - sn * rc4[m];
        const float tr = cc4[m] * cs + cs4[m] * sn, ti = cs4[m] * cs - cc4[m] * sn;
        const float kx = kv[e], ky = kv[e + 1], qx = qv[e], qy = qv[e + 1];
        const float kwx = wr * kx - wi * ky, kwy = wi * kx + wr * ky;
        const float qwx = wr * qx - wi * qy, qwy = wi * qx + wr * qy;
        kc[e] = ep * kwx;
        kc[e + 1] = ep * kwy;
        kb[e] = em * kwx;
        kb[e + 1] = em * kwy;
        qc[e] = ep * qwx;
        qc[e + 1] = ep * qwy;
        qh[e] = eg * (cs * qx + sn * qy);                          // Gamma q
        qh[e + 1] = eg * (cs * qy - sn * qx);
        const float sc = __expf(c8[e] - g8[e]);                    // e^{gamma_C - gamma}
        kt[e] = sc * (tr * kx - ti * ky);                          // Gamma_C^T Gamma^{-T} k
        kt[e + 1] = sc * (ti * kx + tr * ky);
        nn += kx * kx + ky * ky;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float eg = __expf(g8[e]);                                  // e^gamma
        const float ep = __expf(g8[e] - r8[e]), em = __expf(r8[e] - g8[e]);  // e^{+-(gamma - gamma_r)}
        kc[e] = kv[e] * ep;
        kb[e] = kv[e] * em;
        qc[e] = qv[e] * ep;
        qh[e] = qv[e] * eg;
        kt[e] = kv[e] * __expf(c8[e] - g8[e]);  // k e^{gamma_C - gamma}
        nn += kv[e] * kv[e];
      }
    }
    *reinterpret_cast<uint4*>(s.R1 + i * LDD + j * 8) = pack8(kc);
    *reinterpret_cast<uint4*>(s.R2 + i * LDD + j * 8) = pack8(kb);
    *reinterpret_cast<uint4*>(s.R3 + i * LDD + j * 8) = pack8(qc);
    *reinterpret_cast<uint4*>(sv.Qh + cb * C * D + ct_off(i, j * 8, D)) = pack8(qh);
    *reinterpret_cast<uint4*>(sv.Kt + cb * C * D + ct_off(i, j * 8, D)) = pack8(kt);
    nn += __shfl_xor_sync(0xffffffffu, nn, 8);
    nn += __shfl_xor_sync(0xffffffffu, nn, 4);
    nn += __shfl_xor_sync(0xffffffffu, nn, 2);
    nn += __shfl_xor_sync(0xffffffffu, nn, 1);
    if (j == 0) {
      float bb = 0.f;
      if (valid) {
        const float in = beta_in[row_id(p, b, t0 + i, h)];
        bb = (p.beta_mode == kBetaKaczmarz) ? in / (nn + p.eps) : in;
      }
      s.beta[i] = bb;
      sv.beta[cb * C + i] = bb;
      sv.knorm[cb * C + i] = nn;
    }
  }
  if (PHASE) {
    if (tid < D / 2) {
      float sn, cs;
      sincosf(G[(C - 1) * D + 2 * tid + 1], &sn, &cs);
      const float a = __expf(G[(C - 1) * D + 2 * tid]);
      sv.dec[cb * D + 2 * tid] = a * cs;
      sv.dec[cb * D + 2 * tid + 1] = a * sn;
    }
  } else if (tid < D) {
    sv.dec[cb * D + tid] = __expf(gk == D ? G[(C - 1) * D + tid] : G[C - 1]);
  }
#pragma unroll
  for (int it = 0; it < ITEMS; ++it) {
    const int idx = tid + it * NT, i = idx >> 4, j = idx & 15;
    vr[it] = i < nvalid
                 ? *reinterpret_cast<const uint4*>(v + row_id(p, b, t0 + i, h) * D + j * 8)
                 : make_uint4(0, 0, 0, 0);
  }
  __syncthreads();

  // [A ; M] = [K^c ; Q^c] Kb^c^T: warps 0-3 -> A rows 16w.., warps 4-7 -> M rows 16(w-4)..
  const int rb = warp & 3;
  float gram[8][4];
  frag::zero(gram);
  frag::mm_rows<8, 8, false>(gram, warp < 4 ? s.R1 : s.R3, LDD, rb * 16, s.R2, LDD);
  if (warp >= 4) {
#pragma unroll
    for (int jt = 0; jt < 8; ++jt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = rb * 16 + lr + (e >> 1) * 8, jj = jt * 8 + lc + (e & 1);
        if (jj > i) gram[jt][e] = 0.f;
      }
    st_c_global(gram, sv.M + cb * C * C, C, rb * 16, 0);
  }
  __syncthreads();  // K^c, Kb^c, Q^c consumed
  if (warp < 4) {
#pragma unroll
    for (int jt = 0; jt < 8; ++jt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = rb * 16 + lr + (e >> 1) * 8, jj = jt * 8 + lc + (e & 1);
        sA[i * LDA + jj] = (jj < i) ? s.beta[i] * gram[jt][e] : 0.f;
      }
  }
  for (int idx = tid; idx < C * LDA; idx += NT) sT[idx] = 0.f;
  // beta k e^gamma into R1 (k kept in registers)
#pragma unroll
  for (int it = 0; it < ITEMS; ++it) {
    const int idx = tid + it * NT, i = idx >> 4, j = idx & 15;
    float kv[8], g8[8];
    unpack8(kr[it], kv);
    gate8(G, gk, i, j * 8, g8);
    const float bi = s.beta[i];
    if (PHASE) {
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        float sn, cs;
        sincosf(g8[2 * m + 1], &sn, &cs);
        const float a = bi * __expf(g8[2 * m]), kx = kv[2 * m], ky = kv[2 * m + 1];
        kv[2 * m] = a * (cs * kx + sn * ky);                 // beta Gamma k
        kv[2 * m + 1] = a * (cs * ky - sn * kx);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) kv[e] *= bi * __expf(g8[e]);
    }
    *reinterpret_cast<uint4*>(s.R1 + i * LDD + j * 8) = pack8(kv);
  }
  __syncthreads();  // A ready; the gate is no longer needed

  // T = (I + A)^{-1}: diagonal 16 x 16 blocks (warps 0-3, lane l < 16 owns column l)
  if (warp < 4) {
    if (lane < 16) {
      const int base = warp * 16, l = lane;
      float t[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) t[i] = (i == l) ? 1.f : 0.f;
#pragma unroll
      for (int i = 1; i < 16; ++i) {
        if (i > l) {
          float acc = 0.f;
#pragma unroll
          for (int m = 0; m < 15; ++m)
            if (m >= l && m < i) acc += sA[(base + i) * LDA + base + m] * t[m];
          t[i] = -acc;
        }
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) sT[(base + i) * LDA + base + l] = t[i];
    }
  }
  __syncthreads();
  // beta v into the freed gate region (v kept in registers); read after the solve
#pragma unroll
  for (int it = 0; it < ITEMS; ++it) {
    const int idx = tid + it * NT, i = idx >> 4, j = idx & 15;
    float vv[8];
    unpack8(vr[it], vv);
    const float bi = s.beta[i];
#pragma unroll
    for (int e = 0; e < 8; ++e) vv[e] *= bi;
    *reinterpret_cast<uint4*>(sBV + i * LDD + j * 8) = pack8(vv);
  }
  // Off-diagonal blocks, block row bi = 1..3, tf32 tensor cores:
  //   X_j = sum_{m = 16j}^{16bi - 1} A[16bi.., m] T[m, 16j..]  (warp j < bi),
  //   T[bi, j] = -T[bi, bi] X_j
  for (int bi = 1; bi < 4; ++bi) {
    if (warp < bi) {
      const int j = warp, w = 16 * bi;
      float x[2][4] = {};
      frag::mm16x16_tf32(x, sA, LDA, w, sT, LDA, 16 * j, 16 * j, w - 16 * j);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        s.X[lr * 48 + 16 * j + nt * 8 + lc] = x[nt][0];
        s.X[lr * 48 + 16 * j + nt * 8 + lc + 1] = x[nt][1];
        s.X[(lr + 8) * 48 + 16 * j + nt * 8 + lc] = x[nt][2];
        s.X[(lr + 8) * 48 + 16 * j + nt * 8 + lc + 1] = x[nt][3];
      }
      __syncwarp();
      float y[2][4] = {};
      frag::mm16x16_tf32(y, sT + w, LDA, w, s.X + 16 * j, 48, 0, 0, 16);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        sT[(w + lr) * LDA + 16 * j + nt * 8 + lc] = -y[nt][0];
        sT[(w + lr) * LDA + 16 * j + nt * 8 + lc + 1] = -y[nt][1];
        sT[(w + lr + 8) * LDA + 16 * j + nt * 8 + lc] = -y[nt][2];
        sT[(w + lr + 8) * LDA + 16 * j + nt * 8 + lc + 1] = -y[nt][3];
      }
    }
    __syncthreads();
  }
  // T -> bf16: global and the tensor-core A operand (over the dead A tile)
  for (int idx = tid; idx < C * C / 8; idx += NT) {
    const int i = ct_row(idx, C), j8 = ct_col(idx, C);
    const uint4 val = pack8(sT + i * LDA + j8);
    *reinterpret_cast<uint4*>(sv.T + cb * C * C + 8 * idx) = val;  // core-tiled
    *reinterpret_cast<uint4*>(sTb + i * LDC + j8) = val;
  }
  __syncthreads();
  // W = T (beta k e^gamma) (warps 0-3), U' = T (beta v) (warps 4-7): rows 16rb.., 128 columns
  {
    float acc[16][4];
    frag::zero(acc);
    frag::mm_rows<16, 4, true>(acc, sTb, LDC, rb * 16, warp < 4 ? s.R1 : sBV, LDD);
    st_c_global(acc, (warp < 4 ? sv.W : sv.Up) + cb * C * D, D, rb * 16, 0);
  }
}

}  // namespace

cudaError_t launch_prep(const Problem& p, const bf16* q, const bf16* k, const bf16* v,
                        const float* beta, const float* g, const Saved& sv, cudaStream_t st) {
  const size_t sm = sizeof(PrepSmem);
  const bool phase = p.gate == kGatePhase;
  cudaError_t e = cudaFuncSetAttribute(phase ? k_prep<true> : k_prep<false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const double nb = (double)p.B * p.H * p.NC, ntok = nb * C;
  // reads q, k, v, g, beta (the operator's inputs); writes T, beta, dec, W, U', M, Qh, Kt
  const double io = ntok * (3 * D * 2 + p.gk * 4 + 4);
  const double bytes =
      io + nb * ((double)kTBytes + 2 * kBetaBytes + kDecBytes + 4.0 * kTileBytes + kMBytes);
  const double flops = nb * (2.0 * 2 * C * C * D + 2.0 * 2 * C * C * D);  // [A;M] Gram, W|U'
  prof_begin(kKTcIntraFwd, io, bytes, flops, st);
  if (phase)
    k_prep<true><<<dim3(p.NC, p.H, p.B), NT, sm, st>>>(p, q, k, v, beta, g, sv);
  else
    k_prep<false><<<dim3(p.NC, p.H, p.B), NT, sm, st>>>(p, q, k, v, beta, g, sv);
  e = cudaGetLastError();
  prof_end(st);
  return e;
}

}  // namespace fast
}  // namespace dr
