// fast_fwd.cu -- tensor-core forward for bf16 storage, d_k = d_v = 128, C = 64.
//
// tc_prep (chunk-parallel, one CTA per (b, h, chunk)):
//   gamma = inclusive cumulative log-gate, beta (Kaczmarz step applied),
//   A = diag(beta) strict_tril(K^c Kb^c^T) on tensor cores (centred factors
//   K^c = k e^{gamma - gamma_r}, Kb^c = k e^{gamma_r - gamma}),
//   T = (I + A)^{-1} by blocked forward substitution in fp32 (16 x 16 diagonal
//   blocks per warp, then three levels of off-diagonal block products).
//   Writes T (bf16, row-major 64 x 64) and beta per chunk.
// tc_fwd_scan (sequential over chunks, one CTA per (b, h, 64-wide value tile)):
//   per chunk, recomputes from q, k, v, g, T:
//     M = tril(Q^c Kb^c^T), W = T diag(beta) (k e^gamma), U' = T diag(beta) V,
//   then with the fp32 state S (registers) and its bf16 copy (shared memory):
//     U = U' - W S^T,  O = (q e^gamma) S^T + M U,  S <- S Diag(e^{gamma_C}) + U^T Kt
//   (Kt = k e^{gamma_C - gamma}).  Optionally saves each chunk's start state
//   (bf16) and U (bf16) for the backward.  The raw inputs of chunk n+1 are
//   fetched with cp.async while chunk n's state products run.

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
constexpr int NTH = 128;     // threads per CTA (4 warps x 16 rows)

__device__ __forceinline__ int centre_row(int nvalid) { return (nvalid - 1) / 2; }

// In-place inclusive cumulative sum down the 64 rows of column `col` of a
// [C][ld] fp32 tile: all loads first, then the scan in registers.
__device__ __forceinline__ void cumsum_col(float* G, int ld, int col) {
  float v[C];
#pragma unroll
  for (int i = 0; i < C; ++i) v[i] = G[i * ld + col];
#pragma unroll
  for (int i = 1; i < C; ++i) v[i] += v[i - 1];
#pragma unroll
  for (int i = 0; i < C; ++i) G[i * ld + col] = v[i];
}

// Eight consecutive gate values of row i starting at channel c (scalar gate:
// broadcast of the row's value).
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

// ---------------------------------------------------------------------------
// tc_prep
struct PrepSmem {
  bf16 Kc[C * LDD];
  bf16 Kb[C * LDD];
  float A[C * LDA];
  float T[C * LDA];
  float X[16 * 48];
  float beta[C];
  float G[1];  // [C][gk], dynamic tail
};

__global__ void __launch_bounds__(NTH) k_prep(Problem p, const bf16* __restrict__ k,
                                              const float* __restrict__ beta_in,
                                              const float* __restrict__ g,
                                              bf16* __restrict__ Tout,
                                              float* __restrict__ beta_out) {
  extern __shared__ __align__(16) unsigned char smraw[];
  PrepSmem& s = *reinterpret_cast<PrepSmem*>(smraw);
  const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int gk = p.gk, t0 = n * C, nvalid = min(C, p.T - t0);
  const size_t cb = chunk_id(p, b, h, n);
  float* G = s.G;

  // gate -> shared, then inclusive cumulative sum per channel
  if (gk == D) {
    for (int idx = tid; idx < C * D / 4; idx += NTH) {
      const int i = idx / (D / 4), c4 = idx % (D / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < nvalid && p.gate != kGateNone)
        v = *reinterpret_cast<const float4*>(g + row_id(p, b, t0 + i, h) * D + c4 * 4);
      *reinterpret_cast<float4*>(G + i * D + c4 * 4) = v;
    }
  } else if (tid < C) {
    G[tid] = (tid < nvalid && p.gate != kGateNone) ? g[row_id(p, b, t0 + tid, h)] : 0.f;
  }
  for (int idx = tid; idx < C * LDA; idx += NTH) s.T[idx] = 0.f;
  __syncthreads();
  if (tid < gk) cumsum_col(G, gk, tid);
  __syncthreads();

  // centred key factors (bf16) and beta
  const int r = centre_row(nvalid);
#pragma unroll 1
  for (int pass = 0; pass < C * (D / 8) / NTH; ++pass) {
    const int idx = tid + pass * NTH;
    const int i = idx >> 4, j = idx & 15;
    const bool valid = i < nvalid;
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (valid) raw = *reinterpret_cast<const uint4*>(k + row_id(p, b, t0 + i, h) * D + j * 8);
    const uint32_t* rw = reinterpret_cast<const uint32_t*>(&raw);
    float kv[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = frag::unpack(rw[e]);
      kv[2 * e] = f.x;
      kv[2 * e + 1] = f.y;
    }
    float nn = 0.f;
    uint32_t oc[4], ob[4];
    float gi[8], gr[8];
    gate8(G, gk, i, j * 8, gi);
    gate8(G, gk, r, j * 8, gr);
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      oc[e / 2] = frag::pack(kv[e] * __expf(gi[e] - gr[e]), kv[e + 1] * __expf(gi[e + 1] - gr[e + 1]));
      ob[e / 2] = frag::pack(kv[e] * __expf(gr[e] - gi[e]), kv[e + 1] * __expf(gr[e + 1] - gi[e + 1]));
      nn += kv[e] * kv[e] + kv[e + 1] * kv[e + 1];
    }
    *reinterpret_cast<uint4*>(s.Kc + i * LDD + j * 8) = make_uint4(oc[0], oc[1], oc[2], oc[3]);
    *reinterpret_cast<uint4*>(s.Kb + i * LDD + j * 8) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
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
      beta_out[cb * C + i] = bb;
    }
  }
  __syncthreads();

  // Gram on tensor cores: warp w owns rows 16w..16w+15, all 64 columns.
  const int warp = tid >> 5, lane = tid & 31;
  {
    float acc[8][4];
    frag::zero(acc);
    frag::mm_rows<8, 8, false>(acc, s.Kc, LDD, warp * 16, s.Kb, LDD);
    const int r0 = warp * 16 + (lane >> 2), c0 = 2 * (lane & 3);
#pragma unroll
    for (int jt = 0; jt < 8; ++jt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = r0 + (e >> 1) * 8, jj = jt * 8 + c0 + (e & 1);
        s.A[i * LDA + jj] = (jj < i) ? s.beta[i] * acc[jt][e] : 0.f;
      }
    }
  }
  __syncthreads();

  // Diagonal 16 x 16 blocks: warp w inverts block w; lane l < 16 owns column l.
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
          if (m >= l && m < i) acc += s.A[(base + i) * LDA + base + m] * t[m];
        t[i] = -acc;
      }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) s.T[(base + i) * LDA + base + l] = t[i];
  }
  __syncthreads();
  // Off-diagonal blocks, block row bi = 1..3, on tensor cores (tf32):
  //   X_j = sum_{m = 16j}^{16bi - 1} A[16bi.., m] T[m, 16j..]   (warp j < bi)
  //   T[bi, j] = -T[bi, bi] X_j
  for (int bi = 1; bi < 4; ++bi) {
    if (warp < bi) {
      const int j = warp, w = 16 * bi;
      float x[2][4] = {};
      frag::mm16x16_tf32(x, s.A, LDA, w, s.T, LDA, 16 * j, 16 * j, w - 16 * j);
      const int g = lane >> 2, t = lane & 3;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        s.X[g * 48 + 16 * j + nt * 8 + 2 * t] = x[nt][0];
        s.X[g * 48 + 16 * j + nt * 8 + 2 * t + 1] = x[nt][1];
        s.X[(g + 8) * 48 + 16 * j + nt * 8 + 2 * t] = x[nt][2];
        s.X[(g + 8) * 48 + 16 * j + nt * 8 + 2 * t + 1] = x[nt][3];
      }
      __syncwarp();
      float y[2][4] = {};
      frag::mm16x16_tf32(y, s.T + w, LDA, w, s.X + 16 * j, 48, 0, 0, 16);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        s.T[(w + g) * LDA + 16 * j + nt * 8 + 2 * t] = -y[nt][0];
        s.T[(w + g) * LDA + 16 * j + nt * 8 + 2 * t + 1] = -y[nt][1];
        s.T[(w + g + 8) * LDA + 16 * j + nt * 8 + 2 * t] = -y[nt][2];
        s.T[(w + g + 8) * LDA + 16 * j + nt * 8 + 2 * t + 1] = -y[nt][3];
      }
    }
    __syncthreads();
  }
  // T -> global (bf16, row-major)
  for (int idx = tid; idx < C * C / 8; idx += NTH) {
    const int i = idx >> 3, j = idx & 7;
    const float* src = s.T + i * LDA + j * 8;
    uint4 v = make_uint4(frag::pack(src[0], src[1]), frag::pack(src[2], src[3]),
                         frag::pack(src[4], src[5]), frag::pack(src[6], src[7]));
    *reinterpret_cast<uint4*>(Tout + cb * C * C + i * C + j * 8) = v;
  }
}

// ---------------------------------------------------------------------------
// tc_fwd_scan
constexpr int BV = 64;  // value columns per CTA

struct FwdSmem {
  // raw inputs of the current chunk (refilled by cp.async for the next chunk)
  bf16 q[C * LDD];
  bf16 k[C * LDD];
  bf16 v[C * LDC];
  bf16 T[C * LDC];
  float beta[C];
  // operand tiles
  bf16 Qc[C * LDD];   // q e^{gamma - gamma_r}
  bf16 Kb[C * LDD];   // k e^{gamma_r - gamma}
  bf16 BK[C * LDD];   // beta k e^{gamma}          ([j][c], B operand, k-rows)
  bf16 Qh[C * LDD];   // q e^{gamma}
  bf16 Kt[C * LDD];   // k e^{gamma_C - gamma}     ([i][c], B operand, k-rows)
  bf16 BV_[C * LDC];  // beta v                    ([j][a])
  bf16 U[C * LDC];    // pseudo-values U           ([i][a])
  bf16 S[BV * LDD];   // bf16 copy of the state    ([a][c])
  float dec[D];       // e^{gamma_C}
  float G[1];         // [C][gk] raw gate, then cumulative (dynamic tail)
};

// Issue the cp.async loads of chunk n's raw inputs (one commit group).
__device__ void fwd_load_chunk(const Problem& p, FwdSmem& s, const bf16* q, const bf16* k,
                               const bf16* v, const float* g, const bf16* T,
                               const float* beta, int b, int h, int n, int a0) {
  const int tid = threadIdx.x, gk = p.gk, t0 = n * C, nvalid = min(C, p.T - t0);
  const int NTH = blockDim.x;
  const size_t cb = chunk_id(p, b, h, n);
  for (int idx = tid; idx < C * (D / 8); idx += NTH) {
    const int i = idx >> 4, j = idx & 15;
    const bool ok = i < nvalid;
    const size_t rr = row_id(p, b, t0 + (ok ? i : 0), h) * D + j * 8;
    frag::cp16(s.q + i * LDD + j * 8, q + rr, ok);
    frag::cp16(s.k + i * LDD + j * 8, k + rr, ok);
  }
  for (int idx = tid; idx < C * (BV / 8); idx += NTH) {
    const int i = idx >> 3, j = idx & 7;
    const bool ok = i < nvalid;
    frag::cp16(s.v + i * LDC + j * 8, v + row_id(p, b, t0 + (ok ? i : 0), h) * D + a0 + j * 8, ok);
    frag::cp16(s.T + i * LDC + j * 8, T + cb * C * C + i * C + j * 8, true);
  }
  if (gk == D) {
    for (int idx = tid; idx < C * (D / 4); idx += NTH) {
      const int i = idx >> 5, j = idx & 31;
      const bool ok = i < nvalid && p.gate != kGateNone;
      frag::cp16(s.G + i * D + j * 4, g + row_id(p, b, t0 + (ok ? i : 0), h) * D + j * 4, ok);
    }
  }
  if (tid < C / 4) frag::cp16(s.beta + tid * 4, beta + cb * C + tid * 4, true);
  frag::cp_commit();
  if (gk == 1 && tid < C) {
    // scalar gate: plain loads (4 bytes per row)
    s.G[tid] = (tid < nvalid && p.gate != kGateNone) ? g[row_id(p, b, t0 + tid, h)] : 0.f;
  }
}

constexpr int NTS = 256;  // threads of the scan CTA: 8 warps = 4 row blocks x 2 halves

__global__ void __launch_bounds__(NTS, 1)
    k_fwd_scan(Problem p, const bf16* __restrict__ q, const bf16* __restrict__ k,
               const bf16* __restrict__ v, const float* __restrict__ g,
               const bf16* __restrict__ Tg, const float* __restrict__ beta,
               const float* __restrict__ S0, bf16* __restrict__ o, float* __restrict__ ST,
               bf16* __restrict__ hsave, bf16* __restrict__ Usave) {
  extern __shared__ __align__(16) unsigned char smraw[];
  FwdSmem& s = *reinterpret_cast<FwdSmem*>(smraw);
  bf16* sW = s.BK;  // W  [i][c], written once beta K e^gamma is consumed
  bf16* sM = s.Qc;  // M  [i][j] (stride LDC), written once Q^c is consumed
  const int h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, gk = p.gk;
  const int rb = warp & 3, hf = warp >> 2;  // row block (16 rows), column half
  const int a0 = blockIdx.x * BV;
  const int lr = lane >> 2, lc = 2 * (lane & 3);
  const size_t sbase = ((size_t)b * p.H + h) * D * D;

  // fp32 state rows a0 + 16rb + .., key columns 64hf .. 64hf+63
  float S[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int a = rb * 16 + lr + (e >> 1) * 8, c = hf * 64 + j * 8 + lc + (e & 1);
      S[j][e] = S0 ? S0[sbase + (size_t)(a0 + a) * D + c] : 0.f;
    }
  frag::st_c(S, s.S, LDD, rb * 16, hf * 64);

  fwd_load_chunk(p, s, q, k, v, g, Tg, beta, b, h, 0, a0);
  for (int n = 0; n < p.NC; ++n) {
    const int t0 = n * C, nvalid = min(C, p.T - t0);
    const size_t cb = chunk_id(p, b, h, n);
    frag::cp_wait<0>();
    __syncthreads();
    if (tid < gk) cumsum_col(s.G, gk, tid);
    __syncthreads();
    const int r = centre_row(nvalid);
    for (int idx = tid; idx < C * (D / 8); idx += NTS) {
      const int i = idx >> 4, j = idx & 15;
      const uint4 rq = *reinterpret_cast<const uint4*>(s.q + i * LDD + j * 8);
      const uint4 rk = *reinterpret_cast<const uint4*>(s.k + i * LDD + j * 8);
      const uint32_t* wq = reinterpret_cast<const uint32_t*>(&rq);
      const uint32_t* wk = reinterpret_cast<const uint32_t*>(&rk);
      const float bi = s.beta[i];
      uint32_t oqc[4], okb[4], obk[4], oqh[4], okt[4];
      float g8[8], r8[8], c8[8];
      gate8(s.G, gk, i, j * 8, g8);
      gate8(s.G, gk, r, j * 8, r8);
      gate8(s.G, gk, C - 1, j * 8, c8);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fq = frag::unpack(wq[e]), fk = frag::unpack(wk[e]);
        const float gi0 = g8[2 * e], gi1 = g8[2 * e + 1];
        const float ep0 = __expf(gi0 - r8[2 * e]), ep1 = __expf(gi1 - r8[2 * e + 1]);
        const float em0 = __expf(r8[2 * e] - gi0), em1 = __expf(r8[2 * e + 1] - gi1);
        const float ea0 = __expf(gi0), ea1 = __expf(gi1);
        const float et0 = __expf(c8[2 * e] - gi0), et1 = __expf(c8[2 * e + 1] - gi1);
        oqc[e] = frag::pack(fq.x * ep0, fq.y * ep1);
        okb[e] = frag::pack(fk.x * em0, fk.y * em1);
        obk[e] = frag::pack(bi * fk.x * ea0, bi * fk.y * ea1);
        oqh[e] = frag::pack(fq.x * ea0, fq.y * ea1);
        okt[e] = frag::pack(fk.x * et0, fk.y * et1);
      }
      *reinterpret_cast<uint4*>(s.Qc + i * LDD + j * 8) = make_uint4(oqc[0], oqc[1], oqc[2], oqc[3]);
      *reinterpret_cast<uint4*>(s.Kb + i * LDD + j * 8) = make_uint4(okb[0], okb[1], okb[2], okb[3]);
      *reinterpret_cast<uint4*>(s.BK + i * LDD + j * 8) = make_uint4(obk[0], obk[1], obk[2], obk[3]);
      *reinterpret_cast<uint4*>(s.Qh + i * LDD + j * 8) = make_uint4(oqh[0], oqh[1], oqh[2], oqh[3]);
      *reinterpret_cast<uint4*>(s.Kt + i * LDD + j * 8) = make_uint4(okt[0], okt[1], okt[2], okt[3]);
    }
    for (int idx = tid; idx < C * (BV / 8); idx += NTS) {
      const int i = idx >> 3, j = idx & 7;
      const uint4 rv = *reinterpret_cast<const uint4*>(s.v + i * LDC + j * 8);
      const uint32_t* wv = reinterpret_cast<const uint32_t*>(&rv);
      const float bi = s.beta[i];
      uint32_t ov[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = frag::unpack(wv[e]);
        ov[e] = frag::pack(bi * f.x, bi * f.y);
      }
      *reinterpret_cast<uint4*>(s.BV_ + i * LDC + j * 8) = make_uint4(ov[0], ov[1], ov[2], ov[3]);
    }
    if (tid < D) s.dec[tid] = __expf((gk == D) ? s.G[(C - 1) * D + tid] : s.G[C - 1]);
    __syncthreads();

    // State-independent products for rows 16rb..: W (key half hf), M (column
    // half hf, inclusive causal mask), U' (value half hf).
    float Wc[8][4], Mc[4][4], Up[4][4];
    frag::zero(Wc);
    frag::mm_rows<8, 4, true>(Wc, s.T, LDC, rb * 16, s.BK, LDD, hf * 64);
    frag::zero(Mc);
    frag::mm_rows<4, 8, false>(Mc, s.Qc, LDD, rb * 16, s.Kb, LDD, hf * 32);
#pragma unroll
    for (int jt = 0; jt < 4; ++jt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = rb * 16 + lr + (e >> 1) * 8, jj = hf * 32 + jt * 8 + lc + (e & 1);
        if (jj > i) Mc[jt][e] = 0.f;
      }
    frag::zero(Up);
    frag::mm_rows<4, 4, true>(Up, s.T, LDC, rb * 16, s.BV_, LDC, hf * 32);
    __syncthreads();  // Q^c, Kb^c, beta K e^gamma, T, beta V and the raw tiles are consumed
    frag::st_c(Wc, sW, LDD, rb * 16, hf * 64);
    frag::st_c(Mc, sM, LDC, rb * 16, hf * 32);
    if (n + 1 < p.NC) fwd_load_chunk(p, s, q, k, v, g, Tg, beta, b, h, n + 1, a0);
    if (hsave)
      for (int idx = tid; idx < BV * (D / 8); idx += NTS) {
        const int a = idx >> 4, j = idx & 15;
        *reinterpret_cast<uint4*>(hsave + cb * D * D + (size_t)(a0 + a) * D + j * 8) =
            *reinterpret_cast<const uint4*>(s.S + a * LDD + j * 8);
      }
    __syncthreads();

    // U = U' - W S^T and the inter-chunk part of O, rows 16rb.., values 32hf..
    float oc[4][4];
    {
      float ws[4][4];
      frag::zero(ws);
      frag::mm_rows<4, 8, false>(ws, sW, LDD, rb * 16, s.S, LDD, hf * 32);
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) Up[j][e] -= ws[j][e];
      frag::st_c(Up, s.U, LDC, rb * 16, hf * 32);
      frag::zero(oc);
      frag::mm_rows<4, 8, false>(oc, s.Qh, LDD, rb * 16, s.S, LDD, hf * 32);
    }
    __syncthreads();
    if (Usave)
      for (int idx = tid; idx < C * (BV / 8); idx += NTS) {
        const int i = idx >> 3, j = idx & 7;
        *reinterpret_cast<uint4*>(Usave + (cb * C + i) * D + a0 + j * 8) =
            *reinterpret_cast<const uint4*>(s.U + i * LDC + j * 8);
      }
    // O += M U
    frag::mm_rows<4, 4, true>(oc, sM, LDC, rb * 16, s.U, LDC, hf * 32);
    if (o) {
#pragma unroll
      for (int jt = 0; jt < 4; ++jt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int i = rb * 16 + lr + hh * 8;
          if (i < nvalid)
            *reinterpret_cast<uint32_t*>(o + row_id(p, b, t0 + i, h) * D + a0 + hf * 32 + jt * 8 + lc) =
                frag::pack(oc[jt][2 * hh], oc[jt][2 * hh + 1]);
        }
    }
    // S <- S Diag(e^{gamma_C}) + U^T Kt for state rows 16rb.., key columns 64hf..
    {
      float ds[8][4];
      frag::zero(ds);
      frag::mm_rows_at<8, 4, true>(ds, s.U, LDC, rb * 16, s.Kt, LDD, hf * 64);
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          S[j][e] = S[j][e] * s.dec[hf * 64 + j * 8 + lc + (e & 1)] + ds[j][e];
    }
    __syncthreads();  // every warp is done with the bf16 state and the tiles
    frag::st_c(S, s.S, LDD, rb * 16, hf * 64);
  }
  if (ST) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int a = rb * 16 + lr + (e >> 1) * 8, c = hf * 64 + j * 8 + lc + (e & 1);
        ST[sbase + (size_t)(a0 + a) * D + c] = S[j][e];
      }
  }
}

}  // namespace

size_t prep_smem(const Problem& p) { return sizeof(PrepSmem) + sizeof(float) * (C * p.gk); }
size_t fwd_scan_smem(const Problem& p) { return sizeof(FwdSmem) + sizeof(float) * (C * p.gk); }

cudaError_t launch_prep(const Problem& p, const bf16* k, const float* beta, const float* g,
                        bf16* T, float* beta_eff, cudaStream_t st) {
  const size_t sm = prep_smem(p);
  cudaError_t e = cudaFuncSetAttribute(k_prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const double nb = (double)p.B * p.H * p.NC, ntok = nb * C;
  const double bytes = ntok * (D * 2 + p.gk * 4 + 4) + nb * C * C * 2 + ntok * 4;
  const double flops = nb * 2.0 * C * C * D;
  prof_begin(kKTcIntraFwd, bytes, flops, st);
  k_prep<<<dim3(p.NC, p.H, p.B), NTH, sm, st>>>(p, k, beta, g, T, beta_eff);
  e = cudaGetLastError();
  prof_end(st);
  return e;
}

cudaError_t launch_fwd_scan(const Problem& p, const bf16* q, const bf16* k, const bf16* v,
                            const float* g, const bf16* T, const float* beta_eff,
                            const float* S0, bf16* o, float* ST, bf16* hsave, bf16* Usave,
                            cudaStream_t st) {
  const size_t sm = fwd_scan_smem(p);
  cudaError_t e =
      cudaFuncSetAttribute(k_fwd_scan, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const double nb = (double)p.B * p.H * p.NC, ntok = nb * C, heads = (double)p.B * p.H;
  double bytes = ntok * (2 * D * 2 + D * 2 + p.gk * 4 + 4) + nb * C * C * 2;
  if (o) bytes += ntok * D * 2;
  if (hsave) bytes += nb * D * D * 2;
  if (Usave) bytes += ntok * D * 2;
  bytes += heads * D * D * 4 * ((S0 ? 1 : 0) + (ST ? 1 : 0));
  const double per_tile = 2.0 * C * C * D * 2 + 2.0 * C * C * BV * 2 + 2.0 * C * BV * D * 3;
  const double flops = nb * (D / BV) * per_tile;
  prof_begin(kKTcScanFwd, bytes, flops, st);
  k_fwd_scan<<<dim3(D / BV, p.H, p.B), NTS, sm, st>>>(p, q, k, v, g, T, beta_eff, S0, o, ST,
                                                      hsave, Usave);
  e = cudaGetLastError();
  prof_end(st);
  return e;
}

}  // namespace fast
}  // namespace dr
