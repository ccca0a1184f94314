// generic.cu -- fp32 CUDA-core implementation of the chunkwise forward and
// backward, for any supported head size and for fp32 or bf16 storage.
//
// Every product here is an fp32 FMA loop over shared memory; this path serves
// fp32 inputs (whose tolerance rules out bf16 tensor-core operands) and every
// head size the tensor-core path does not take.  Chunk math (per head, chunk of
// C = 64 rows, gamma = inclusive within-chunk cumulative log-gate):
//   A_ij = beta_i sum_c k_ic k_jc e^{gamma_ic - gamma_jc} (j < i),
//   M_ij = sum_c q_ic k_jc e^{gamma_ic - gamma_jc} (j <= i)           (decayed Grams)
//   T = (I + A)^{-1};  W = T diag(beta) (k e^{gamma});  U' = T diag(beta) V
//   U = U' - W S^T;  O = (q e^{gamma}) S^T + M U
//   S <- S Diag(e^{gamma_C}) + U^T (k e^{gamma_C - gamma})
// Each pair's factor e^{gamma_i - gamma_j} (j <= i) is evaluated directly, so it
// is at most 1 and never overflows whatever the decay; where it underflows the
// exact term is below fp32 resolution.  The backward's gate-scaled products
// are formed the same way.

#include "dr_common.cuh"

namespace dr {

__device__ int g_device_error = 0;

int* device_error_word() {
  int* ptr = nullptr;
  if (cudaGetSymbolAddress((void**)&ptr, g_device_error) != cudaSuccess) return nullptr;
  return ptr;
}

cudaError_t read_and_clear_device_error(int* flag) {
  cudaError_t e = cudaMemcpyFromSymbol(flag, g_device_error, sizeof(int));
  if (e != cudaSuccess || *flag == 0) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
}

namespace {

constexpr int C = kC;
constexpr int NT = kThreads;
constexpr int LDC = C + 1;  // padded stride of C x C tiles


// gamma of row i, key channel c (gk == 1: scalar gate broadcast).
__device__ __forceinline__ float gam_at(const float* sG, int gk, int i, int c) {
  return sG[i * gk + (gk == 1 ? 0 : c)];
}

// ---------------------------------------------------------------------------
// Intra-chunk forward: gamma, beta, centred Grams, T = (I + A)^{-1}, W, U'.
// grid (NC, H, B), block NT.
template <typename TIn>
__global__ void __launch_bounds__(NT) k_intra_fwd(Problem p, const TIn* __restrict__ q,
                                                  const TIn* __restrict__ k,
                                                  const TIn* __restrict__ v,
                                                  const float* __restrict__ beta,
                                                  const float* __restrict__ g, Ws ws) {
  extern __shared__ float sm[];
  const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int dk = p.dk, dv = p.dv, gk = p.gk;
  const int LD = (dk > dv ? dk : dv) + 1;
  const int t0 = n * C;
  const int nvalid = min(C, p.T - t0);
  const size_t cb = chunk_id(p, b, h, n);

  float* sK = sm;              // [C][LD] raw k
  float* sQc = sK + C * LD;    // [C][LD] raw q, later beta k e^{gamma}
  float* sKc = sQc + C * LD;   // [C][LD] beta v
  float* sA = sKc + C * LD;    // [C][LDC]
  float* sT = sA + C * LDC;    // [C][LDC]
  float* sG = sT + C * LDC;    // [C][gk]
  float* sB = sG + C * gk;     // [C]

  for (int idx = tid; idx < C * dk; idx += NT) {
    const int i = idx / dk, c = idx % dk;
    sK[i * LD + c] = (i < nvalid) ? load_f(k + row_id(p, b, t0 + i, h) * dk + c) : 0.f;
  }
  for (int idx = tid; idx < C * gk; idx += NT) {
    const int i = idx / gk, c = idx % gk;
    sG[idx] = (i < nvalid && p.gate != kGateNone) ? g[row_id(p, b, t0 + i, h) * gk + c] : 0.f;
  }
  __syncthreads();
  for (int c = tid; c < gk; c += NT) {
    float s = 0.f;
    for (int i = 0; i < C; ++i) {
      s += sG[i * gk + c];
      sG[i * gk + c] = s;
    }
  }
  for (int i = tid; i < C; i += NT) {
    float nn = 0.f;
    for (int c = 0; c < dk; ++c) nn += sK[i * LD + c] * sK[i * LD + c];
    float bb = 0.f;
    if (i < nvalid) {
      const float in = beta[row_id(p, b, t0 + i, h)];
      bb = (p.beta_mode == kBetaKaczmarz) ? in / (nn + p.eps) : in;
    }
    sB[i] = bb;
    ws.beff[cb * C + i] = bb;
    ws.kn[cb * C + i] = nn;
  }
  __syncthreads();
  for (int idx = tid; idx < C * gk; idx += NT) ws.gam[cb * C * gk + idx] = sG[idx];

  for (int idx = tid; idx < C * dk; idx += NT) {
    const int i = idx / dk, c = idx % dk;
    sQc[i * LD + c] = (i < nvalid) ? load_f(q + row_id(p, b, t0 + i, h) * dk + c) : 0.f;
  }
  __syncthreads();

  // Gram products: A (strictly lower, beta-scaled) and M (inclusive lower),
  // with each pair's factor e^{gamma_i - gamma_j} <= 1 evaluated directly.
  for (int idx = tid; idx < C * C; idx += NT) {
    const int i = idx / C, j = idx % C;
    float a = 0.f, m = 0.f;
    if (j <= i) {
      if (gk == 1) {
        for (int c = 0; c < dk; ++c) {
          const float kj = sK[j * LD + c];
          a += sK[i * LD + c] * kj;
          m += sQc[i * LD + c] * kj;
        }
        const float f = expf(sG[i] - sG[j]);
        a *= f;
        m *= f;
      } else {
        for (int c = 0; c < dk; ++c) {
          const float kj = sK[j * LD + c] * expf(sG[i * gk + c] - sG[j * gk + c]);
          a += sK[i * LD + c] * kj;
          m += sQc[i * LD + c] * kj;
        }
      }
    }
    sA[i * LDC + j] = (j < i) ? sB[i] * a : 0.f;
    ws.Mm[cb * C * C + idx] = (j <= i) ? m : 0.f;
  }
  __syncthreads();

  // T = (I + A)^{-1} by forward substitution, one column per 4 lanes:
  // T_ij = -sum_{m=j}^{i-1} A_im T_mj for i > j, T_jj = 1.
  {
    const int j = tid >> 2, part = tid & 3;
    if (part == 0)
      for (int i = 0; i < C; ++i) sT[i * LDC + j] = (i == j) ? 1.f : 0.f;
    __syncwarp();
    for (int i = 1; i < C; ++i) {
      float s = 0.f;
      if (i > j)
        for (int m = j + part; m < i; m += 4) s += sA[i * LDC + m] * sT[m * LDC + j];
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (part == 0 && i > j) sT[i * LDC + j] = -s;
      __syncwarp();
    }
  }
  __syncthreads();

  // Right-hand sides: beta k e^{gamma} into sQc, beta v into sKc.
  for (int idx = tid; idx < C * dk; idx += NT) {
    const int i = idx / dk, c = idx % dk;
    sQc[i * LD + c] = sB[i] * sK[i * LD + c] * expf(gam_at(sG, gk, i, c));
  }
  for (int idx = tid; idx < C * dv; idx += NT) {
    const int i = idx / dv, a = idx % dv;
    sKc[i * LD + a] =
        (i < nvalid) ? sB[i] * load_f(v + row_id(p, b, t0 + i, h) * dv + a) : 0.f;
  }
  for (int idx = tid; idx < C * C; idx += NT)
    ws.Tm[cb * C * C + idx] = sT[(idx / C) * LDC + idx % C];
  __syncthreads();

  for (int col = tid; col < dk + dv; col += NT) {
    const bool isw = col < dk;
    const float* rhs = isw ? sQc + col : sKc + (col - dk);
    for (int i = 0; i < C; ++i) {
      float acc = 0.f;
      for (int j = 0; j <= i; ++j) acc += sT[i * LDC + j] * rhs[j * LD];
      if (isw)
        ws.W[(cb * C + i) * dk + col] = acc;
      else
        ws.Up[(cb * C + i) * dv + (col - dk)] = acc;
    }
  }
}

// Load the per-chunk operands shared by the two scans: W, q e^{gamma},
// k e^{gamma_C - gamma}, the output Gram M and the chunk decay e^{gamma_C}.
template <typename TIn>
__device__ void load_scan_chunk(const Problem& p, const TIn* q, const TIn* k, const Ws& ws,
                                int b, int h, int n, int LDk, float* sW, float* sQ,
                                float* sKt, float* sM, float* sDec) {
  const int dk = p.dk, gk = p.gk, tid = threadIdx.x;
  const int t0 = n * C, nvalid = min(C, p.T - t0);
  const size_t cb = chunk_id(p, b, h, n);
  const float* gam = ws.gam + cb * C * gk;
  for (int idx = tid; idx < C * dk; idx += NT) {
    const int i = idx / dk, c = idx % dk;
    const int cg = (gk == 1) ? 0 : c;
    const float gi = gam[i * gk + cg], gC = gam[(C - 1) * gk + cg];
    float qv = 0.f, kv = 0.f;
    if (i < nvalid) {
      const size_t rr = row_id(p, b, t0 + i, h) * dk + c;
      qv = load_f(q + rr);
      kv = load_f(k + rr);
    }
    sW[i * LDk + c] = ws.W[cb * C * dk + idx];
    sQ[i * LDk + c] = qv * expf(gi);
    sKt[i * LDk + c] = kv * expf(gC - gi);
  }
  for (int c = tid; c < dk; c += NT) sDec[c] = expf(gam[(C - 1) * gk + (gk == 1 ? 0 : c)]);
  for (int idx = tid; idx < C * C; idx += NT) sM[(idx / C) * LDC + idx % C] = ws.Mm[cb * C * C + idx];
}

// ---------------------------------------------------------------------------
// Forward state scan + output.  grid (dv / BV, H, B), block NT.  The fp32
// state tile S[a0:a0+BV, :] stays in shared memory for the whole sequence.
template <typename TIn>
__global__ void __launch_bounds__(NT) k_scan_fwd(Problem p, int BV, const TIn* __restrict__ q,
                                                 const TIn* __restrict__ k,
                                                 const float* __restrict__ S0,
                                                 TIn* __restrict__ o, float* __restrict__ ST,
                                                 float* __restrict__ hsave, Ws ws) {
  extern __shared__ float sm[];
  const int h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int dk = p.dk, dv = p.dv, LDk = dk + 1, LDv = BV + 1;
  const int a0 = blockIdx.x * BV;
  float* sS = sm;                // [BV][LDk]
  float* sW = sS + BV * LDk;     // [C][LDk]
  float* sQ = sW + C * LDk;      // [C][LDk]
  float* sKt = sQ + C * LDk;     // [C][LDk]
  float* sU = sKt + C * LDk;     // [C][LDv]
  float* sM = sU + C * LDv;      // [C][LDC]
  float* sDec = sM + C * LDC;    // [dk]
  const size_t sbase = ((size_t)b * p.H + h) * dv * dk;

  for (int idx = tid; idx < BV * dk; idx += NT) {
    const int a = idx / dk, c = idx % dk;
    sS[a * LDk + c] = S0 ? S0[sbase + (size_t)(a0 + a) * dk + c] : 0.f;
  }
  for (int n = 0; n < p.NC; ++n) {
    const int t0 = n * C, nvalid = min(C, p.T - t0);
    const size_t cb = chunk_id(p, b, h, n);
    __syncthreads();
    load_scan_chunk(p, q, k, ws, b, h, n, LDk, sW, sQ, sKt, sM, sDec);
    for (int idx = tid; idx < C * BV; idx += NT) {
      const int i = idx / BV, a = idx % BV;
      sU[i * LDv + a] = ws.Up[(cb * C + i) * dv + a0 + a];
    }
    if (hsave)
      for (int idx = tid; idx < BV * dk; idx += NT) {
        const int a = idx / dk, c = idx % dk;
        hsave[cb * dv * dk + (size_t)(a0 + a) * dk + c] = sS[a * LDk + c];
      }
    __syncthreads();
    // U = U' - W S^T
    for (int idx = tid; idx < C * BV; idx += NT) {
      const int i = idx / BV, a = idx % BV;
      float acc = 0.f;
      for (int c = 0; c < dk; ++c) acc += sW[i * LDk + c] * sS[a * LDk + c];
      sU[i * LDv + a] -= acc;
    }
    __syncthreads();
    // O = (q e^{gamma}) S^T + M U
    if (o) {
      for (int idx = tid; idx < C * BV; idx += NT) {
        const int i = idx / BV, a = idx % BV;
        if (i >= nvalid) continue;
        float acc = 0.f;
        for (int c = 0; c < dk; ++c) acc += sQ[i * LDk + c] * sS[a * LDk + c];
        for (int j = 0; j <= i; ++j) acc += sM[i * LDC + j] * sU[j * LDv + a];
        store_f(o + row_id(p, b, t0 + i, h) * dv + a0 + a, acc);
      }
      __syncthreads();
    }
    // S <- S Diag(e^{gamma_C}) + U^T (k e^{gamma_C - gamma})
    for (int idx = tid; idx < BV * dk; idx += NT) {
      const int a = idx / dk, c = idx % dk;
      float acc = sS[a * LDk + c] * sDec[c];
      for (int i = 0; i < C; ++i) acc += sU[i * LDv + a] * sKt[i * LDk + c];
      sS[a * LDk + c] = acc;
    }
  }
  __syncthreads();
  if (ST)
    for (int idx = tid; idx < BV * dk; idx += NT) {
      const int a = idx / dk, c = idx % dk;
      ST[sbase + (size_t)(a0 + a) * dk + c] = sS[a * LDk + c];
    }
}

// ---------------------------------------------------------------------------
// Reverse state-gradient scan.  grid (dv / BV, H, B).  Emits dh (gradient of
// each chunk's end state), dU and dS0.
//   dU = M^T dO + Kt dS^T;   dS <- dS Diag(e^{gamma_C}) + dO^T (q e^{gamma}) - dU^T W
template <typename TIn>
__global__ void __launch_bounds__(NT) k_scan_bwd(Problem p, int BV, const TIn* __restrict__ q,
                                                 const TIn* __restrict__ k,
                                                 const TIn* __restrict__ dO,
                                                 const float* __restrict__ dST,
                                                 float* __restrict__ dS0, Ws ws) {
  extern __shared__ float sm[];
  const int h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int dk = p.dk, dv = p.dv, LDk = dk + 1, LDv = BV + 1;
  const int a0 = blockIdx.x * BV;
  float* sdS = sm;               // [BV][LDk]
  float* sW = sdS + BV * LDk;    // [C][LDk]
  float* sQ = sW + C * LDk;      // [C][LDk]
  float* sKt = sQ + C * LDk;     // [C][LDk]
  float* sdO = sKt + C * LDk;    // [C][LDv]
  float* sdU = sdO + C * LDv;    // [C][LDv]
  float* sM = sdU + C * LDv;     // [C][LDC]
  float* sDec = sM + C * LDC;    // [dk]
  const size_t sbase = ((size_t)b * p.H + h) * dv * dk;

  for (int idx = tid; idx < BV * dk; idx += NT) {
    const int a = idx / dk, c = idx % dk;
    sdS[a * LDk + c] = dST ? dST[sbase + (size_t)(a0 + a) * dk + c] : 0.f;
  }
  for (int n = p.NC - 1; n >= 0; --n) {
    const int t0 = n * C, nvalid = min(C, p.T - t0);
    const size_t cb = chunk_id(p, b, h, n);
    __syncthreads();
    load_scan_chunk(p, q, k, ws, b, h, n, LDk, sW, sQ, sKt, sM, sDec);
    for (int idx = tid; idx < C * BV; idx += NT) {
      const int i = idx / BV, a = idx % BV;
      sdO[i * LDv + a] = (i < nvalid) ? load_f(dO + row_id(p, b, t0 + i, h) * dv + a0 + a) : 0.f;
    }
    for (int idx = tid; idx < BV * dk; idx += NT) {
      const int a = idx / dk, c = idx % dk;
      ws.dh[cb * dv * dk + (size_t)(a0 + a) * dk + c] = sdS[a * LDk + c];
    }
    __syncthreads();
    for (int idx = tid; idx < C * BV; idx += NT) {
      const int i = idx / BV, a = idx % BV;
      float acc = 0.f;
      for (int i2 = i; i2 < C; ++i2) acc += sM[i2 * LDC + i] * sdO[i2 * LDv + a];
      for (int c = 0; c < dk; ++c) acc += sKt[i * LDk + c] * sdS[a * LDk + c];
      sdU[i * LDv + a] = acc;
      ws.dU[(cb * C + i) * dv + a0 + a] = acc;
    }
    __syncthreads();
    for (int idx = tid; idx < BV * dk; idx += NT) {
      const int a = idx / dk, c = idx % dk;
      float acc = sdS[a * LDk + c] * sDec[c];
      for (int i = 0; i < C; ++i)
        acc += sdO[i * LDv + a] * sQ[i * LDk + c] - sdU[i * LDv + a] * sW[i * LDk + c];
      sdS[a * LDk + c] = acc;
    }
  }
  __syncthreads();
  if (dS0)
    for (int idx = tid; idx < BV * dk; idx += NT) {
      const int a = idx / dk, c = idx % dk;
      dS0[sbase + (size_t)(a0 + a) * dk + c] = sdS[a * LDk + c];
    }
}

// ---------------------------------------------------------------------------
// Per-chunk products with the chunk's start state S = h_n and end-state
// gradient dS' = dh_n.  grid (NC, H, B).
//   U = U' - W S^T;  dQs = dO S;  dWs = -dU S;  dKt = U dS';
//   dgC = e^{gamma_C} * colsum(dS' .* S)
template <typename TIn>
__global__ void __launch_bounds__(NT) k_state_grads(Problem p, const TIn* __restrict__ dO,
                                                    const float* __restrict__ hst, Ws ws) {
  extern __shared__ float sm[];
  const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int dk = p.dk, dv = p.dv, gk = p.gk, LDk = dk + 1, LDv = dv + 1;
  const int t0 = n * C, nvalid = min(C, p.T - t0);
  const size_t cb = chunk_id(p, b, h, n);
  float* sS = sm;               // [dv][LDk]   S, later dS'
  float* sX = sS + dv * LDk;    // [C][max(LDk, LDv)]  W, later dO
  const int LDx = LDk > LDv ? LDk : LDv;
  float* sU = sX + C * LDx;     // [C][LDv]
  float* sdU = sU + C * LDv;    // [C][LDv]
  const float* Sg = hst + cb * dv * dk;
  const float* dSg = ws.dh + cb * dv * dk;

  for (int idx = tid; idx < dv * dk; idx += NT) sS[(idx / dk) * LDk + idx % dk] = Sg[idx];
  for (int idx = tid; idx < C * dk; idx += NT)
    sX[(idx / dk) * LDx + idx % dk] = ws.W[cb * C * dk + idx];
  for (int idx = tid; idx < C * dv; idx += NT)
    sdU[(idx / dv) * LDv + idx % dv] = ws.dU[cb * C * dv + idx];
  __syncthreads();
  for (int idx = tid; idx < C * dv; idx += NT) {
    const int i = idx / dv, a = idx % dv;
    float acc = 0.f;
    for (int c = 0; c < dk; ++c) acc += sX[i * LDx + c] * sS[a * LDk + c];
    const float u = ws.Up[cb * C * dv + idx] - acc;
    sU[i * LDv + a] = u;
    ws.U[cb * C * dv + idx] = u;
  }
  // e^{gamma_C} * colsum(dS' .* S)
  for (int c = tid; c < dk; c += NT) {
    float acc = 0.f;
    for (int a = 0; a < dv; ++a) acc += dSg[(size_t)a * dk + c] * sS[a * LDk + c];
    ws.dgC[cb * dk + c] = acc * expf(ws.gam[(cb * C + C - 1) * gk + (gk == 1 ? 0 : c)]);
  }
  __syncthreads();
  for (int idx = tid; idx < C * dv; idx += NT) {
    const int i = idx / dv, a = idx % dv;
    sX[i * LDx + a] = (i < nvalid) ? load_f(dO + row_id(p, b, t0 + i, h) * dv + a) : 0.f;
  }
  __syncthreads();
  for (int idx = tid; idx < C * dk; idx += NT) {
    const int i = idx / dk, c = idx % dk;
    float aq = 0.f, aw = 0.f;
    for (int a = 0; a < dv; ++a) {
      const float s = sS[a * LDk + c];
      aq += sX[i * LDx + a] * s;
      aw += sdU[i * LDv + a] * s;
    }
    ws.dQs[cb * C * dk + idx] = aq;
    ws.dWs[cb * C * dk + idx] = -aw;
  }
  __syncthreads();
  for (int idx = tid; idx < dv * dk; idx += NT) sS[(idx / dk) * LDk + idx % dk] = dSg[idx];
  __syncthreads();
  for (int idx = tid; idx < C * dk; idx += NT) {
    const int i = idx / dk, c = idx % dk;
    float acc = 0.f;
    for (int a = 0; a < dv; ++a) acc += sU[i * LDv + a] * sS[a * LDk + c];
    ws.dKt[cb * C * dk + idx] = acc;
  }
}

// ---------------------------------------------------------------------------
// Intra-chunk backward (triangular residual system).  grid (NC, H, B).
// Threads [0, dk) own key channels, threads [dk, dk + dv) own value channels.
template <typename TIn>
__global__ void __launch_bounds__(NT) k_intra_bwd(Problem p, const TIn* __restrict__ q,
                                                  const TIn* __restrict__ k,
                                                  const TIn* __restrict__ v,
                                                  const TIn* __restrict__ dO,
                                                  const float* __restrict__ beta_in,
                                                  TIn* __restrict__ dq, TIn* __restrict__ dk_out,
                                                  TIn* __restrict__ dv_out,
                                                  float* __restrict__ dbeta,
                                                  float* __restrict__ dg, Ws ws) {
  extern __shared__ float sm[];
  const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int dk = p.dk, dv = p.dv, gk = p.gk;
  const int LD = (dk > dv ? dk : dv) + 1;
  const int t0 = n * C, nvalid = min(C, p.T - t0);
  const size_t cb = chunk_id(p, b, h, n);
  float* sKc = sm;               // [C][LD] raw k
  float* sM1 = sKc + C * LD;     // [C][LDC] T
  float* sM2 = sM1 + C * LDC;    // [C][LDC] dM, later dA
  float* sR0 = sM2 + C * LDC;    // [C][LD] dO | raw q | Lambda half
  float* sR1 = sR0 + C * LD;     // [C][LD] U | dX half | X half
  float* sG = sR1 + C * LD;      // [C][gk]
  float* sB = sG + C * gk;       // [C]
  float* sdb = sB + C;           // [C] dbeta accumulator
  float* sdgs = sdb + C;         // [C] scalar-gate dg accumulator
  float* dk_acc = ws.dk_acc + cb * C * dk;
  float* dg_acc = ws.dg_acc + cb * C * dk;
  const float* gamg = ws.gam + cb * C * gk;

  for (int idx = tid; idx < C * gk; idx += NT) sG[idx] = gamg[idx];
  for (int i = tid; i < C; i += NT) {
    sB[i] = ws.beff[cb * C + i];
    sdb[i] = 0.f;
    sdgs[i] = 0.f;
  }
  // P0: dM = tril(dO U^T)
  for (int idx = tid; idx < C * dv; idx += NT) {
    const int i = idx / dv, a = idx % dv;
    sR0[i * LD + a] = (i < nvalid) ? load_f(dO + row_id(p, b, t0 + i, h) * dv + a) : 0.f;
    sR1[i * LD + a] = ws.U[cb * C * dv + idx];
  }
  __syncthreads();
  for (int idx = tid; idx < C * C; idx += NT) {
    const int i = idx / C, j = idx % C;
    float acc = 0.f;
    if (j <= i)
      for (int a = 0; a < dv; ++a) acc += sR0[i * LD + a] * sR1[j * LD + a];
    sM2[i * LDC + j] = acc;
  }
  __syncthreads();
  // P1: raw q into sR0 and raw k into sKc; each gate-scaled product below forms
  // its pair factor e^{gamma_i - gamma_j} (<= 1) directly.
  for (int idx = tid; idx < C * dk; idx += NT) {
    const int i = idx / dk, c = idx % dk;
    float kv = 0.f, qv = 0.f;
    if (i < nvalid) {
      const size_t rr = row_id(p, b, t0 + i, h) * dk + c;
      kv = load_f(k + rr);
      qv = load_f(q + rr);
    }
    sR0[i * LD + c] = qv;
    sKc[i * LD + c] = kv;
  }
  __syncthreads();
  if (tid < dk) {
    const int c = tid;
    for (int i = 0; i < C; ++i) {
      // dq of the intra-chunk term: sum_{j <= i} dM_ij k_j e^{gamma_i - gamma_j}
      const float gi = gam_at(sG, gk, i, c);
      float dqm = 0.f;
      for (int j = 0; j <= i; ++j)
        dqm += sM2[i * LDC + j] * sKc[j * LD + c] * expf(gi - gam_at(sG, gk, j, c));
      const float eg = expf(gi);
      const float dqs = ws.dQs[(cb * C + i) * dk + c];
      ws.dQs[(cb * C + i) * dk + c] = 0.f;  // reused below as this column's dbeta terms
      const float qv = sR0[i * LD + c];
      if (i < nvalid) store_f(dq + row_id(p, b, t0 + i, h) * dk + c, dqm + eg * dqs);
      dg_acc[i * dk + c] = qv * dqm + qv * eg * dqs;
    }
    for (int j = 0; j < C; ++j) {
      // the write-key side: sum_{i >= j} dM_ij q_i e^{gamma_i - gamma_j}
      const float gj = gam_at(sG, gk, j, c);
      float dkbm = 0.f;
      for (int i = j; i < C; ++i)
        dkbm += sM2[i * LDC + j] * sR0[i * LD + c] * expf(gam_at(sG, gk, i, c) - gj);
      dk_acc[j * dk + c] = dkbm;
      dg_acc[j * dk + c] -= sKc[j * LD + c] * dkbm;
    }
  }
  // P2: Lambda = T^T [dU | dW]; dA = -strict_tril(Lambda X^T), X = [U' | W].
  for (int idx = tid; idx < C * C; idx += NT)
    sM1[(idx / C) * LDC + idx % C] = ws.Tm[cb * C * C + idx];
  __syncthreads();
  for (int idx = tid; idx < C * dv; idx += NT)
    sR1[(idx / dv) * LD + idx % dv] = ws.dU[cb * C * dv + idx];
  __syncthreads();
  if (tid >= dk && tid < dk + dv) {
    const int a = tid - dk;
    for (int i = 0; i < C; ++i) {
      float lam = 0.f;
      for (int m = i; m < C; ++m) lam += sM1[m * LDC + i] * sR1[m * LD + a];
      sR0[i * LD + a] = lam;
      float dbt = 0.f;
      if (i < nvalid) {
        const size_t rr = row_id(p, b, t0 + i, h) * dv + a;
        store_f(dv_out + rr, sB[i] * lam);
        dbt = lam * load_f(v + rr);
      }
      ws.dU[(cb * C + i) * dv + a] = dbt;  // dU is in shared memory now; reuse for dbeta terms
    }
  }
  __syncthreads();
  for (int idx = tid; idx < C * dv; idx += NT)
    sR1[(idx / dv) * LD + idx % dv] = ws.Up[cb * C * dv + idx];
  __syncthreads();
  for (int idx = tid; idx < C * C; idx += NT) {
    const int i = idx / C, j = idx % C;
    float acc = 0.f;
    if (j < i)
      for (int a = 0; a < dv; ++a) acc += sR0[i * LD + a] * sR1[j * LD + a];
    sM2[i * LDC + j] = -acc;
  }
  __syncthreads();
  for (int idx = tid; idx < C * dk; idx += NT)
    sR1[(idx / dk) * LD + idx % dk] = ws.dWs[cb * C * dk + idx];
  __syncthreads();
  if (tid < dk) {
    const int c = tid;
    for (int i = 0; i < C; ++i) {
      float lam = 0.f;
      for (int m = i; m < C; ++m) lam += sM1[m * LDC + i] * sR1[m * LD + c];
      sR0[i * LD + c] = lam;
      // R = diag(beta) k e^{gamma}: dk += e^{gamma} beta Lambda_W; dgamma += Kh beta Lambda_W
      const float eg = expf(gam_at(sG, gk, i, c));
      const float kv = (i < nvalid) ? load_f(k + row_id(p, b, t0 + i, h) * dk + c) : 0.f;
      dk_acc[i * dk + c] += eg * sB[i] * lam;
      dg_acc[i * dk + c] += kv * eg * sB[i] * lam;
      ws.dQs[(cb * C + i) * dk + c] += lam * kv * eg;
    }
  }
  __syncthreads();
  for (int idx = tid; idx < C * dk; idx += NT)
    sR1[(idx / dk) * LD + idx % dk] = ws.W[cb * C * dk + idx];
  __syncthreads();
  for (int idx = tid; idx < C * C; idx += NT) {
    const int i = idx / C, j = idx % C;
    float acc = 0.f;
    if (j < i)
      for (int c = 0; c < dk; ++c) acc += sR0[i * LD + c] * sR1[j * LD + c];
    sM2[i * LDC + j] -= acc;
  }
  __syncthreads();
  // P4: A_ij = beta_i sum_c k_ic k_jc e^{gamma_ic - gamma_jc} (j < i):
  //   x_i = sum_{j<i} dA_ij k_j e^{gamma_i - gamma_j},  y_i = sum_{i2>i} dA_i2,i beta_i2 k_i2 e^{gamma_i2 - gamma_i}
  //   dk += beta x + y;  dgamma += k (beta x - y);  dbeta += k . x
  if (tid < dk) {
    const int c = tid;
    for (int i = 0; i < C; ++i) {
      const float gi = gam_at(sG, gk, i, c);
      float x = 0.f, y = 0.f;
      for (int j = 0; j < i; ++j)
        x += sM2[i * LDC + j] * sKc[j * LD + c] * expf(gi - gam_at(sG, gk, j, c));
      for (int i2 = i + 1; i2 < C; ++i2)
        y += sM2[i2 * LDC + i] * sB[i2] * sKc[i2 * LD + c] * expf(gam_at(sG, gk, i2, c) - gi);
      const float kv = sKc[i * LD + c];
      dk_acc[i * dk + c] += sB[i] * x + y;
      dg_acc[i * dk + c] += kv * (sB[i] * x - y);
      ws.dQs[(cb * C + i) * dk + c] += kv * x;
    }
    // P5: state-update key term Kt = k e^{gamma_C - gamma}, then reverse cumsum.
    const float gC = gam_at(sG, gk, C - 1, c);
    float sumkt = 0.f;
    for (int i = 0; i < C; ++i) {
      const float gi = gam_at(sG, gk, i, c);
      const float e = expf(gC - gi);
      const float kv = (i < nvalid) ? load_f(k + row_id(p, b, t0 + i, h) * dk + c) : 0.f;
      const float dkt = ws.dKt[(cb * C + i) * dk + c];
      dk_acc[i * dk + c] += e * dkt;
      dg_acc[i * dk + c] -= kv * e * dkt;
      sumkt += kv * e * dkt;
    }
    dg_acc[(C - 1) * dk + c] += sumkt + ws.dgC[cb * dk + c];
    float run = 0.f;
    for (int i = C - 1; i >= 0; --i) {
      run += dg_acc[i * dk + c];
      dg_acc[i * dk + c] = run;
      if (i < nvalid && p.gate == kGateChannel) dg[row_id(p, b, t0 + i, h) * dk + c] = run;
    }
  }
  __syncthreads();
  // Row reductions in a fixed order (no atomics, so results are bit-reproducible).
  for (int i = tid; i < C; i += NT) {
    float db = 0.f, gs = 0.f;
    for (int a = 0; a < dv; ++a) db += ws.dU[(cb * C + i) * dv + a];
    for (int c = 0; c < dk; ++c) {
      db += ws.dQs[(cb * C + i) * dk + c];
      gs += dg_acc[i * dk + c];
    }
    sdb[i] = db;
    sdgs[i] = gs;
  }
  __syncthreads();
  if (tid < dk) {
    const int c = tid;
    for (int i = 0; i < nvalid; ++i) {
      const size_t rr = row_id(p, b, t0 + i, h) * dk + c;
      float acc = dk_acc[i * dk + c];
      if (p.beta_mode == kBetaKaczmarz) {
        const float den = ws.kn[cb * C + i] + p.eps;
        acc += -2.f * sB[i] * sdb[i] * load_f(k + rr) / den;
      }
      store_f(dk_out + rr, acc);
    }
  }
  for (int i = tid; i < nvalid; i += NT) {
    const size_t rr = row_id(p, b, t0 + i, h);
    float db = sdb[i];
    if (p.beta_mode == kBetaKaczmarz) db /= (ws.kn[cb * C + i] + p.eps);
    dbeta[rr] = db;
    if (p.gate == kGateScalar) dg[rr] = sdgs[i];
  }
  (void)beta_in;
}

size_t intra_fwd_smem(const Problem& p) {
  const int LD = (p.dk > p.dv ? p.dk : p.dv) + 1;
  return sizeof(float) * ((size_t)3 * C * LD + 2 * C * LDC + C * p.gk + C);
}
size_t scan_smem(const Problem& p, int BV) {
  const int LDk = p.dk + 1;
  return sizeof(float) * ((size_t)BV * LDk + 3 * C * LDk + 2 * C * (BV + 1) + C * LDC + p.dk);
}
size_t state_grads_smem(const Problem& p) {
  const int LDk = p.dk + 1, LDv = p.dv + 1, LDx = LDk > LDv ? LDk : LDv;
  return sizeof(float) * ((size_t)p.dv * LDk + C * LDx + 2 * C * LDv);
}
size_t intra_bwd_smem(const Problem& p) {
  const int LD = (p.dk > p.dv ? p.dk : p.dv) + 1;
  return sizeof(float) * ((size_t)3 * C * LD + 2 * C * LDC + C * p.gk + 3 * C);
}

int pick_bv(const Problem& p) { return (p.dv % 32 == 0) ? 32 : 16; }

// Work models per launch (whole grid): io_bytes = the operator's inputs and
// outputs the kernel reads or writes, each once (algorithmic); bytes = every
// tensor it must read or write once, including the workspace tensors it
// exchanges with the other kernels; FLOPs = 2 x multiply-adds of its products,
// triangular products counted at their triangle.
struct Work {
  double io_bytes, bytes, flops;
};
Work work_of(int kernel, const Problem& p, int es, bool states_io) {
  const double nb = (double)p.B * p.H * p.NC, C = kC, dk = p.dk, dv = p.dv, gk = p.gk;
  const double ntok = nb * C;  // padded token-heads
  const double grid_in = ntok * (gk * 4 + 4);          // g, beta
  const double st = nb * dv * dk * 4;                  // one fp32 state per chunk
  Work w{0, 0, 0};
  switch (kernel) {
    case kKIntraFwd:
      w.io_bytes = ntok * (2 * dk + dv) * es + grid_in;
      w.bytes = ntok * (2 * dk + dv) * es + grid_in +
                ntok * (gk * 4 + 8) + nb * C * C * 8 + ntok * (dk + dv) * 4;
      w.flops = nb * (2 * C * C * dk + C * C * C / 3 + C * C * (dk + dv));
      break;
    case kKScanFwd:
      w.io_bytes = ntok * (2 * dk + dv) * es;
      w.bytes = ntok * ((dk + dv) * 4 + gk * 4 + 2 * dk * es) + nb * C * C * 4 +
                ntok * dv * es + (states_io ? st : 0);
      w.flops = nb * (6 * C * dk * dv + C * C * dv);
      break;
    case kKScanBwd:
      w.io_bytes = ntok * (2 * dk + dv) * es;
      w.bytes = ntok * (dk * 4 + gk * 4 + 2 * dk * es + dv * es) + nb * C * C * 4 + st +
                ntok * dv * 4;
      w.flops = nb * (6 * C * dk * dv + C * C * dv);
      break;
    case kKStateGrads:
      w.io_bytes = ntok * dv * es;
      w.bytes = 2 * st + ntok * (dk * 4 + 2 * dv * 4 + dv * es) + ntok * (dv * 4 + 3 * dk * 4) +
                nb * dk * 4;
      w.flops = nb * 8 * C * dk * dv;
      break;
    case kKIntraBwd:
      w.io_bytes = ntok * ((2 * dk + 2 * dv) * es + gk * 4 + 4) +
                   ntok * ((2 * dk + dv) * es + gk * 4 + 4);
      w.bytes = ntok * ((2 * dk + 2 * dv) * es + gk * 4 + 12) + nb * C * C * 4 +
                ntok * (3 * dv + 4 * dk) * 4 + nb * dk * 4 + ntok * ((2 * dk + dv) * es + gk * 4 + 4);
      w.flops = nb * (C * C * dv + 2 * C * C * dk + 2 * C * C * (dk + dv) + 2 * C * C * dk);
      break;
  }
  return w;
}

template <typename F>
cudaError_t timed_launch(int kernel, const Problem& p, int es, bool states_io, cudaStream_t st,
                         F&& launch) {
  const Work w = work_of(kernel, p, es, states_io);
  prof_begin(kernel, w.io_bytes, w.bytes, w.flops, st);
  launch();
  cudaError_t e = cudaGetLastError();
  prof_end(st);
  return e;
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace

template <typename TIn>
cudaError_t launch_generic_fwd(const Problem& p, const TIn* q, const TIn* k, const TIn* v,
                               const float* beta, const float* g, const float* S0, TIn* o,
                               float* ST, float* hsave, const Ws& ws, cudaStream_t st) {
  cudaError_t e;
  const int es = sizeof(TIn);
  const size_t s1 = intra_fwd_smem(p);
  if ((e = set_smem(k_intra_fwd<TIn>, s1)) != cudaSuccess) return e;
  e = timed_launch(kKIntraFwd, p, es, false, st, [&] {
    k_intra_fwd<TIn><<<dim3(p.NC, p.H, p.B), NT, s1, st>>>(p, q, k, v, beta, g, ws);
  });
  if (e != cudaSuccess) return e;
  const int BV = pick_bv(p);
  const size_t s2 = scan_smem(p, BV);
  if ((e = set_smem(k_scan_fwd<TIn>, s2)) != cudaSuccess) return e;
  return timed_launch(kKScanFwd, p, es, hsave != nullptr, st, [&] {
    k_scan_fwd<TIn><<<dim3(p.dv / BV, p.H, p.B), NT, s2, st>>>(p, BV, q, k, S0, o, ST, hsave,
                                                               ws);
  });
}

template <typename TIn>
cudaError_t launch_generic_bwd(const Problem& p, const TIn* q, const TIn* k, const TIn* v,
                               const float* beta, const float* g, const float* S0,
                               const TIn* dO, const float* dST, const float* hsaved,
                               TIn* dq, TIn* dk, TIn* dv, float* dbeta, float* dg,
                               float* dS0, const Ws& ws, cudaStream_t st) {
  cudaError_t e;
  const int es = sizeof(TIn);
  const size_t s1 = intra_fwd_smem(p);
  if ((e = set_smem(k_intra_fwd<TIn>, s1)) != cudaSuccess) return e;
  e = timed_launch(kKIntraFwd, p, es, false, st, [&] {
    k_intra_fwd<TIn><<<dim3(p.NC, p.H, p.B), NT, s1, st>>>(p, q, k, v, beta, g, ws);
  });
  if (e != cudaSuccess) return e;
  const int BV = pick_bv(p);
  const size_t s2 = scan_smem(p, BV);
  const float* hst = hsaved;
  if (!hst) {
    if ((e = set_smem(k_scan_fwd<TIn>, s2)) != cudaSuccess) return e;
    e = timed_launch(kKScanFwd, p, es, true, st, [&] {
      k_scan_fwd<TIn><<<dim3(p.dv / BV, p.H, p.B), NT, s2, st>>>(p, BV, q, k, S0, nullptr,
                                                                 nullptr, ws.h, ws);
    });
    if (e != cudaSuccess) return e;
    hst = ws.h;
  }
  if ((e = set_smem(k_scan_bwd<TIn>, s2)) != cudaSuccess) return e;
  e = timed_launch(kKScanBwd, p, es, true, st, [&] {
    k_scan_bwd<TIn><<<dim3(p.dv / BV, p.H, p.B), NT, s2, st>>>(p, BV, q, k, dO, dST, dS0, ws);
  });
  if (e != cudaSuccess) return e;
  const size_t s3 = state_grads_smem(p);
  if ((e = set_smem(k_state_grads<TIn>, s3)) != cudaSuccess) return e;
  e = timed_launch(kKStateGrads, p, es, true, st, [&] {
    k_state_grads<TIn><<<dim3(p.NC, p.H, p.B), NT, s3, st>>>(p, dO, hst, ws);
  });
  if (e != cudaSuccess) return e;
  const size_t s4 = intra_bwd_smem(p);
  if ((e = set_smem(k_intra_bwd<TIn>, s4)) != cudaSuccess) return e;
  return timed_launch(kKIntraBwd, p, es, true, st, [&] {
    k_intra_bwd<TIn><<<dim3(p.NC, p.H, p.B), NT, s4, st>>>(p, q, k, v, dO, beta, dq, dk, dv,
                                                           dbeta, dg, ws);
  });
}

template cudaError_t launch_generic_fwd<float>(const Problem&, const float*, const float*,
                                               const float*, const float*, const float*,
                                               const float*, float*, float*, float*, const Ws&,
                                               cudaStream_t);
template cudaError_t launch_generic_fwd<__nv_bfloat16>(
    const Problem&, const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*,
    const float*, const float*, const float*, __nv_bfloat16*, float*, float*, const Ws&,
    cudaStream_t);
template cudaError_t launch_generic_bwd<float>(const Problem&, const float*, const float*,
                                               const float*, const float*, const float*,
                                               const float*, const float*, const float*,
                                               const float*, float*, float*, float*, float*,
                                               float*, float*, const Ws&, cudaStream_t);
template cudaError_t launch_generic_bwd<__nv_bfloat16>(
    const Problem&, const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*,
    const float*, const float*, const float*, const __nv_bfloat16*, const float*,
    const float*, __nv_bfloat16*, __nv_bfloat16*, __nv_bfloat16*, float*, float*, float*,
    const Ws&, cudaStream_t);

}  // namespace dr
