// fast_scan_tc.cu -- the forward state scan on tcgen05 tensor cores (bf16
// storage, d_k = d_v = 128, C = 64): one CTA per (b, h, value tile of BV
// rows of the state), 256 threads, sequential over the chunks of the head.
//
// Per chunk n, with the chunk tiles the prep kernel produced (W, q e^gamma,
// k e^{gamma_C - gamma}, M = tril(Q^c Kb^c^T), U', the chunk decay):
//   MMA-A  D_A   = [W ; q e^gamma] S_n^T                 (M = 128, N = BV, K = 128)
//   epilogue 1   U = U' - D_A[0:64]       (bf16 operand tile, saved for the backward)
//   MMA-B  D_A[64:128] += M U    (A = [0 ; M], so the W rows are left untouched)
//   MMA-C  D_S   = (k e^{gamma_C - gamma})^T U           (M = 128 keys, N = BV)
//   epilogue 2   S_{n+1}^T = Diag(e^{gamma_C}) S_n^T + D_S   (fp32, registers)
// and o_n = D_A[64:128].  The state lives in registers transposed, one key
// column per TMEM lane, so the per-channel decay is one scalar per thread; the
// bf16 copy of S^T in shared memory is the MN-major B operand of the next
// MMA-A.  o_{n-1} is written to global memory while MMA-A of chunk n runs, the
// chunk-start state h_n while MMA-B and MMA-C run.  D_A is double-buffered in tensor memory for
// that reason.  Chunk tiles stream through a two-stage pipeline of bulk copies
// (issued by the lanes of one warp, one mbarrier per stage) into the canonical
// no-swizzle core-matrix layouts.
//
// This is the affine state transfer of the chunkwise (WY/UT) form:
//   S_{n+1} = S_n Diag(e^{gamma_C}) + (U' - W S_n^T)^T K~,
//   O_n     = Q^ S_n^T + (M o L) (U' - W S_n^T).

#include "dr_common.cuh"
#include "fast.cuh"
#include "frag.cuh"
#include "tc.cuh"

namespace dr {
namespace fast {

using frag::bf16;

namespace {

constexpr int C = 64, D = 128;
constexpr int NTF = 256;
constexpr uint32_t kSpinScan = 1u << 22;

template <int BV>
struct ScanStage {
  bf16 AWQ[128 * D];   // [W ; q e^gamma], K-major (rows i | 64 + i, K = key c)
  bf16 KT[C * D];      // k e^{gamma_C - gamma} as the MN-major A of MMA-C ([K = i][M = c])
  bf16 MZ[128 * C];    // [0 ; M], K-major (K = j); the zero half is written once
  bf16 UP[C * BV];     // U'[:, a0 .. a0 + BV), core-tiled
  float dec[D];        // e^{gamma_C} per key column
};

template <int BV>
struct ScanSmem {
  ScanStage<BV> st[2];
  bf16 SB[D * BV];     // bf16 S^T, MN-major B of MMA-A ([K = c][N = a])
  bf16 UB[C * BV];     // bf16 U, MN-major B of MMA-B / MMA-C ([K = i][N = a])
  uint64_t barA, barB, barO, full[2];
  uint32_t tmem;
};

// Bytes of one stage fill's bulk copies.
__host__ __device__ constexpr uint32_t scan_fill_bytes(bool with_o) {
  return (uint32_t)(sizeof(bf16) * (2 * C * D + (with_o ? C * D + C * C : 0)) + sizeof(float) * D);
}

// Fills a stage, called by every thread: the chunk tiles, stored core-tiled in
// HBM (the layout of the operands here), by bulk copies from lane 0 of warps 1,
// 4 and 5 (the warps that neither issue MMA-A nor store o at the top of a step;
// a bulk copy holds its issuing thread while the copy engine takes it),
// completing on `full` (whose transaction count thread 0 has set with
// scan_fill_bytes before a barrier that precedes this), and U'[:, a0 .. a0 + BV)
// (one run of BV / 8 core matrices per block of 8 rows) by cp.async from every
// thread, one group (committed also when empty).
// The stage's M tile was last read by the output product (MMA-B) of the step
// two chunks back, which completes on its own barrier: when `mb_parity` >= 0 the
// copy of M waits (bounded) for that phase of `barO` first.
template <int BV>
__device__ __forceinline__ void scan_fill(ScanStage<BV>& s, uint64_t* full, const Saved& sv,
                                          size_t cb, int a0, bool with_o, bool with_up,
                                          int warp, int lane, uint64_t* barO, int mb_parity) {
  constexpr uint32_t kT = sizeof(bf16) * C * D, kM = sizeof(bf16) * C * C;
  if (lane == 0) {
    switch (warp) {
      case 1:
        tc::bulk_g2s(s.AWQ, sv.W + cb * C * D, kT, full);
        tc::bulk_g2s(s.KT, sv.Kt + cb * C * D, kT, full);
        break;
      case 4:
        if (with_o) {
          tc::bulk_g2s(s.AWQ + C * D, sv.Qh + cb * C * D, kT, full);
          if (mb_parity < 0 || tc::mbar_wait(barO, (uint32_t)(mb_parity & 1), kSpinScan))
            tc::bulk_g2s(s.MZ + C * C, sv.M + cb * C * C, kM, full);
        }
        break;
      case 5: tc::bulk_g2s(s.dec, sv.dec + cb * D, sizeof(float) * D, full); break;
      default: break;
    }
  }
  if (with_up) cp_ct_cols<NTF>(s.UP, sv.Up + cb * C * D, C, a0, BV, threadIdx.x);
  frag::cp_commit();
}

// Writes this thread's HB state values x[u] (value rows a0h + u of key c; one
// key per lane) as bf16 into a core-tiled state tile stored transposed, [key
// c][value a] (the K-major B operand of the chunk backward's products with the
// state): a thread's values are 16-byte runs of its own row, and a warp writes
// four whole 128-byte core matrices per store.
template <int HB>
__device__ __forceinline__ void store_state_ct(bf16* dst, const float* x, int a0h, int c) {
#pragma unroll
  for (int u8 = 0; u8 < HB / 8; ++u8) {
    const float* v = x + 8 * u8;
    *reinterpret_cast<uint4*>(dst + ct_off(c, a0h + 8 * u8, D)) =
        make_uint4(frag::pack(v[0], v[1]), frag::pack(v[2], v[3]), frag::pack(v[4], v[5]),
                   frag::pack(v[6], v[7]));
  }
}

__device__ __forceinline__ uint32_t lane_addr(uint32_t base, int warp, int col) {
  return base + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)col;
}


// PHASE: the SFDA rotation-decay gate.  The chunk decay then mixes the key
// pair (2j, 2j + 1) of every state row as the complex product
// (dec[2j] + i dec[2j+1]) (x + i y); the pair's two keys sit on adjacent lanes.
template <int BV, bool PHASE>
__global__ void __launch_bounds__(NTF, 1)
    k_fwd_scan_tc(Problem p, Saved sv, ScanSeg sg, bf16* __restrict__ o, int save,
                  int* __restrict__ err) {
  constexpr int HB = BV / 2;             // value columns per thread in the state epilogue
  constexpr int TCOLS = 3 * BV;          // tensor memory columns: D_A x 2, D_S
  constexpr int TALLOC = TCOLS <= 256 ? 256 : 512;
  extern __shared__ __align__(1024) unsigned char smraw[];
  ScanSmem<BV>& s = *reinterpret_cast<ScanSmem<BV>*>(smraw);
  const int h = blockIdx.y, b = blockIdx.z / sg.G, seg = blockIdx.z % sg.G, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  int mode = sg.mode, xb = blockIdx.x;
  float* __restrict__ ST = sg.ST;
  if (mode == 3) {  // transfer matrices (first D/BV x-blocks) and offsets (the rest)
    mode = xb < D / BV ? 1 : 2;
    if (mode == 2) {
      ST = sg.ST2;
      xb -= D / BV;
    }
  }
  const int a0 = xb * BV;
  const int n0 = seg * sg.L, n1 = min(p.NC, n0 + sg.L);
  if (n0 >= n1) return;
  const bool with_o = o != nullptr;
  const bool with_up = mode != 1;
  const float* __restrict__ S0 = mode == 0 ? sg.S0 : nullptr;
  const size_t sbase = (((size_t)b * sg.G + seg) * p.H + h) * D * D;
  // state epilogue ownership: key column c (= TMEM lane), value columns ah*HB ..
  const int c = 32 * (warp & 3) + lane, ah = warp >> 2;
  const uint32_t T_S = 2 * BV;  // D_A buffers at columns 0 and BV

  if (warp == 0) tc::tmem_alloc(&s.tmem, TALLOC);
  if (tid == 0) {
    tc::mbar_init(&s.barA, 1);
    tc::mbar_init(&s.barB, 1);
    tc::mbar_init(&s.barO, 1);
    tc::mbar_init(&s.full[0], 1);
    tc::mbar_init(&s.full[1], 1);
    tc::fence_mbar_init();
  }
  // zero halves of [0 ; M] in both stages
  for (int idx = tid; idx < 2 * C * C / 8; idx += NTF) {
    const int stg = idx / (C * C / 8), e = idx % (C * C / 8);
    *reinterpret_cast<uint4*>(s.st[stg].MZ + 8 * e) = make_uint4(0, 0, 0, 0);
  }
  // fp32 state S^T[c][a0 + ah*HB + u]
  float S[HB];
#pragma unroll
  for (int u = 0; u < HB; ++u) {
    const int a = a0 + ah * HB + u;
    S[u] = mode == 1 ? (a == c ? 1.f : 0.f) : (S0 ? S0[sbase + (size_t)a * D + c] : 0.f);
  }

  auto write_sb = [&]() {
#pragma unroll
    for (int u8 = 0; u8 < HB / 8; ++u8) {
      float f[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = S[8 * u8 + e];
      *reinterpret_cast<uint4*>(s.SB + tc::mnmaj_off(c, ah * HB + 8 * u8, BV)) =
          make_uint4(frag::pack(f[0], f[1]), frag::pack(f[2], f[3]), frag::pack(f[4], f[5]),
                     frag::pack(f[6], f[7]));
    }
  };
  // h_n (bf16, core-tiled [c][a]) from the registers
  auto store_h = [&](size_t cbn) {
    store_state_ct<HB>(sv.h + cbn * D * D, S, a0 + ah * HB, c);
  };
  // o rows of chunk nn from D_A buffer `buf` (warps on lanes 64 .. 127)
  auto store_o = [&](int nn, int buf, int ph) -> bool {
    if ((warp & 3) < 2) return true;
    if (!tc::mbar_wait(&s.barO, (uint32_t)(ph & 1), kSpinScan)) return false;
    tc::fence_after_sync();
    const int i = 32 * ((warp & 3) - 2) + lane;
    const int t0 = nn * C, nvalid = min(C, p.T - t0);
    uint32_t r[HB];
#pragma unroll
    for (int q16 = 0; q16 < HB / 16; ++q16)
      tc::tmem_ld16_nowait(lane_addr(s.tmem, warp, buf * BV + ah * HB + 16 * q16), r + 16 * q16);
    tc::tmem_wait_ld();
    // the row's HB values as bf16 pairs, 16-byte block e8 = w[4 e8 .. 4 e8 + 3];
    // blocks transposed across each quad of lanes (four consecutive rows), so that
    // one store instruction writes 64 contiguous bytes of each of 8 rows instead
    // of 16 bytes of each of 32
    uint32_t w[HB / 2];
#pragma unroll
    for (int q = 0; q < HB / 2; ++q) {
      const float* f = reinterpret_cast<const float*>(r);
      w[q] = frag::pack(f[2 * q], f[2 * q + 1]);
    }
    const int lq = lane & 3, iq = i - lq;  // the quad's first row
#pragma unroll
    for (int bg = 0; bg < HB / 32; ++bg)
#pragma unroll
      for (int pw = 0; pw < 4; ++pw) {
        uint32_t a[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) a[j] = w[4 * (4 * bg + j) + pw];
        frag::quad_transpose(a, lq);
#pragma unroll
        for (int j = 0; j < 4; ++j) w[4 * (4 * bg + j) + pw] = a[j];
      }
    // now w[4 (4 bg + k) .. + 3] is block 4 bg + lq of row iq + k
#pragma unroll
    for (int bg = 0; bg < HB / 32; ++bg)
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (iq + k < nvalid) {
          bf16* op = o + row_id(p, b, t0 + iq + k, h) * D + a0 + ah * HB + 8 * (4 * bg + lq);
          const int q0 = 4 * (4 * bg + k);
          *reinterpret_cast<uint4*>(op) = make_uint4(w[q0], w[q0 + 1], w[q0 + 2], w[q0 + 3]);
        }
    return true;
  };

  write_sb();
  tc::fence_before_sync();
  __syncthreads();  // barriers initialised
  tc::fence_after_sync();
  int fills[2] = {0, 0};  // bulk fills issued per stage (uniform over the CTA)
  constexpr int NTW = NTF / 32;
  static_assert(NTW == 8, "the stage fill spreads its copies over eight warps");
  const uint32_t fill_tx = scan_fill_bytes(with_o);
  if (tid == 0) {
    tc::mbar_arrive_expect_tx(&s.full[0], fill_tx);
    if (n0 + 1 < n1) tc::mbar_arrive_expect_tx(&s.full[1], fill_tx);
  }
  __syncthreads();
  scan_fill<BV>(s.st[0], &s.full[0], sv, chunk_id(p, b, h, n0), a0, with_o, with_up, warp, lane,
                &s.barO, -1);
  fills[0] = 1;
  frag::cp_wait<0>();
  bool ok = tc::mbar_wait(&s.full[0], 0u, kSpinScan);
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  ok = __syncthreads_or(ok ? 0 : 1) == 0;
  tc::fence_after_sync();
  const uint32_t tbase = s.tmem;
  const uint32_t idA = tc::idesc_bf16(128, BV, false, true);
  const uint32_t idC = tc::idesc_bf16(128, BV, true, true);
  // descriptors: per-k-step advance of the start address (in 16-byte units)
  const uint64_t dSB = tc::sdesc_mnmaj(s.SB, BV, 0), dUB = tc::sdesc_mnmaj(s.UB, BV, 0);
  constexpr uint32_t kSB = 2 * (BV / 8) * 128 / 16, kUB = kSB, kKM = 256 / 16;
  constexpr uint32_t kKT = 2 * (D / 8) * 128 / 16;
  for (int n = n0; n < n1 && ok; ++n) {
    const int it = n - n0;
    const size_t cb = chunk_id(p, b, h, n);
    ScanStage<BV>& st = s.st[it & 1];
    const int buf = it & 1;
    const float dc = st.dec[PHASE ? (c & ~1) : c];  // read before the stage is refilled below
    const float di = PHASE ? ((c & 1) ? st.dec[c] : -st.dec[c | 1]) : 0.f;
    // MMA-A: [W ; q e^gamma] S^T
    if (tid == 0) {
      const uint64_t dA = tc::sdesc_kmaj(st.AWQ, D, 0);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        tc::mma(tbase + buf * BV, dA + ks * kKM, dSB + ks * kSB, idA, ks > 0 ? 1u : 0u);
      tc::commit(&s.barA);
    }
    // while it runs: the next chunk's tiles into the other stage (consumed by the
    // previous step; it lands by the end of this one) and the previous chunk's output
    if (n + 1 < n1) {
      scan_fill<BV>(s.st[(it + 1) & 1], &s.full[(it + 1) & 1], sv, chunk_id(p, b, h, n + 1), a0,
                    with_o, with_up, warp, lane, &s.barO, it - 1);
      ++fills[(it + 1) & 1];
    } else {
      frag::cp_commit();  // empty group
    }
    bool bad = false;
    if (with_o && it > 0) bad = !store_o(n - 1, buf ^ 1, it - 1);
    // each thread waits for MMA-A itself; the barrier after epilogue 1 settles a
    // failed wait for the whole CTA
    bad = !tc::mbar_wait(&s.barA, (uint32_t)(it & 1), kSpinScan) || bad;
    tc::fence_after_sync();
    // epilogue 1: U = U' - W S^T (rows i = lanes 0 .. 63)
    uint4 usave[HB / 8];
    if ((warp & 3) < 2) {
      const int i = c;  // lanes 0 .. 63
      uint32_t r[HB];
#pragma unroll
      for (int q16 = 0; q16 < HB / 16; ++q16)
        tc::tmem_ld16_nowait(lane_addr(tbase, warp, buf * BV + ah * HB + 16 * q16), r + 16 * q16);
      tc::tmem_wait_ld();
#pragma unroll
      for (int e8 = 0; e8 < HB / 8; ++e8) {
        const int a = ah * HB + 8 * e8;
        const uint4 u8 = with_up ? *reinterpret_cast<const uint4*>(st.UP + ct_off(i, a, BV))
                                 : make_uint4(0, 0, 0, 0);
        const uint32_t* w8 = reinterpret_cast<const uint32_t*>(&u8);
        const float* f = reinterpret_cast<const float*>(r + 8 * e8);
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x = frag::unpack(w8[e]);
          pk[e] = frag::pack(x.x - f[2 * e], x.y - f[2 * e + 1]);
        }
        usave[e8] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(s.UB + tc::mnmaj_off(i, a, BV)) = usave[e8];
      }
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    ok = __syncthreads_or(bad ? 1 : 0) == 0;
    tc::fence_after_sync();
    if (!ok) break;
    // MMA-C (state increment, thread 0) and MMA-B (output, thread 32, its own
    // barrier: only the next step's output store waits for it)
    if (tid == 0) {
      const uint64_t dK = tc::sdesc_mnmaj(st.KT, D, 0);
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks)
        tc::mma(tbase + T_S, dK + ks * kKT, dUB + ks * kUB, idC, ks > 0 ? 1u : 0u);
      tc::commit(&s.barB);
    } else if (with_o && tid == 32) {
      const uint64_t dM = tc::sdesc_kmaj(st.MZ, C, 0);
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks)
        tc::mma(tbase + buf * BV, dM + ks * kKM, dUB + ks * kUB, idA, 1u);
      tc::commit(&s.barO);
    }
    // while they run: U and the chunk-start state to global memory
    if (save) {
      if ((warp & 3) < 2) {
        bf16* up = sv.U + cb * C * D;
#pragma unroll
        for (int e8 = 0; e8 < HB / 8; ++e8)
          *reinterpret_cast<uint4*>(up + ct_off(c, a0 + ah * HB + 8 * e8, D)) = usave[e8];
      }
      store_h(cb);
    }
    // each thread waits for MMA-C itself (the barrier at the end of the step
    // settles a failed wait)
    const bool badB = !tc::mbar_wait(&s.barB, (uint32_t)(it & 1), kSpinScan);
    tc::fence_after_sync();
    // this stage is consumed: the transaction count of its refill (chunk n + 2,
    // whose copies the next step issues after the barrier below)
    if (tid == 0 && n + 2 < n1) tc::mbar_arrive_expect_tx(&s.full[it & 1], fill_tx);
    // epilogue 2: S^T <- Diag(e^{gamma_C}) S^T + D_S
    {
      uint32_t r[HB];
#pragma unroll
      for (int q16 = 0; q16 < HB / 16; ++q16)
        tc::tmem_ld16_nowait(lane_addr(tbase, warp, T_S + ah * HB + 16 * q16), r + 16 * q16);
      tc::tmem_wait_ld();
      if (PHASE) {
        // own key c: Re (even c) or Im (odd c) of (dec_re + i dec_im)(x + i y)
#pragma unroll
        for (int e = 0; e < HB; ++e) {
          const float partner = __shfl_xor_sync(0xffffffffu, S[e], 1);
          S[e] = S[e] * dc + di * partner + __uint_as_float(r[e]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < HB; ++e) S[e] = S[e] * dc + __uint_as_float(r[e]);
      }
      write_sb();
    }
    // the next chunk's stage (filled at the top of this step)
    bool okF = true;
    frag::cp_wait<0>();
    if (n + 1 < n1) okF = tc::mbar_wait(&s.full[(it + 1) & 1], (uint32_t)(((it + 1) >> 1) & 1), kSpinScan);
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    ok = __syncthreads_or((okF && !badB) ? 0 : 1) == 0;
    tc::fence_after_sync();
  }
  if (ok) {
    if (with_o && !store_o(n1 - 1, (n1 - 1 - n0) & 1, n1 - 1 - n0) && err) atomicExch(err, 1);
    if (ST) {
#pragma unroll
      for (int u = 0; u < HB; ++u) ST[sbase + (size_t)(a0 + ah * HB + u) * D + c] = S[u];
    }
  } else if (tid == 0 && err) {
    atomicExch(err, 1);
  }
  // fills still in flight (only after a failed wait) land before exit
  frag::cp_wait<0>();
  if (tid == 0) {
    if (fills[0] > 0) tc::mbar_wait(&s.full[0], (uint32_t)((fills[0] - 1) & 1), kSpinScan);
    if (fills[1] > 0) tc::mbar_wait(&s.full[1], (uint32_t)((fills[1] - 1) & 1), kSpinScan);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, TALLOC);
}

template <int BV>
cudaError_t launch_fwd_scan_tc_bv(const Problem& p, const Saved& sv, const ScanSeg& sg, bf16* o,
                                  bool save, cudaStream_t st) {
  const float* S0 = sg.mode == 0 ? sg.S0 : nullptr;
  float* ST = sg.ST;
  const int maps = sg.mode == 3 ? 2 : 1;  // mode 3 runs both map kinds
  const size_t sm = sizeof(ScanSmem<BV>) + 1024;
  const bool phase = p.gate == kGatePhase;
  cudaError_t e = cudaFuncSetAttribute(phase ? k_fwd_scan_tc<BV, true> : k_fwd_scan_tc<BV, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const double nb = (double)p.B * p.H * p.NC, ntok = nb * C, heads = (double)p.B * p.H;
  // reads W, Kt, U' (not for a transfer-matrix pass), dec (+ q e^gamma, M with the
  // output); writes h, U (saving), o, and the segment start / end states
  double bytes = nb * (2.0 * kTileBytes + (sg.mode == 1 ? 0.0 : (double)kTileBytes) + kDecBytes);
  if (o) bytes += nb * ((double)kTileBytes + kMBytes) + ntok * D * 2;
  if (save) bytes += nb * ((double)kStateBytes + kUBytes);
  bytes += heads * sg.G * D * D * 4 * ((S0 ? 1 : 0) + (ST ? maps : 0));
  // operator I/O: o, and S0 / S_T when they are the operator's own (unsegmented)
  const double io = (o ? ntok * D * 2 : 0.0) +
                    (sg.G == 1 ? heads * D * D * 4.0 * ((S0 ? 1 : 0) + (ST ? 1 : 0)) : 0.0);
  const double flops =
      maps * nb * (2.0 * C * D * D * (o ? 3 : 2) + (o ? 2.0 * C * C * D : 0.0));
  prof_begin(kKTcScanFwd, io, bytes, flops, st);
  const dim3 grid(maps * (D / BV), p.H, p.B * sg.G);
  if (phase)
    k_fwd_scan_tc<BV, true><<<grid, NTF, sm, st>>>(p, sv, sg, o, save ? 1 : 0, device_error_word());
  else
    k_fwd_scan_tc<BV, false><<<grid, NTF, sm, st>>>(p, sv, sg, o, save ? 1 : 0,
                                                    device_error_word());
  e = cudaGetLastError();
  prof_end(st);
  return e;
}

// ---------------------------------------------------------------------------
// The reverse state-gradient scan on tcgen05.  Per chunk n, from the last to
// the first, with dS = dS_{n+1} (the gradient of the chunk's end state):
//   MMA-1  D_U  = M^T dO + (k e^{gamma_C - gamma}) dS^T     (M = 64, N = BV)
//   MMA-2a D_S  = (q e^gamma)^T dO                           (M = 128 keys)
//   epilogue 1   dU = D_U (bf16, saved for the chunk kernel; -dU is the operand)
//   MMA-2b D_S += W^T (-dU)
//   epilogue 2   dS_n^T = Diag(e^{gamma_C}) dS^T + D_S       (fp32, registers)
// dh_n = dS_{n+1} is written out (bf16) while MMA-1 runs.  Each CTA owns the
// value columns a0 .. a0 + BV of dS; the state gradient is held transposed,
// one key per TMEM lane.  The dS-free half of MMA-1 (M^T dO) of the next chunk
// is issued under epilogue 2 into the other D_U buffer, so a step's critical
// path holds only the dS-dependent products.  The chunk tiles arrive by bulk
// copies (one thread, the stage's mbarrier); the dO slice by cp.async.
template <int BV>
struct BScanStage {
  bf16 QH[C * D];     // q e^gamma, core-tiled [j][c]: MN-major A (M = key c, K = j)
  bf16 KT[C * D];     // k e^{gamma_C - gamma}, core-tiled [i][c]: K-major A (M = i, K = c)
  bf16 W[C * D];      // W, core-tiled [i][c]: MN-major A (M = key c, K = i)
  bf16 M[C * C];      // M, core-tiled [j][i]: MN-major A of M^T (M = i, K = j)
  bf16 DO[C * BV];    // dO[:, a0 .. a0 + BV), core-tiled [j][a]: MN-major B
  float dec[D];
};
template <int BV>
struct BScanSmem {
  BScanStage<BV> st[2];
  bf16 DSB[D * BV];   // bf16 dS^T, core-tiled [c][a]: MN-major B of MMA-1
  bf16 DUB[C * BV];   // bf16 -dU, core-tiled [i][a]: MN-major B of MMA-2b
  uint64_t barA, barB, full[2];
  uint32_t tmem;
};

// Fills a stage: the core-tiled chunk tiles by bulk copies from thread 0
// (completing on `full`), the dO slice by cp.async from every thread (the
// caller commits the group).
template <int BV>
__device__ __forceinline__ void bscan_fill(const Problem& p, BScanStage<BV>& s, uint64_t* full,
                                           const Saved& sv, const bf16* __restrict__ dO, int b,
                                           int h, int n, int a0) {
  const int tid = threadIdx.x;
  const size_t cb = chunk_id(p, b, h, n);
  const int t0 = n * C, nvalid = min(C, p.T - t0);
  if (tid == 0) {
    constexpr uint32_t kT = C * D * 2, kM = C * C * 2, kDec = D * 4;
    tc::mbar_arrive_expect_tx(full, 3 * kT + kM + kDec);
    tc::bulk_g2s(s.QH, sv.Qh + cb * C * D, kT, full);
    tc::bulk_g2s(s.KT, sv.Kt + cb * C * D, kT, full);
    tc::bulk_g2s(s.W, sv.W + cb * C * D, kT, full);
    tc::bulk_g2s(s.M, sv.M + cb * C * C, kM, full);
    tc::bulk_g2s(s.dec, sv.dec + cb * D, kDec, full);
  }
  for (int idx = tid; idx < C * BV / 8; idx += NTF) {
    const int j = ct_row(idx, BV), col = ct_col(idx, BV);
    const bool ok = j < nvalid;
    frag::cp16(s.DO + 8 * idx, dO + row_id(p, b, t0 + (ok ? j : 0), h) * D + a0 + col, ok);
  }
}

// PHASE: the SFDA rotation-decay gate.  The forward decay multiplies each
// state row's key pair by dec = dec[2j] + i dec[2j+1] (the conjugate of the
// chunk's cumulative complex decay), so the gradient goes back through the
// adjoint, multiplication by conj(dec); the pair's keys sit on adjacent lanes.
template <int BV, bool PHASE>
__global__ void __launch_bounds__(NTF, 1)
    k_bwd_scan_tc(Problem p, Saved sv, const bf16* __restrict__ dO, ScanSeg sg,
                  bf16* __restrict__ dUout, bf16* __restrict__ dhout, int* __restrict__ err) {
  constexpr int HB = BV / 2;
  constexpr int TALLOC = 3 * BV <= 256 ? 256 : 512;  // D_U x 2, D_S
  extern __shared__ __align__(1024) unsigned char smraw[];
  BScanSmem<BV>& s = *reinterpret_cast<BScanSmem<BV>*>(smraw);
  const int h = blockIdx.y, b = blockIdx.z / sg.G, seg = blockIdx.z % sg.G, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int a0 = blockIdx.x * BV;
  const int n0 = seg * sg.L, n1 = min(p.NC, n0 + sg.L);
  if (n0 >= n1) return;
  const bool outputs = sg.mode == 0;
  const float* __restrict__ dST = outputs ? sg.S0 : nullptr;
  float* __restrict__ dS0 = sg.ST;
  const size_t sbase = (((size_t)b * sg.G + seg) * p.H + h) * D * D;
  const int c = 32 * (warp & 3) + lane, ah = warp >> 2;  // key (TMEM lane), value half
  const uint32_t T_S = 2 * BV;  // D_U buffers at columns 0 and BV

  if (warp == 0) tc::tmem_alloc(&s.tmem, TALLOC);
  if (tid == 0) {
    tc::mbar_init(&s.barA, 1);
    tc::mbar_init(&s.barB, 1);
    tc::mbar_init(&s.full[0], 1);
    tc::mbar_init(&s.full[1], 1);
    tc::fence_mbar_init();
  }
  float dS[HB];  // dS^T[c][a0 + ah*HB + u]
#pragma unroll
  for (int u = 0; u < HB; ++u)
    dS[u] = dST ? dST[sbase + (size_t)(a0 + ah * HB + u) * D + c] : 0.f;
  auto write_dsb = [&]() {
#pragma unroll
    for (int u8 = 0; u8 < HB / 8; ++u8) {
      const float* f = dS + 8 * u8;
      *reinterpret_cast<uint4*>(s.DSB + tc::mnmaj_off(c, ah * HB + 8 * u8, BV)) =
          make_uint4(frag::pack(f[0], f[1]), frag::pack(f[2], f[3]), frag::pack(f[4], f[5]),
                     frag::pack(f[6], f[7]));
    }
  };
  // dh (bf16, core-tiled [c][a]) from the registers
  auto store_dh = [&](size_t cbn) {
    store_state_ct<HB>(dhout + cbn * D * D, dS, a0 + ah * HB, c);
  };

  write_dsb();
  tc::fence_before_sync();
  __syncthreads();  // barriers initialised
  tc::fence_after_sync();
  bscan_fill<BV>(p, s.st[0], &s.full[0], sv, dO, b, h, n1 - 1, a0);
  frag::cp_commit();
  if (n1 - 2 >= n0) bscan_fill<BV>(p, s.st[1], &s.full[1], sv, dO, b, h, n1 - 2, a0);
  frag::cp_commit();
  int fills0 = 1, fills1 = n1 - 2 >= n0 ? 1 : 0;  // bulk fills issued per stage (uniform)
  frag::cp_wait<1>();
  bool ok = tc::mbar_wait(&s.full[0], 0u, kSpinScan);
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  ok = __syncthreads_or(ok ? 0 : 1) == 0;
  tc::fence_after_sync();
  const uint32_t tbase = s.tmem;

  const uint32_t id1a = tc::idesc_bf16(64, BV, true, true);    // M^T dO
  const uint32_t id1b = tc::idesc_bf16(64, BV, false, true);   // Kt dS^T
  const uint32_t id2 = tc::idesc_bf16(128, BV, true, true);    // Qh^T dO, W^T (-dU)
  const uint64_t dDSB = tc::sdesc_mnmaj(s.DSB, BV, 0), dDUB = tc::sdesc_mnmaj(s.DUB, BV, 0);
  constexpr uint32_t kB = 2 * (BV / 8) * 128 / 16;   // MN-major B k-step (16-byte units)
  constexpr uint32_t kA64 = 2 * (C / 8) * 128 / 16;  // MN-major A k-step, 64 wide
  constexpr uint32_t kA128 = 2 * (D / 8) * 128 / 16; // MN-major A k-step, 128 wide
  constexpr uint32_t kK = 256 / 16;                  // K-major k-step
  // epilogue-1 ownership (M = 64 accumulator layout): row i = 16 (warp % 4) + lane, lane < 16
  const int ri = 16 * (warp & 3) + (lane & 15);
  // M^T dO of the chunk in stage `sg` into D_U buffer `ub` (overwrites it)
  auto issue_mtdo = [&](int sg, int ub) {
    const uint64_t dM = tc::sdesc_mnmaj(s.st[sg].M, C, 0), dDO = tc::sdesc_mnmaj(s.st[sg].DO, BV, 0);
#pragma unroll
    for (int ks = 0; ks < C / 16; ++ks)
      tc::mma(tbase + ub * BV, dM + ks * kA64, dDO + ks * kB, id1a, ks > 0 ? 1u : 0u);
  };
  if (ok && tid == 0) issue_mtdo(0, 0);
  for (int it = 0; it < n1 - n0 && ok; ++it) {
    const int n = n1 - 1 - it;
    const size_t cb = chunk_id(p, b, h, n);
    BScanStage<BV>& st = s.st[it & 1];
    const uint32_t T_U = (uint32_t)((it & 1) * BV);
    const float dc = st.dec[PHASE ? (c & ~1) : c];  // read before the stage is refilled below
    const float di = PHASE ? ((c & 1) ? -st.dec[c] : st.dec[c | 1]) : 0.f;
    if (tid == 0) {
      const uint64_t dKT = tc::sdesc_kmaj(st.KT, D, 0), dQH = tc::sdesc_mnmaj(st.QH, D, 0);
      const uint64_t dDO = tc::sdesc_mnmaj(st.DO, BV, 0);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        tc::mma(tbase + T_U, dKT + ks * kK, dDSB + ks * kB, id1b, 1u);
      tc::commit(&s.barA);  // dU is complete; the dU-free half of D_S runs under epilogue 1
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks)
        tc::mma(tbase + T_S, dQH + ks * kA128, dDO + ks * kB, id2, ks > 0 ? 1u : 0u);
    }
    if (outputs) store_dh(cb);
    // each thread waits for MMA-1 itself; the barrier after epilogue 1 settles a
    // failed wait for the whole CTA
    const bool badA = !tc::mbar_wait(&s.barA, (uint32_t)(it & 1), kSpinScan);
    tc::fence_after_sync();
    // epilogue 1: dU rows ri, value columns ah*HB ..
    uint4 dusave[HB / 8];
    {
      uint32_t r[HB];
#pragma unroll
      for (int q16 = 0; q16 < HB / 16; ++q16)
        tc::tmem_ld16_nowait(lane_addr(tbase, warp, T_U + ah * HB + 16 * q16), r + 16 * q16);
      tc::tmem_wait_ld();
#pragma unroll
      for (int e8 = 0; e8 < HB / 8; ++e8) {
        const float* f = reinterpret_cast<const float*>(r + 8 * e8);
        dusave[e8] = make_uint4(frag::pack(f[0], f[1]), frag::pack(f[2], f[3]),
                                frag::pack(f[4], f[5]), frag::pack(f[6], f[7]));
        if (lane < 16)
          *reinterpret_cast<uint4*>(s.DUB + tc::mnmaj_off(ri, ah * HB + 8 * e8, BV)) =
              make_uint4(frag::pack(-f[0], -f[1]), frag::pack(-f[2], -f[3]),
                         frag::pack(-f[4], -f[5]), frag::pack(-f[6], -f[7]));
      }
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    ok = __syncthreads_or(badA ? 1 : 0) == 0;
    tc::fence_after_sync();
    if (!ok) break;
    if (tid == 0) {
      const uint64_t dW = tc::sdesc_mnmaj(st.W, D, 0);
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks)
        tc::mma(tbase + T_S, dW + ks * kA128, dDUB + ks * kB, id2, 1u);
      tc::commit(&s.barB);
    }
    if (outputs && lane < 16) {
      bf16* up = dUout + cb * C * D;
#pragma unroll
      for (int e8 = 0; e8 < HB / 8; ++e8)
        *reinterpret_cast<uint4*>(up + ct_off(ri, a0 + ah * HB + 8 * e8, D)) = dusave[e8];
    }
    // the next chunk's stage (filled one step ago) must be complete before the
    // barrier below, so that its M^T dO can be issued under epilogue 2
    bool okF = true;
    if (n - 1 >= n0) {
      frag::cp_wait<0>();
      okF = tc::mbar_wait(&s.full[(it + 1) & 1], (uint32_t)(((it + 1) >> 1) & 1), kSpinScan);
      tc::fence_smem_to_async();
    }
    {
      const bool okB = tc::mbar_wait(&s.barB, (uint32_t)(it & 1), kSpinScan);
      ok = __syncthreads_or((okB && okF) ? 0 : 1) == 0;
      tc::fence_after_sync();
    }
    if (!ok) break;
    if (tid == 0 && n - 1 >= n0) issue_mtdo((it + 1) & 1, (it + 1) & 1);
    // every read of this stage is done: refill it with chunk n - 2
    if (n - 2 >= n0) {
      bscan_fill<BV>(p, st, &s.full[it & 1], sv, dO, b, h, n - 2, a0);
      ++((it & 1) ? fills1 : fills0);
    }
    frag::cp_commit();
    // epilogue 2: dS^T <- Diag(e^{gamma_C}) dS^T + D_S
    {
      uint32_t r[HB];
#pragma unroll
      for (int q16 = 0; q16 < HB / 16; ++q16)
        tc::tmem_ld16_nowait(lane_addr(tbase, warp, T_S + ah * HB + 16 * q16), r + 16 * q16);
      tc::tmem_wait_ld();
      if (PHASE) {
        // own key c: Re (even c) or Im (odd c) of conj(dec_re + i dec_im) (x + i y)
#pragma unroll
        for (int e = 0; e < HB; ++e) {
          const float partner = __shfl_xor_sync(0xffffffffu, dS[e], 1);
          dS[e] = dS[e] * dc + di * partner + __uint_as_float(r[e]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < HB; ++e) dS[e] = dS[e] * dc + __uint_as_float(r[e]);
      }
      write_dsb();
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
  }
  if (ok) {
    if (dS0) {
#pragma unroll
      for (int u = 0; u < HB; ++u) dS0[sbase + (size_t)(a0 + ah * HB + u) * D + c] = dS[u];
    }
  } else if (tid == 0 && err) {
    atomicExch(err, 1);
  }
  // copies still in flight (only after a failed wait) land before exit
  frag::cp_wait<0>();
  if (tid == 0) {
    if (fills0 > 0) tc::mbar_wait(&s.full[0], (uint32_t)((fills0 - 1) & 1), kSpinScan);
    if (fills1 > 0) tc::mbar_wait(&s.full[1], (uint32_t)((fills1 - 1) & 1), kSpinScan);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, TALLOC);
}

template <int BV>
cudaError_t launch_bwd_scan_tc_bv(const Problem& p, const Saved& sv, const bf16* dO,
                                  const ScanSeg& sg, bf16* dU, bf16* dh, cudaStream_t st) {
  const float* dST = sg.mode == 0 ? sg.S0 : nullptr;
  float* dS0 = sg.ST;
  const size_t sm = sizeof(BScanSmem<BV>) + 1024;
  auto kern = p.gate == kGatePhase ? k_bwd_scan_tc<BV, true> : k_bwd_scan_tc<BV, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const double nb = (double)p.B * p.H * p.NC, ntok = nb * C, heads = (double)p.B * p.H;
  // reads W, Qh, Kt, M, dec, dO; writes dU, dh (output pass) and the segment
  // end / start gradients
  const double bytes = nb * (3.0 * kTileBytes + kMBytes + kDecBytes) + ntok * D * 2 +
                       (sg.mode == 0 ? nb * ((double)kUBytes + kStateBytes) : 0.0) +
                       heads * sg.G * D * D * 4 * ((dST ? 1 : 0) + (dS0 ? 1 : 0));
  // operator I/O: dO, and dS_T / dS0 when they are the operator's own (unsegmented)
  const double io = ntok * D * 2 +
                    (sg.G == 1 ? heads * D * D * 4.0 * ((dST ? 1 : 0) + (dS0 ? 1 : 0)) : 0.0);
  const double flops = nb * (2.0 * C * C * D + 2.0 * C * D * D * 3);
  prof_begin(kKTcScanBwd, io, bytes, flops, st);
  kern<<<dim3(D / BV, p.H, p.B * sg.G), NTF, sm, st>>>(p, sv, dO, sg, dU, dh,
                                                       device_error_word());
  e = cudaGetLastError();
  prof_end(st);
  return e;
}

}  // namespace

cudaError_t launch_fwd_scan_tc(const Problem& p, const Saved& sv, const float* S0, bf16* o,
                               float* ST, bool save, cudaStream_t st) {
  // One CTA per (b, h, value tile): 64-row tiles while two per head still fit one wave
  // of the 148 SMs, whole-state tiles otherwise.
  const ScanSeg sg{1, p.NC, 0, S0, ST, nullptr};
  if ((long)p.B * p.H * 2 <= 148) return launch_fwd_scan_tc_bv<64>(p, sv, sg, o, save, st);
  return launch_fwd_scan_tc_bv<128>(p, sv, sg, o, save, st);
}

cudaError_t launch_fwd_scan_tc_seg(const Problem& p, const Saved& sv, const ScanSeg& sg, bf16* o,
                                   bool save, int bv, cudaStream_t st) {
  return bv == 64 ? launch_fwd_scan_tc_bv<64>(p, sv, sg, o, save, st)
                  : launch_fwd_scan_tc_bv<128>(p, sv, sg, o, save, st);
}

cudaError_t launch_bwd_scan_tc(const Problem& p, const Saved& sv, const bf16* dO,
                               const float* dST, float* dS0, bf16* dU, bf16* dh,
                               cudaStream_t st) {
  const ScanSeg sg{1, p.NC, 0, dST, dS0, nullptr};
  if ((long)p.B * p.H * 2 <= 148) return launch_bwd_scan_tc_bv<64>(p, sv, dO, sg, dU, dh, st);
  return launch_bwd_scan_tc_bv<128>(p, sv, dO, sg, dU, dh, st);
}

cudaError_t launch_bwd_scan_tc_seg(const Problem& p, const Saved& sv, const bf16* dO,
                                   const ScanSeg& sg, bf16* dU, bf16* dh, int bv,
                                   cudaStream_t st) {
  return bv == 64 ? launch_bwd_scan_tc_bv<64>(p, sv, dO, sg, dU, dh, st)
                  : launch_bwd_scan_tc_bv<128>(p, sv, dO, sg, dU, dh, st);
}

}  // namespace fast
}  // namespace dr
