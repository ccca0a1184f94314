// fast_bwd_hy.cu -- chunk-parallel backward with the products on tcgen05 and
// the element-wise work on all 16 warps (bf16 storage, d_k = d_v = 128, C = 64).
//
// Persistent, one CTA per SM, looping over the (b, h, chunk) tiles.  From the
// chunk's saved tiles (T, W, U', the chunk-start state S = h_n, the
// pseudo-values U) and the state-gradient scan's dU and dS' (the gradient of
// the chunk's end state):
//   level 1  dQs = dO S, dW = -dU S, dKt = U dS', dM = tril(dO U^T)  (its diagonal
//            kept apart in fp32: it enters dq and dk with the factor 1 and cancels in dg)
//   level 2  Lambda = T^T [dU | dW]             (dv = diag(beta) Lambda_U)
//   level 3  dA = -strict_tril(Lambda_U U'^T + Lambda_W W^T)
//   level 4  the gate-scaled products of dM and dA with the keys and queries:
//            F1_i = sum_{j<=i} dM_ij k_j e^{g_i - g_j},  F2_i = sum_{j<i} dA_ij k_j e^{g_i - g_j},
//            G_j  = sum_{i>=j} (dM_ij q_i + dA_ij beta_i k_i) e^{g_i - g_j}
//            (g: the within-chunk cumulative log-gate of each key channel)
// which give dq, dk, dgamma and dbeta in a register epilogue, then the gate's
// reverse cumulative sum (in registers) and the Kaczmarz chain rule.  The chunk correction is
// differentiated as the triangular residual system (I + A)[U' | W] = diag(beta)
// [V | k e^g] (ReWY abstract): one transposed triangular product (level 2), no
// adjoint of the inverse.
//
// Reference rows.  The gate factors of level 4 are exponentials of differences
// of cumulative gates.  Every row i uses the reference row rho of its own
// 32-row half (rows 15 and 47), e^{g_i - g_j} = e^{g_i - g_rho} e^{g_rho - g_j}:
// the first factor spans at most 16 rows of decay, and the second does too for
// j in the same half, while for j in the earlier half it is at most 1 (an
// underflow there drops a term that is negligible against the kept ones).  So
// no factor overflows unless the gates decay by more than about 5.5 nats per
// token over 16 consecutive tokens ("centered matrix contractions", ReWY
// abstract).  A factor that crosses halves is applied in two steps through the
// half boundary, each at most 1 in size, so it underflows only where the
// exact product would.  Products whose reference differs between output rows are split:
// F1 and F2 read dM and dA through row-masked copies (rows of the other half
// zero) against per-half key tiles, accumulating into one tensor-memory tile;
// G (whose output rows are the keys) has one accumulator per half.
//
// PHASE: the SFDA rotation-decay gate ("Semidirect Fourier Delta Attention"
// explainer, Kernarchitektur).  Key channels pair up as complex numbers, the
// chunk's cumulative decay of a pair is zeta_i = e^{g_i - i Theta_i} (g, Theta:
// the cumulative sums at the pair's even and odd channels), and every real
// factor above becomes a per-pair complex one: u_i = zeta_i / zeta_rho scales
// queries and read keys, 1 / conj(u_i) the write keys.  Gradients map back by
// the conjugate factors, d/dg of a pair is Re(.) and d/dTheta is Im(.) of the
// same products (with the write-key and chunk-end terms of opposite sign in g).
//
// Overlap: the level-1 tiles of the CTA's next chunk (dO, dU, U, S, dS', T;
// 120 KB) are loaded while the epilogue of this one runs, into the tiles that
// level 4 has released, so a chunk starts with its first products; q, k, v and
// the gate (which the epilogue still reads) load, and the gate's cumulative sum
// runs, on warps 1..15 while warp 0 issues level 1; for real gates warps 1..4
// form the state tiles' column sums while those copies land.  Likewise the tile builds
// under levels 3 and 4 leave warp 0 to its MMA issue.
//
// Each level is a set of tcgen05.mma (M = 64, operands in shared memory in the
// canonical core-matrix layout, fp32 accumulators in tensor memory) issued by
// one thread (thread 0).  An M = 64 accumulator occupies lanes 16 q .. 16 q + 15 of each
// 32-lane quadrant q, and tcgen05.ld.16x256b returns it to the warps of that
// quadrant in the register fragment of a warp-level m16n8 product (thread t:
// row t / 4 and t / 4 + 8, columns 2 (t % 4), + 1 of each 8-column group), so
// warp w = 4 qt + rb owns rows 16 rb .., columns 32 qt ..; a thread's two
// columns are one key pair.

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
constexpr uint32_t kSpinHy = 1u << 22;
// Polls of the injected wait (dr_inject_timeout): short, so the test that
// drives the timeout path ends within milliseconds.
constexpr uint32_t kSpinInjected = 256;
constexpr int kRho0 = 15, kRho1 = 47;  // reference rows of the two halves
// rows of HySmem::grow
constexpr int kGR0 = 0, kGR1 = 1, kG31 = 2, kG32 = 3, kGC = 4;
__device__ __forceinline__ int grow_slot(int i) {
  return i == kRho0 ? kGR0 : i == kRho1 ? kGR1 : i == 31 ? kG31 : i == 32 ? kG32 : i == 63 ? kGC : -1;
}

// Gate tile element (i, c): 8-column groups XOR-swizzled by row.
__device__ __forceinline__ int gsw(int i, int c) { return i * D + (c ^ ((i & 7) << 3)); }
// v tile element (i, a) (bf16): 16-byte chunks XOR-swizzled by row, so that the
// fragment reads (8 rows, 4 consecutive pairs) hit distinct banks.
__device__ __forceinline__ int vsw(int i, int a) { return i * D + (a ^ ((i & 7) << 3)); }

// Tensor memory columns (512 allocated): each level reuses the columns whose
// accumulators the previous levels have read back.
constexpr uint32_t T_ZQ = 0, T_ADW = 128, T_AKT = 256, T_ADM = 384;  // level 1
constexpr uint32_t T_LU = 0, T_LW = 128;                             // level 2
constexpr uint32_t T_DA = 256;  // level 3: four 64-column partial sums of dA
constexpr uint32_t T_F1 = 0, T_G0 = 128, T_F2 = 256, T_G1 = 384;     // level 4

// Row-masked copy of a 64 x 64 matrix for level 4 ("X tile"): core-tiled
// K-major (8 x 8 blocks of 128 bytes, rows of blocks 1 KB apart), rows 0..31
// at bytes [0, 4K), zeros at [4K, 8K), rows 32..63 at [8K, 12K).  Read from
// byte 0 it is the matrix with rows 32..63 zeroed, from byte 4K the matrix with
// rows 0..31 zeroed; read by k-steps of 16 rows that skip the zero block, its
// transpose.
constexpr int kXElems = 3 * C * C / 2;  // 12 KB

struct HySmem {
  bf16 SS[D * D];   // S = h_n stored [c][a] (level 1);  Lambda_U | Lambda_W (levels 2-3);
                    // beta k^{rho0} (level 4);  at the end the fp32 dgamma tile (with SD)
  bf16 SD[D * D];   // dS' stored [c][a];  then W | U' (level 3)
  bf16 DO[C * D];   // dO [i][a] (K-major A);  then dW [j][c] (level 2);  then Kb^{rho1} (level 4)
  bf16 DU[C * D];   // dU [j][a];  then q^{rho0} (level 4)
  bf16 UU[2 * kXElems];  // U [j][a] (level 1, first 16 KB);  then the X tiles of dM and dA
  bf16 QC[C * D];   // v (rows of 16-byte chunks XOR-swizzled by row, for dv and dbeta);
                    // then Kb^{rho0} rows 0..31 | q^{rho1} rows 32..63 (level 4)
  bf16 QR[C * LDD]; // raw q, row-major padded
  bf16 k[C * LDD];  // raw k, row-major padded
  bf16 TT[C * C];   // T [i][j], core-tiled (MN-major A of T^T);  then beta k^{rho1} rows 32..63
  float G[C * D];   // cumulative gate (gsw), then the factor u_i of each element
  alignas(16) float beta[C];
  alignas(16) float knorm[C];
  float dbp[C * 4];
  alignas(16) float dgc[4 * D];  // colsum(conj(dS') S) (real gates: the first D; phase gate:
                                 // four slots per key) and the gate scan's scratch
  float ktk[4 * D];
  float er[2 * D];   // per half: conj(zeta_rho)                (real gates: e^{g_rho})
  float erc[2 * D];  // per half: zeta_C / zeta_rho             (real gates: e^{g_C - g_rho})
  // cross-half factors, each spanning at most 17 rows: write keys of the first
  // half against the second reference, conj(zeta_31 / zeta_rho0) conj(zeta_rho1 / zeta_31),
  // and queries / keys of the second half against the first reference,
  // (zeta_rho1 / zeta_32) (zeta_32 / zeta_rho0); applied one after the other, so
  // that no intermediate underflows where the product does not
  alignas(16) float xk[2 * D];
  alignas(16) float xq[2 * D];
  float dmd[C];      // the diagonal of dM (fp32), added outside the level-4 products
  float blk[4 * D];  // dgamma totals of each 16-row block (scalar gate: row partial sums)
  // the cumulative gate at rows 15, 47 (the references), 31, 32 and 63, kept apart
  // from the gate tile (which the factor pass overwrites in place); a scalar gate
  // uses column 0
  alignas(16) float grow[5][D];
  uint64_t bar;
  uint64_t full;    // the chunk tiles' bulk copies
  uint64_t never;   // fault injection: a barrier that nothing ever arrives on
  uint32_t tmem;
};

static_assert(sizeof(bf16) * C * D <= sizeof(bf16) * 2 * kXElems, "U fits the X-tile region");
static_assert(offsetof(HySmem, ktk) == offsetof(HySmem, dgc) + sizeof(float) * 4 * D,
              "the gate scan's segment totals span the adjacent dgc and ktk tiles");

// --- complex helpers (a key pair as x + i y) -------------------------------
struct cf {
  float x, y;
};
__device__ __forceinline__ cf cmul(cf a, cf b) { return {a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x}; }
// conj(a) b
__device__ __forceinline__ cf cmulc(cf a, cf b) { return {a.x * b.x + a.y * b.y, a.x * b.y - a.y * b.x}; }
__device__ __forceinline__ cf cconj(cf a) { return {a.x, -a.y}; }
// 1 / u, scaled so that |u|^2 is never formed (|u| up to e^{+-80} stays finite)
__device__ __forceinline__ cf cinv(cf u) {
  const float s = __fdividef(1.f, fmaxf(fabsf(u.x), fabsf(u.y)));
  const float a = u.x * s, b = u.y * s;
  const float t = __fdividef(s, a * a + b * b);
  return {a * t, -b * t};
}

// Barrier among `count` threads (whole warps) on hardware barrier `id` (1..15;
// barrier 0 is __syncthreads).
__device__ __forceinline__ void named_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void mma_step(uint32_t tm, uint64_t a, uint64_t b, uint32_t id,
                                         uint32_t acc) {
  tc::mma(tm, a, b, id, acc);
}

// The raw registers of frag_ld4 / frag_ld2 (below) without the wait: several
// loads are issued back to back, then one tc::tmem_wait_ld(), then frag_of.
__device__ __forceinline__ void frag_ld4_raw(uint32_t col, int warp, uint32_t (&r)[16]) {
  const uint32_t ta = col + ((uint32_t)(32 * (warp & 3)) << 16);
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(ta));
}
__device__ __forceinline__ void frag_ld2_raw(uint32_t col, int warp, uint32_t (&r)[8]) {
  const uint32_t ta = col + ((uint32_t)(32 * (warp & 3)) << 16);
  asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(ta));
}
template <int NT>
__device__ __forceinline__ void frag_of(const uint32_t (&r)[4 * NT], float (&f)[NT][4]) {
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) f[j][e] = __uint_as_float(r[4 * j + e]);
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
__device__ __forceinline__ bool hy_wait(uint64_t* bar, int phase, uint32_t limit = kSpinHy) {
  const bool ok = tc::mbar_wait(bar, (uint32_t)(phase & 1), limit);
  const int bad = __syncthreads_or(ok ? 0 : 1);
  tc::fence_after_sync();
  return bad == 0;
}

// Bounded wait for the commit of level `phase` by this thread alone (no
// barrier): a failure is carried to the next barrier the chunk needs anyway.
__device__ __forceinline__ bool hy_wait_local(uint64_t* bar, int phase) {
  const bool ok = tc::mbar_wait(bar, (uint32_t)(phase & 1), kSpinHy);
  tc::fence_after_sync();
  return ok;
}

// The wait for a level's MMAs.  Real gates: each thread alone (hy_wait_local),
// a failure settled at the next barrier the chunk needs.  The phase gate, whose
// per-element work is heavier, runs faster with the CTA held at a barrier after
// each level (hy_wait; measured on the SFDA workload: 1195 against 1090 us).
template <bool PHASE>
__device__ __forceinline__ bool level_wait_t(uint64_t* bar, int phase) {
  return PHASE ? hy_wait(bar, phase) : hy_wait_local(bar, phase);
}

// Descriptors: K-major [rows][K = 64] tiles (X tiles, row groups 1 KB apart),
// MN-major [K][N = 128] tiles (the level-4 key and query tiles), MN-major
// [K][M = 64] (an X tile read as its transpose).
__device__ __forceinline__ uint64_t dk64(const bf16* t, uint32_t byte_off) {
  return tc::sdesc(tc::smem_u32(t) + byte_off, 128, 1024);
}
__device__ __forceinline__ uint64_t dmn128(const bf16* t, uint32_t byte_off) {
  return tc::sdesc(tc::smem_u32(t) + byte_off, 2048, 128);
}
__device__ __forceinline__ uint64_t dmn64(const bf16* t, uint32_t byte_off) {
  return tc::sdesc(tc::smem_u32(t) + byte_off, 1024, 128);
}
// Byte offset of k-step ks (rows 16 ks .. 16 ks + 15) of an X tile's transpose.
__device__ __forceinline__ uint32_t xt_off(int ks) {
  return ks < 2 ? ks * 2048u : 8192u + (ks - 2) * 2048u;
}

template <bool PHASE>
__global__ void __launch_bounds__(NTB, 1)
    k_bwd_chunk_hy(Problem p, const bf16* __restrict__ q, const bf16* __restrict__ k,
                   const bf16* __restrict__ v, const bf16* __restrict__ dO,
                   const float* __restrict__ g, const bf16* __restrict__ Tg,
                   const float* __restrict__ beta, const bf16* __restrict__ hst,
                   const bf16* __restrict__ dhst, const bf16* __restrict__ Ug,
                   const bf16* __restrict__ dUg, const bf16* __restrict__ Wg,
                   const bf16* __restrict__ Upg, const float* __restrict__ knorm_g,
                   bf16* __restrict__ dq, bf16* __restrict__ dk, bf16* __restrict__ dv,
                   float* __restrict__ dbeta, float* __restrict__ dg, int* __restrict__ err,
                   int inject_timeout) {
  extern __shared__ __align__(1024) unsigned char smraw[];
  HySmem& s = *reinterpret_cast<HySmem*>(smraw);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, gk = p.gk;
  auto level_wait = [](uint64_t* bar, int phase) { return level_wait_t<PHASE>(bar, phase); };
  const int rb = warp & 3, qt = warp >> 2;
  const int hf = rb >> 1;  // the half of this warp's fragment rows
  const int lr = lane >> 2, lc = 2 * (lane & 3);
  bf16* const sLU = s.SS;          // Lambda_U, after the first level
  bf16* const sLW = s.SS + C * D;  // Lambda_W
  bf16* const sW = s.SD;           // W, U' for the third level
  bf16* const sUp = s.SD + C * D;
  bf16* const sdW = s.DO;          // dW, after the first level
  bf16* const XM = s.UU;           // X tile of dM
  bf16* const XA = s.UU + kXElems; // X tile of dA
  // level-4 key and query tiles (MN-major [K][N = 128], core-tiled [rows][128])
  bf16* const Kb1 = s.DO;              // k_j / conj(zeta_j / zeta_rho1), rows 0..63
  bf16* const Q0 = s.DU;               // (zeta_i / zeta_rho0) q_i, rows 0..63
  bf16* const Kb0 = s.QC;              // k_j / conj(zeta_j / zeta_rho0), rows 0..31
  bf16* const Q1 = s.QC + 32 * D;      // (zeta_i / zeta_rho1) q_i, rows 32..63
  bf16* const B0 = s.SS;               // beta_i (zeta_i / zeta_rho0) k_i, rows 0..63
  bf16* const B1 = s.TT;               // beta_i (zeta_i / zeta_rho1) k_i, rows 32..63

  // The level-1 tiles of chunk L (launch order: chunks, then heads, then
  // batches): dU, U, S, dS' and T by bulk copies, one from lane 0 of each of
  // warps 1..5, completing on `full` (whose transaction count thread 0 has set
  // before the barrier that precedes them: expect_tiles), and dO by cp.async from
  // every thread (one group).  Issued one chunk ahead, into the tiles level 4
  // has released.
  constexpr uint32_t kTileTx = sizeof(bf16) * (2 * C * D + 2 * D * D + C * C);
  auto issue_tiles = [&](int n, int h, int b) {
    const int t0 = n * C, nvalid = min(C, p.T - t0);
    const size_t cb = chunk_id(p, b, h, n);
    if (lane == 0 && warp >= 1 && warp <= 5) {
      if (warp == 1) tc::bulk_g2s(s.DU, dUg + cb * C * D, sizeof(bf16) * C * D, &s.full);
      if (warp == 2) tc::bulk_g2s(s.UU, Ug + cb * C * D, sizeof(bf16) * C * D, &s.full);
      if (warp == 3) tc::bulk_g2s(s.SS, hst + cb * D * D, sizeof(bf16) * D * D, &s.full);
      if (warp == 4) tc::bulk_g2s(s.SD, dhst + cb * D * D, sizeof(bf16) * D * D, &s.full);
      if (warp == 5) tc::bulk_g2s(s.TT, Tg + cb * C * C, sizeof(bf16) * C * C, &s.full);
    }
    tc::cp_core_tile<NTB>(s.DO, dO + row_id(p, b, t0, h) * D, (size_t)p.H * D, C, D, nvalid, tid);
    frag::cp_commit();
  };

  if (warp == 0) tc::tmem_alloc(&s.tmem, 512);
  if (tid == 0) {
    tc::mbar_init(&s.bar, 1);
    tc::mbar_init(&s.never, 1);
    tc::mbar_init(&s.full, 1);
    tc::fence_mbar_init();
  }
  // the zero block of the dA tile (outside the U region; nothing overwrites it)
  for (int idx = tid; idx < C * C / 16; idx += NTB)
    *reinterpret_cast<uint4*>(XA + C * C / 2 + 8 * idx) = make_uint4(0, 0, 0, 0);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tb = s.tmem;
  bool ok = true, pending = false;
  uint32_t fph = 0;  // phase of `full`
  // this CTA's chunks: (n, h, b) from blockIdx.x, then every gridDim.x-th in
  // launch order (advanced without divisions)
  int n = blockIdx.x % p.NC, h = (blockIdx.x / p.NC) % p.H, b = blockIdx.x / (p.NC * p.H);
  auto advance = [&](int& an, int& ah, int& ab) {
    an += gridDim.x;
    while (an >= p.NC) {
      an -= p.NC;
      if (++ah == p.H) {
        ah = 0;
        ++ab;
      }
    }
  };
  int nn = n, nh = h, nb = b;  // the chunk after this one
  advance(nn, nh, nb);
  if (b < p.B) {
    if (tid == 0) tc::mbar_arrive_expect_tx(&s.full, kTileTx);
    __syncthreads();
    issue_tiles(n, h, b);
    pending = true;
  }
  // Persistent: one CTA per SM.  A bounded wait that gives up leaves the loop (break).
  for (bool first = true; b < p.B; n = nn, h = nh, b = nb, advance(nn, nh, nb), first = false) {
  const int t0 = n * C, nvalid = min(C, p.T - t0);
  const size_t cb = chunk_id(p, b, h, n);
  frag::cp_wait<0>();  // dO
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  ok = hy_wait(&s.full, (int)fph);
  if (!ok) break;
  pending = false;
  fph ^= 1u;

  // Fault injection (dr_inject_timeout): wait, with a short limit, on a barrier
  // that nothing arrives on.  Every copy has landed and no MMA has been issued,
  // so the timeout path below leaves nothing in flight.
  if (inject_timeout && first) {
    ok = hy_wait(&s.never, 0, kSpinInjected);
    if (!ok) break;
  }
  bool bad = false;  // a level wait of this thread gave up (settled at the next barrier)

  // ---- level 1 (tensor memory): dQs = dO S, dW' = dU S, dKt = U dS', dM = dO U^T
  // (descriptors are built once; a k-step adds its byte offset / 16 to the start
  // address field, which stays below 2^14 for any shared-memory address)
  if (tid == 0) {
    const uint32_t id128 = tc::idesc_bf16(64, 128, false, false);  // B = the state, K-major [c][a]
    const uint32_t id64 = tc::idesc_bf16(64, 64, false, false);
    const uint64_t aDO = tc::sdesc_kmaj(s.DO, D, 0), aDU = tc::sdesc_kmaj(s.DU, D, 0);
    const uint64_t aUU = tc::sdesc_kmaj(s.UU, D, 0);
    const uint64_t bSS = tc::sdesc_kmaj(s.SS, D, 0), bSD = tc::sdesc_kmaj(s.SD, D, 0);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const uint32_t acc = ks > 0 ? 1u : 0u;
      const uint64_t ka = 16u * ks;  // K-major k-step, 16-byte units
      mma_step(tb + T_ZQ, aDO + ka, bSS + ka, id128, acc);
      mma_step(tb + T_ADW, aDU + ka, bSS + ka, id128, acc);
      mma_step(tb + T_AKT, aUU + ka, bSD + ka, id128, acc);
      mma_step(tb + T_ADM, aDO + ka, aUU + ka, id64, acc);
    }
    tc::commit(&s.bar);
  }
  // q, k, v, the gate, beta and ||k||^2 of this chunk by warps 1..15, then the
  // gate's cumulative sum by warps 8..15, while warp 0 issues level 1 (named
  // barriers 1 and 2 hold only the warps that take part)
  float dsc[4];  // real gates, warps 1..4: colsum(dS' S) of this lane's keys (lanes 0..7)
  if (warp > 0) {
    const int lt = tid - 32;
    constexpr int NL = NTB - 32;
    for (int idx = lt; idx < C * (D / 8); idx += NL) {
      const int i = idx >> 4, j = idx & 15;
      const bool ok = i < nvalid;
      const size_t rr = row_id(p, b, t0 + (ok ? i : 0), h) * D + j * 8;
      frag::cp16(s.QR + i * LDD + j * 8, q + rr, ok);
      frag::cp16(s.k + i * LDD + j * 8, k + rr, ok);
      frag::cp16(s.QC + vsw(i, 8 * j), v + rr, ok);
    }
    if (gk == D) {
      for (int idx = lt; idx < C * (D / 4); idx += NL) {
        const int i = idx >> 5, j = idx & 31;
        const bool ok = i < nvalid && p.gate != kGateNone;
        frag::cp16(s.G + gsw(i, j * 4), g + row_id(p, b, t0 + (ok ? i : 0), h) * D + j * 4, ok);
      }
    } else if (lt < C) {
      s.G[lt] = (lt < nvalid && p.gate != kGateNone) ? g[row_id(p, b, t0 + lt, h)] : 0.f;
    }
    if (lt >= C && lt < C + C / 4)
      frag::cp16(s.beta + 4 * (lt - C), beta + cb * C + 4 * (lt - C), true);
    else if (lt >= C + C / 4 && lt < C + C / 2)
      frag::cp16(s.knorm + 4 * (lt - C - C / 4), knorm_g + cb * C + 4 * (lt - C - C / 4), true);
    frag::cp_commit();
    // real gates: colsum(dS' S) on warps 1..4 while the copies land (per key
    // channel c the sum over a of dS'[c][a] S[c][a]; the state tiles are stored
    // [c][a]).  Lane: row r of the core matrices (key c = 8 kb + r) and 16-byte
    // chunk j = 4 jh + (lane / 8) of 8 values a; a warp takes key blocks
    // kb = warp - 1 + 4 m, sums its four chunks per lane, then over the lanes.
    // (The phase gate's cross term needs a shuffle per element pair: its sums run
    // on all 16 warps after the gate scan.)
    if (!PHASE && warp <= 4) {
      const int r = lane & 7, jl = lane >> 3;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int c = (warp - 1 + 4 * m) * 8 + r;
        float pr = 0.f, pr2 = 0.f;  // two sums: shorter dependency chains
        uint4 xs[4], ys[4];
#pragma unroll
        for (int jh = 0; jh < 4; ++jh) {
          const int o = ct_off(c, 8 * (4 * jh + jl), D);
          xs[jh] = *reinterpret_cast<const uint4*>(s.SS + o);
          ys[jh] = *reinterpret_cast<const uint4*>(s.SD + o);
        }
#pragma unroll
        for (int jh = 0; jh < 4; ++jh) {
          const uint32_t* wx = reinterpret_cast<const uint32_t*>(&xs[jh]);
          const uint32_t* wy = reinterpret_cast<const uint32_t*>(&ys[jh]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 fx = frag::unpack(wx[e]), fy = frag::unpack(wy[e]);
            pr += fx.x * fy.x;
            pr2 += fx.y * fy.y;
          }
        }
        pr += pr2;
        pr += __shfl_xor_sync(0xffffffffu, pr, 8);
        pr += __shfl_xor_sync(0xffffffffu, pr, 16);
        dsc[m] = pr;
      }
    }
    frag::cp_wait<0>();
    named_sync(1, NTB - 32);  // warps 1..15: their copies have landed
    if (gk == D) {
      if (warp >= 8) {
        // thread: channels 4 lane .. + 3 (16 bytes; the swizzle keeps them
        // together), rows 8 sg .. 8 sg + 7 (sg = warp - 8), scanned in registers;
        // then the totals of the earlier row segments through the dgc | ktk tiles
        const int sg = warp - 8, c4 = 4 * lane;
        float4* segtot = reinterpret_cast<float4*>(s.dgc);  // [8 segments][32 channel quads]
        float4 x[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) x[r] = *reinterpret_cast<const float4*>(s.G + gsw(8 * sg + r, c4));
#pragma unroll
        for (int r = 1; r < 8; ++r) {
          x[r].x += x[r - 1].x;
          x[r].y += x[r - 1].y;
          x[r].z += x[r - 1].z;
          x[r].w += x[r - 1].w;
        }
        segtot[sg * 32 + lane] = x[7];
        named_sync(2, NTB / 2);  // warps 8..15
        float4 off = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s2 = 0; s2 < sg; ++s2) {
          const float4 t = segtot[s2 * 32 + lane];
          off.x += t.x, off.y += t.y, off.z += t.z, off.w += t.w;
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const float4 y = make_float4(x[r].x + off.x, x[r].y + off.y, x[r].z + off.z, x[r].w + off.w);
          *reinterpret_cast<float4*>(s.G + gsw(8 * sg + r, c4)) = y;
          const int slot = grow_slot(8 * sg + r);
          if (slot >= 0) *reinterpret_cast<float4*>(&s.grow[slot][c4]) = y;
        }
      }
    } else if (warp == 1) {
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
      const int so = grow_slot(2 * lane + 1), se = grow_slot(2 * lane);
      if (so >= 0) s.grow[so][0] = x;
      if (se >= 0) s.grow[se][0] = x - a1v;
    }
  }
  __syncthreads();
  // real gates: the colsum into dgc (after the barrier: the gate scan used it as scratch)
  if (!PHASE && warp >= 1 && warp <= 4 && lane < 8) {
#pragma unroll
    for (int m = 0; m < 4; ++m) s.dgc[(warp - 1 + 4 * m) * 8 + lane] = dsc[m];
  }
  // element (i, c) of the gate tile
  auto gat = [&](int i, int c) -> float& { return gk == D ? s.G[gsw(i, c)] : s.G[i]; };

  // per-channel reference factors (phase gate: per pair, complex, at the pair's two channels)
  if (PHASE) {
    if (tid < D / 2) {
      const int c = 2 * tid;
      const float gC = s.grow[kGC][c], tC = s.grow[kGC][c + 1];
      float gr[2], tr[2];
      gr[0] = s.grow[kGR0][c], tr[0] = s.grow[kGR0][c + 1];
      gr[1] = s.grow[kGR1][c], tr[1] = s.grow[kGR1][c + 1];
      const float g31 = s.grow[kG31][c], t31 = s.grow[kG31][c + 1];
      const float g32 = s.grow[kG32][c], t32 = s.grow[kG32][c + 1];
      float sn, cs;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        sincosf(tr[hh], &sn, &cs);
        const float m = __expf(gr[hh]);
        s.er[hh * D + c] = m * cs;  // conj(zeta_rho) = e^{g_rho} e^{+i Theta_rho}
        s.er[hh * D + c + 1] = m * sn;
        sincosf(tC - tr[hh], &sn, &cs);
        const float mc = __expf(gC - gr[hh]);
        s.erc[hh * D + c] = mc * cs;  // zeta_C / zeta_rho
        s.erc[hh * D + c + 1] = -mc * sn;
      }
      // zeta_a / zeta_b = e^{g_a - g_b} e^{-i (Theta_a - Theta_b)}; the write-key
      // factors are conjugated
      sincosf(t31 - tr[0], &sn, &cs);
      float m = __expf(g31 - gr[0]);
      s.xk[c] = m * cs, s.xk[c + 1] = m * sn;
      sincosf(tr[1] - t31, &sn, &cs);
      m = __expf(gr[1] - g31);
      s.xk[D + c] = m * cs, s.xk[D + c + 1] = m * sn;
      sincosf(tr[1] - t32, &sn, &cs);
      m = __expf(gr[1] - g32);
      s.xq[c] = m * cs, s.xq[c + 1] = -m * sn;
      sincosf(t32 - tr[0], &sn, &cs);
      m = __expf(g32 - gr[0]);
      s.xq[D + c] = m * cs, s.xq[D + c + 1] = -m * sn;
    }
  } else if (tid < D) {
    const int cg = (gk == D) ? tid : 0;
    const float g0 = s.grow[kGR0][cg], g1 = s.grow[kGR1][cg], gC = s.grow[kGC][cg];
    const float g31 = s.grow[kG31][cg], g32 = s.grow[kG32][cg];
    s.er[tid] = __expf(g0);
    s.er[D + tid] = __expf(g1);
    s.erc[tid] = __expf(gC - g0);
    s.erc[D + tid] = __expf(gC - g1);
    s.xk[tid] = __expf(g31 - g0);
    s.xk[D + tid] = __expf(g1 - g31);
    s.xq[tid] = __expf(g1 - g32);
    s.xq[D + tid] = __expf(g32 - g0);
  }
  // gate tile -> factor u_i = zeta_i / zeta_rho (real gates: e^{g_i - g_rho}), rho the
  // reference row of row i's half (the references from the snapshot: each thread
  // rewrites only the elements it reads)
  if (PHASE) {
#pragma unroll
    for (int u = 0; u < C * D / NTB / 2; ++u) {
      const int idx = tid + u * NTB;  // a key pair of one row
      const int i = idx >> 6, c = 2 * (idx & 63), rs = i < 32 ? kGR0 : kGR1;
      float sn, cs;
      sincosf(gat(i, c + 1) - s.grow[rs][c + 1], &sn, &cs);
      const float m = __expf(gat(i, c) - s.grow[rs][c]);
      gat(i, c) = m * cs;
      gat(i, c + 1) = -m * sn;
    }
  } else if (gk == D) {
    // thread: channels c4 .. c4 + 3 of rows i4 + 16 u (16-byte accesses; the
    // swizzle keeps groups of 4 channels contiguous)
    const int c4 = 4 * (tid & 31), i4 = tid >> 5;
    const float4 r0 = *reinterpret_cast<const float4*>(&s.grow[kGR0][c4]);
    const float4 r1 = *reinterpret_cast<const float4*>(&s.grow[kGR1][c4]);
    float4 v[C * D / NTB / 4];
#pragma unroll
    for (int u = 0; u < C * D / NTB / 4; ++u)
      v[u] = *reinterpret_cast<const float4*>(s.G + gsw(i4 + 16 * u, c4));
#pragma unroll
    for (int u = 0; u < C * D / NTB / 4; ++u) {
      const int i = i4 + 16 * u;
      const float4 r = i < 32 ? r0 : r1;
      *reinterpret_cast<float4*>(s.G + gsw(i, c4)) =
          make_float4(frag::ex2_approx((v[u].x - r.x) * frag::kLog2e),
                      frag::ex2_approx((v[u].y - r.y) * frag::kLog2e),
                      frag::ex2_approx((v[u].z - r.z) * frag::kLog2e),
                      frag::ex2_approx((v[u].w - r.w) * frag::kLog2e));
    }
  } else if (tid < C) {
    s.G[tid] = __expf(s.G[tid] - s.grow[tid < 32 ? kGR0 : kGR1][0]);
  }
  // factor u at (i, c), (i, c + 1), c even (phase gate: the pair's complex u)
  auto ep2 = [&](int i, int c) -> float2 {
    if (gk == D) return *reinterpret_cast<const float2*>(s.G + gsw(i, c));
    const float x = s.G[i];
    return make_float2(x, x);
  };
  auto ep4 = [&](int i, int c) -> float4 {
    if (gk == D) return *reinterpret_cast<const float4*>(s.G + gsw(i, c));
    const float x = s.G[i];
    return make_float4(x, x, x, x);
  };
  // raw keys / queries (i, c), (i, c + 1)
  auto k2 = [&](int i, int c) -> float2 {
    return frag::unpack(*reinterpret_cast<const uint32_t*>(s.k + i * LDD + c));
  };
  auto q2 = [&](int i, int c) -> float2 {
    return frag::unpack(*reinterpret_cast<const uint32_t*>(s.QR + i * LDD + c));
  };
  // Level-4 key/query tiles for the 8 channels c .. c + 7 of row i (a warp's
  // rows lie in one half).  first: the tiles built under level 3 -- rows of the
  // first half: the write keys against both references and the queries; of the
  // second half: the write keys, the queries against both references and the
  // beta keys; otherwise the beta keys against the first reference.  Each case
  // forms only the factors it stores.
  auto build_row = [&](int idx, bool first) {
    const int i = ct_row(idx, D), c = ct_col(idx, D);
    const bool h1 = i >= 32;
    const uint4 rk = *reinterpret_cast<const uint4*>(s.k + i * LDD + c);
    const float bi = s.beta[i];
    const float4 f0 = ep4(i, c), f1 = ep4(i, c + 4);
    const float f[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
    const uint32_t* wk = reinterpret_cast<const uint32_t*>(&rk);
    // core-tiled offset of row i (idx) and of row i - 32 in a 32-row tile
    const int o = 8 * idx, o32 = 8 * idx - 32 * D;
    auto st4 = [](bf16* dst, const uint32_t (&w)[4]) {
      *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    };
    if (first) {
      const uint4 rq = *reinterpret_cast<const uint4*>(s.QR + i * LDD + c);
      const uint32_t* wq = reinterpret_cast<const uint32_t*>(&rq);
      uint32_t okb[4], oq[4], ox[4], obk[4];
      // the cross-half factors of these 8 channels (real gates): write keys of
      // the first half, queries of the second
      float xa[8], xb[8];
      if (!PHASE) {
        frag::load8((h1 ? s.xq : s.xk) + c, xa);
        frag::load8((h1 ? s.xq : s.xk) + D + c, xb);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 kk = frag::unpack(wk[e]), qq = frag::unpack(wq[e]);
        const int cc = c + 2 * e;
        if (PHASE) {
          const cf uu{f[2 * e], f[2 * e + 1]}, kc{kk.x, kk.y}, qc{qq.x, qq.y};
          const cf kb = cmul(kc, cconj(cinv(uu)));  // k / conj(u)
          const cf qf = cmul(uu, qc);
          okb[e] = frag::pack(kb.x, kb.y);
          oq[e] = frag::pack(qf.x, qf.y);
          if (!h1) {
            const cf kbx = cmul(cmul(kb, cf{s.xk[cc], s.xk[cc + 1]}), cf{s.xk[D + cc], s.xk[D + cc + 1]});
            ox[e] = frag::pack(kbx.x, kbx.y);
          } else {
            const cf xq0{s.xq[cc], s.xq[cc + 1]}, xq1{s.xq[D + cc], s.xq[D + cc + 1]};
            const cf qx = cmul(cmul(qf, xq0), xq1);
            const cf bk = cmul(uu, kc);
            ox[e] = frag::pack(qx.x, qx.y);
            obk[e] = frag::pack(bi * bk.x, bi * bk.y);
          }
        } else {
          const float kb0 = __fdividef(kk.x, f[2 * e]), kb1 = __fdividef(kk.y, f[2 * e + 1]);
          const float qf0 = qq.x * f[2 * e], qf1 = qq.y * f[2 * e + 1];
          okb[e] = frag::pack(kb0, kb1);
          oq[e] = frag::pack(qf0, qf1);
          if (!h1) {
            ox[e] = frag::pack(kb0 * xa[2 * e] * xb[2 * e], kb1 * xa[2 * e + 1] * xb[2 * e + 1]);
          } else {
            ox[e] = frag::pack(qf0 * xa[2 * e] * xb[2 * e], qf1 * xa[2 * e + 1] * xb[2 * e + 1]);
            obk[e] = frag::pack(bi * kk.x * f[2 * e], bi * kk.y * f[2 * e + 1]);
          }
        }
      }
      if (!h1) {
        st4(Kb0 + o, okb);
        st4(Kb1 + o, ox);
        st4(Q0 + o, oq);
      } else {
        st4(Kb1 + o, okb);
        st4(Q0 + o, ox);
        st4(Q1 + o32, oq);
        st4(B1 + o32, obk);
      }
    } else {
      uint32_t ob[4];
      float xa[8], xb[8];  // the queries' cross-half factors (second half, real gates)
      if (!PHASE && h1) {
        frag::load8(s.xq + c, xa);
        frag::load8(s.xq + D + c, xb);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 kk = frag::unpack(wk[e]);
        const int cc = c + 2 * e;
        if (PHASE) {
          cf bk = cmul(cf{f[2 * e], f[2 * e + 1]}, cf{kk.x, kk.y});
          if (h1) bk = cmul(cmul(bk, cf{s.xq[cc], s.xq[cc + 1]}), cf{s.xq[D + cc], s.xq[D + cc + 1]});
          ob[e] = frag::pack(bi * bk.x, bi * bk.y);
        } else {
          float b0 = bi * kk.x * f[2 * e], b1 = bi * kk.y * f[2 * e + 1];
          if (h1) {
            b0 = b0 * xa[2 * e] * xb[2 * e];
            b1 = b1 * xa[2 * e + 1] * xb[2 * e + 1];
          }
          ob[e] = frag::pack(b0, b1);
        }
      }
      st4(B0 + o, ob);
    }
  };

  // phase gate: colsum(conj(dS') S) while level 1 runs.  Thread: row r of the
  // core matrices of row blocks 4 q .. 4 q + 3 (keys c), 16-byte chunk j (8
  // values a); eight lanes read one whole core matrix.  Partial sums reduce over
  // the warp's four chunks, then land in one of four slots per key (warp % 4),
  // summed by the reader.
  if (PHASE) {
    const int r = tid & 7, j = (tid >> 3) & 15, q = tid >> 7;
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int c = (4 * q + rr) * 8 + r;
      const int o = ct_off(c, 8 * j, D);
      const uint4 x = *reinterpret_cast<const uint4*>(s.SS + o);
      const uint4 y = *reinterpret_cast<const uint4*>(s.SD + o);
      const uint32_t* wx = reinterpret_cast<const uint32_t*>(&x);
      const uint32_t* wy = reinterpret_cast<const uint32_t*>(&y);
      float pr = 0.f, cross = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fx = frag::unpack(wx[e]), fy = frag::unpack(wy[e]);
        pr += fx.x * fy.x + fx.y * fy.y;
        // the pair's odd key (lane ^ 1) for the cross term of conj(dS') S:
        // Im = sum_a (dx sy - dy sx), x the even key, y the odd one
        const float2 gx = frag::unpack(__shfl_xor_sync(0xffffffffu, wx[e], 1));
        const float2 gy = frag::unpack(__shfl_xor_sync(0xffffffffu, wy[e], 1));
        cross += fy.x * gx.x + fy.y * gx.y - gy.x * fx.x - gy.y * fx.y;
      }
      pr += __shfl_xor_sync(0xffffffffu, pr, 8);
      pr += __shfl_xor_sync(0xffffffffu, pr, 16);
      cross += __shfl_xor_sync(0xffffffffu, cross, 8);
      cross += __shfl_xor_sync(0xffffffffu, cross, 16);
      const float po = __shfl_xor_sync(0xffffffffu, pr, 1);
      if ((lane >> 3) == 0 && (r & 1) == 0) {
        s.dgc[(warp & 3) * D + c] = pr + po;     // Re: dx sx + dy sy
        s.dgc[(warp & 3) * D + c + 1] = cross;  // Im
      }
    }
  }
  bad = !level_wait(&s.bar, 0) || bad;
  float zq[4][4], adw[4][4], akt[4][4], adm[2][4];
  {
    uint32_t rz[16], rw[16], rk[16], rm[8];
    frag_ld4_raw(tb + T_ZQ + 32 * qt, warp, rz);
    frag_ld4_raw(tb + T_ADW + 32 * qt, warp, rw);
    frag_ld4_raw(tb + T_AKT + 32 * qt, warp, rk);
    frag_ld2_raw(tb + T_ADM + 16 * qt, warp, rm);
    tc::tmem_wait_ld();
    frag_of<4>(rz, zq);
    frag_of<4>(rw, adw);
    frag_of<4>(rk, akt);
    frag_of<2>(rm, adm);
  }
  // dW = -dW', and dM masked (inclusive lower) into its X tile (rows of the
  // second half 4 KB further on, after the zero block written here)
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
        if (jj == i) s.dmd[i] = adm[jt][e];
        if (jj >= i) adm[jt][e] = 0.f;
      }
    frag::st_c(adm, XM, -C, rb * 16 + (hf ? 32 : 0), qt * 16);
    if (tid < C * C / 16)
      *reinterpret_cast<uint4*>(XM + C * C / 2 + 8 * tid) = make_uint4(0, 0, 0, 0);
  }
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  ok = __syncthreads_or(bad ? 1 : 0) == 0;
  tc::fence_after_sync();
  if (!ok) break;
  // W and U' into the dS' tile: level 1 and every thread's colsum have read it
  // (the barrier above; a thread's own level-1 wait alone does not cover the
  // other threads' colsum reads)
  cp_linear<NTB>(sW, Wg + cb * C * D, C * D, tid);
  cp_linear<NTB>(sUp, Upg + cb * C * D, C * D, tid);
  frag::cp_commit();
  // ---- level 2: Lambda = T^T [dU | dW]; dv = diag(beta) Lambda_U (runs under the dKt pass)
  if (tid == 0) {
    const uint32_t id = tc::idesc_bf16(64, 128, true, true);
    const uint64_t aT = tc::sdesc_mnmaj(s.TT, C, 0);
    const uint64_t bU = tc::sdesc_mnmaj(s.DU, D, 0), bW = tc::sdesc_mnmaj(sdW, D, 0);
#pragma unroll
    for (int ks = 0; ks < C / 16; ++ks) {
      const uint32_t acc = ks > 0 ? 1u : 0u;
      mma_step(tb + T_LU, aT + 128u * ks, bU + 256u * ks, id, acc);
      mma_step(tb + T_LW, aT + 128u * ks, bW + 256u * ks, id, acc);
    }
    tc::commit(&s.bar);
  }

  // The per-element epilogue works on three accumulators at this thread's
  // fragment positions (rows i0, i0 + 8 of half hf; key columns c, c + 1, one
  // pair), with u the row's factor relative to its half's reference rho:
  //   Z = conj(zeta_rho) dQs + F1                  -> dq = conj(u) Z
  //   P = (zeta_C / zeta_rho) dKt + G              -> t2 = P / u
  //   Q = conj(zeta_rho) Lambda_W + F2             -> t1 = conj(u) Q
  // so that dk = beta t1 + t2, d(beta) = Lambda_U . v + k . t1, and, with
  // E1 = conj(dq) q + beta conj(t1) k, E2 = conj(t2) k: dg = Re(E1 - E2) (real
  // gates: q dq + k (beta t1 - t2)) and d Theta = Im(E1 + E2).
  const int i0 = rb * 16 + lr;
  const size_t rowg[2] = {row_id(p, b, t0 + min(i0, nvalid - 1), h) * D,
                          row_id(p, b, t0 + min(i0 + 8, nvalid - 1), h) * D};
  float(&Z)[4][4] = zq;
  float(&P)[4][4] = akt;
  // colsum(conj(dKt) K~) for the chunk-end gate term, then the reference scalings
  {
    float cs[4][2] = {};
#pragma unroll
    for (int jt = 0; jt < 4; ++jt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int i = i0 + hh * 8, c = qt * 32 + jt * 8 + lc;
        const float2 kk = k2(i, c), f = ep2(i, c);
        if (PHASE) {  // conj(dKt) (k / conj(u))
          const cf kb = cmul(cf{kk.x, kk.y}, cconj(cinv(cf{f.x, f.y})));
          const cf t = cmulc(cf{akt[jt][2 * hh], akt[jt][2 * hh + 1]}, kb);
          cs[jt][0] += t.x;
          cs[jt][1] += t.y;
        } else {
          cs[jt][0] += kk.x * __fdividef(akt[jt][2 * hh], f.x);
          cs[jt][1] += kk.y * __fdividef(akt[jt][2 * hh + 1], f.y);
        }
      }
#pragma unroll
    for (int jt = 0; jt < 4; ++jt) {
      const int c = qt * 32 + jt * 8 + lc;
      const float2 fr = *reinterpret_cast<const float2*>(s.er + hf * D + c);
      const float2 frc = *reinterpret_cast<const float2*>(s.erc + hf * D + c);
      float x[2];
      if (PHASE) {  // K~ = conj(zeta_C / zeta_rho) (k / conj(u))
        const cf t = cmulc(cf{frc.x, frc.y}, cf{cs[jt][0], cs[jt][1]});
        x[0] = t.x, x[1] = t.y;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const cf z = cmul(cf{fr.x, fr.y}, cf{Z[jt][2 * hh], Z[jt][2 * hh + 1]});
          const cf pp = cmul(cf{frc.x, frc.y}, cf{P[jt][2 * hh], P[jt][2 * hh + 1]});
          Z[jt][2 * hh] = z.x, Z[jt][2 * hh + 1] = z.y;
          P[jt][2 * hh] = pp.x, P[jt][2 * hh + 1] = pp.y;
        }
      } else {
        x[0] = cs[jt][0] * frc.x, x[1] = cs[jt][1] * frc.y;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          Z[jt][2 * hh] *= fr.x, Z[jt][2 * hh + 1] *= fr.y;
          P[jt][2 * hh] *= frc.x, P[jt][2 * hh + 1] *= frc.y;
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float y = x[u];
        y += __shfl_xor_sync(0xffffffffu, y, 4);
        y += __shfl_xor_sync(0xffffffffu, y, 8);
        y += __shfl_xor_sync(0xffffffffu, y, 16);
        if (lr == 0) s.ktk[rb * D + c + u] = y;
      }
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
        vv[jt][hh] = *reinterpret_cast<const uint32_t*>(s.QC + vsw(i0 + 8 * hh, qt * 32 + jt * 8 + lc));
    bad = !level_wait(&s.bar, 1) || bad;
    float lu[4][4];
    frag_ld4(tb + T_LU + 32 * qt, warp, lu);
#pragma unroll
    for (int jt = 0; jt < 4; ++jt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const float2 vf = frag::unpack(vv[jt][hh]);
        dbrow[hh] += lu[jt][2 * hh] * vf.x + lu[jt][2 * hh + 1] * vf.y;
      }
    // dv = diag(beta) Lambda_U.  Real gates: transposed across the quad of lanes
    // that share a row into one 16-byte store per row and lane; the phase gate
    // (short of registers here) stores its pairs directly.
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int i = i0 + hh * 8;
      const float bi = s.beta[i];
      uint32_t dvp[4];
#pragma unroll
      for (int jt = 0; jt < 4; ++jt) dvp[jt] = frag::pack(bi * lu[jt][2 * hh], bi * lu[jt][2 * hh + 1]);
      if (PHASE) {
#pragma unroll
        for (int jt = 0; jt < 4; ++jt)
          if (i < nvalid) *reinterpret_cast<uint32_t*>(dv + rowg[hh] + qt * 32 + jt * 8 + lc) = dvp[jt];
      } else {
        frag::quad_transpose(dvp, lane & 3);
        if (i < nvalid)
          *reinterpret_cast<uint4*>(dv + rowg[hh] + qt * 32 + 8 * (lane & 3)) =
              make_uint4(dvp[0], dvp[1], dvp[2], dvp[3]);
      }
    }
    frag::st_c(lu, sLU, -D, rb * 16, qt * 32);
    frag_ld4(tb + T_LW + 32 * qt, warp, Q);
    frag::st_c(Q, sLW, -D, rb * 16, qt * 32);
#pragma unroll
    for (int jt = 0; jt < 4; ++jt) {
      const float2 fr = *reinterpret_cast<const float2*>(s.er + hf * D + qt * 32 + jt * 8 + lc);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (PHASE) {
          const cf z = cmul(cf{fr.x, fr.y}, cf{Q[jt][2 * hh], Q[jt][2 * hh + 1]});
          Q[jt][2 * hh] = z.x, Q[jt][2 * hh + 1] = z.y;
        } else {
          Q[jt][2 * hh] *= fr.x, Q[jt][2 * hh + 1] *= fr.y;
        }
      }
    }
  }

  frag::cp_wait<0>();  // W, U'
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  ok = __syncthreads_or(bad ? 1 : 0) == 0;
  tc::fence_after_sync();
  if (!ok) break;

  // ---- level 3: dA = -strict_tril(Lambda_U U'^T + Lambda_W W^T): four partial sums
  if (tid == 0) {
    const uint32_t id = tc::idesc_bf16(64, 64, false, false);
    const uint64_t aLU = tc::sdesc_kmaj(sLU, D, 0), aLW = tc::sdesc_kmaj(sLW, D, 0);
    const uint64_t bUp = tc::sdesc_kmaj(sUp, D, 0), bW = tc::sdesc_kmaj(sW, D, 0);
#pragma unroll
    for (int j = 0; j < D / 32; ++j)
#pragma unroll
      for (int part = 0; part < 4; ++part) {
        const uint64_t ko = 16u * (2 * j + (part & 1));
        mma_step(tb + T_DA + 64 * part, (part < 2 ? aLU : aLW) + ko, (part < 2 ? bUp : bW) + ko,
                 id, j > 0 ? 1u : 0u);
      }
    tc::commit(&s.bar);
  }
  // ---- under level 3: the dA-free level-4 operands (warps 1..15: warp 0 issues
  //      level 3), then their products F1 = dM Kb (per-half references) and the
  //      dM half of G for the first half
  if (warp > 0)
    for (int idx = tid - 32; idx < C * (D / 8); idx += NTB - 32) build_row(idx, true);
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t idF = tc::idesc_bf16(64, 128, false, true);
  const uint32_t idG = tc::idesc_bf16(64, 128, true, true);
  // level-4 descriptors (k-step offsets in 16-byte units are added below)
  const uint64_t xmK = dk64(XM, 0), xaK = dk64(XA, 0), xmT = dmn64(XM, 0), xaT = dmn64(XA, 0);
  const uint64_t dKb0 = dmn128(Kb0, 0), dKb1 = dmn128(Kb1, 0), dQ0 = dmn128(Q0, 0);
  const uint64_t dQ1 = dmn128(Q1, 0), dB0 = dmn128(B0, 0), dB1 = dmn128(B1, 0);
  bad = !level_wait(&s.bar, 2) || bad;
  // level 4, dM part (thread 0, after the barrier above: the other warps go on
  // to the dA readout without waiting for the issue)
  if (tid == 0) {
    // F1: rows of the first half against Kb^{rho0} (k-steps 0, 1), rows of the
    // second half against Kb^{rho1} (k-steps 0..3); one accumulator
    mma_step(tb + T_F1, xmK, dKb0, idF, 0u);
    mma_step(tb + T_G0, xmT + xt_off(0) / 16, dQ0, idG, 0u);
    mma_step(tb + T_F1, xmK + 16, dKb0 + 256, idF, 1u);
    mma_step(tb + T_G0, xmT + xt_off(1) / 16, dQ0 + 256, idG, 1u);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      mma_step(tb + T_F1, xmK + 256 + 16 * ks, dKb1 + 256 * ks, idF, 1u);
      if (ks >= 2) mma_step(tb + T_G0, xmT + xt_off(ks) / 16, dQ0 + 256 * ks, idG, 1u);
    }
  }
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
    frag::st_c(da, XA, -C, rb * 16 + (hf ? 32 : 0), qt * 16);
  }
  // beta k of the first reference into the Lambda tiles (level 3 has read them;
  // warps 1..15: warp 0 issued the dM part of level 4)
  if (warp > 0)
    for (int idx = tid - 32; idx < C * (D / 8); idx += NTB - 32) build_row(idx, false);
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  ok = __syncthreads_or(bad ? 1 : 0) == 0;
  tc::fence_after_sync();
  if (!ok) break;
  // ---- level 4, dA part: F2 = dA Kb; G += dA^T beta k (first half); G of the second half
  if (tid == 0) {
    mma_step(tb + T_F2, xaK, dKb0, idF, 0u);
    mma_step(tb + T_G1, xmT + xt_off(2) / 16, dQ1, idG, 0u);
    mma_step(tb + T_G0, xaT + xt_off(0) / 16, dB0, idG, 1u);
    mma_step(tb + T_F2, xaK + 16, dKb0 + 256, idF, 1u);
    mma_step(tb + T_G1, xmT + xt_off(3) / 16, dQ1 + 256, idG, 1u);
    mma_step(tb + T_G0, xaT + xt_off(1) / 16, dB0 + 256, idG, 1u);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      mma_step(tb + T_F2, xaK + 256 + 16 * ks, dKb1 + 256 * ks, idF, 1u);
      if (ks >= 2) {
        mma_step(tb + T_G0, xaT + xt_off(ks) / 16, dB0 + 256 * ks, idG, 1u);
        mma_step(tb + T_G1, xaT + xt_off(ks) / 16, dB1 + 256 * (ks - 2), idG, 1u);
      }
    }
    tc::commit(&s.bar);
    if (nb < p.B) tc::mbar_arrive_expect_tx(&s.full, kTileTx);
  }
  bad = !level_wait(&s.bar, 3) || bad;
  // the next chunk's level-1 tiles into the tiles level 4 has released
  if (nb < p.B) {
    issue_tiles(nn, nh, nb);
    pending = true;
  }
  {
    uint32_t r1[16], r2[16], r3[16];
    frag_ld4_raw(tb + T_F1 + 32 * qt, warp, r1);
    frag_ld4_raw(tb + T_F2 + 32 * qt, warp, r2);
    frag_ld4_raw(tb + (hf ? T_G1 : T_G0) + 32 * qt, warp, r3);
    tc::tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        Z[j][e] += __uint_as_float(r1[4 * j + e]);
        Q[j][e] += __uint_as_float(r2[4 * j + e]);
        P[j][e] += __uint_as_float(r3[4 * j + e]);
      }
  }

  // ---- per-element epilogue: dq out; P <- dk (before the Kaczmarz term), Q <- dgamma
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    uint32_t dqp[4];  // dq pairs of this row (column group jt), stored after a quad transpose
#pragma unroll
    for (int jt = 0; jt < 4; ++jt) {
      const int i = i0 + hh * 8, c = qt * 32 + jt * 8 + lc;
      const float bi = s.beta[i];
      const float2 kk = k2(i, c), qq = q2(i, c), f = ep2(i, c);
      const int e0 = 2 * hh, e1 = 2 * hh + 1;
      // the diagonal of dM enters dq and t2 with the factor 1 and cancels in dg
      // exactly, so it is kept out of the bf16 products and of dg
      const float dmi = s.dmd[i];
      float dqo[2], dko[2], dgo[2];
      if (PHASE) {
        const cf uu{f.x, f.y}, kc{kk.x, kk.y}, qc{qq.x, qq.y};
        const cf dqc = cmulc(uu, cf{Z[jt][e0], Z[jt][e1]});   // conj(u) Z
        const cf t1 = cmulc(uu, cf{Q[jt][e0], Q[jt][e1]});    // conj(u) Q
        const cf t2 = cmul(cf{P[jt][e0], P[jt][e1]}, cinv(uu));  // P / u
        const cf a1 = cmulc(dqc, qc), a2 = cmulc(t1, kc), a3 = cmulc(t2, kc);
        dgo[0] = a1.x + bi * a2.x - a3.x;  // Re(E1 - E2)
        dgo[1] = a1.y + bi * a2.y + a3.y;  // Im(E1 + E2)
        dqo[0] = dqc.x + dmi * kc.x, dqo[1] = dqc.y + dmi * kc.y;
        dko[0] = bi * t1.x + t2.x + dmi * qc.x, dko[1] = bi * t1.y + t2.y + dmi * qc.y;
        dbrow[hh] += kc.x * t1.x + kc.y * t1.y;
      } else {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int e = 2 * hh + u;
          const float ep = u ? f.y : f.x, kv = u ? kk.y : kk.x, qv = u ? qq.y : qq.x;
          const float t1 = ep * Q[jt][e], t2 = __fdividef(P[jt][e], ep);
          const float dqs = ep * Z[jt][e];
          dgo[u] = qv * dqs + kv * (bi * t1 - t2);
          dqo[u] = dqs + dmi * kv;
          dko[u] = bi * t1 + t2 + dmi * qv;
          dbrow[hh] += kv * t1;
        }
      }
      if (i == C - 1) {
        // chunk-end gate term: colsum(conj(dKt) K~) + conj(zeta_C) colsum(conj(dS') S)
        float kt[2], gs[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int cc = c + u;
          kt[u] = s.ktk[cc] + s.ktk[D + cc] + s.ktk[2 * D + cc] + s.ktk[3 * D + cc];
          gs[u] = PHASE ? s.dgc[cc] + s.dgc[D + cc] + s.dgc[2 * D + cc] + s.dgc[3 * D + cc]
                        : s.dgc[cc];
        }
        const float2 fr = *reinterpret_cast<const float2*>(s.er + D + c);
        const float2 frc = *reinterpret_cast<const float2*>(s.erc + D + c);
        if (PHASE) {
          const cf dec = cmul(cf{fr.x, fr.y}, cconj(cf{frc.x, frc.y}));  // conj(zeta_C)
          const cf ps = cmul(dec, cf{gs[0], gs[1]});
          dgo[0] += kt[0] + ps.x;
          dgo[1] -= kt[1] + ps.y;
        } else {
          dgo[0] += kt[0] + fr.x * frc.x * gs[0];
          dgo[1] += kt[1] + fr.y * frc.y * gs[1];
        }
      }
      dqp[jt] = frag::pack(dqo[0], dqo[1]);
      P[jt][e0] = dko[0], P[jt][e1] = dko[1];
      Q[jt][e0] = dgo[0], Q[jt][e1] = dgo[1];
    }
    // after the quad transpose lane lq holds channels qt * 32 + 8 lq .. + 7 of
    // the row (one 16-byte store instead of four 4-byte ones)
    frag::quad_transpose(dqp, lane & 3);
    if (i0 + 8 * hh < nvalid)
      *reinterpret_cast<uint4*>(dq + rowg[hh] + qt * 32 + 8 * (lane & 3)) =
          make_uint4(dqp[0], dqp[1], dqp[2], dqp[3]);
  }
  // d(beta_eff) partials: reduce the 4 lanes that share a row, one slot per column quarter
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    float xx = dbrow[hh];
    xx += __shfl_xor_sync(0xffffffffu, xx, 1);
    xx += __shfl_xor_sync(0xffffffffu, xx, 2);
    if ((lane & 3) == 0) s.dbp[(i0 + hh * 8) * 4 + qt] = xx;
  }
  // dgamma: reverse cumulative sum over the chunk's rows.  Within this warp's
  // 16 rows (rows i0 = 16 rb + lr and i0 + 8, lr = lane / 4 on the lanes that
  // share its columns): suffix sums down the 8 lane rows by shuffles, the
  // second 8 rows' total added to the first; the later row blocks' totals
  // follow through shared memory.
  if (gk == D) {
#pragma unroll
    for (int jt = 0; jt < 4; ++jt)
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float lo = Q[jt][u], hi = Q[jt][2 + u];
#pragma unroll
        for (int d = 1; d < 8; d <<= 1) {
          const float yl = __shfl_down_sync(0xffffffffu, lo, 4 * d);
          const float yh = __shfl_down_sync(0xffffffffu, hi, 4 * d);
          if (lr + d < 8) {
            lo += yl;
            hi += yh;
          }
        }
        lo += __shfl_sync(0xffffffffu, hi, lane & 3);
        Q[jt][u] = lo;
        Q[jt][2 + u] = hi;
        if (lr == 0) s.blk[rb * D + qt * 32 + jt * 8 + lc + u] = lo;
      }
  } else {
    // scalar gate: the row sums of dgamma, one slot per column quarter
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float xx = 0.f;
#pragma unroll
      for (int jt = 0; jt < 4; ++jt) xx += Q[jt][2 * hh] + Q[jt][2 * hh + 1];
      xx += __shfl_xor_sync(0xffffffffu, xx, 1);
      xx += __shfl_xor_sync(0xffffffffu, xx, 2);
      if ((lane & 3) == 0) s.blk[(i0 + hh * 8) * 4 + qt] = xx;
    }
  }
  ok = __syncthreads_or(bad ? 1 : 0) == 0;
  if (!ok) break;
  float dbt = 0.f;
  if (tid < C) {
    dbt = s.dbp[tid * 4] + s.dbp[tid * 4 + 1] + s.dbp[tid * 4 + 2] + s.dbp[tid * 4 + 3];
    s.dbp[tid * 4] = dbt;  // total d(beta_eff) of row tid (read back by this thread only)
  }
  if (gk == D) {
#pragma unroll
    for (int jt = 0; jt < 4; ++jt) {
      const int c = qt * 32 + jt * 8 + lc;
      float later[2] = {0.f, 0.f};
      for (int r2 = rb + 1; r2 < 4; ++r2) {
        const float2 t = *reinterpret_cast<const float2*>(s.blk + r2 * D + c);
        later[0] += t.x;
        later[1] += t.y;
      }
      if (i0 < nvalid)
        *reinterpret_cast<float2*>(dg + rowg[0] + c) =
            make_float2(Q[jt][0] + later[0], Q[jt][1] + later[1]);
      if (i0 + 8 < nvalid)
        *reinterpret_cast<float2*>(dg + rowg[1] + c) =
            make_float2(Q[jt][2] + later[0], Q[jt][3] + later[1]);
    }
  } else if (p.gate != kGateNone && warp == 0) {
    // rows 2 lane, 2 lane + 1: suffix sums across the warp
    const int ia = 2 * lane, ib = ia + 1;
    const float a0 = s.blk[ia * 4] + s.blk[ia * 4 + 1] + s.blk[ia * 4 + 2] + s.blk[ia * 4 + 3];
    const float a1 = s.blk[ib * 4] + s.blk[ib * 4 + 1] + s.blk[ib * 4 + 2] + s.blk[ib * 4 + 3];
    float x = a0 + a1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_down_sync(0xffffffffu, x, o);
      if (lane + o < 32) x += y;
    }
    if (ia < nvalid) dg[row_id(p, b, t0 + ia, h)] = x;
    if (ib < nvalid) dg[row_id(p, b, t0 + ib, h)] = x - a0;
  }
  __syncthreads();
  // dk (with the Kaczmarz chain rule; quad-transposed into 16-byte stores) and dbeta
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    uint32_t dkp[4];
#pragma unroll
    for (int jt = 0; jt < 4; ++jt) {
      const int i = i0 + hh * 8, c = qt * 32 + jt * 8 + lc;
      float o0 = P[jt][2 * hh], o1 = P[jt][2 * hh + 1];
      if (p.beta_mode == kBetaKaczmarz) {
        const float f = -2.f * s.beta[i] * s.dbp[i * 4] / (s.knorm[i] + p.eps);
        const float2 kk = k2(i, c);
        o0 += f * kk.x;
        o1 += f * kk.y;
      }
      dkp[jt] = frag::pack(o0, o1);
    }
    frag::quad_transpose(dkp, lane & 3);
    if (i0 + 8 * hh < nvalid)
      *reinterpret_cast<uint4*>(dk + rowg[hh] + qt * 32 + 8 * (lane & 3)) =
          make_uint4(dkp[0], dkp[1], dkp[2], dkp[3]);
  }
  if (tid < nvalid) {
    if (p.beta_mode == kBetaKaczmarz) dbt /= (s.knorm[tid] + p.eps);
    dbeta[row_id(p, b, t0 + tid, h)] = dbt;
  }
  }
  if (!ok) {
    // a bounded wait gave up: record it and let the copies in flight land
    if (tid == 0 && err) atomicExch(err, 1);
    frag::cp_wait<0>();
    if (pending && tid == 0) tc::mbar_wait(&s.full, fph, kSpinHy);
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
  const bool phase = p.gate == kGatePhase;
  auto kern = phase ? k_bwd_chunk_hy<true> : k_bwd_chunk_hy<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const double nb = (double)p.B * p.H * p.NC, ntok = nb * C;
  // operator I/O: reads q, k, v, dO, g, beta; writes dq, dk, dv, dbeta, dg
  const double io = ntok * (4 * D * 2 + p.gk * 4 + 4) + ntok * (3 * D * 2 + p.gk * 4 + 4);
  // and by design the chunk tiles T, h, dh, U, dU, W, U' (and beta, ||k||^2 from the saved set)
  const double bytes = io + nb * C * C * 2 + nb * 2.0 * D * D * 2 + ntok * 4 * D * 2 + ntok * 4;
  // level 1: 3 (C x D x D) + C^2 D; level 2: 2 C^2 D; level 3: 2 C^2 D;
  // level 4 as issued: 24 products of 64 x 16 x 128
  const double mac = 3.0 * C * D * D + (double)C * C * D + 2.0 * C * C * D + 2.0 * C * C * D +
                     24.0 * 64 * 16 * 128;
  prof_begin(kKTcChunkBwd, io, bytes, nb * 2.0 * mac, st);
  // persistent: one CTA per SM (its shared memory allows no second one)
  const long nchunks = (long)p.NC * p.H * p.B;
  const int grid = (int)(nchunks < sm_count() ? nchunks : sm_count());
  kern<<<grid, NTB, sm, st>>>(
      p, q, k, v, dO, g, sv.T, sv.beta, sv.h, dh, sv.U, dU, sv.W, sv.Up, sv.knorm, dq, dk, dv,
      dbeta, dg, device_error_word(), take_injected_timeout() ? 1 : 0);
  e = cudaGetLastError();
  prof_end(st);
  return e;
}

}  // namespace fast
}  // namespace dr
