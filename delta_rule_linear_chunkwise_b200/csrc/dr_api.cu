// dr_api.cu -- the C ABI declared in include/dr.h: argument validation,
// workspace carving and kernel dispatch.  No device memory is allocated here.

#include <atomic>

#include "../../include/dr.h"
#include "dr_common.cuh"
#include "fast.cuh"

namespace dr {

namespace {
std::atomic<int> g_injected_timeouts{0};
}  // namespace

int sm_count() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

bool take_injected_timeout() {
  int n = g_injected_timeouts.load();
  while (n > 0)
    if (g_injected_timeouts.compare_exchange_weak(n, n - 1)) return true;
  return false;
}

}  // namespace dr

namespace {

using dr::Problem;
using dr::Ws;

constexpr size_t kAlign = 256;

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return p == nullptr || ((uintptr_t)p & 15u) == 0; }

dr_status validate(const dr_problem* in, Problem* out) {
  if (!in) return DR_ERR_INVALID_ARG;
  if (in->B < 1 || in->H < 1 || in->T < 1 || in->dk < 1 || in->dv < 1)
    return DR_ERR_INVALID_ARG;
  if (in->dtype != DR_F32 && in->dtype != DR_BF16) return DR_ERR_INVALID_ARG;
  if (in->gate < DR_GATE_NONE || in->gate > DR_GATE_PHASE) return DR_ERR_INVALID_ARG;
  if (in->beta_mode != DR_BETA_DIRECT && in->beta_mode != DR_BETA_KACZMARZ)
    return DR_ERR_INVALID_ARG;
  if (!(in->eps >= 0.f)) return DR_ERR_INVALID_ARG;
  if (in->chunk != dr::kC) return DR_ERR_UNSUPPORTED;
  if (in->dk % 16 || in->dv % 16 || in->dk > 128 || in->dv > 128) return DR_ERR_UNSUPPORTED;
  // Index arithmetic uses size_t throughout, but grid dims are 16-bit in y/z.
  if (in->H > 65535 || in->B > 65535) return DR_ERR_UNSUPPORTED;
  out->B = in->B;
  out->H = in->H;
  out->T = in->T;
  out->dk = in->dk;
  out->dv = in->dv;
  out->NC = (in->T + dr::kC - 1) / dr::kC;
  out->gate = in->gate;
  out->beta_mode = in->beta_mode;
  out->gk = (in->gate == DR_GATE_CHANNEL || in->gate == DR_GATE_PHASE) ? in->dk : 1;
  out->eps = in->eps;
  return DR_OK;
}

// Region sizes in floats, in carving order.  pass 0 = forward, 1 = backward.
struct Layout {
  size_t off[17];
  size_t total;
};

Layout layout(const Problem& p, int pass) {
  const size_t nb = (size_t)p.B * p.H * p.NC;  // (b, h, chunk) blocks
  const size_t C = dr::kC;
  size_t sz[17] = {
      nb * C * p.gk,       // gam
      nb * C,              // beff
      nb * C,              // kn
      nb * C * C,          // Tm
      nb * C * C,          // Mm
      nb * C * p.dk,       // W
      nb * C * p.dv,       // Up
      0,                   // U
      0,                   // h
      0, 0, 0, 0, 0, 0, 0, 0};
  if (pass == 1) {
    sz[7] = nb * C * p.dv;          // U
    sz[8] = nb * p.dv * p.dk;       // h (used when no saved buffer is given)
    sz[9] = nb * p.dv * p.dk;       // dh
    sz[10] = nb * C * p.dv;         // dU
    sz[11] = nb * C * p.dk;         // dQs
    sz[12] = nb * C * p.dk;         // dWs
    sz[13] = nb * C * p.dk;         // dKt
    sz[14] = nb * p.dk;             // dgC
    sz[15] = nb * C * p.dk;         // dk_acc
    sz[16] = nb * C * p.dk;         // dg_acc
  }
  Layout L;
  size_t o = 0;
  for (int i = 0; i < 17; ++i) {
    L.off[i] = o;
    o += round_up(sz[i] * sizeof(float));
  }
  // The tensor-core path carves its own regions from the same workspace.
  const size_t nb2 = (size_t)p.B * p.H * p.NC;
  size_t fast = round_up(dr::fast::saved_bytes(p));
  if (pass == 1)
    fast += round_up(nb2 * dr::fast::kUBytes) + round_up(nb2 * dr::fast::kStateBytes);
  // segmented (affine) scans: two [B][G][H] state buffers
  fast += 2 * round_up(dr::fast::affine_map_bytes(p, dr::fast::affine_segments(p)));
  L.total = o > fast ? o : fast;
  return L;
}

Ws carve(const Layout& L, void* base, int pass) {
  char* b = (char*)base;
  auto at = [&](int i) { return (float*)(b + L.off[i]); };
  Ws w;
  w.gam = at(0);
  w.beff = at(1);
  w.kn = at(2);
  w.Tm = at(3);
  w.Mm = at(4);
  w.W = at(5);
  w.Up = at(6);
  w.U = pass ? at(7) : nullptr;
  w.h = pass ? at(8) : nullptr;
  w.dh = pass ? at(9) : nullptr;
  w.dU = pass ? at(10) : nullptr;
  w.dQs = pass ? at(11) : nullptr;
  w.dWs = pass ? at(12) : nullptr;
  w.dKt = pass ? at(13) : nullptr;
  w.dgC = pass ? at(14) : nullptr;
  w.dk_acc = pass ? at(15) : nullptr;
  w.dg_acc = pass ? at(16) : nullptr;
  return w;
}

// Segments of the chunk-parallel affine scan for this problem (1 = sequential).
int scan_segments(const Problem& P) { return dr::fast::affine_segments(P); }

// The forward state scan, plain or segmented.  Segmented: the transfer
// matrices (into the saved tiles) and offsets of all segments in one
// parallel pass, their composition into segment start states, then the
// output pass of all segments in parallel.  aff: two affine buffers.
cudaError_t fwd_scan_any(const Problem& P, const dr::fast::Saved& sv, const float* S0,
                         __nv_bfloat16* o, float* ST, bool save, char* aff, cudaStream_t st) {
  const int G = scan_segments(P);
  if (G == 1) return dr::fast::launch_fwd_scan_tc(P, sv, S0, o, ST, save, st);
  const int L = dr::fast::affine_seg_len(P, G);
  float* Bm = (float*)aff;
  float* Sst = (float*)(aff + round_up(dr::fast::affine_map_bytes(P, G)));
  const int bv_maps = (long)4 * P.B * P.H * G <= 148 ? 64 : 128;
  cudaError_t e = dr::fast::launch_fwd_scan_tc_seg(
      P, sv, dr::fast::ScanSeg{G, L, 3, nullptr, sv.Pseg, Bm}, nullptr, false, bv_maps, st);
  if (e == cudaSuccess) e = dr::fast::launch_affine_compose_fwd(P, G, S0, sv.Pseg, Bm, Sst, ST, st);
  if (e == cudaSuccess)
    e = dr::fast::launch_fwd_scan_tc_seg(P, sv, dr::fast::ScanSeg{G, L, 0, Sst, nullptr, nullptr},
                                         o, save, 64, st);
  return e;
}

// The backward state-gradient scan, plain or segmented (the segment offsets C
// in parallel, their composition with the saved transfer matrices into
// segment end gradients and dS0, then the output pass in parallel).
cudaError_t bwd_scan_any(const Problem& P, const dr::fast::Saved& sv, const __nv_bfloat16* dO,
                         const float* dST, float* dS0, __nv_bfloat16* dU, __nv_bfloat16* dh,
                         char* aff, cudaStream_t st) {
  const int G = scan_segments(P);
  if (G == 1) return dr::fast::launch_bwd_scan_tc(P, sv, dO, dST, dS0, dU, dh, st);
  const int L = dr::fast::affine_seg_len(P, G);
  float* Cm = (float*)aff;
  float* dSe = (float*)(aff + round_up(dr::fast::affine_map_bytes(P, G)));
  cudaError_t e = dr::fast::launch_bwd_scan_tc_seg(
      P, sv, dO, dr::fast::ScanSeg{G, L, 1, nullptr, Cm, nullptr}, nullptr, nullptr, 64, st);
  if (e == cudaSuccess)
    e = dr::fast::launch_affine_compose_bwd(P, G, dST, sv.Pseg, Cm, dSe, dS0, st);
  if (e == cudaSuccess)
    e = dr::fast::launch_bwd_scan_tc_seg(P, sv, dO,
                                         dr::fast::ScanSeg{G, L, 0, dSe, nullptr, nullptr}, dU,
                                         dh, 64, st);
  return e;
}

size_t saved_bytes(const Problem& p) {
  const size_t generic = (size_t)p.B * p.H * p.NC * p.dv * p.dk * sizeof(float);
  const size_t fast = dr::fast::saved_bytes(p);
  return round_up(generic > fast ? generic : fast);
}

}  // namespace

extern "C" {

dr_status dr_workspace_size(const dr_problem* p, int pass, size_t* bytes) {
  Problem P;
  if (!bytes || (pass != 0 && pass != 1)) return DR_ERR_INVALID_ARG;
  dr_status s = validate(p, &P);
  if (s != DR_OK) return s;
  *bytes = layout(P, pass).total;
  return DR_OK;
}

dr_status dr_saved_size(const dr_problem* p, size_t* bytes) {
  Problem P;
  if (!bytes) return DR_ERR_INVALID_ARG;
  dr_status s = validate(p, &P);
  if (s != DR_OK) return s;
  *bytes = saved_bytes(P);
  return DR_OK;
}

dr_status dr_chunk_fwd(const dr_problem* p, const void* q, const void* k, const void* v,
                       const float* beta, const float* g, const float* S0, void* o,
                       float* ST, void* saved, void* ws, size_t ws_bytes, void* stream) {
  Problem P;
  dr_status s = validate(p, &P);
  if (s != DR_OK) return s;
  if (!q || !k || !v || !beta || !o) return DR_ERR_INVALID_ARG;
  if ((P.gate == DR_GATE_NONE) != (g == nullptr)) return DR_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, beta, g, S0, o, ST, saved};
  for (const void* x : ptrs)
    if (!aligned16(x)) return DR_ERR_INVALID_ARG;
  const Layout L = layout(P, 0);
  if (!ws || ws_bytes < L.total || ((uintptr_t)ws % kAlign)) return DR_ERR_WORKSPACE;
  const Ws w = carve(L, ws, 0);
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if (P.gate == DR_GATE_NONE) g = nullptr;
  const bool fast = dr::fast::eligible(P, p->dtype == DR_BF16);
  // the phase gate runs on the tensor-core path only
  if (P.gate == DR_GATE_PHASE && !fast) return DR_ERR_UNSUPPORTED;
  if (fast) {
    // Tensor-core path: the per-chunk tiles go to the saved buffer when given
    // (the backward reuses them), else to the workspace.
    dr::fast::Saved sv = dr::fast::carve_saved(P, saved ? saved : ws);
    using bf = __nv_bfloat16;
    char* aff = (char*)ws + round_up(dr::fast::saved_bytes(P));
    e = dr::fast::launch_prep(P, (const bf*)q, (const bf*)k, (const bf*)v, beta, g, sv, st);
    if (e == cudaSuccess)
      e = fwd_scan_any(P, sv, S0, (bf*)o, ST, saved != nullptr, aff, st);
    return e == cudaSuccess ? DR_OK : DR_ERR_CUDA;
  }
  if (p->dtype == DR_F32)
    e = dr::launch_generic_fwd<float>(P, (const float*)q, (const float*)k, (const float*)v,
                                      beta, g, S0, (float*)o, ST, (float*)saved, w, st);
  else
    e = dr::launch_generic_fwd<__nv_bfloat16>(
        P, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, beta,
        g, S0, (__nv_bfloat16*)o, ST, (float*)saved, w, st);
  return e == cudaSuccess ? DR_OK : DR_ERR_CUDA;
}

dr_status dr_decode_step(const dr_problem* p, const void* q, const void* k, const void* v,
                         const float* beta, const float* g, float* S, void* o, void* stream) {
  Problem P;
  dr_status s = validate(p, &P);
  if (s != DR_OK) return s;
  if (p->T != 1) return DR_ERR_INVALID_ARG;
  if (!q || !k || !v || !beta || !S || !o) return DR_ERR_INVALID_ARG;
  if ((P.gate == DR_GATE_NONE) != (g == nullptr)) return DR_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, beta, g, S, o};
  for (const void* x : ptrs)
    if (!aligned16(x)) return DR_ERR_INVALID_ARG;
  const cudaError_t e = dr::launch_decode_step(P, p->dtype == DR_BF16, q, k, v, beta, g, S, o,
                                               (cudaStream_t)stream);
  return e == cudaSuccess ? DR_OK : DR_ERR_CUDA;
}

dr_status dr_chunk_bwd(const dr_problem* p, const void* q, const void* k, const void* v,
                       const float* beta, const float* g, const float* S0, const void* dO,
                       const float* dST, const void* saved, void* dq, void* dk, void* dv,
                       float* dbeta, float* dg, float* dS0, void* ws, size_t ws_bytes,
                       void* stream) {
  Problem P;
  dr_status s = validate(p, &P);
  if (s != DR_OK) return s;
  if (!q || !k || !v || !beta || !dO || !dq || !dk || !dv || !dbeta)
    return DR_ERR_INVALID_ARG;
  if ((P.gate == DR_GATE_NONE) != (g == nullptr)) return DR_ERR_INVALID_ARG;
  if (P.gate != DR_GATE_NONE && !dg) return DR_ERR_INVALID_ARG;
  // the phase gate runs on the tensor-core path only
  if (P.gate == DR_GATE_PHASE && !dr::fast::eligible(P, p->dtype == DR_BF16))
    return DR_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k, v, beta, g, S0, dO, dST, saved, dq, dk, dv, dbeta, dg, dS0};
  for (const void* x : ptrs)
    if (!aligned16(x)) return DR_ERR_INVALID_ARG;
  const Layout L = layout(P, 1);
  if (!ws || ws_bytes < L.total || ((uintptr_t)ws % kAlign)) return DR_ERR_WORKSPACE;
  const Ws w = carve(L, ws, 1);
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if (dr::fast::eligible(P, p->dtype == DR_BF16)) {
    using bf = __nv_bfloat16;
    // The forward's per-chunk tensors come from its saved buffer or are
    // recomputed into the workspace.
    char* wsb = (char*)ws + round_up(dr::fast::saved_bytes(P));
    const size_t nb = (size_t)P.B * P.H * P.NC;
    bf* dU = (bf*)wsb;
    bf* dh = (bf*)(wsb + round_up(nb * dr::fast::kUBytes));
    char* aff = wsb + round_up(nb * dr::fast::kUBytes) + round_up(nb * dr::fast::kStateBytes);
    dr::fast::Saved sv;
    if (saved) {
      sv = dr::fast::carve_saved(P, (void*)saved);
    } else {
      sv = dr::fast::carve_saved(P, ws);
      e = dr::fast::launch_prep(P, (const bf*)q, (const bf*)k, (const bf*)v, beta, g, sv, st);
      if (e == cudaSuccess) e = fwd_scan_any(P, sv, S0, nullptr, nullptr, true, aff, st);
      if (e != cudaSuccess) return DR_ERR_CUDA;
    }
    e = bwd_scan_any(P, sv, (const bf*)dO, dST, dS0, dU, dh, aff, st);
    if (e == cudaSuccess) {
      e = dr::fast::launch_bwd_chunk_hy(P, (const bf*)q, (const bf*)k, (const bf*)v, (const bf*)dO, g, sv, dh, dU,
                 (bf*)dq, (bf*)dk, (bf*)dv, dbeta, dg, st);
    }
    return e == cudaSuccess ? DR_OK : DR_ERR_CUDA;
  }
  if (p->dtype == DR_F32)
    e = dr::launch_generic_bwd<float>(P, (const float*)q, (const float*)k, (const float*)v,
                                      beta, g, S0, (const float*)dO, dST,
                                      (const float*)saved, (float*)dq, (float*)dk, (float*)dv,
                                      dbeta, dg, dS0, w, st);
  else
    e = dr::launch_generic_bwd<__nv_bfloat16>(
        P, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, beta,
        g, S0, (const __nv_bfloat16*)dO, dST, (const float*)saved, (__nv_bfloat16*)dq,
        (__nv_bfloat16*)dk, (__nv_bfloat16*)dv, dbeta, dg, dS0, w, st);
  return e == cudaSuccess ? DR_OK : DR_ERR_CUDA;
}

const char* dr_status_string(dr_status s) {
  switch (s) {
    case DR_OK: return "ok";
    case DR_ERR_INVALID_ARG: return "invalid argument";
    case DR_ERR_UNSUPPORTED: return "unsupported problem (chunk must be 64; dk, dv multiples of 16 up to 128; phase gate: bf16, dk = dv = 128)";
    case DR_ERR_WORKSPACE: return "workspace or saved buffer missing, misaligned or too small";
    case DR_ERR_CUDA: return "CUDA error";
    case DR_ERR_TIMEOUT: return "a bounded device-side wait timed out";
  }
  return "unknown status";
}

dr_status dr_last_device_error(void* stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return DR_ERR_CUDA;
  int flag = 0;
  if (dr::read_and_clear_device_error(&flag) != cudaSuccess) return DR_ERR_CUDA;
  return flag ? DR_ERR_TIMEOUT : DR_OK;
}

dr_status dr_inject_timeout(int launches) {
  if (launches < 0) return DR_ERR_INVALID_ARG;
  dr::g_injected_timeouts.store(launches);
  return DR_OK;
}

int dr_version(void) { return 200; }

}  // extern "C"
