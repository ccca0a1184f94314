// profile.cu -- opt-in per-kernel timing with CUDA events on the launch stream.
//
// While enabled, every kernel launch the library makes is bracketed by two
// events recorded on the stream it is launched on; dr_profile_read sums the
// elapsed times per kernel together with the kernel's work model (algorithmic
// HBM bytes and FLOPs per launch, supplied by the launcher).  Events are
// created once, when profiling is first enabled; no device memory is allocated.

#include <mutex>
#include <string.h>

#include "../../include/dr.h"
#include "dr_common.cuh"

namespace dr {
namespace {

constexpr int kMaxRecords = 8192;

struct Record {
  int kernel;
  double io_bytes, bytes, flops;
  cudaEvent_t start, stop;
};

std::mutex g_mu;
bool g_enabled = false;
bool g_events_made = false;
Record g_rec[kMaxRecords];
int g_nrec = 0;
int g_open = -1;

}  // namespace

const char* kernel_name(int id) {
  switch (id) {
    case kKIntraFwd: return "intra_fwd";
    case kKScanFwd: return "scan_fwd";
    case kKScanBwd: return "scan_bwd";
    case kKStateGrads: return "state_grads";
    case kKIntraBwd: return "intra_bwd";
    case kKTcIntraFwd: return "tc_intra_fwd";
    case kKTcScanFwd: return "tc_scan_fwd";
    case kKTcScanBwd: return "tc_scan_bwd";
    case kKTcChunkBwd: return "tc_chunk_bwd";
    case kKDecode: return "decode_step";
    case kKAffine: return "affine_compose";
  }
  return "unknown";
}

void prof_begin(int kernel, double io_bytes, double bytes, double flops, cudaStream_t st) {
  if (!g_enabled) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_nrec >= kMaxRecords) return;
  Record& r = g_rec[g_nrec];
  r.kernel = kernel;
  r.io_bytes = io_bytes;
  r.bytes = bytes;
  r.flops = flops;
  cudaEventRecord(r.start, st);
  g_open = g_nrec;
}

void prof_end(cudaStream_t st) {
  if (!g_enabled) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_open < 0) return;
  cudaEventRecord(g_rec[g_open].stop, st);
  g_open = -1;
  ++g_nrec;
}

}  // namespace dr

extern "C" {

dr_status dr_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(dr::g_mu);
  if (on && !dr::g_events_made) {
    for (int i = 0; i < dr::kMaxRecords; ++i) {
      if (cudaEventCreate(&dr::g_rec[i].start) != cudaSuccess ||
          cudaEventCreate(&dr::g_rec[i].stop) != cudaSuccess)
        return DR_ERR_CUDA;
    }
    dr::g_events_made = true;
  }
  dr::g_enabled = on != 0;
  dr::g_nrec = 0;
  dr::g_open = -1;
  return DR_OK;
}

int dr_profile_read(dr_kernel_time* out, int max_out) {
  std::lock_guard<std::mutex> lk(dr::g_mu);
  int n = 0;
  for (int i = 0; i < dr::g_nrec; ++i) {
    const dr::Record& r = dr::g_rec[i];
    float ms = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess ||
        cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess)
      return -1;
    int j = 0;
    while (j < n && strcmp(out[j].name, dr::kernel_name(r.kernel)) != 0) ++j;
    if (j == n) {
      if (n >= max_out) continue;
      memset(&out[n], 0, sizeof(out[n]));
      strncpy(out[n].name, dr::kernel_name(r.kernel), sizeof(out[n].name) - 1);
      ++n;
    }
    // running means over the kernel's launches (its launches may differ, e.g.
    // the transfer-matrix and output passes of a segmented scan)
    const double c = out[j].launches, w = 1.0 / (c + 1.0);
    out[j].launches += 1;
    out[j].ms_total += ms;
    out[j].bytes_per_launch += (r.io_bytes - out[j].bytes_per_launch) * w;
    out[j].flops_per_launch += (r.flops - out[j].flops_per_launch) * w;
    out[j].design_bytes_per_launch += (r.bytes - out[j].design_bytes_per_launch) * w;
  }
  dr::g_nrec = 0;
  return n;
}

}  // extern "C"
