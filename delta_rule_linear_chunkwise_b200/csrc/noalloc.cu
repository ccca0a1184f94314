// noalloc.cu -- dr_chunk_fwd_static: the chunkwise forward for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all, and so cannot hand the library
// a workspace: a plugin running inside a host framework that owns every device
// allocation through its own pool and forbids others, or a latency-critical
// path where cudaMalloc's implicit device synchronisation is not acceptable.
// For them the forward's scratch lives in the file-scope device array below,
// DR_STATIC_SCRATCH_BYTES bytes that every GPU which loads this library holds
// until the process exits.  The caller still passes inputs and outputs.

#include <mutex>

#include "../../include/dr.h"
#include "dr_common.cuh"

namespace {

// The shared scratch.  In host code this name is only a host-side stand-in
// for the device array, never a device address: kernels receive the address
// that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_static_scratch[DR_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Set-up, once per device, with that device current: look up the device
// address of the scratch array (no allocation happens here).
dr_status scratch_of_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DR_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
      return DR_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return DR_OK;
}

}  // namespace

extern "C" dr_status dr_chunk_fwd_static(const dr_problem* p, const void* q, const void* k,
                                         const void* v, const float* beta, const float* g,
                                         const float* S0, void* o, float* ST, void* stream) {
  size_t need = 0;
  dr_status s = dr_workspace_size(p, 0, &need);
  if (s != DR_OK) return s;
  if (need > (size_t)DR_STATIC_SCRATCH_BYTES) return DR_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((s = scratch_of_current_device(&scratch)) != DR_OK) return s;
  // Every region the forward reads is written earlier in the same call, so
  // the previous call's leftovers in the shared scratch need no clearing.
  return dr_chunk_fwd(p, q, k, v, beta, g, S0, o, ST, nullptr, scratch,
                      (size_t)DR_STATIC_SCRATCH_BYTES, stream);
}
