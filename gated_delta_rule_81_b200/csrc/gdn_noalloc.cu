// gdn_prefill_noalloc: the uniform-length prefill for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc or any allocating library routine: code
// that runs inside a fixed memory budget handed to it by a host framework, an
// allocator hook that must not re-enter the allocator, or a pre-planned
// inference runtime whose memory plan is fixed before the first launch.  For
// them this entry point takes the same inputs and outputs as gdn_prefill but
// no workspace: the prefill's scratch lives in a file-scope device array of
// GDN_NOALLOC_SCRATCH_BYTES that the CUDA runtime places on every GPU that
// loads this library, and that stays there until the process exits.
//
// The array's name in host code is only a host-side stand-in for the device
// symbol, so its device address is looked up with cudaGetSymbolAddress, once
// per device, with that device current, on the first call made on that
// device; the lookup's return code is checked.
#include <mutex>

#include "../../include/gdn.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[GDN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDevices] = {};

// device address of the scratch array on the current device (set up on first use)
gdn_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GDN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GDN_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return GDN_OK;
}

}  // namespace

extern "C" gdn_status gdn_prefill_noalloc(const gdn_inputs* in, int B, int T, const float* state_in,
                                          float* state_out, const void* conv_in, void* conv_out, void* out,
                                          int* err, void* stream) {
  if (!in || B < 0 || T < 0) return GDN_ERR_INVALID_ARG;
  const long long n_chunks = static_cast<long long>(B) * ((T + GDN_CHUNK - 1) / GDN_CHUNK);
  const size_t need = gdn_prefill_workspace_size(in->H_k, in->H_v, B, n_chunks);
  if (need == 0) return GDN_ERR_INVALID_ARG;
  if (need > static_cast<size_t>(GDN_NOALLOC_SCRATCH_BYTES)) return GDN_ERR_WORKSPACE;
  void* scratch = nullptr;
  const gdn_status st = scratch_for_current_device(&scratch);
  if (st != GDN_OK) return st;
  // No byte of the scratch has to start at zero: every byte the kernels read
  // is written earlier in the same call.
  return gdn_prefill(in, B, T, state_in, state_out, conv_in, conv_out, out, scratch,
                     static_cast<size_t>(GDN_NOALLOC_SCRATCH_BYTES), err, stream);
}
