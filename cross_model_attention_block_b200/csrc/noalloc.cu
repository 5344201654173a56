// Block statistics for callers that cannot allocate device memory.
//
// Some callers have no way to hand this library a workspace: a serving engine
// that reserved all free HBM for its KV-cache pool at start-up has nothing
// left to cudaMalloc, and a plain C host program with a fixed memory plan may
// have no device allocator at all.  mf_block_stats_noalloc runs the same
// kernels as mf_block_stats, with the scratch space taken from one array that
// the library keeps in device memory for its whole lifetime.
#include <cuda_runtime.h>

#include <mutex>

#include "mf_internal.h"

namespace {

// Scratch of mf_block_stats_noalloc.  Every GPU that loads the library holds
// these bytes until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[64] = {nullptr};

// Device address of the scratch array on the current device, looked up once per
// device.  Host code must not use the symbol itself: on the host it only names
// a stand-in, not device memory.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

size_t mf_block_stats_noalloc_max_workspace(void) { return kNoAllocScratchBytes; }

mf_status mf_block_stats_noalloc(const mf_attn_desc* desc, const void* Q, const void* K,
                                 float* lse, float* mass, mf_stream_t stream) {
  const size_t need = mf_block_stats_workspace(desc);
  if (need == 0) {
    // the descriptor is invalid: let the regular entry point report why
    return mf_block_stats(desc, Q, K, lse, mass, nullptr, 0, stream);
  }
  if (need > kNoAllocScratchBytes) {
    mf::set_last_error(
        "mf_block_stats_noalloc: this context needs more scratch than the 8 MiB the "
        "library holds (Hs * causal blocks * 4 bytes plus metadata); use mf_block_stats "
        "with a caller workspace");
    return MF_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) {
    mf::set_last_error("mf_block_stats_noalloc: cudaGetSymbolAddress of the scratch failed");
    return MF_ERR_CUDA;
  }
  return mf_block_stats(desc, Q, K, lse, mass, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
