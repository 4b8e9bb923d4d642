// nectar_cache_attn_lse_static: exact cached-token attention without any
// caller-provided or library-allocated workspace.
//
// Some callers cannot create device buffers of their own: code embedded in a
// host application or serving runtime whose memory manager owns the whole
// device pool (a stray cudaMalloc there fails or fragments the pool), plugin
// interfaces that hand over only input and output pointers, and decode loops
// on a latency budget that cannot afford cudaMalloc, which may synchronise
// the device.  This entry point serves them with a scratch area that is part
// of the library's own device image: a file-scope __device__ array of
// kStaticScratchBytes, which every GPU that loads the library holds until
// the process exits.
//
// The array's name in host code is only a host-side handle, not a device
// address, so the address is looked up with cudaGetSymbolAddress (with the
// device current) on the first call in each CUDA context, and the kernels
// get that device address.  A new context on the device (after
// cudaDeviceReset, say) has a new id, and its first call looks the address
// up again.
#include <cuda_runtime.h>
#include <stdio.h>

#include <mutex>

#include "../../include/nectar.h"
#include "kernels.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(NECTAR_STATIC_SCRATCH_BYTES);

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
struct ScratchAddr {
  unsigned long long ctx = 0;   // id of the context the address belongs to
  void* addr = nullptr;
};
ScratchAddr g_scratch_addr[kMaxDevices];

}  // namespace

extern "C" {

NECTAR_API size_t nectar_static_scratch_bytes(void) { return kStaticScratchBytes; }

NECTAR_API nectar_status nectar_cache_attn_lse_static(nectar_dims dims, const nectar_bf16* K, const nectar_bf16* V,
                                                      int64_t n, const nectar_bf16* Q, int64_t nq, float scale,
                                                      float* alpha, float* A, nectar_stream_t stream) {
  // Same validation and kernels as nectar_cache_attn_lse; only the scratch differs.
  const size_t need = nectar_cache_attn_workspace_size(dims, n, nq);
  if (need > kStaticScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof msg,
             "nectar_cache_attn_lse_static: this call needs %zu bytes of scratch, the static area holds %zu "
             "(use nectar_cache_attn_lse with a caller workspace)",
             need, kStaticScratchBytes);
    nectar::set_last_error(msg);
    return NECTAR_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if (need > 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
      nectar::set_last_error("nectar_cache_attn_lse_static: no usable current CUDA device");
      return NECTAR_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    ScratchAddr& c = g_scratch_addr[dev];
    const unsigned long long ctx = nectar::current_context_id();
    if (c.addr == nullptr || ctx == 0 || c.ctx != ctx) {
      void* addr = nullptr;
      // also makes the device's primary context current if none is
      const cudaError_t e = cudaGetSymbolAddress(&addr, g_static_scratch);
      if (e != cudaSuccess || addr == nullptr) {
        char msg[256];
        snprintf(msg, sizeof msg, "nectar_cache_attn_lse_static: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        nectar::set_last_error(msg);
        return NECTAR_ERR_CUDA;
      }
      c.addr = addr;
      c.ctx = nectar::current_context_id();
    }
    scratch = c.addr;
  }
  return nectar_cache_attn_lse(dims, K, V, n, Q, nq, scale, alpha, A, scratch, need > 0 ? kStaticScratchBytes : 0,
                               stream);
}

}  // extern "C"
