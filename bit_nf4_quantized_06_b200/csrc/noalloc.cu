// qlora_linear_fwd_noalloc: the forward for callers that cannot provide a
// workspace.
//
// Some callers have no way to hand the library a scratch buffer: a runtime
// whose device memory is entirely owned by its own pool allocator, code that
// runs where a device allocation is forbidden or would stall other work
// (cudaMalloc may synchronise the device), or a plain C caller without a
// device allocator of its own. This entry point serves them with scratch
// memory the library owns: one file-scope device array of a fixed size that
// every GPU loading the library keeps until the process exits.
//
// The array's host-side name is only a stand-in for the symbol, not a device
// address, so the host resolves the real address with cudaGetSymbolAddress
// (with the device current) and passes that pointer to the existing forward
// as its workspace. The address is cached per device together with the CUDA
// context it was resolved in; when the current context differs (after a
// cudaDeviceReset the runtime makes a new primary context and loads the
// module again) it is resolved anew. Nothing here allocates or frees.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/qlora.h"
#include "kernels.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[QLORA_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
struct Resolved {
  CUcontext ctx;
  void* ptr;
};
Resolved g_noalloc[64] = {};

// Device address of the scratch array in the current device's current
// context. Returns nullptr on failure (nothing is cached then).
void* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return nullptr;
  }
  // the device check that runs before this has made the runtime's context
  // current, so this is the context the launches will use
  CUcontext ctx = qlora::current_context();
  if (ctx == nullptr) return nullptr;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  Resolved& r = g_noalloc[dev];
  if (r.ptr == nullptr || r.ctx != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      r = Resolved{nullptr, nullptr};
      return nullptr;
    }
    r = Resolved{ctx, p};
  }
  return r.ptr;
}

}  // namespace

extern "C" qlora_status_t qlora_linear_fwd_noalloc(const qlora_nf4_t* q, const void* x_bf16, int64_t m,
                                                   const void* a_bf16, const void* b_bf16, int32_t r, float alpha,
                                                   void* y_bf16, void* u_out_bf16, void* stream) {
  if (q == nullptr) return QLORA_ERR_INVALID_ARG;
  if (m == 0) {
    return qlora_linear_fwd(q, x_bf16, m, a_bf16, b_bf16, r, alpha, y_bf16, u_out_bf16, nullptr, 0, stream);
  }
  const size_t need = qlora_fwd_workspace_bytes(m, q->n_out, q->k_in, r);
  if (need == 0) return QLORA_ERR_SHAPE;
  if (need > QLORA_NOALLOC_SCRATCH_BYTES) return QLORA_ERR_WORKSPACE;  // problem too large for the fixed scratch
  // the device check every entry point runs, before the symbol lookup (which
  // fails without an sm_100 image of this module)
  const int dst = qlora::check_current_device_status();
  if (dst != QLORA_OK) return static_cast<qlora_status_t>(dst);
  void* ws = scratch_address();
  if (ws == nullptr) return QLORA_ERR_CUDA;
  return qlora_linear_fwd(q, x_bf16, m, a_bf16, b_bf16, r, alpha, y_bf16, u_out_bf16, ws,
                          QLORA_NOALLOC_SCRATCH_BYTES, stream);
}
