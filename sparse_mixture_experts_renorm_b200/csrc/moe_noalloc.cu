// moe_noalloc.cu — moe_forward_noalloc: the whole layer for callers that
// cannot allocate device memory, with its scratch in a fixed-size array that
// lives in this library's device image.
//
// Some callers can't call cudaMalloc while they run the layer: code inside an
// engine or plugin whose host framework owns every device allocation, or a
// serving loop that forbids allocation after warm-up so that memory use stays
// fixed. They still own the inputs and outputs; only the scratch moves into
// the static array below. Every GPU that loads the library keeps the array
// for as long as the process lives.
#include <cudaTypedefs.h>

#include <mutex>

#include "moe_internal.h"

namespace moe {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

// Device address of the array, per device, together with the unique id of
// the CUDA context it was looked up in. In host code the array's name is only
// a host-side stand-in, so the address is looked up (with that device and
// context current) and passed to the kernels as a plain pointer. A context
// that is destroyed and created again (cudaDeviceReset, or a caller that
// switches to its own context) loads the module again, possibly at another
// address, and gets a new id, so the lookup is then repeated.
struct ScratchAddr {
  unsigned long long ctx_id;
  void* addr;
};
std::mutex g_mu;
ScratchAddr g_scratch_addr[64] = {};

// The driver's cuCtxGetCurrent and cuCtxGetId through the runtime's entry
// point query (the library links only the runtime).
struct CtxFns {
  PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  PFN_cuCtxGetId_v12000 get_id = nullptr;
};
const CtxFns& ctx_fns() {
  static CtxFns f;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  return f;
}

// Unique id of the calling thread's current context, or 0 when there is none
// yet (or the driver cannot say).
unsigned long long current_ctx_id() {
  const CtxFns& f = ctx_fns();
  if (!f.get_current || !f.get_id) return 0;
  CUcontext ctx = nullptr;
  if (f.get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  unsigned long long id = 0;
  if (f.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_forward_noalloc(const void* x, const void* w_router, const float* b_router,
                                          const void* w_gate, const void* w_up, const void* w_down, int T, int d,
                                          int E, int k, int I, int renorm, moe_dtype dtype, float* out,
                                          int32_t* topk_idx, float* topk_gate, int32_t* counts, float* aux,
                                          int32_t* status_dev, void* stream) {
  const size_t need = moe_workspace_size(T, d, E, k, I, dtype);
  if (need == 0)  // invalid or unsupported shape: moe_forward reports which, before launching anything
    return moe_forward(x, w_router, b_router, w_gate, w_up, w_down, T, d, E, k, I, renorm, dtype, out, topk_idx,
                       topk_gate, counts, aux, nullptr, 0, status_dev, stream);
  if (need > (size_t)MOE_NOALLOC_SCRATCH_BYTES) {
    set_error_detail("moe_forward_noalloc: this shape needs %zu bytes of scratch but the static scratch holds %zu; "
                     "use moe_forward with a caller workspace",
                     need, (size_t)MOE_NOALLOC_SCRATCH_BYTES);
    return MOE_ERR_WORKSPACE;
  }
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) {
    set_error_detail("moe_forward_noalloc: cudaGetDevice: %s", cudaGetErrorString(err));
    return MOE_ERR_CUDA;
  }
  if (dev < 0 || dev >= 64) {
    set_error_detail("moe_forward_noalloc: device ordinal %d out of range", dev);
    return MOE_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    const unsigned long long id = current_ctx_id();
    ScratchAddr& slot = g_scratch_addr[dev];
    if (!slot.addr || id == 0 || slot.ctx_id != id) {
      void* p = nullptr;
      err = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // also makes the device's primary context current
      if (err != cudaSuccess || !p) {
        set_error_detail("moe_forward_noalloc: cudaGetSymbolAddress of the static scratch failed: %s",
                         cudaGetErrorString(err));
        return MOE_ERR_CUDA;
      }
      slot.addr = p;
      slot.ctx_id = current_ctx_id();
    }
    scratch = slot.addr;
  }
  return moe_forward(x, w_router, b_router, w_gate, w_up, w_down, T, d, E, k, I, renorm, dtype, out, topk_idx,
                     topk_gate, counts, aux, scratch, (size_t)MOE_NOALLOC_SCRATCH_BYTES, status_dev, stream);
}
