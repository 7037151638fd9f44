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
#include <mutex>

#include "moe_internal.h"

namespace moe {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

// Device address of the array on each device. In host code the array's name
// is only a host-side stand-in, so the address is looked up once per device
// (with that device current) and passed to the kernels as a plain pointer.
std::mutex g_mu;
void* g_scratch_addr[64] = {};

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
    if (!g_scratch_addr[dev]) {
      void* p = nullptr;
      err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (err != cudaSuccess || !p) {
        set_error_detail("moe_forward_noalloc: cudaGetSymbolAddress of the static scratch failed: %s",
                         cudaGetErrorString(err));
        return MOE_ERR_CUDA;
      }
      g_scratch_addr[dev] = p;
    }
    scratch = g_scratch_addr[dev];
  }
  return moe_forward(x, w_router, b_router, w_gate, w_up, w_down, T, d, E, k, I, renorm, dtype, out, topk_idx,
                     topk_gate, counts, aux, scratch, (size_t)MOE_NOALLOC_SCRATCH_BYTES, status_dev, stream);
}
