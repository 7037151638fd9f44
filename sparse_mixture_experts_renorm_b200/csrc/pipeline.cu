// pipeline.cu — moe_pipeline_*: repeated calls of one layer on batches that
// live in host memory, with the copies of neighbouring batches overlapped
// with the compute (host-side runtime; the kernels are moe_forward_ex's).
//
// Three streams: copy-in, compute (the caller's), copy-out. Two device
// staging slots (x, out, aux; supplied by the caller) alternate between
// batches, so batch i+1 is copied in and batch i-1 copied out while batch i
// computes. Events order the streams:
//   copy-in of batch i   waits until batch i-2 no longer reads its x slot
//   compute of batch i   waits for its copy-in, and for the copy-out of
//                        batch i-2 (which read the same out slot)
//   copy-out of batch i  waits for its compute
// The library allocates no device memory here either: streams and events
// are the only resources it creates, and moe_pipeline_destroy releases them.
#include <new>

#include "moe_internal.h"

struct moe_pipeline {
  moe_layer_desc desc;
  moe_options opt;
  bool has_opt;
  size_t x_bytes, out_bytes;
  cudaStream_t compute, h2d, d2h;
  cudaEvent_t in_ready[2], computed[2], out_free[2];
  long long n;  // batches submitted
};

namespace {

using moe::set_error_detail;

moe_status cuda_fail(cudaError_t err, const char* what) {
  set_error_detail("%s: %s (%s)", what, cudaGetErrorName(err), cudaGetErrorString(err));
  return MOE_ERR_CUDA;
}

void release(moe_pipeline* p) {
  for (int b = 0; b < 2; ++b) {
    if (p->in_ready[b]) cudaEventDestroy(p->in_ready[b]);
    if (p->computed[b]) cudaEventDestroy(p->computed[b]);
    if (p->out_free[b]) cudaEventDestroy(p->out_free[b]);
  }
  if (p->h2d) cudaStreamDestroy(p->h2d);
  if (p->d2h) cudaStreamDestroy(p->d2h);
  delete p;
}

}  // namespace

extern "C" {

moe_status moe_pipeline_create(const moe_layer_desc* desc, void* compute_stream, moe_pipeline** out) {
  if (!out) {
    set_error_detail("moe_pipeline_create: out is NULL");
    return MOE_ERR_INVALID_ARG;
  }
  *out = nullptr;
  if (!desc || desc->struct_bytes < sizeof(moe_layer_desc)) {
    set_error_detail("moe_pipeline_create: desc is NULL or its struct_bytes is below %zu", sizeof(moe_layer_desc));
    return MOE_ERR_INVALID_ARG;
  }
  // the shape, options and buffers go through the same checks as a call
  if (moe_launch_plan(desc->T, desc->d, desc->E, desc->k, desc->I, desc->dtype, desc->opt) < 0)
    return MOE_ERR_INVALID_ARG;
  for (int b = 0; b < 2; ++b)
    if (desc->T > 0 && (!desc->x_dev[b] || !desc->out_dev[b] || !desc->aux_dev[b])) {
      set_error_detail("moe_pipeline_create: the device slots x_dev, out_dev and aux_dev must not be NULL");
      return MOE_ERR_INVALID_ARG;
    }
  moe_pipeline* p = new (std::nothrow) moe_pipeline();
  if (!p) {
    set_error_detail("moe_pipeline_create: out of host memory");
    return MOE_ERR_INVALID_ARG;
  }
  p->desc = *desc;
  p->has_opt = desc->opt != nullptr;
  if (p->has_opt) p->opt = *desc->opt;  // the caller's struct need not outlive the call
  p->desc.opt = nullptr;
  p->x_bytes = (size_t)desc->T * desc->d * (desc->dtype == MOE_BF16 ? 2 : 4);
  p->out_bytes = (size_t)desc->T * desc->d * sizeof(float);
  p->compute = static_cast<cudaStream_t>(compute_stream);
  cudaError_t err = cudaStreamCreateWithFlags(&p->h2d, cudaStreamNonBlocking);
  if (err == cudaSuccess) err = cudaStreamCreateWithFlags(&p->d2h, cudaStreamNonBlocking);
  for (int b = 0; b < 2 && err == cudaSuccess; ++b) {
    err = cudaEventCreateWithFlags(&p->in_ready[b], cudaEventDisableTiming);
    if (err == cudaSuccess) err = cudaEventCreateWithFlags(&p->computed[b], cudaEventDisableTiming);
    if (err == cudaSuccess) err = cudaEventCreateWithFlags(&p->out_free[b], cudaEventDisableTiming);
  }
  if (err != cudaSuccess) {
    release(p);
    return cuda_fail(err, "moe_pipeline_create");
  }
  *out = p;
  return MOE_OK;
}

moe_status moe_pipeline_submit(moe_pipeline* p, const void* x_host, float* out_host, float* aux_host) {
  if (!p || (p->desc.T > 0 && (!x_host || !out_host))) {
    set_error_detail("moe_pipeline_submit: pipeline, x_host and out_host must not be NULL");
    return MOE_ERR_INVALID_ARG;
  }
  const moe_layer_desc& L = p->desc;
  const int b = (int)(p->n & 1);
  cudaError_t err = cudaSuccess;
  if (p->n >= 2) err = cudaStreamWaitEvent(p->h2d, p->computed[b], 0);  // slot b's x no longer read
  if (err == cudaSuccess && p->x_bytes)
    err = cudaMemcpyAsync(L.x_dev[b], x_host, p->x_bytes, cudaMemcpyHostToDevice, p->h2d);
  if (err == cudaSuccess) err = cudaEventRecord(p->in_ready[b], p->h2d);
  if (err == cudaSuccess) err = cudaStreamWaitEvent(p->compute, p->in_ready[b], 0);
  if (err == cudaSuccess && p->n >= 2) err = cudaStreamWaitEvent(p->compute, p->out_free[b], 0);
  if (err != cudaSuccess) return cuda_fail(err, "moe_pipeline_submit (copy in)");
  const moe_status st = moe_forward_ex(L.x_dev[b], L.w_router, L.b_router, L.w_gate, L.w_up, L.w_down, L.T, L.d, L.E,
                                       L.k, L.I, L.renorm, L.dtype, p->has_opt ? &p->opt : nullptr, L.out_dev[b],
                                       L.topk_idx, L.topk_gate, L.counts, L.aux_dev[b], L.workspace,
                                       L.workspace_bytes, L.status_dev, p->compute, nullptr, 0);
  if (st != MOE_OK) return st;
  err = cudaEventRecord(p->computed[b], p->compute);
  if (err == cudaSuccess) err = cudaStreamWaitEvent(p->d2h, p->computed[b], 0);
  if (err == cudaSuccess && p->out_bytes)
    err = cudaMemcpyAsync(out_host, L.out_dev[b], p->out_bytes, cudaMemcpyDeviceToHost, p->d2h);
  if (err == cudaSuccess && aux_host)
    err = cudaMemcpyAsync(aux_host, L.aux_dev[b], sizeof(float), cudaMemcpyDeviceToHost, p->d2h);
  if (err == cudaSuccess) err = cudaEventRecord(p->out_free[b], p->d2h);
  if (err != cudaSuccess) return cuda_fail(err, "moe_pipeline_submit (copy out)");
  ++p->n;
  return MOE_OK;
}

moe_status moe_pipeline_synchronize(moe_pipeline* p) {
  if (!p) {
    set_error_detail("moe_pipeline_synchronize: pipeline is NULL");
    return MOE_ERR_INVALID_ARG;
  }
  cudaError_t err = cudaStreamSynchronize(p->d2h);
  if (err == cudaSuccess) err = cudaStreamSynchronize(p->compute);
  if (err == cudaSuccess) err = cudaStreamSynchronize(p->h2d);
  return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_pipeline_synchronize");
}

void* moe_pipeline_stream(const moe_pipeline* p, int which) {
  if (!p) return nullptr;
  switch (which) {
    case MOE_PIPELINE_COPY_IN: return p->h2d;
    case MOE_PIPELINE_COMPUTE: return p->compute;
    case MOE_PIPELINE_COPY_OUT: return p->d2h;
    default: return nullptr;
  }
}

moe_status moe_pipeline_destroy(moe_pipeline* p) {
  if (!p) return MOE_OK;
  const moe_status st = moe_pipeline_synchronize(p);
  release(p);
  return st;
}

}  // extern "C"
