// moe_api.cu — the C ABI (include/moe.h): argument validation, the workspace
// layout, TMA tensor-map encoding and the launch sequence
//   router -> scan -> permute -> gate/up GEMM + SwiGLU -> down GEMM -> combine
// on the caller's stream. Nothing here synchronises the host or allocates.
#include <cudaTypedefs.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <string>

#include "moe_internal.h"

namespace moe {
namespace {

thread_local std::string g_last_error;

moe_status fail(moe_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

moe_status fail_cuda(cudaError_t err, const char* what) {
  return fail(MOE_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(err), cudaGetErrorString(err));
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape checks shared by every entry point.
moe_status check_shape(int T, int d, int E, int k, int I, moe_dtype dtype) {
  if (dtype != MOE_F32 && dtype != MOE_BF16) return fail(MOE_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T must be >= 0 (got %d)", T);
  if (d <= 0 || I <= 0 || E <= 0)
    return fail(MOE_ERR_INVALID_ARG, "d, I and E must be positive (got d=%d I=%d E=%d)", d, I, E);
  if (k <= 0) return fail(MOE_ERR_INVALID_ARG, "top_k must be positive (got %d)", k);
  if (k > E) return fail(MOE_ERR_INVALID_ARG, "top_k (%d) must be <= num_experts (%d)", k, E);
  if (E > kMaxExperts) return fail(MOE_ERR_UNSUPPORTED, "E=%d exceeds the supported maximum %d", E, kMaxExperts);
  if (k > kMaxTopK) return fail(MOE_ERR_UNSUPPORTED, "top_k=%d exceeds the supported maximum %d", k, kMaxTopK);
  if ((long long)T * k >= (1ll << 31)) return fail(MOE_ERR_UNSUPPORTED, "T*k must be < 2^31");
  if ((long long)d * I >= (1ll << 31) || (long long)E * I >= (1ll << 31) || (long long)E * d >= (1ll << 31))
    return fail(MOE_ERR_UNSUPPORTED, "d*I, E*I and E*d must be < 2^31");
  if (dtype == MOE_BF16) {
    if (d % 64 != 0 || I % 64 != 0)
      return fail(MOE_ERR_UNSUPPORTED, "bf16 path needs d %% 64 == 0 and I %% 64 == 0 (got d=%d I=%d)", d, I);
  } else {
    if (d % 4 != 0) return fail(MOE_ERR_UNSUPPORTED, "fp32 path needs d %% 4 == 0 (got d=%d)", d);
    if ((long long)T * k / kSimtBM + E > 65535)
      return fail(MOE_ERR_UNSUPPORTED, "fp32 path supports T*k up to %d", (65535 - E) * kSimtBM);
  }
  return MOE_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

void set_error_detail(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
}

Workspace workspace_layout(int T, int d, int E, int k, int I, moe_dtype dtype) {
  const size_t R = (size_t)T * k;
  const size_t nb = (size_t)router_blocks(T, MOE_F32);  // the finer blocking of the two routers
  const size_t el = dtype == MOE_BF16 ? 2 : 4;
  Workspace w;
  size_t o = 0;
  w.status = o;   o = align256(o + 4);
  w.offsets = o;  o = align256(o + 4 * (size_t)(E + 1));
  w.counts = o;   o = align256(o + 4 * (size_t)E);
  w.mtile = o;    o = align256(o + 4 * (size_t)(E + 1));
  w.aux = o;      o = align256(o + 4);
  w.blk_cnt = o;  o = align256(o + 4 * nb * E);
  w.blk_psum = o; o = align256(o + 4 * nb * E);
  w.lrank = o;    o = align256(o + 4 * R);
  w.perm_tok = o; o = align256(o + 4 * R);
  w.inv = o;      o = align256(o + 4 * R);
  w.rgate = o;    o = align256(o + 4 * R);
  w.xp = o;       o = align256(o + el * R * (size_t)d);
  w.h = o;        o = align256(o + el * R * (size_t)I);
  w.y = o;        o = align256(o + 4 * R * (size_t)d);
  w.total = o;
  return w;
}

bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode_fn();
  if (!encode) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_size(int T, int d, int E, int k, int I, moe_dtype dtype) {
  if (check_shape(T, d, E, k, I, dtype) != MOE_OK) return 0;
  return workspace_layout(T, d, E, k, I, dtype).total;
}

size_t moe_last_error_detail(char* buf, size_t n) {
  const std::string& s = g_last_error;
  if (buf && n) {
    const size_t m = s.size() < n - 1 ? s.size() : n - 1;
    memcpy(buf, s.data(), m);
    buf[m] = '\0';
  }
  return s.size();
}

namespace {

struct EventMarks {
  void* const* events;
  int n;
  int next = 0;
  cudaError_t mark(cudaStream_t s) {
    if (!events || next >= n) return cudaSuccess;
    return cudaEventRecord(static_cast<cudaEvent_t>(events[next++]), s);
  }
};

moe_status forward_impl(const void* x, const void* w_router, const float* b_router, const void* w_gate,
                        const void* w_up, const void* w_down, int T, int d, int E, int k, int I, int renorm,
                        moe_dtype dtype, float* out, int32_t* topk_idx, float* topk_gate, int32_t* counts,
                        float* aux, void* workspace, size_t workspace_bytes, int32_t* status_dev, void* stream_ptr,
                        EventMarks marks) {
  moe_status st = check_shape(T, d, E, k, I, dtype);
  if (st != MOE_OK) return st;
  if (renorm != 0 && renorm != 1) return fail(MOE_ERR_INVALID_ARG, "renorm must be 0 or 1 (got %d)", renorm);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  if (T > 0) {
    if (!x || !w_router || !w_gate || !w_up || !w_down || !out || !topk_idx || !topk_gate)
      return fail(MOE_ERR_INVALID_ARG, "a required pointer (x, weights, out, topk_idx, topk_gate) is NULL");
    if (!aligned16(x) || !aligned16(w_router) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) ||
        !aligned16(out))
      return fail(MOE_ERR_INVALID_ARG, "x, weights and out must be 16-byte aligned");
  }
  const Workspace w = workspace_layout(T, d, E, k, I, dtype);
  if (!workspace || workspace_bytes < w.total)
    return fail(MOE_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu%s)", w.total, workspace_bytes,
                workspace ? "" : ", NULL");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(MOE_ERR_INVALID_ARG, "workspace must be 256-byte aligned");

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* status = status_dev ? status_dev : reinterpret_cast<int32_t*>(ws + w.status);
  int32_t* cnt = counts ? counts : reinterpret_cast<int32_t*>(ws + w.counts);
  float* aux_p = aux ? aux : reinterpret_cast<float*>(ws + w.aux);
  cudaError_t err;
  if (!status_dev) {
    err = cudaMemsetAsync(status, 0, sizeof(int32_t), stream);
    if (err != cudaSuccess) return fail_cuda(err, "clearing the status word");
  }
  if (T == 0) {
    err = cudaMemsetAsync(ws + w.offsets, 0, sizeof(int32_t) * (E + 1), stream);
    if (err == cudaSuccess) err = cudaMemsetAsync(cnt, 0, sizeof(int32_t) * E, stream);
    if (err == cudaSuccess) err = cudaMemsetAsync(aux_p, 0, sizeof(float), stream);
    if (err != cudaSuccess) return fail_cuda(err, "zeroing counts/aux for T=0");
    return MOE_OK;
  }

  int32_t* offsets = reinterpret_cast<int32_t*>(ws + w.offsets);
  int32_t* mtile = reinterpret_cast<int32_t*>(ws + w.mtile);
  int32_t* blk_cnt = reinterpret_cast<int32_t*>(ws + w.blk_cnt);
  float* blk_psum = reinterpret_cast<float*>(ws + w.blk_psum);
  int32_t* lrank = reinterpret_cast<int32_t*>(ws + w.lrank);
  int32_t* perm_tok = reinterpret_cast<int32_t*>(ws + w.perm_tok);
  int32_t* inv = reinterpret_cast<int32_t*>(ws + w.inv);
  void* xp = ws + w.xp;
  void* h = ws + w.h;
  float* y = reinterpret_cast<float*>(ws + w.y);
  const int R = T * k;

  err = marks.mark(stream);
  if (err != cudaSuccess) return fail_cuda(err, "recording a timing event");
  err = launch_router(dtype, x, w_router, b_router, T, d, E, k, renorm, topk_idx, topk_gate, lrank, blk_cnt, blk_psum,
                      status, stream);
  if (err != cudaSuccess) return fail_cuda(err, "router kernel");
  marks.mark(stream);
  err = launch_route_scan(router_blocks(T, dtype), T, E, k, blk_cnt, blk_psum, cnt, offsets, mtile, aux_p, stream);
  if (err != cudaSuccess) return fail_cuda(err, "routing scan kernel");
  marks.mark(stream);
  // With k = 2 the bf16 path folds the combine into the down GEMM's epilogue
  // (two fp32 adds into a zeroed row commute, so the result stays
  // deterministic); otherwise a separate combine kernel sums the k rows.
  const bool fused_combine = dtype == MOE_BF16 && k == 2;
  float* rgate = reinterpret_cast<float*>(ws + w.rgate);
  err = launch_permute(dtype, x, T, d, E, k, router_block_tokens(dtype), topk_idx, lrank, blk_cnt, perm_tok, inv, xp,
                       topk_gate, rgate, fused_combine ? out : nullptr, status, stream);
  if (err != cudaSuccess) return fail_cuda(err, "permute kernel");

  if (dtype == MOE_BF16) {
    // weights are the UMMA M operand (64 gate + 64 up rows, or 128 down rows
    // per CTA), dispatched tokens the N operand (128-row boxes, 16-row boxes
    // for tiles of at most 32 tokens)
    CUtensorMap tm_wg, tm_wu, tm_wd, tm_xp, tm_xp_s, tm_h, tm_h_s;
    if (!make_tmap_bf16_2d(&tm_wg, w_gate, (uint64_t)E * I, (uint64_t)d, 64) ||
        !make_tmap_bf16_2d(&tm_wu, w_up, (uint64_t)E * I, (uint64_t)d, 64) ||
        !make_tmap_bf16_2d(&tm_wd, w_down, (uint64_t)E * d, (uint64_t)I, 128) ||
        !make_tmap_bf16_2d(&tm_xp, xp, (uint64_t)R, (uint64_t)d, 128) ||
        !make_tmap_bf16_2d(&tm_xp_s, xp, (uint64_t)R, (uint64_t)d, 16) ||
        !make_tmap_bf16_2d(&tm_h, h, (uint64_t)R, (uint64_t)I, 128) ||
        !make_tmap_bf16_2d(&tm_h_s, h, (uint64_t)R, (uint64_t)I, 16))
      return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point unavailable or bad pointer)");
    marks.mark(stream);
    err = launch_gemm_gateup_tc2(tm_wg, tm_wu, tm_xp, tm_xp_s, offsets, mtile, R, E, I, d, h, status, stream);
    if (err != cudaSuccess) return fail_cuda(err, "gate/up grouped GEMM");
    marks.mark(stream);
    err = launch_gemm_down_tc2(tm_wd, tm_h, tm_h_s, offsets, mtile, R, E, I, d, y, perm_tok, rgate,
                               fused_combine ? out : nullptr, status, stream);
    if (err != cudaSuccess) return fail_cuda(err, "down grouped GEMM");
  } else {
    marks.mark(stream);
    err = launch_gemm_gateup_simt(static_cast<const float*>(xp), static_cast<const float*>(w_gate),
                                  static_cast<const float*>(w_up), offsets, R, E, I, d, static_cast<float*>(h), stream);
    if (err != cudaSuccess) return fail_cuda(err, "gate/up grouped GEMM (fp32)");
    marks.mark(stream);
    err = launch_gemm_down_simt(static_cast<const float*>(h), static_cast<const float*>(w_down), offsets, R, E, I, d, y,
                                stream);
    if (err != cudaSuccess) return fail_cuda(err, "down grouped GEMM (fp32)");
  }
  marks.mark(stream);
  if (!fused_combine) {
    err = launch_combine(T, d, k, y, inv, topk_gate, out, status, stream);
    if (err != cudaSuccess) return fail_cuda(err, "combine kernel");
  }
  err = marks.mark(stream);
  if (err != cudaSuccess) return fail_cuda(err, "recording a timing event");
  return MOE_OK;
}

}  // namespace

moe_status moe_forward(const void* x, const void* w_router, const float* b_router, const void* w_gate,
                       const void* w_up, const void* w_down, int T, int d, int E, int k, int I, int renorm,
                       moe_dtype dtype, float* out, int32_t* topk_idx, float* topk_gate, int32_t* counts, float* aux,
                       void* workspace, size_t workspace_bytes, int32_t* status_dev, void* stream) {
  return forward_impl(x, w_router, b_router, w_gate, w_up, w_down, T, d, E, k, I, renorm, dtype, out, topk_idx,
                      topk_gate, counts, aux, workspace, workspace_bytes, status_dev, stream, EventMarks{nullptr, 0});
}

moe_status moe_forward_events(const void* x, const void* w_router, const float* b_router, const void* w_gate,
                              const void* w_up, const void* w_down, int T, int d, int E, int k, int I, int renorm,
                              moe_dtype dtype, float* out, int32_t* topk_idx, float* topk_gate, int32_t* counts,
                              float* aux, void* workspace, size_t workspace_bytes, int32_t* status_dev, void* stream,
                              void* const* events, int n_events) {
  if (!events || n_events < MOE_NUM_KERNELS + 1)
    return fail(MOE_ERR_INVALID_ARG, "moe_forward_events needs %d events (got %d)", MOE_NUM_KERNELS + 1, n_events);
  for (int i = 0; i < MOE_NUM_KERNELS + 1; ++i)
    if (!events[i]) return fail(MOE_ERR_INVALID_ARG, "event %d is NULL", i);
  return forward_impl(x, w_router, b_router, w_gate, w_up, w_down, T, d, E, k, I, renorm, dtype, out, topk_idx,
                      topk_gate, counts, aux, workspace, workspace_bytes, status_dev, stream,
                      EventMarks{events, MOE_NUM_KERNELS + 1});
}

const char* moe_kernel_name(int i) {
  static const char* names[MOE_NUM_KERNELS] = {"router_topk", "route_scan", "permute",
                                               "grouped_gemm_gateup_swiglu", "grouped_gemm_down", "combine"};
  return (i >= 0 && i < MOE_NUM_KERNELS) ? names[i] : nullptr;
}

moe_status moe_get_permutation(const void* workspace, size_t workspace_bytes, int T, int d, int E, int k, int I,
                               moe_dtype dtype, int32_t* offsets, int32_t* perm_tok, int32_t* inv, void* stream_ptr) {
  moe_status st = check_shape(T, d, E, k, I, dtype);
  if (st != MOE_OK) return st;
  const Workspace w = workspace_layout(T, d, E, k, I, dtype);
  if (!workspace || workspace_bytes < w.total)
    return fail(MOE_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", w.total, workspace_bytes);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  const uint8_t* ws = static_cast<const uint8_t*>(workspace);
  const size_t R = (size_t)T * k;
  cudaError_t err = cudaSuccess;
  if (offsets)
    err = cudaMemcpyAsync(offsets, ws + w.offsets, 4 * (size_t)(E + 1), cudaMemcpyDeviceToDevice, stream);
  if (err == cudaSuccess && perm_tok && R)
    err = cudaMemcpyAsync(perm_tok, ws + w.perm_tok, 4 * R, cudaMemcpyDeviceToDevice, stream);
  if (err == cudaSuccess && inv && R) err = cudaMemcpyAsync(inv, ws + w.inv, 4 * R, cudaMemcpyDeviceToDevice, stream);
  if (err != cudaSuccess) return fail_cuda(err, "copying the permutation");
  return MOE_OK;
}

}  // extern "C"
