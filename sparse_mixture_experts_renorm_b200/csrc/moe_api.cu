// moe_api.cu — the C ABI (include/moe.h): argument validation, the workspace
// layout, TMA tensor-map encoding and the launch sequence
//   router -> scan -> permute -> gate/up GEMM + SwiGLU -> down GEMM -> combine
// on the caller's stream. Nothing here synchronises the host or allocates.
#include <cudaTypedefs.h>
#include <math.h>
#include <nvtx3/nvToolsExt.h>
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

Workspace workspace_layout(int T, int d, int E, int k, int I, moe_dtype dtype, int n_shared, bool norm) {
  const size_t R = (size_t)T * k;
  const size_t Rx = R + (n_shared > 0 ? (size_t)T : 0);  // dispatched rows + one copy for the shared experts
  const size_t Rh = R + (size_t)n_shared * T;             // hidden / output rows: routed, then shared
  const size_t nb = (size_t)router_blocks(T, MOE_F32);    // the finer blocking of the two routers
  const size_t el = dtype == MOE_BF16 ? 2 : 4;
  Workspace w;
  size_t o = 0;
  w.status = o;   o = align256(o + 4);
  w.offsets = o;  o = align256(o + 4 * (size_t)(E + 1));
  w.counts = o;   o = align256(o + 4 * (size_t)E);
  w.mtile = o;    o = align256(o + 4 * (size_t)(E + 1 + kMaxShared));
  w.aux = o;      o = align256(o + 4);
  w.blk_cnt = o;  o = align256(o + 4 * nb * E);
  w.blk_psum = o; o = align256(o + 4 * nb * E);
  w.lrank = o;    o = align256(o + 4 * R);
  w.perm_tok = o; o = align256(o + 4 * R);
  w.inv = o;      o = align256(o + 4 * R);
  w.rgate = o;    o = align256(o + 4 * R);
  w.xp = o;       o = align256(o + el * Rx * (size_t)d);
  w.h = o;        o = align256(o + el * Rh * (size_t)I);
  w.y = o;        o = align256(o + 4 * Rh * (size_t)d);
  w.blk_z = o;    o = align256(o + 4 * nb);
  w.zloss = o;    o = align256(o + 4);
  w.dropped = o;  o = align256(o + 4);
  w.rnorm = o;    o = align256(o + (norm ? 4 * (size_t)T : 0));
  w.wr_hi = o;    o = align256(o + (norm && dtype == MOE_BF16 ? 2 * (size_t)E * d : 0));
  w.wr_lo = o;    o = align256(o + (norm && dtype == MOE_BF16 ? 2 * (size_t)E * d : 0));
  // token tiles of both GEMMs: at most (rows / 256) + one partial tile per group
  w.n_mt = (R + (size_t)kMaxShared * T) / kTileM + (size_t)E + kMaxShared + 1;
  w.mt_done = o;  o = align256(o + 4 * w.n_mt);
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

namespace {

// The options after validation (defaults: the plain layer).
struct Opts {
  int norm_form = 0;
  float norm_eps = 0.f;
  const void* norm_w = nullptr;
  int n_shared = 0;
  const void* sg = nullptr;
  const void* su = nullptr;
  const void* sd = nullptr;
  double cf = 0.0;
  int32_t* dropped = nullptr;
  float* zloss = nullptr;
  bool fold_combine = false;
};

moe_status parse_options(const moe_options* opt, int T, int d, int k, int I, Opts* o) {
  *o = Opts();
  if (!opt) return MOE_OK;
  if (opt->struct_bytes < sizeof(moe_options))
    return fail(MOE_ERR_INVALID_ARG, "moe_options.struct_bytes is %zu, expected %zu", opt->struct_bytes,
                sizeof(moe_options));
  if (opt->norm_form != MOE_NORM_NONE && opt->norm_form != MOE_NORM_RMS && opt->norm_form != MOE_NORM_RMS_EPS_OUTSIDE)
    return fail(MOE_ERR_INVALID_ARG, "unknown norm_form %d", opt->norm_form);
  if (opt->norm_form != MOE_NORM_NONE && !(opt->norm_eps >= 0.f && opt->norm_eps <= 3.0e38f))
    return fail(MOE_ERR_INVALID_ARG, "norm_eps must be finite and >= 0");
  if (opt->norm_form != MOE_NORM_NONE && opt->norm_weight && !aligned16(opt->norm_weight))
    return fail(MOE_ERR_INVALID_ARG, "norm_weight must be 16-byte aligned");
  if (opt->n_shared < 0 || opt->n_shared > MOE_MAX_SHARED)
    return fail(MOE_ERR_INVALID_ARG, "n_shared must be within 0..%d (got %d)", MOE_MAX_SHARED, opt->n_shared);
  if (opt->n_shared > 0 && T > 0) {
    if (!opt->shared_gate || !opt->shared_up || !opt->shared_down)
      return fail(MOE_ERR_INVALID_ARG, "shared expert weights must not be NULL when n_shared > 0");
    if (!aligned16(opt->shared_gate) || !aligned16(opt->shared_up) || !aligned16(opt->shared_down))
      return fail(MOE_ERR_INVALID_ARG, "shared expert weights must be 16-byte aligned");
  }
  if ((long long)T * (k + opt->n_shared) >= (1ll << 31) || (long long)opt->n_shared * I * d >= (1ll << 31))
    return fail(MOE_ERR_UNSUPPORTED, "T*(k+n_shared) and n_shared*I*d must be < 2^31");
  if (!(opt->capacity_factor >= 0.0 && opt->capacity_factor <= 1e300))
    return fail(MOE_ERR_INVALID_ARG, "capacity_factor must be finite and >= 0");
  o->norm_form = opt->norm_form;
  o->norm_eps = opt->norm_eps;
  o->norm_w = opt->norm_form != MOE_NORM_NONE ? opt->norm_weight : nullptr;
  o->n_shared = opt->n_shared;
  o->sg = opt->shared_gate;
  o->su = opt->shared_up;
  o->sd = opt->shared_down;
  o->cf = opt->capacity_factor;
  o->dropped = opt->dropped;
  o->zloss = opt->z_loss;
  o->fold_combine = opt->fold_combine != 0;
  return MOE_OK;
}

// The combine runs in the down GEMM's epilogue as fp32 atomic adds into the
// zeroed output (bf16 path, no shared experts, whose rows the combine kernel
// adds): always for k = 2, where the two additions into zero commute and the
// result is deterministic, and for every k when the caller allows the
// run-to-run order of the additions (fold_combine).
bool combine_folded(moe_dtype dtype, int k, const Opts& o) {
  return dtype == MOE_BF16 && o.n_shared == 0 && (k == 2 || o.fold_combine);
}

// Assignments an expert keeps: ceil(cf * T * k / E), clamped to T (an expert
// never receives more than T); -1 without a capacity.
int capacity_of(double cf, int T, int k, int E) {
  if (!(cf > 0.0)) return -1;
  const double c = ceil(cf * (double)T * (double)k / (double)E);
  return c >= (double)T ? T : (int)c;
}

// NVTX range on the host thread for one call and one range per kernel
// launch, so a timeline tool (Nsight Systems) can tie each kernel to the call
// and step that issued it. Without an attached tool the push and pop return
// at once.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

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
                        moe_dtype dtype, const Opts& o, float* out, int32_t* topk_idx, float* topk_gate,
                        int32_t* counts, float* aux, void* workspace, size_t workspace_bytes, int32_t* status_dev,
                        void* stream_ptr, EventMarks marks) {
  NvtxRange call_range("moe_forward");
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
  const bool norm = o.norm_form != MOE_NORM_NONE;
  const Workspace w = workspace_layout(T, d, E, k, I, dtype, o.n_shared, norm);
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
    if (err == cudaSuccess && o.zloss) err = cudaMemsetAsync(o.zloss, 0, sizeof(float), stream);
    if (err == cudaSuccess && o.dropped) err = cudaMemsetAsync(o.dropped, 0, sizeof(int32_t), stream);
    if (err != cudaSuccess) return fail_cuda(err, "zeroing counts and statistics for T=0");
    return MOE_OK;
  }

  int32_t* offsets = reinterpret_cast<int32_t*>(ws + w.offsets);
  int32_t* mtile = reinterpret_cast<int32_t*>(ws + w.mtile);
  int32_t* blk_cnt = reinterpret_cast<int32_t*>(ws + w.blk_cnt);
  float* blk_psum = reinterpret_cast<float*>(ws + w.blk_psum);
  int32_t* lrank = reinterpret_cast<int32_t*>(ws + w.lrank);
  int32_t* perm_tok = reinterpret_cast<int32_t*>(ws + w.perm_tok);
  int32_t* inv = reinterpret_cast<int32_t*>(ws + w.inv);
  float* rgate = reinterpret_cast<float*>(ws + w.rgate);
  void* xp = ws + w.xp;
  void* h = ws + w.h;
  float* y = reinterpret_cast<float*>(ws + w.y);
  float* rnorm = norm ? reinterpret_cast<float*>(ws + w.rnorm) : nullptr;
  const int R = T * k;
  const int Rx = R + (o.n_shared > 0 ? T : 0);
  const int Rh = R + o.n_shared * T;
  const int cap = capacity_of(o.cf, T, k, E);

  err = marks.mark(stream);
  if (err != cudaSuccess) return fail_cuda(err, "recording a timing event");
  RouterNorm rn;
  rn.form = o.norm_form;
  rn.eps = o.norm_eps;
  rn.w = dtype == MOE_F32 ? o.norm_w : nullptr;
  rn.w_hi = nullptr;
  rn.w_lo = nullptr;
  rn.rnorm = rnorm;
  if (norm && dtype == MOE_BF16 && o.norm_w) {
    rn.w_hi = ws + w.wr_hi;
    rn.w_lo = ws + w.wr_lo;
    NvtxRange r("split_router_weight");
    err = launch_split_router_weight(w_router, o.norm_w, E, d, ws + w.wr_hi, ws + w.wr_lo, stream);
    if (err != cudaSuccess) return fail_cuda(err, "router weight split kernel");
  }
  float* blk_z = o.zloss ? reinterpret_cast<float*>(ws + w.blk_z) : nullptr;
  const bool fused_gemms = gemms_fused(T, dtype);
  int32_t* mt_done = fused_gemms ? reinterpret_cast<int32_t*>(ws + w.mt_done) : nullptr;
  // a batch of one router block: the router also does the routing scan
  const bool router_scan = router_does_scan(T, E, dtype);
  RouterScan rs;
  rs.counts = cnt;
  rs.offsets = offsets;
  rs.mtile = mtile;
  rs.aux = aux_p;
  rs.zloss = o.zloss;
  rs.dropped = o.dropped;
  rs.mt_done = mt_done;
  rs.n_mt = mt_done ? (int)w.n_mt : 0;
  rs.cap = cap;
  rs.n_shared = o.n_shared;
  {
    NvtxRange r("router_topk");
    err = launch_router(dtype, x, w_router, b_router, T, d, E, k, renorm, rn, topk_idx, topk_gate, lrank, blk_cnt,
                        blk_psum, blk_z, rs, status, stream);
  }
  if (err != cudaSuccess) return fail_cuda(err, "router kernel");
  marks.mark(stream);
  const int nb = router_blocks(T, dtype);
  const bool permute_scan = !router_scan && permute_does_scan(nb, E);
  PermuteScanArgs ps;
  if (permute_scan) {
    ps.nb = nb;
    ps.cap = cap;
    ps.n_shared = o.n_shared;
    ps.n_mt = mt_done ? (int)w.n_mt : 0;
    ps.blk_psum = blk_psum;
    ps.blk_z = blk_z;
    ps.counts = cnt;
    ps.offsets = offsets;
    ps.mtile = mtile;
    ps.aux = aux_p;
    ps.zloss = o.zloss;
    ps.dropped = o.dropped;
    ps.mt_done = mt_done;
  }
  if (!router_scan && !permute_scan) {
    NvtxRange r("route_scan");
    err = launch_route_scan(router_blocks(T, dtype), T, E, k, cap, o.n_shared, blk_cnt, blk_psum, blk_z, cnt,
                            offsets, mtile, aux_p, o.zloss, o.dropped, mt_done, (int)w.n_mt, stream);
  }
  if (err != cudaSuccess) return fail_cuda(err, "routing scan kernel");
  marks.mark(stream);
  // With k = 2 (and no shared experts) the bf16 path folds the combine into
  // the down GEMM's epilogue (two fp32 adds into a zeroed row commute, so the
  // result stays deterministic), and for any k with fold_combine; otherwise a
  // separate combine kernel sums the rows in a fixed order.
  const bool fused_combine = combine_folded(dtype, k, o);
  {
    NvtxRange r("permute");
    err = launch_permute(dtype, x, T, d, E, k, router_block_tokens(dtype), topk_idx, lrank, blk_cnt, offsets,
                         cap >= 0 ? 1 : 0, perm_tok, inv, xp, topk_gate, rgate, fused_combine ? out : nullptr, rnorm,
                         o.norm_w, o.n_shared > 0 ? R : -1, ps, status, stream);
  }
  if (err != cudaSuccess) return fail_cuda(err, "permute kernel");

  // shared experts: gate/up read the one copy of x at rows R..R+T-1 and write
  // hidden rows R + s*T; down reads and writes rows R + s*T
  const SharedGroups sh_up{o.n_shared, T, R, 0, R};
  const SharedGroups sh_down{o.n_shared, T, R, T, R};
  if (dtype == MOE_BF16) {
    // weights are the UMMA M operand (64 gate + 64 up rows, or 128 down rows
    // per CTA), dispatched tokens the N operand (128-row boxes, 16-row boxes
    // for tiles of at most 32 tokens)
    CUtensorMap tm_wg, tm_wu, tm_wd, tm_sg, tm_su, tm_sd, tm_xp, tm_xp_s, tm_h, tm_h_s;
    const bool sh = o.n_shared > 0;
    const uint64_t ns = (uint64_t)(sh ? o.n_shared : E);
    if (!make_tmap_bf16_2d(&tm_wg, w_gate, (uint64_t)E * I, (uint64_t)d, 64) ||
        !make_tmap_bf16_2d(&tm_wu, w_up, (uint64_t)E * I, (uint64_t)d, 64) ||
        !make_tmap_bf16_2d(&tm_wd, w_down, (uint64_t)E * d, (uint64_t)I, 128) ||
        !make_tmap_bf16_2d(&tm_sg, sh ? o.sg : w_gate, ns * I, (uint64_t)d, 64) ||
        !make_tmap_bf16_2d(&tm_su, sh ? o.su : w_up, ns * I, (uint64_t)d, 64) ||
        !make_tmap_bf16_2d(&tm_sd, sh ? o.sd : w_down, ns * d, (uint64_t)I, 128) ||
        !make_tmap_bf16_2d(&tm_xp, xp, (uint64_t)Rx, (uint64_t)d, 128) ||
        !make_tmap_bf16_2d(&tm_xp_s, xp, (uint64_t)Rx, (uint64_t)d, 16) ||
        !make_tmap_bf16_2d(&tm_h, h, (uint64_t)Rh, (uint64_t)I, 128) ||
        !make_tmap_bf16_2d(&tm_h_s, h, (uint64_t)Rh, (uint64_t)I, 16))
      return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point unavailable or bad pointer)");
    marks.mark(stream);
    if (fused_gemms) {
      // both projections in one launch (the down slot of the timing events
      // is then empty)
      {
        NvtxRange r("grouped_gemm_gateup_down");
        err = launch_gemm_fused_tc2(tm_wg, tm_wu, tm_sg, tm_su, tm_xp_s, tm_wd, tm_sd, tm_h_s, offsets, mtile, Rh, E,
                                    sh_up, sh_down, I, d, h, y, perm_tok, rgate, fused_combine ? out : nullptr,
                                    mt_done, status, stream);
      }
      if (err != cudaSuccess) return fail_cuda(err, "fused gate/up + down grouped GEMMs");
      marks.mark(stream);
    } else {
      {
        NvtxRange r("grouped_gemm_gateup_swiglu");
        err = launch_gemm_gateup_tc2(tm_wg, tm_wu, tm_sg, tm_su, tm_xp, tm_xp_s, offsets, mtile, Rh, E, sh_up, I, d,
                                     h, status, stream);
      }
      if (err != cudaSuccess) return fail_cuda(err, "gate/up grouped GEMM");
      marks.mark(stream);
      {
        NvtxRange r("grouped_gemm_down");
        err = launch_gemm_down_tc2(tm_wd, tm_sd, tm_h, tm_h_s, offsets, mtile, Rh, E, sh_down, I, d, y, perm_tok,
                                   rgate, fused_combine ? out : nullptr, status, stream);
      }
      if (err != cudaSuccess) return fail_cuda(err, "down grouped GEMM");
    }
  } else {
    marks.mark(stream);
    {
      NvtxRange r("grouped_gemm_gateup_swiglu");
      err = launch_gemm_gateup_simt(static_cast<const float*>(xp), static_cast<const float*>(w_gate),
                                    static_cast<const float*>(w_up), static_cast<const float*>(o.sg),
                                    static_cast<const float*>(o.su), offsets, Rh, E, sh_up, I, d,
                                    static_cast<float*>(h), stream);
    }
    if (err != cudaSuccess) return fail_cuda(err, "gate/up grouped GEMM (fp32)");
    marks.mark(stream);
    {
      NvtxRange r("grouped_gemm_down");
      err = launch_gemm_down_simt(static_cast<const float*>(h), static_cast<const float*>(w_down),
                                  static_cast<const float*>(o.sd), offsets, Rh, E, sh_down, I, d, y, stream);
    }
    if (err != cudaSuccess) return fail_cuda(err, "down grouped GEMM (fp32)");
  }
  marks.mark(stream);
  if (!fused_combine) {
    NvtxRange r("combine");
    err = launch_combine(T, d, k, y, inv, topk_gate, cap >= 0 ? 1 : 0, o.n_shared, R, out, status, stream);
    if (err != cudaSuccess) return fail_cuda(err, "combine kernel");
  }
  err = marks.mark(stream);
  if (err != cudaSuccess) return fail_cuda(err, "recording a timing event");
  return MOE_OK;
}

moe_status check_events(void* const* events, int n_events) {
  if (!events || n_events < MOE_NUM_KERNELS + 1)
    return fail(MOE_ERR_INVALID_ARG, "timing needs %d events (got %d)", MOE_NUM_KERNELS + 1, n_events);
  for (int i = 0; i < MOE_NUM_KERNELS + 1; ++i)
    if (!events[i]) return fail(MOE_ERR_INVALID_ARG, "event %d is NULL", i);
  return MOE_OK;
}

}  // namespace

extern "C" {

size_t moe_workspace_size(int T, int d, int E, int k, int I, moe_dtype dtype) {
  if (check_shape(T, d, E, k, I, dtype) != MOE_OK) return 0;
  return workspace_layout(T, d, E, k, I, dtype).total;
}

size_t moe_workspace_size_ex(int T, int d, int E, int k, int I, moe_dtype dtype, const moe_options* opt) {
  if (check_shape(T, d, E, k, I, dtype) != MOE_OK) return 0;
  Opts o;
  if (parse_options(opt, T, d, k, I, &o) != MOE_OK) return 0;
  return workspace_layout(T, d, E, k, I, dtype, o.n_shared, o.norm_form != MOE_NORM_NONE).total;
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

moe_status moe_forward(const void* x, const void* w_router, const float* b_router, const void* w_gate,
                       const void* w_up, const void* w_down, int T, int d, int E, int k, int I, int renorm,
                       moe_dtype dtype, float* out, int32_t* topk_idx, float* topk_gate, int32_t* counts, float* aux,
                       void* workspace, size_t workspace_bytes, int32_t* status_dev, void* stream) {
  return forward_impl(x, w_router, b_router, w_gate, w_up, w_down, T, d, E, k, I, renorm, dtype, Opts(), out,
                      topk_idx, topk_gate, counts, aux, workspace, workspace_bytes, status_dev, stream,
                      EventMarks{nullptr, 0});
}

moe_status moe_forward_events(const void* x, const void* w_router, const float* b_router, const void* w_gate,
                              const void* w_up, const void* w_down, int T, int d, int E, int k, int I, int renorm,
                              moe_dtype dtype, float* out, int32_t* topk_idx, float* topk_gate, int32_t* counts,
                              float* aux, void* workspace, size_t workspace_bytes, int32_t* status_dev, void* stream,
                              void* const* events, int n_events) {
  moe_status st = check_events(events, n_events);
  if (st != MOE_OK) return st;
  return forward_impl(x, w_router, b_router, w_gate, w_up, w_down, T, d, E, k, I, renorm, dtype, Opts(), out,
                      topk_idx, topk_gate, counts, aux, workspace, workspace_bytes, status_dev, stream,
                      EventMarks{events, MOE_NUM_KERNELS + 1});
}

moe_status moe_forward_ex(const void* x, const void* w_router, const float* b_router, const void* w_gate,
                          const void* w_up, const void* w_down, int T, int d, int E, int k, int I, int renorm,
                          moe_dtype dtype, const moe_options* opt, float* out, int32_t* topk_idx, float* topk_gate,
                          int32_t* counts, float* aux, void* workspace, size_t workspace_bytes, int32_t* status_dev,
                          void* stream, void* const* events, int n_events) {
  moe_status st = check_shape(T, d, E, k, I, dtype);
  if (st != MOE_OK) return st;
  Opts o;
  st = parse_options(opt, T, d, k, I, &o);
  if (st != MOE_OK) return st;
  if (events || n_events) {
    st = check_events(events, n_events);
    if (st != MOE_OK) return st;
  }
  return forward_impl(x, w_router, b_router, w_gate, w_up, w_down, T, d, E, k, I, renorm, dtype, o, out, topk_idx,
                      topk_gate, counts, aux, workspace, workspace_bytes, status_dev, stream,
                      EventMarks{events, events ? MOE_NUM_KERNELS + 1 : 0});
}

int moe_launch_plan(int T, int d, int E, int k, int I, moe_dtype dtype, const moe_options* opt) {
  if (check_shape(T, d, E, k, I, dtype) != MOE_OK) return -1;
  Opts o;
  if (parse_options(opt, T, d, k, I, &o) != MOE_OK) return -1;
  int plan = 0;
  if (combine_folded(dtype, k, o)) plan |= MOE_PLAN_FUSED_COMBINE;
  if (gemms_fused(T, dtype)) plan |= MOE_PLAN_FUSED_GEMMS;
  if (router_does_scan(T, E, dtype))
    plan |= MOE_PLAN_FUSED_SCAN;
  else if (T > 0 && permute_does_scan(router_blocks(T, dtype), E))
    plan |= MOE_PLAN_PERMUTE_SCAN;
  if (dtype == MOE_BF16 && o.norm_form != MOE_NORM_NONE && o.norm_w) plan |= MOE_PLAN_ROUTER_WEIGHT_SPLIT;
  return plan;
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
