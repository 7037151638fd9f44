// permute.cu — kernel (b), the dispatch: every (token, slot) gets its row in
// the expert-contiguous order (experts ascending, tokens ascending within an
// expert, axonml-nn layers/moe.rs, MoELayer::forward "gather tokens for this
// expert"), and the token's row of x is copied to each of its k rows; and
// kernel (d), the combine: out[t] = sum_j gate[t,j] * Y[row(t,j)] (same page,
// "Scatter weighted outputs back", each expert weighted by its own gate).
#include "common.cuh"

namespace moe {
namespace {

// One warp per token. Lanes j < k compute the row of slot j from the
// per-block base row of its expert plus its rank inside the router block;
// then the warp copies the token's row of x (16-byte vectors, read once) to
// each of its k rows.
__global__ void __launch_bounds__(256) permute_kernel(const uint4* __restrict__ x, int T, int nvec, int E, int k,
                                                      int R, const int32_t* __restrict__ topk_idx,
                                                      const int32_t* __restrict__ lrank,
                                                      const int32_t* __restrict__ blk_base,
                                                      int32_t* __restrict__ perm_tok, int32_t* __restrict__ inv,
                                                      uint4* __restrict__ xp, int32_t* status) {
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  int row = -1;
  if (lane < k) {
    const int e = topk_idx[(size_t)t * k + lane];
    if (e >= 0 && e < E) row = blk_base[(size_t)(t / kRouterTokens) * E + e] + lrank[(size_t)t * k + lane];
    if (row < 0 || row >= R) {
      atomicOr(status, MOE_DEV_INTERNAL);
      row = -1;
    } else {
      perm_tok[row] = t;
      inv[(size_t)t * k + lane] = row;
    }
  }
  int rows[kMaxTopK];
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) rows[j] = __shfl_sync(0xffffffffu, row, j);
  const uint4* src = x + (size_t)t * nvec;
  for (int i = lane; i < nvec; i += 32) {
    const uint4 v = __ldg(src + i);
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j)
      if (j < k && rows[j] >= 0) xp[(size_t)rows[j] * nvec + i] = v;
  }
}

// One warp per token; fp32 accumulation over the k slots in slot order.
__global__ void __launch_bounds__(256) combine_kernel(const float4* __restrict__ y, int T, int nvec4, int k, int R,
                                                      const int32_t* __restrict__ inv,
                                                      const float* __restrict__ gate, float4* __restrict__ out,
                                                      int32_t* status) {
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  int row = 0;
  float g = 0.f;
  if (lane < k) {
    row = inv[(size_t)t * k + lane];
    g = gate[(size_t)t * k + lane];
    if (row < 0 || row >= R) {
      atomicOr(status, MOE_DEV_INTERNAL);
      row = 0;
      g = 0.f;
    }
  }
  int rows[kMaxTopK];
  float gs[kMaxTopK];
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    rows[j] = __shfl_sync(0xffffffffu, row, j);
    gs[j] = __shfl_sync(0xffffffffu, g, j);
  }
  for (int i = lane; i < nvec4; i += 32) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j < k) {
        const float4 v = __ldg(y + (size_t)rows[j] * nvec4 + i);
        acc.x = fmaf(gs[j], v.x, acc.x);
        acc.y = fmaf(gs[j], v.y, acc.y);
        acc.z = fmaf(gs[j], v.z, acc.z);
        acc.w = fmaf(gs[j], v.w, acc.w);
      }
    }
    out[(size_t)t * nvec4 + i] = acc;
  }
}

}  // namespace

cudaError_t launch_permute(moe_dtype dtype, const void* x, int T, int d, int E, int k, const int32_t* topk_idx,
                           const int32_t* lrank, const int32_t* blk_base, int32_t* perm_tok, int32_t* inv, void* xp,
                           int32_t* status, cudaStream_t stream) {
  const int elem = dtype == MOE_BF16 ? 2 : 4;
  const int nvec = d * elem / 16;
  const int blocks = (T + 7) / 8;
  permute_kernel<<<blocks, 256, 0, stream>>>(static_cast<const uint4*>(x), T, nvec, E, k, T * k, topk_idx, lrank,
                                             blk_base, perm_tok, inv, static_cast<uint4*>(xp), status);
  return cudaGetLastError();
}

cudaError_t launch_combine(int T, int d, int k, const float* y, const int32_t* inv, const float* topk_gate, float* out,
                           int32_t* status, cudaStream_t stream) {
  const int blocks = (T + 7) / 8;
  combine_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<const float4*>(y), T, d / 4, k, T * k, inv, topk_gate,
                                             reinterpret_cast<float4*>(out), status);
  return cudaGetLastError();
}

}  // namespace moe
