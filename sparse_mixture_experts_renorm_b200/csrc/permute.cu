// permute.cu — kernel (b), the dispatch: every (token, slot) gets its row in
// the expert-contiguous order (experts ascending, tokens ascending within an
// expert, axonml-nn layers/moe.rs, MoELayer::forward "gather tokens for this
// expert"), and the token's row of x is copied to each of its k rows; and
// kernel (d), the combine: out[t] = sum_j gate[t,j] * Y[row(t,j)] (same page,
// "Scatter weighted outputs back", each expert weighted by its own gate).
#include "common.cuh"

namespace moe {
namespace {

constexpr int kCopyThreads = 256;  // 16-byte vectors per block (4 KB of a row)

// Block (token t, chunk c): threads j < k compute the row of slot j from the
// per-block base row of its expert plus its rank inside the router block
// (chunk 0 also records perm_tok / inv); then every thread copies one 16-byte
// vector of x[t] to each of the token's k rows.
__global__ void __launch_bounds__(kCopyThreads) permute_kernel(const uint4* __restrict__ x, int nvec, int E, int k,
                                                              int rb, int R, const int32_t* __restrict__ topk_idx,
                                                              const int32_t* __restrict__ lrank,
                                                              const int32_t* __restrict__ blk_base,
                                                              int32_t* __restrict__ perm_tok, int32_t* __restrict__ inv,
                                                              uint4* __restrict__ xp, const float* __restrict__ gate,
                                                              float* __restrict__ rgate, float4* __restrict__ zero_out,
                                                              int nout4, int32_t* status) {
  const int t = blockIdx.x;
  __shared__ int s_rows[kMaxTopK];
  pdl_wait();
  if (threadIdx.x < k) {
    const int j = threadIdx.x;
    const int e = topk_idx[(size_t)t * k + j];
    int row = -1;
    if (e >= 0 && e < E) row = blk_base[(size_t)(t / rb) * E + e] + lrank[(size_t)t * k + j];
    if (row < 0 || row >= R) {
      atomicOr(status, MOE_DEV_INTERNAL);
      row = -1;
    } else if (blockIdx.y == 0) {
      perm_tok[row] = t;
      inv[(size_t)t * k + j] = row;
      rgate[row] = gate[(size_t)t * k + j];
    }
    s_rows[j] = row;
  }
  __syncthreads();
  if (zero_out) {  // the output row this block's x chunk maps to, for a combine done by atomics
    const int per = (nout4 + gridDim.y - 1) / gridDim.y;
    for (int o = blockIdx.y * per + threadIdx.x; o < min(nout4, (int)(blockIdx.y + 1) * per); o += kCopyThreads)
      zero_out[(size_t)t * nout4 + o] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const int i = blockIdx.y * kCopyThreads + threadIdx.x;
  if (i >= nvec) return;
  const uint4 v = __ldg(x + (size_t)t * nvec + i);
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j)
    if (j < k && s_rows[j] >= 0) xp[(size_t)s_rows[j] * nvec + i] = v;
}

// Block (token t, chunk c): every thread sums one float4 of its token's k
// expert rows, weighted by the gates, in slot order (fp32).
__global__ void __launch_bounds__(kCopyThreads) combine_kernel(const float4* __restrict__ y, int nvec4, int k, int R,
                                                              const int32_t* __restrict__ inv,
                                                              const float* __restrict__ gate,
                                                              float4* __restrict__ out, int32_t* status) {
  const int t = blockIdx.x;
  __shared__ int s_rows[kMaxTopK];
  __shared__ float s_g[kMaxTopK];
  pdl_wait();
  if (threadIdx.x < k) {
    const int j = threadIdx.x;
    int row = inv[(size_t)t * k + j];
    float g = gate[(size_t)t * k + j];
    if (row < 0 || row >= R) {
      atomicOr(status, MOE_DEV_INTERNAL);
      row = 0;
      g = 0.f;
    }
    s_rows[j] = row;
    s_g[j] = g;
  }
  __syncthreads();
  const int i = blockIdx.y * kCopyThreads + threadIdx.x;
  if (i >= nvec4) return;
  float4 v[kMaxTopK];
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j)
    if (j < k) v[j] = __ldg(y + (size_t)s_rows[j] * nvec4 + i);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    if (j < k) {
      const float g = s_g[j];
      acc.x = fmaf(g, v[j].x, acc.x);
      acc.y = fmaf(g, v[j].y, acc.y);
      acc.z = fmaf(g, v[j].z, acc.z);
      acc.w = fmaf(g, v[j].w, acc.w);
    }
  }
  out[(size_t)t * nvec4 + i] = acc;
}

}  // namespace

cudaError_t launch_permute(moe_dtype dtype, const void* x, int T, int d, int E, int k, int rb, const int32_t* topk_idx,
                           const int32_t* lrank, const int32_t* blk_base, int32_t* perm_tok, int32_t* inv, void* xp,
                           const float* topk_gate, float* rgate, float* zero_out, int32_t* status,
                           cudaStream_t stream) {
  const int elem = dtype == MOE_BF16 ? 2 : 4;
  const int nvec = d * elem / 16;
  const dim3 grid(T, (nvec + kCopyThreads - 1) / kCopyThreads);
  return launch_pdl(permute_kernel, grid, dim3(kCopyThreads), 0, stream, static_cast<const uint4*>(x), nvec, E, k, rb,
                    T * k, topk_idx, lrank, blk_base, perm_tok, inv, static_cast<uint4*>(xp), topk_gate, rgate,
                    reinterpret_cast<float4*>(zero_out), d / 4, status);
}

cudaError_t launch_combine(int T, int d, int k, const float* y, const int32_t* inv, const float* topk_gate, float* out,
                           int32_t* status, cudaStream_t stream) {
  const int nvec4 = d / 4;
  const dim3 grid(T, (nvec4 + kCopyThreads - 1) / kCopyThreads);
  return launch_pdl(combine_kernel, grid, dim3(kCopyThreads), 0, stream, reinterpret_cast<const float4*>(y), nvec4, k,
                    T * k, inv, topk_gate, reinterpret_cast<float4*>(out), status);
}

}  // namespace moe
