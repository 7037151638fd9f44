// router.cu — kernel (a): router logits, softmax over E, top-k with ties to
// the lower expert index, gates (optionally renormalised), per-block expert
// histogram, per-block rank of every assignment and per-block sums of the
// probabilities; then the single-CTA scan that turns the per-block counts into
// expert offsets, per-block base rows, the tcgen05 tile schedule and the
// load-balancing statistic.
//
// Method: axonml-nn layers/moe.rs, MoERouter::route (Linear -> softmax ->
// stable descending sort -> first k -> renormalise, 1/k if the sum is not
// positive), MoELayer::forward ("Track expert utilization") and
// load_balancing_loss (E * sum_i f_i * P_i); Model Architecture Patterns,
// "Top-K Router" (raw top-k softmax gates when not renormalised).
#include <math.h>

#include "common.cuh"

namespace moe {
namespace {

__device__ __forceinline__ uint32_t u4_get(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Logits of the CTA's 32 tokens against every expert, bf16 inputs, fp32
// accumulation on the tensor cores (m16n8k16). The 4 warps split d into
// interleaved 64-column chunks; their partial sums are added in warp order.
// Inside a chunk the k-slots of the MMA fragments are assigned to physical
// columns so that every thread reads 16 contiguous bytes of x and of W_r;
// A and B use the same assignment, so each product pairs x[t,c] with W_r[e,c].
__device__ void router_logits_bf16(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ wr,
                                   int T, int d, int E, int tok0, float* s_logit, int ld, float* s_part) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;
  for (int e0 = 0; e0 < E; e0 += 64) {
    const int EC = min(64, E - e0);
    const int NT = (EC + 7) >> 3;
    float acc[2][8][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[mt][nt][i] = 0.f;

    for (int kc = warp * 64; kc < d; kc += 4 * 64) {
      uint4 a[2][2][2];  // [m-tile][row g / row g+8][32-column half]
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int t = tok0 + mt * 16 + hr * 8 + g;
          if (t < T) {
            const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d + kc + tq * 8);
            a[mt][hr][0] = __ldg(src);
            a[mt][hr][1] = __ldg(src + 4);
          } else {
            a[mt][hr][0] = make_uint4(0, 0, 0, 0);
            a[mt][hr][1] = make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        if (nt < NT) {
          const int e = e0 + nt * 8 + g;
          uint4 b[2];
          if (e < E) {
            const uint4* src = reinterpret_cast<const uint4*>(wr + (size_t)e * d + kc + tq * 8);
            b[0] = __ldg(src);
            b[1] = __ldg(src + 4);
          } else {
            b[0] = make_uint4(0, 0, 0, 0);
            b[1] = make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int half = 0; half < 2; ++half)
#pragma unroll
            for (int s = 0; s < 2; ++s) {
              const uint32_t b0 = u4_get(b[half], 2 * s), b1 = u4_get(b[half], 2 * s + 1);
#pragma unroll
              for (int mt = 0; mt < 2; ++mt)
                mma_bf16_16816(acc[mt][nt], u4_get(a[mt][0][half], 2 * s), u4_get(a[mt][1][half], 2 * s),
                               u4_get(a[mt][0][half], 2 * s + 1), u4_get(a[mt][1][half], 2 * s + 1), b0, b1);
            }
        }
      }
    }
    // accumulator (row g, cols 2tq..2tq+1) and (row g+8, same cols)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int row = mt * 16 + g, col = nt * 8 + 2 * tq;
        float* p0 = s_part + (warp * 32 + row) * 64 + col;
        float* p1 = s_part + (warp * 32 + row + 8) * 64 + col;
        p0[0] = acc[mt][nt][0];
        p0[1] = acc[mt][nt][1];
        p1[0] = acc[mt][nt][2];
        p1[1] = acc[mt][nt][3];
      }
    __syncthreads();
    for (int i = threadIdx.x; i < kRouterTokens * EC; i += blockDim.x) {
      const int row = i / EC, col = i - row * EC;
      float s = s_part[(0 * 32 + row) * 64 + col];
      s += s_part[(1 * 32 + row) * 64 + col];
      s += s_part[(2 * 32 + row) * 64 + col];
      s += s_part[(3 * 32 + row) * 64 + col];
      s_logit[row * ld + e0 + col] = s;
    }
    __syncthreads();
  }
}

// fp32 logits with plain FFMA (the fp32 workload is small; TF32 tensor cores
// would not meet its 1e-4 tolerance).
__device__ void router_logits_f32(const float* __restrict__ x, const float* __restrict__ wr, int T, int d, int E,
                                  int tok0, float* s_logit, int ld) {
  for (int i = threadIdx.x; i < kRouterTokens * E; i += blockDim.x) {
    const int e = i / kRouterTokens, row = i - e * kRouterTokens;
    const int t = tok0 + row;
    float s = 0.f;
    if (t < T) {
      const float* xr = x + (size_t)t * d;
      const float* wrow = wr + (size_t)e * d;
      for (int c = 0; c < d; ++c) s = fmaf(xr[c], wrow[c], s);
    }
    s_logit[row * ld + e] = s;
  }
  __syncthreads();
}

template <typename Tin>
__global__ void __launch_bounds__(kRouterThreads) router_kernel(
    const Tin* __restrict__ x, const Tin* __restrict__ wr, const float* __restrict__ br, int T, int d, int E, int k,
    int renorm, int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate, int32_t* __restrict__ lrank,
    int32_t* __restrict__ blk_cnt, float* __restrict__ blk_psum, int32_t* status) {
  extern __shared__ float smem[];
  const int ld = E + 1;
  float* s_p = smem;                         // [32][E+1] logits, then probabilities
  float* s_part = smem + kRouterTokens * ld; // [4][32][64] per-warp partial logits (bf16 path)
  __shared__ int32_t s_idx[kRouterTokens][kMaxTopK];

  const int tok0 = blockIdx.x * kRouterTokens;
  const int ntok = min(kRouterTokens, T - tok0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if constexpr (sizeof(Tin) == 2)
    router_logits_bf16(x, wr, T, d, E, tok0, s_p, ld, s_part);
  else
    router_logits_f32(x, wr, T, d, E, tok0, s_p, ld);

  // ---- softmax, top-k and gates: one warp per token --------------------
  const int NE = (E + 31) >> 5;  // values per lane (<= 8)
  for (int row = warp; row < kRouterTokens; row += kRouterThreads / 32) {
    if (row >= ntok) {
      if (lane < kMaxTopK) s_idx[row][lane] = -1;
      for (int e = lane; e < E; e += 32) s_p[row * ld + e] = 0.f;
      continue;
    }
    const int t = tok0 + row;
    float v[8];
    float m = -INFINITY;
    bool finite = true;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      v[i] = -INFINITY;
      if (i < NE && e < E) {
        float l = s_p[row * ld + e];
        if (br) l += br[e];
        finite = finite && isfinite(l);
        v[i] = l;
        m = fmaxf(m, l);
      }
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      const float ex = (i < NE && e < E) ? expf(v[i] - m) : 0.f;
      v[i] = ex;
      s += ex;
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      v[i] = v[i] / s;
      if (i < NE && e < E) s_p[row * ld + e] = v[i];
    }
    if (!__all_sync(0xffffffffu, finite) && lane == 0) atomicOr(status, MOE_DEV_NONFINITE);

    // k rounds of a warp arg-max under (p descending, index ascending); a
    // NaN probability ranks as -inf so every token still gets k distinct,
    // valid experts.
    uint32_t taken = 0;
    float pk[kMaxTopK];
    int ek[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      pk[j] = 0.f;
      ek[j] = 0;
      if (j < k) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int e = lane + 32 * i;
          if (i < NE && e < E && !((taken >> i) & 1u)) {
            float pv = v[i];
            if (pv != pv) pv = -INFINITY;
            if (pv > bv || (pv == bv && e < be)) {
              bv = pv;
              be = e;
            }
          }
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
          const int oe = __shfl_xor_sync(0xffffffffu, be, off);
          if (ov > bv || (ov == bv && oe < be)) {
            bv = ov;
            be = oe;
          }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        pk[j] = bv;
        ek[j] = be;
      }
    }
    float psel = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j)
      if (j < k) psel += pk[j];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j < k && lane == j) {
        float gsel;
        if (!renorm)
          gsel = pk[j];
        else if (psel > 0.f)
          gsel = pk[j] / psel;
        else
          gsel = 1.0f / (float)k;
        topk_idx[(size_t)t * k + j] = ek[j];
        topk_gate[(size_t)t * k + j] = gsel;
        s_idx[row][j] = ek[j];
      }
    }
  }
  __syncthreads();

  // ---- per-block histogram and the rank of each assignment ---------------
  for (int e = warp; e < E; e += kRouterThreads / 32) {
    int jhit = -1;
    if (lane < ntok) {
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j)
        if (j < k && s_idx[lane][j] == e) jhit = j;
    }
    const uint32_t mask = __ballot_sync(0xffffffffu, jhit >= 0);
    if (jhit >= 0) lrank[(size_t)(tok0 + lane) * k + jhit] = __popc(mask & ((1u << lane) - 1u));
    if (lane == 0) blk_cnt[(size_t)blockIdx.x * E + e] = __popc(mask);
  }
  // ---- per-block sums of the probabilities, in token order ---------------
  for (int e = threadIdx.x; e < E; e += kRouterThreads) {
    float s = 0.f;
    for (int row = 0; row < ntok; ++row) s += s_p[row * ld + e];
    blk_psum[(size_t)blockIdx.x * E + e] = s;
  }
}

// One CTA of 1024 threads. Thread (e, slice) reduces a contiguous range of
// router blocks for expert e; slices are then scanned in order, so every
// result is deterministic.
__global__ void __launch_bounds__(1024) route_scan_kernel(int nb, int T, int E, int k, int32_t* __restrict__ blk_cnt,
                                                          const float* __restrict__ blk_psum,
                                                          int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                          int32_t* __restrict__ mtile128, float* __restrict__ aux) {
  __shared__ int s_cnt[1024];
  __shared__ double s_ps[1024];
  __shared__ int s_tot[kMaxExperts];
  __shared__ double s_ptot[kMaxExperts];
  __shared__ int s_off[kMaxExperts + 1];
  const int S = max(1, (int)blockDim.x / E);
  const int tid = threadIdx.x;
  const int e = tid % E, sl = tid / E;
  const bool active = sl < S;
  const int chunk = (nb + S - 1) / S;
  const int b0 = min(nb, sl * chunk), b1 = min(nb, b0 + chunk);
  if (active) {
    int c = 0;
    double ps = 0.0;
    for (int b = b0; b < b1; ++b) {
      c += blk_cnt[(size_t)b * E + e];
      ps += (double)blk_psum[(size_t)b * E + e];
    }
    s_cnt[sl * E + e] = c;
    s_ps[sl * E + e] = ps;
  }
  __syncthreads();
  if (tid < E) {
    int run = 0;
    double p = 0.0;
    for (int s2 = 0; s2 < S; ++s2) {
      const int v = s_cnt[s2 * E + tid];
      s_cnt[s2 * E + tid] = run;
      run += v;
      p += s_ps[s2 * E + tid];
    }
    s_tot[tid] = run;
    s_ptot[tid] = p;
  }
  __syncthreads();
  if (tid == 0) {
    int off = 0, mt = 0;
    double a = 0.0;
    for (int ee = 0; ee < E; ++ee) {
      s_off[ee] = off;
      offsets[ee] = off;
      mtile128[ee] = mt;
      if (counts) counts[ee] = s_tot[ee];
      a += ((double)s_tot[ee] / ((double)T * (double)k)) * (s_ptot[ee] / (double)T);
      off += s_tot[ee];
      mt += (s_tot[ee] + kBM - 1) / kBM;
    }
    offsets[E] = off;
    mtile128[E] = mt;
    s_off[E] = off;
    if (aux) *aux = (float)((double)E * a);
  }
  __syncthreads();
  if (active) {
    int run = s_off[e] + s_cnt[sl * E + e];
    for (int b = b0; b < b1; ++b) {
      const int v = blk_cnt[(size_t)b * E + e];
      blk_cnt[(size_t)b * E + e] = run;
      run += v;
    }
  }
}

}  // namespace

size_t router_smem_bytes(moe_dtype dtype, int E) {
  size_t b = (size_t)kRouterTokens * (E + 1) * sizeof(float);
  if (dtype == MOE_BF16) b += (size_t)4 * 32 * 64 * sizeof(float);
  return b;
}

cudaError_t launch_router(moe_dtype dtype, const void* x, const void* w_router, const float* b_router, int T, int d,
                          int E, int k, int renorm, int32_t* topk_idx, float* topk_gate, int32_t* lrank,
                          int32_t* blk_cnt, float* blk_psum, int32_t* status, cudaStream_t stream) {
  const int nb = router_blocks(T);
  const size_t smem = router_smem_bytes(dtype, E);
  if (dtype == MOE_BF16) {
    auto kern = router_kernel<__nv_bfloat16>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    kern<<<nb, kRouterThreads, smem, stream>>>(static_cast<const __nv_bfloat16*>(x),
                                               static_cast<const __nv_bfloat16*>(w_router), b_router, T, d, E, k,
                                               renorm, topk_idx, topk_gate, lrank, blk_cnt, blk_psum, status);
  } else {
    auto kern = router_kernel<float>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    kern<<<nb, kRouterThreads, smem, stream>>>(static_cast<const float*>(x), static_cast<const float*>(w_router),
                                               b_router, T, d, E, k, renorm, topk_idx, topk_gate, lrank, blk_cnt,
                                               blk_psum, status);
  }
  return cudaGetLastError();
}

cudaError_t launch_route_scan(int T, int E, int k, int32_t* blk_cnt, const float* blk_psum, int32_t* counts,
                              int32_t* offsets, int32_t* mtile128, float* aux, cudaStream_t stream) {
  route_scan_kernel<<<1, 1024, 0, stream>>>(router_blocks(T), T, E, k, blk_cnt, blk_psum, counts, offsets, mtile128,
                                            aux);
  return cudaGetLastError();
}

}  // namespace moe
