// router.cu — kernel (a) for fp32 (the bf16 router is router_tc.cu): router
// logits, softmax over E, top-k with ties to the lower expert index, gates
// (optionally renormalised), per-block expert histogram, per-block rank of
// every assignment and per-block sums of the probabilities; then, for both
// dtypes, the single-CTA scan that turns the per-block counts into expert
// offsets, per-block base rows, the tcgen05 tile schedule and the
// load-balancing statistic.
//
// Method: axonml-nn layers/moe.rs, MoERouter::route (Linear -> softmax ->
// stable descending sort -> first k -> renormalise, 1/k if the sum is not
// positive), MoELayer::forward (its per-expert utilization counts) and
// load_balancing_loss (E * sum_i f_i * P_i); Model Architecture Patterns,
// "Top-K Router" (raw top-k softmax gates when not renormalised).
#include <math.h>

#include "common.cuh"

namespace moe {
namespace {

// fp32 logits with plain FFMA (the fp32 workload is small; TF32 tensor cores
// would not meet its 1e-4 tolerance). With the RMSNorm, s_r[row] holds the
// token's scale and the logit is r * sum_c x[c] * (w[c] * W_r[e,c]).
// Thread pair (row, e) keeps its sum in a register while 32-column slices of
// the block's x rows and of up to 32 router rows pass through shared memory
// (coalesced loads, all of a slice in flight at once); each sum still runs
// over c in index order. Experts beyond 32 take further passes.
constexpr int kRC = 32;  // columns per staged slice
constexpr int kRP = 8;   // (token, expert) pairs per thread and pass: 32 experts per pass

__device__ void router_logits_f32(const float* __restrict__ x, const float* __restrict__ wr,
                                  const float* __restrict__ nw, bool norm, const float* s_r, int T, int d, int E,
                                  int tok0, float* s_logit, int ld) {
  __shared__ float s_x[kRouterTokensSimt][kRC + 1];
  __shared__ float s_w[kRouterThreads * kRP / kRouterTokensSimt][kRC + 1];
  constexpr int kPassE = kRouterThreads * kRP / kRouterTokensSimt;
  for (int e0 = 0; e0 < E; e0 += kPassE) {
    const int ne = min(kPassE, E - e0);
    float acc[kRP];
#pragma unroll
    for (int j = 0; j < kRP; ++j) acc[j] = 0.f;
    for (int c0 = 0; c0 < d; c0 += kRC) {
      const int w = min(kRC, d - c0);
      __syncthreads();  // the previous slice has been consumed
#pragma unroll
      for (int i0 = 0; i0 < kRouterTokensSimt * kRC; i0 += kRouterThreads) {
        const int i = i0 + threadIdx.x;
        const int row = i / kRC, c = i % kRC;
        const int t = tok0 + row;
        s_x[row][c] = (t < T && c < w) ? x[(size_t)t * d + c0 + c] : 0.f;
      }
#pragma unroll
      for (int i0 = 0; i0 < kPassE * kRC; i0 += kRouterThreads) {
        const int i = i0 + threadIdx.x;
        const int el = i / kRC, c = i % kRC;
        float v = 0.f;
        if (el < ne && c < w) {
          v = wr[(size_t)(e0 + el) * d + c0 + c];
          if (nw) v = nw[c0 + c] * v;
        }
        s_w[el][c] = v;
      }
      __syncthreads();
#pragma unroll
      for (int j = 0; j < kRP; ++j) {
        const int il = threadIdx.x + j * kRouterThreads;  // a warp shares el, lanes are rows
        const int el = il / kRouterTokensSimt, row = il % kRouterTokensSimt;
        if (el < ne) {
          float s = acc[j];
          for (int c = 0; c < w; ++c) s = fmaf(s_x[row][c], s_w[el][c], s);
          acc[j] = s;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kRP; ++j) {
      const int il = threadIdx.x + j * kRouterThreads;
      const int el = il / kRouterTokensSimt, row = il % kRouterTokensSimt;
      if (el < ne) {
        float s = 0.f;
        if (tok0 + row < T) s = norm ? acc[j] * s_r[row] : acc[j];
        s_logit[row * ld + e0 + el] = s;
      }
    }
  }
  __syncthreads();
}

// kNE: probabilities per lane (E <= 32 * kNE), so that the per-token loops
// hold no predicated-off copies for small E.
template <int kNE>
__global__ void __launch_bounds__(kRouterThreads) router_kernel(
    const float* __restrict__ x, const float* __restrict__ wr, const float* __restrict__ br, int T, int d, int E, int k,
    int renorm, int norm_form, float norm_eps, const float* __restrict__ nw, float* __restrict__ rnorm,
    int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate, int32_t* __restrict__ lrank,
    int32_t* __restrict__ blk_cnt, float* __restrict__ blk_psum, float* __restrict__ blk_z, int32_t* status) {
  extern __shared__ float smem[];
  const int ld = E + 1;
  float* s_p = smem;  // [32][E+1] logits, then probabilities
  __shared__ int32_t s_idx[kRouterTokensSimt][kMaxTopK];
  __shared__ float s_r[kRouterTokensSimt];  // RMSNorm scale per token
  __shared__ float s_z[kRouterTokensSimt];  // logsumexp^2 per token

  const int tok0 = blockIdx.x * kRouterTokensSimt;
  const int ntok = min(kRouterTokensSimt, T - tok0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  pdl_wait();
  if (norm_form) {
    // one thread per token: the sum of x^2 in 32-element pieces
    if (threadIdx.x < kRouterTokensSimt) {
      const int t = tok0 + threadIdx.x;
      float r = 1.0f;
      if (t < T) {
        const float* xr = x + (size_t)t * d;
        float ss = 0.f;
        for (int c0 = 0; c0 < d; c0 += 32) {
          float part = 0.f;
          for (int c = c0; c < min(d, c0 + 32); ++c) part = fmaf(xr[c], xr[c], part);
          ss += part;
        }
        const float ms = ss / (float)d;
        r = norm_form == MOE_NORM_RMS ? 1.0f / sqrtf(ms + norm_eps) : 1.0f / (sqrtf(ms) + norm_eps);
        rnorm[t] = r;
      }
      s_r[threadIdx.x] = r;
    }
    __syncthreads();
  }
  router_logits_f32(x, wr, nw, norm_form != 0, s_r, T, d, E, tok0, s_p, ld);

  // ---- softmax, top-k and gates: one warp per token --------------------
  constexpr int NE = kNE;
  for (int row = warp; row < kRouterTokensSimt; row += kRouterThreads / 32) {
    if (row >= ntok) {
      if (lane < kMaxTopK) s_idx[row][lane] = -1;
      if (lane == 0) s_z[row] = 0.f;
      for (int e = lane; e < E; e += 32) s_p[row * ld + e] = 0.f;
      continue;
    }
    const int t = tok0 + row;
    float v[kNE];
    float m = -INFINITY;
    bool finite = true;
#pragma unroll
    for (int i = 0; i < kNE; ++i) {
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
    for (int i = 0; i < kNE; ++i) {
      const int e = lane + 32 * i;
      const float ex = (i < NE && e < E) ? expf(v[i] - m) : 0.f;
      v[i] = ex;
      s += ex;
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) {
      const float lse = m + logf(s);
      s_z[row] = lse * lse;
    }
#pragma unroll
    for (int i = 0; i < kNE; ++i) {
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
        for (int i = 0; i < kNE; ++i) {
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
  if (blk_z && threadIdx.x == 0) {
    float z = 0.f;
    for (int row = 0; row < ntok; ++row) z += s_z[row];
    blk_z[blockIdx.x] = z;
  }
}

// One CTA of 1024 threads. Thread (slice, e) sums the counts and
// probability sums of a contiguous range of router blocks for expert e (the
// loads of neighbouring threads are neighbouring experts of one block, so they
// coalesce). One warp per expert then scans its slice sums with shuffles;
// warp 0 scans the expert totals (kept counts under a capacity: an expert
// keeps min(count, cap) rows, and a row computed past that is a dropped slot)
// into the offsets and the tile schedule, the shared experts following the
// routed ones with T rows each, and the balance statistic; warp 1 sums the
// per-block z-loss partials. Finally every thread walks its slice once more,
// writing each block's base row. Every sum runs in a fixed order (fp64 for
// the probabilities, the statistic and the z-loss), so the results are
// deterministic.
__global__ void __launch_bounds__(1024) route_scan_kernel(int nb, int T, int E, int k, int cap, int n_shared,
                                                          int32_t* __restrict__ blk_cnt,
                                                          const float* __restrict__ blk_psum,
                                                          const float* __restrict__ blk_z,
                                                          int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                          int32_t* __restrict__ mtile, float* __restrict__ aux,
                                                          float* __restrict__ zloss, int32_t* __restrict__ dropped,
                                                          int32_t* __restrict__ mt_done, int n_mt) {
  __shared__ int s_cnt[1024];      // [slice][E] slice sums, then exclusive slice prefixes
  __shared__ double s_ps[1024];    // [slice][E] probability slice sums
  __shared__ int s_tot[kMaxExperts];
  __shared__ double s_ptot[kMaxExperts];
  __shared__ int s_off[kMaxExperts + 1];
  const unsigned full = 0xffffffffu;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
  const int S = max(1, min((int)blockDim.x / E, nb));  // slices
  const int e = tid % E, sl = tid / E;
  const bool active = sl < S;
  const int chunk = (nb + S - 1) / S;
  const int b0 = min(nb, sl * chunk), b1 = min(nb, b0 + chunk);
  pdl_wait();
  if (mt_done)  // the fused GEMMs' per-token-tile counters start from zero every call
    for (int i = tid; i < n_mt; i += blockDim.x) mt_done[i] = 0;
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
  for (int ee = warp; ee < E; ee += nw) {  // one warp per expert: scan over the slices
    int carry = 0;
    double ps = 0.0;
    for (int s0 = 0; s0 < S; s0 += 32) {
      const int s1 = s0 + lane;
      const int c = s1 < S ? s_cnt[s1 * E + ee] : 0;
      double p = s1 < S ? s_ps[s1 * E + ee] : 0.0;
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(full, incl, o);
        if (lane >= o) incl += n;
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) p += __shfl_xor_sync(full, p, o);
      if (s1 < S) s_cnt[s1 * E + ee] = carry + incl - c;
      carry += __shfl_sync(full, incl, 31);
      ps += p;
    }
    if (lane == 0) {
      s_tot[ee] = carry;
      s_ptot[ee] = ps;
    }
  }
  __syncthreads();
  if (warp == 0) {
    int run = 0, mt = 0, drop = 0;
    double a = 0.0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int ee = e0 + lane;
      const int tot = ee < E ? s_tot[ee] : 0;
      const int kept = cap >= 0 ? min(tot, cap) : tot;
      const int tiles = (kept + kTileM - 1) / kTileM;
      int ik = kept, it = tiles;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n1 = __shfl_up_sync(full, ik, o), n2 = __shfl_up_sync(full, it, o);
        if (lane >= o) {
          ik += n1;
          it += n2;
        }
      }
      double ae = ee < E ? ((double)tot / ((double)T * (double)k)) * (s_ptot[ee] / (double)T) : 0.0;
      int dr = tot - kept;
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        ae += __shfl_xor_sync(full, ae, o);
        dr += __shfl_xor_sync(full, dr, o);
      }
      if (ee < E) {
        const int off = run + ik - kept;
        offsets[ee] = off;
        s_off[ee] = off;
        mtile[ee] = mt + it - tiles;
        if (counts) counts[ee] = tot;
      }
      run += __shfl_sync(full, ik, 31);
      mt += __shfl_sync(full, it, 31);
      a += ae;
      drop += dr;
    }
    if (lane == 0) {
      offsets[E] = run;
      s_off[E] = run;
      mtile[E] = mt;
      for (int s2 = 0; s2 < n_shared; ++s2) {
        mt += (T + kTileM - 1) / kTileM;
        mtile[E + 1 + s2] = mt;
      }
      if (aux) *aux = (float)((double)E * a);
      if (dropped) *dropped = drop;
    }
  }
  if (zloss && warp == 1) {
    double z = 0.0;
    for (int b = lane; b < nb; b += 32) z += (double)blk_z[b];
#pragma unroll
    for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(full, z, o);
    if (lane == 0) *zloss = (float)(z / (double)T);
  }
  __syncthreads();
  if (active) {  // base row of every block: expert offset + slice prefix + blocks before it in the slice
    int run = s_off[e] + s_cnt[sl * E + e];
    for (int b = b0; b < b1; ++b) {
      const int v = blk_cnt[(size_t)b * E + e];
      blk_cnt[(size_t)b * E + e] = run;
      run += v;
    }
  }
}

}  // namespace

cudaError_t launch_router(moe_dtype dtype, const void* x, const void* w_router, const float* b_router, int T, int d,
                          int E, int k, int renorm, const RouterNorm& norm, int32_t* topk_idx, float* topk_gate,
                          int32_t* lrank, int32_t* blk_cnt, float* blk_psum, float* blk_z, const RouterScan& scan,
                          int32_t* status, cudaStream_t stream) {
  if (dtype == MOE_BF16)
    return launch_router_tc(x, w_router, b_router, T, d, E, k, renorm, norm, topk_idx, topk_gate, lrank, blk_cnt,
                            blk_psum, blk_z, scan, status, stream);
  const int nb = router_blocks(T, MOE_F32);
  const size_t smem = (size_t)kRouterTokensSimt * (E + 1) * sizeof(float);
  auto kern = E <= 32 ? router_kernel<1> : E <= 64 ? router_kernel<2> : E <= 128 ? router_kernel<4> : router_kernel<8>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  return launch_pdl(kern, dim3(nb), dim3(kRouterThreads), smem, stream, static_cast<const float*>(x),
                    static_cast<const float*>(w_router), b_router, T, d, E, k, renorm, norm.form, norm.eps,
                    static_cast<const float*>(norm.w), norm.rnorm, topk_idx, topk_gate, lrank, blk_cnt, blk_psum,
                    blk_z, status);
}

cudaError_t launch_route_scan(int nb, int T, int E, int k, int cap, int n_shared, int32_t* blk_cnt,
                              const float* blk_psum, const float* blk_z, int32_t* counts, int32_t* offsets,
                              int32_t* mtile, float* aux, float* zloss, int32_t* dropped, int32_t* mt_done, int n_mt,
                              cudaStream_t stream) {
  return launch_pdl(route_scan_kernel, dim3(1), dim3(1024), 0, stream, nb, T, E, k, cap, n_shared, blk_cnt, blk_psum,
                    blk_z, counts, offsets, mtile, aux, zloss, dropped, mt_done, n_mt);
}

}  // namespace moe
