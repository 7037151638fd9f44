// permute.cu — kernel (b), the dispatch: every (token, slot) gets its row in
// the expert-contiguous order (experts ascending, tokens ascending within an
// expert: the order in which axonml-nn layers/moe.rs, MoELayer::forward,
// collects each expert's tokens), and the token's row of x is copied to each
// of its k rows; and kernel (d), the combine: out[t] = sum_j gate[t,j] *
// Y[row(t,j)] (the same function's scatter of the expert outputs back to
// token order, each expert weighted by its own gate).
// Options: the pre-MoE RMSNorm is applied on the copy; with a capacity
// ("moe_capacity_factor", KempnerForge ModelConfig) a slot whose rank in its
// expert reaches the capacity is dropped; shared experts ("moe_shared_experts")
// get every token's row and add their outputs with weight 1.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kCopyThreads = 256;  // 16-byte vectors per block (4 KB of a row)
static_assert(kMaxExperts <= kCopyThreads, "one thread per expert in the permute's scan");

// Exclusive prefix sum of one int per thread over the block (kCopyThreads
// threads, in thread order); *total gets the sum. s_w: kCopyThreads/32 + 1 ints.
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_w, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  constexpr int kW = kCopyThreads / 32;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) s_w[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int x = lane < kW ? s_w[lane] : 0;
    int xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += n;
    }
    if (lane < kW) s_w[lane] = xi - x;
    if (lane == 31) s_w[kW] = xi;
  }
  __syncthreads();
  const int r = s_w[w] + incl - v;
  *total = s_w[kW];
  __syncthreads();  // s_w is reused by the next call
  return r;
}

// x_hat = x * r * w for one 16-byte vector (8 bf16 or 4 fp32), rounded to
// the dtype (the pre-MoE RMSNorm applied on the copy).
__device__ __forceinline__ uint4 scale_vec(uint4 v, uint4 w, float r, bool bf16, bool has_w) {
  uint32_t u[4] = {v.x, v.y, v.z, v.w};
  const uint32_t uw[4] = {w.x, w.y, w.z, w.w};
  if (bf16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float a = __uint_as_float(u[i] << 16) * r, b = __uint_as_float(u[i] & 0xffff0000u) * r;
      if (has_w) {
        a *= __uint_as_float(uw[i] << 16);
        b *= __uint_as_float(uw[i] & 0xffff0000u);
      }
      u[i] = pack_bf16x2(a, b);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float a = __uint_as_float(u[i]) * r;
      if (has_w) a *= __uint_as_float(uw[i]);
      u[i] = __float_as_uint(a);
    }
  }
  return make_uint4(u[0], u[1], u[2], u[3]);
}

// Block (tokens t0 .. t0+G-1, chunk c): threads g*k + j compute the row of
// slot j of token t0+g from the per-block base row of its expert plus its
// rank inside the router block (chunk 0 also records perm_tok / inv); then
// the block copies its chunk of 16-byte vectors of the G rows of x
// (normalised when rnorm is given) to each kept row of its token and, with
// shared experts, to row shared_row0 + t. Several tokens per block put one
// chain of dependent index loads in front of several rows of copying, and
// four vectors in flight per thread.
// The routing scan done by every permute block itself (kScan), for batches
// whose router blocks are few: each block sums the per-block expert counts
// again for its own router block's base rows, and block 0 also writes the
// scan's results (counts, offsets, the GEMMs' tile schedule, the load-balance
// statistic, the z-loss, the dropped count, the fused GEMMs' counters
// cleared). The integer results are route_scan_kernel's exactly (so are the
// rows); the fp64 sums of the statistics run in another fixed order.
struct PermuteScan {
  int nb, cap, n_shared, n_mt;
  const float* blk_psum;
  const float* blk_z;
  int32_t* counts;
  int32_t* offsets;
  int32_t* mtile;
  float* aux;
  float* zloss;
  int32_t* dropped;
  int32_t* mt_done;
};

template <int G, bool kScan>
__global__ void __launch_bounds__(kCopyThreads) permute_kernel(
    const uint4* __restrict__ x, int T, int nvec, int E, int k, int rb, int R, const int32_t* __restrict__ topk_idx,
    const int32_t* __restrict__ lrank, const int32_t* __restrict__ blk_base, const int32_t* __restrict__ offsets,
    int has_cap, int32_t* __restrict__ perm_tok, int32_t* __restrict__ inv, uint4* __restrict__ xp,
    const float* __restrict__ gate, float* __restrict__ rgate, float4* __restrict__ zero_out, int nout4,
    const float* __restrict__ rnorm, const uint4* __restrict__ norm_w, int bf16, int shared_row0, int32_t* status,
    const PermuteScan sc) {
  const int t0 = blockIdx.x * G;
  const int ng = min(G, T - t0);
  __shared__ int s_rows[G][kMaxTopK];
  __shared__ int s_base[kScan ? kMaxExperts : 1];  // first row of each expert for this router block
  __shared__ int s_end[kScan ? kMaxExperts + 1 : 1];  // end of each expert's kept rows
  pdl_wait();
  if constexpr (kScan) {
    __shared__ int s_w[kCopyThreads / 32 + 1];
    const int e = threadIdx.x;  // one expert per thread
    const int bb = t0 / rb;     // this block's router block
    int tot = 0, pre = 0;
    if (e < E)
      for (int b = 0; b < sc.nb; ++b) {
        const int c = blk_base[(size_t)b * E + e];  // per-block counts (the router's histogram)
        tot += c;
        if (b < bb) pre += c;
      }
    const int kept = e < E ? (sc.cap >= 0 ? min(tot, sc.cap) : tot) : 0;
    int run = 0;
    const int off = block_exclusive_scan(kept, s_w, &run);
    if (e < E) {
      s_base[e] = off + pre;
      s_end[e] = off + kept;
    }
    if (blockIdx.x == 0 && blockIdx.y == 0) {
      for (int i = threadIdx.x; i < sc.n_mt; i += kCopyThreads) sc.mt_done[i] = 0;
      const int tiles = (kept + kTileM - 1) / kTileM;
      int mt = 0;
      const int mt_off = block_exclusive_scan(tiles, s_w, &mt);
      // the statistic: E * sum_e (count_e / (T k)) * (sum of p_e / T), in fp64
      double ps = 0.0;
      if (e < E)
        for (int b = 0; b < sc.nb; ++b) ps += (double)sc.blk_psum[(size_t)b * E + e];
      double ae = e < E ? ((double)tot / ((double)T * (double)k)) * (ps / (double)T) : 0.0;
      int dr = e < E ? tot - kept : 0;
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        ae += __shfl_xor_sync(0xffffffffu, ae, o);
        dr += __shfl_xor_sync(0xffffffffu, dr, o);
      }
      __shared__ double s_ae[kCopyThreads / 32];
      __shared__ int s_dr[kCopyThreads / 32];
      if ((threadIdx.x & 31) == 0) {
        s_ae[threadIdx.x >> 5] = ae;
        s_dr[threadIdx.x >> 5] = dr;
      }
      if (e < E) {
        sc.offsets[e] = off;
        sc.mtile[e] = mt_off;
        if (sc.counts) sc.counts[e] = tot;
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        double a = 0.0;
        int drop = 0;
        for (int w = 0; w < kCopyThreads / 32; ++w) {
          a += s_ae[w];
          drop += s_dr[w];
        }
        sc.offsets[E] = run;
        sc.mtile[E] = mt;
        for (int s2 = 0; s2 < sc.n_shared; ++s2) {
          mt += (T + kTileM - 1) / kTileM;
          sc.mtile[E + 1 + s2] = mt;
        }
        if (sc.aux) *sc.aux = (float)((double)E * a);
        if (sc.dropped) *sc.dropped = drop;
        if (sc.zloss) {
          double z = 0.0;
          for (int b = 0; b < sc.nb; ++b) z += (double)sc.blk_z[b];
          *sc.zloss = (float)(z / (double)T);
        }
      }
    }
    __syncthreads();
  }
  if ((int)threadIdx.x < ng * k) {
    const int g = threadIdx.x / k, j = threadIdx.x - g * k;
    const int t = t0 + g;
    const int e = topk_idx[(size_t)t * k + j];
    int row = -1;
    bool bad = e < 0 || e >= E;
    if (!bad) {
      row = (kScan ? s_base[e] : blk_base[(size_t)(t / rb) * E + e]) + lrank[(size_t)t * k + j];
      if (has_cap && row >= (kScan ? s_end[e] : offsets[e + 1])) {
        row = -1;  // past the expert's capacity: this slot is dropped
        if (blockIdx.y == 0) inv[(size_t)t * k + j] = -1;
      } else if (row < 0 || row >= R) {
        bad = true;
      }
    }
    if (bad) {
      atomicOr(status, MOE_DEV_INTERNAL);
      row = -1;
    } else if (row >= 0 && blockIdx.y == 0) {
      perm_tok[row] = t;
      inv[(size_t)t * k + j] = row;
      rgate[row] = gate[(size_t)t * k + j];
    }
    s_rows[g][j] = row;
  }
  __syncthreads();
  if (zero_out) {  // the output rows this block's x chunk maps to, for a combine done by atomics
    const int per = (nout4 + gridDim.y - 1) / gridDim.y;
    const int o0 = blockIdx.y * per, w = min(nout4, o0 + per) - o0;
    for (int idx = threadIdx.x; idx < ng * w; idx += kCopyThreads) {
      const int g = idx / w;
      zero_out[(size_t)(t0 + g) * nout4 + o0 + (idx - g * w)] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  const int c0 = blockIdx.y * kCopyThreads;
  if constexpr (G == 1) {  // one vector per thread (fewer registers: eight blocks per SM)
    const int i = c0 + threadIdx.x;
    if (i >= nvec) return;
    uint4 v = __ldg(x + (size_t)t0 * nvec + i);
    if (rnorm) v = scale_vec(v, norm_w ? __ldg(norm_w + i) : make_uint4(0u, 0u, 0u, 0u), rnorm[t0], bf16 != 0,
                             norm_w != nullptr);
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j)
      if (j < k && s_rows[0][j] >= 0) xp[(size_t)s_rows[0][j] * nvec + i] = v;
    if (shared_row0 >= 0) xp[(size_t)(shared_row0 + t0) * nvec + i] = v;
    return;
  }
  const int cw = min(kCopyThreads, nvec - c0);  // vectors of this chunk in every row
  const int n = ng * cw;
  for (int base = threadIdx.x; base < n; base += 4 * kCopyThreads) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = base + u * kCopyThreads;
      if (idx < n) {
        const int g = idx / cw, i = c0 + idx - g * cw;
        v[u] = __ldg(x + (size_t)(t0 + g) * nvec + i);
        if (rnorm)
          v[u] = scale_vec(v[u], norm_w ? __ldg(norm_w + i) : make_uint4(0u, 0u, 0u, 0u), rnorm[t0 + g], bf16 != 0,
                           norm_w != nullptr);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = base + u * kCopyThreads;
      if (idx < n) {
        const int g = idx / cw, i = c0 + idx - g * cw;
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j)
          if (j < k && s_rows[g][j] >= 0) xp[(size_t)s_rows[g][j] * nvec + i] = v[u];
        if (shared_row0 >= 0) xp[(size_t)(shared_row0 + t0 + g) * nvec + i] = v[u];
      }
    }
  }
}

// Block (token t, chunk c): every thread sums one float4 of its token's k
// expert rows, weighted by the gates, in slot order (fp32), skipping dropped
// slots, then adds the token's rows of the shared experts in order.
// KM: the top-k rounded up to 2, 4, 6 or 8, so a thread holds only the rows
// it can have (fewer registers, more resident blocks for the loads in flight).
template <int KM>
__global__ void __launch_bounds__(kCopyThreads, KM <= 6 ? 6 : 4) combine_kernel(const float4* __restrict__ y, int nvec4, int k, int R,
                                                              int T, const int32_t* __restrict__ inv,
                                                              const float* __restrict__ gate, int has_cap,
                                                              int n_shared, int shared_row0,
                                                              float4* __restrict__ out, int32_t* status) {
  const int t = blockIdx.x;
  __shared__ int s_rows[kMaxTopK];
  __shared__ float s_g[kMaxTopK];
  pdl_wait();
  if (threadIdx.x < k) {
    const int j = threadIdx.x;
    int row = inv[(size_t)t * k + j];
    float g = gate[(size_t)t * k + j];
    if (row < 0 && has_cap) {
      row = -1;  // dropped slot
    } else if (row < 0 || row >= R) {
      atomicOr(status, MOE_DEV_INTERNAL);
      row = -1;
    }
    s_rows[j] = row;
    s_g[j] = g;
  }
  __syncthreads();
  const int i = blockIdx.y * kCopyThreads + threadIdx.x;
  if (i >= nvec4) return;
  float4 v[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j)
    if (j < k && s_rows[j] >= 0) v[j] = __ldg(y + (size_t)s_rows[j] * nvec4 + i);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    if (j < k && s_rows[j] >= 0) {
      const float g = s_g[j];
      acc.x = fmaf(g, v[j].x, acc.x);
      acc.y = fmaf(g, v[j].y, acc.y);
      acc.z = fmaf(g, v[j].z, acc.z);
      acc.w = fmaf(g, v[j].w, acc.w);
    }
  }
  for (int s2 = 0; s2 < n_shared; ++s2) {
    const float4 u = __ldg(y + (size_t)(shared_row0 + s2 * T + t) * nvec4 + i);
    acc.x += u.x;
    acc.y += u.y;
    acc.z += u.z;
    acc.w += u.w;
  }
  out[(size_t)t * nvec4 + i] = acc;
}

}  // namespace

cudaError_t launch_permute(moe_dtype dtype, const void* x, int T, int d, int E, int k, int rb, const int32_t* topk_idx,
                           const int32_t* lrank, const int32_t* blk_base, const int32_t* offsets, int has_cap,
                           int32_t* perm_tok, int32_t* inv, void* xp, const float* topk_gate, float* rgate,
                           float* zero_out, const float* rnorm, const void* norm_w, int shared_row0,
                           const PermuteScanArgs& scan, int32_t* status, cudaStream_t stream) {
  const int elem = dtype == MOE_BF16 ? 2 : 4;
  const int nvec = d * elem / 16;
  // tokens per block: up to 8 while the grid keeps about 512 blocks or more,
  // and fewer as a token's copies grow (measured: with k = 6 rows of 4 KB a
  // token, one token per block copies faster)
  const int copy_bytes = k * nvec * 16;
  const int gmax = copy_bytes <= 8192 ? 8 : copy_bytes <= 16384 ? 4 : 1;
  const int gt = T >= 4096 ? 8 : T >= 2048 ? 4 : T >= 1024 ? 2 : 1;
  const int G = gt < gmax ? gt : gmax;
  const dim3 grid((T + G - 1) / G, (nvec + kCopyThreads - 1) / kCopyThreads);
  const bool in_scan = scan.offsets != nullptr;
  auto kern = in_scan ? (G == 8 ? permute_kernel<8, true> : G == 4 ? permute_kernel<4, true>
                         : G == 2 ? permute_kernel<2, true> : permute_kernel<1, true>)
                      : (G == 8 ? permute_kernel<8, false> : G == 4 ? permute_kernel<4, false>
                         : G == 2 ? permute_kernel<2, false> : permute_kernel<1, false>);
  PermuteScan sc;
  sc.nb = scan.nb;
  sc.cap = scan.cap;
  sc.n_shared = scan.n_shared;
  sc.n_mt = scan.mt_done ? scan.n_mt : 0;
  sc.blk_psum = scan.blk_psum;
  sc.blk_z = scan.blk_z;
  sc.counts = scan.counts;
  sc.offsets = scan.offsets;
  sc.mtile = scan.mtile;
  sc.aux = scan.aux;
  sc.zloss = scan.zloss;
  sc.dropped = scan.dropped;
  sc.mt_done = scan.mt_done;
  return launch_pdl(kern, grid, dim3(kCopyThreads), 0, stream, static_cast<const uint4*>(x), T, nvec, E, k, rb, T * k,
                    topk_idx, lrank, blk_base, offsets, has_cap, perm_tok, inv, static_cast<uint4*>(xp), topk_gate,
                    rgate, reinterpret_cast<float4*>(zero_out), d / 4, rnorm, static_cast<const uint4*>(norm_w),
                    dtype == MOE_BF16 ? 1 : 0, shared_row0, status, sc);
}

cudaError_t launch_combine(int T, int d, int k, const float* y, const int32_t* inv, const float* topk_gate,
                           int has_cap, int n_shared, int shared_row0, float* out, int32_t* status,
                           cudaStream_t stream) {
  const int nvec4 = d / 4;
  const dim3 grid(T, (nvec4 + kCopyThreads - 1) / kCopyThreads);
  auto kern = k <= 2 ? combine_kernel<2> : k <= 4 ? combine_kernel<4> : k <= 6 ? combine_kernel<6> : combine_kernel<8>;
  return launch_pdl(kern, grid, dim3(kCopyThreads), 0, stream, reinterpret_cast<const float4*>(y), nvec4, k,
                    T * k, T, inv, topk_gate, has_cap, n_shared, shared_row0, reinterpret_cast<float4*>(out), status);
}

}  // namespace moe
