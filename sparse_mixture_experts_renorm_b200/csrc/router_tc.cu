// router_tc.cu — kernel (a) for bf16: the router as a 128 x E tile on the
// tcgen05 tensor cores, then softmax, top-k, gates, the per-block histogram,
// the in-block rank of every assignment and the per-block probability sums,
// with one thread per token.
//
// Method: axonml-nn layers/moe.rs, MoERouter::route (Linear -> softmax ->
// stable descending sort -> first k -> renormalise, 1/k if the sum is not
// positive), MoELayer::forward (its per-expert utilization counts),
// load_balancing_loss (E * sum_i f_i * P_i); Model Architecture Patterns,
// "Top-K Router" (raw top-k softmax gates when not renormalised).
//
// A block of 128 tokens (the UMMA M) is owned by a cluster of S CTAs that
// split the d-long K loop (S = 1 when the grid already fills the GPU): each
// CTA's warp 0 streams its share of x and W_r through a shared-memory ring by
// TMA, warp 1 issues 128 x N x 16 UMMAs (N = E rounded up to 16; TMA zero-fills
// the missing router rows), and warps 2-5 read each token's logits from their
// own TMEM lane. The other CTAs of the cluster add their partial logits into
// the leading CTA's shared memory, which finishes the block. For E <= 16 one
// thread per token does the softmax, top-k and gates with its logits in
// registers, then per-warp ballots give the histogram and ranks; for E > 16
// the logits go to shared memory and all six warps take four lanes per token
// (the softmax reduced by two shuffles, per-lane sorted top-k lists merged by
// a four-lane arg-max), the histogram being a bit mask per (expert, 32-token
// chunk). Both end with the block's probability sums and its sum of
// logsumexp^2 for the z-loss.
//
// With the pre-MoE RMSNorm (Mixtral MoE Block, nn.RMSNorm before the MoE;
// Model Architecture Patterns, "RMSNorm") the logits are
//   l[t,e] = r_t * sum_c x[t,c] * (w[c] * W_r[e,c]) + b[e],
// r_t = 1/sqrt(mean x^2 + eps) or 1/(sqrt(mean x^2) + eps): the epilogue
// warps square-sum their token's row of every x tile while the UMMAs run
// (they are extra consumers of the ring), and w * W_r enters as two bf16
// operands hi + lo whose products go to two accumulators, so x is used as
// stored and the weight's product is carried to about 16 bits.
#include <math.h>

#include <atomic>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kRB = kRouterTokensTc;  // 128 tokens per block
constexpr int kRegE = kRouterRegExperts;  // up to this many experts a token's logits stay in registers
constexpr int kSplitE = 64;           // up to this many experts the K loop may be split over a cluster

struct RouterCfg {
  int npad;         // UMMA N
  int lo_col;       // TMEM column of the second (w * W_r low part) accumulator
  int S;            // CTAs per token block (split of the K loop)
  int stages;       // ring depth
  int stage_bytes;  // x tile + W_r tile(s)
  int part_bytes;   // partial-logit (and partial square-sum) buffer of the leading CTA
  int tmem_cols;    // power of two >= max(32, columns read)
  int smem_bytes;   // dynamic shared memory
};

RouterCfg router_cfg(int T, int d, int E, bool norm, bool split, int num_sms) {
  RouterCfg c;
  c.npad = ((E + 15) / 16) * 16;
  c.lo_col = 32 * ((E + 31) / 32);
  c.stage_bytes = kRB * kBK * 2 + (split ? 2 : 1) * c.npad * kBK * 2;
  const int nb = (T + kRB - 1) / kRB;
  const int KB = d / kBK;
  const int per_cta = kRB * (E + (norm ? 1 : 0)) * 4;
  // split K only while the grid leaves SMs idle, the partial logits stay
  // small, and each CTA keeps at least two k-blocks
  c.S = 1;
  if (E <= kSplitE)
    while (c.S < 8 && nb * c.S * 2 <= num_sms && (c.S * 2 - 1) * per_cta <= 64 * 1024 && KB / (c.S * 2) >= 2)
      c.S *= 2;
  c.part_bytes = (c.S - 1) * per_cta;
  c.stages = (192 * 1024 - c.part_bytes) / c.stage_bytes;
  if (c.stages > 8) c.stages = 8;
  const int cols = split ? 2 * c.lo_col : c.lo_col;
  c.tmem_cols = 32;
  while (c.tmem_cols < cols) c.tmem_cols <<= 1;
  c.smem_bytes = c.stages * c.stage_bytes + c.part_bytes + 1024 + 13312;
  return c;
}

// (v, e) ranks ahead of (bv, be): larger probability, or equal and lower index.
__device__ __forceinline__ bool ahead(float v, int e, float bv, int be) { return v > bv || (v == bv && e < be); }

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ uint32_t cta_rank_in_cluster() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Store to the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ void st_cluster_f32(const void* local_in_leader_layout, uint32_t rank, float v) {
  uint32_t addr;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(addr) : "r"(smem_u32(local_in_leader_layout)), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
// The same for four floats at a 16-byte aligned offset.
__device__ __forceinline__ void st_cluster_v4(const void* local_in_leader_layout, uint32_t rank, float a, float b,
                                              float c, float d) {
  uint32_t addr;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(addr) : "r"(smem_u32(local_in_leader_layout)), "r"(rank));
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// Insert (v, e) into the list of the kMaxTopK best, kept sorted best first
// (an element that ranks behind all of them leaves the list unchanged).
// Branch-free: its position is the number of entries ranked ahead of it, and
// every slot then selects its old value, the new one or its predecessor.
__device__ __forceinline__ void topk_insert(float (&bv)[kMaxTopK], int (&be)[kMaxTopK], float v, int e) {
  int pos = 0;
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) pos += ahead(bv[j], be[j], v, e) ? 1 : 0;
#pragma unroll
  for (int j = kMaxTopK - 1; j > 0; --j) {
    const bool shift = j > pos, here = j == pos;
    bv[j] = shift ? bv[j - 1] : (here ? v : bv[j]);
    be[j] = shift ? be[j - 1] : (here ? e : be[j]);
  }
  if (pos == 0) {
    bv[0] = v;
    be[0] = e;
  }
}

// The routing scan of a batch that is a single router block (E <= 32): warp
// lanes are experts. Offsets and the GEMM tile prefix are inclusive shuffle
// scans of the kept counts, the statistic and the dropped count xor-reduced
// over the lanes in fp64, exactly as route_scan_kernel does for one block;
// the block's base rows are the offsets themselves.
__device__ __forceinline__ void single_block_scan(const RouterScan& sc, int T, int E, int k, int tot, float ps,
                                                  float blk_zsum, int32_t* blk_cnt, int lane) {
  const unsigned full = 0xffffffffu;
  const bool has = lane < E;
  if (!has) {
    tot = 0;
    ps = 0.f;
  }
  const int kept = sc.cap >= 0 ? min(tot, sc.cap) : tot;
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
  double p = (double)ps;  // the probability sum of one block, widened as the scan does
  double ae = has ? ((double)tot / ((double)T * (double)k)) * (p / (double)T) : 0.0;
  int dr = tot - kept;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    ae += __shfl_xor_sync(full, ae, o);
    dr += __shfl_xor_sync(full, dr, o);
  }
  if (has) {
    const int off = ik - kept;
    sc.offsets[lane] = off;
    sc.mtile[lane] = it - tiles;
    if (sc.counts) sc.counts[lane] = tot;
    blk_cnt[lane] = off;  // base row of block 0
  }
  const int run = __shfl_sync(full, ik, 31), mt0 = __shfl_sync(full, it, 31);
  if (lane == 0) {
    sc.offsets[E] = run;
    sc.mtile[E] = mt0;
    int mt = mt0;
    for (int s2 = 0; s2 < sc.n_shared; ++s2) {
      mt += (T + kTileM - 1) / kTileM;
      sc.mtile[E + 1 + s2] = mt;
    }
    if (sc.aux) *sc.aux = (float)((double)E * ae);
    if (sc.dropped) *sc.dropped = dr;
    if (sc.zloss) *sc.zloss = (float)((double)blk_zsum / (double)T);
  }
}

// E <= kE: logits in registers (fully unrolled code); kE == 0: E > kRegE,
// logits in shared memory and rolled loops (code executed once per block must
// stay small: unrolled per-expert code for large E thrashes the instruction
// cache)
template <int kE>
__global__ void __launch_bounds__(kGemmThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const __grid_constant__ CUtensorMap tmW2, const float* __restrict__ br, int T, int d, int E,
                     int k, int renorm, int npad, int lo_col, int split, int S, int stages, int stage_bytes,
                     int part_bytes, int tmem_cols, int norm_form, float norm_eps, float* __restrict__ rnorm,
                     int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate, int32_t* __restrict__ lrank,
                     int32_t* __restrict__ blk_cnt, float* __restrict__ blk_psum, float* __restrict__ blk_z,
                     const RouterScan scan, int32_t* status, uint64_t limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  float* part = reinterpret_cast<float*>(smem + stages * stage_bytes);  // [S-1][128][E] (leading CTA)
  float* part_ss = part + (size_t)(S - 1) * kRB * E;                   // [S-1][128] square sums (norm)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + stages * stage_bytes + part_bytes);
  uint64_t* full = bars;           // [stages]
  uint64_t* empty = bars + 8;      // [stages]
  uint64_t* tfull = bars + 16;
  uint64_t* done = bars + 17;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 18);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_idx = reinterpret_cast<int*>(s_tmem + 4);  // [128][kMaxTopK]
  int* s_wcnt = s_idx + kRB * kMaxTopK;              // [4][E] per-warp counts, then exclusive prefix
  float* s_z = reinterpret_cast<float*>(s_wcnt + 4 * E);  // [4] per-warp sums of logsumexp^2
  float* s_bias = s_z + 4;                                 // [E] router bias (leading CTA)
  float* s_rn = s_bias + E;                                // [128] RMSNorm scale per token (E > kRegE)
  float* s_lse2 = s_rn + kRB;                              // [128] logsumexp^2 per token (E > kRegE)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = S > 1 ? cta_rank_in_cluster() : 0u;
  // row stride of the logits in shared memory (E > kRegE): odd, so a warp's
  // 32 token rows fall in 32 banks
  const int ldp = (E + 1) | 1;
  const int blk = blockIdx.x / S;
  const int tok0 = blk * kRB;
  const int KB = d / kBK;
  const int kb0 = (int)rank * KB / S, kb1 = ((int)rank + 1) * KB / S;
  const int a_bytes = kRB * kBK * 2;
  const int w_bytes = npad * kBK * 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      // the UMMA commit, plus the 4 epilogue warps when they read x for the norm
      mbar_init(&empty[s], norm_form ? 5 : 1);
    }
    mbar_init(tfull, 1);
    mbar_init(done, 1);
    *s_abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
    if (split) tma_prefetch_desc(&tmW2);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  pdl_wait();

  constexpr int kL = kE > 0 ? kE : 1;
  float bias_pref = 0.f;  // b_r[r] for the leading CTA's epilogue thread r < E
  float lg[kL];    // this token's logits (register path)
  float ss = 0.f;  // this token's sum of x^2 (RMSNorm)
  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, s_abort, status, limit_ns)) break;
        mbar_arrive_expect_tx(&full[stage], stage_bytes);
        uint8_t* st = ring + stage * stage_bytes;
        tma_load_2d(st, &tmX, &full[stage], kb * kBK, tok0);
        tma_load_2d(st + a_bytes, &tmW, &full[stage], kb * kBK, 0);
        if (split) tma_load_2d(st + a_bytes + w_bytes, &tmW2, &full[stage], kb * kBK, 0);
        ++issued;
        if (++stage == stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      const int n = issued < stages ? issued : stages;
      for (int i = 0; i < n; ++i) {
        if (stage == 0) {
          stage = stages;
          phase ^= 1u;
        }
        --stage;
        mbar_wait(&full[stage], phase, nullptr, status, limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kRB, npad);
      int stage = 0;
      uint32_t phase = 0;
      bool mok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&full[stage], phase, s_abort, status, limit_ns)) {
          mok = false;
          break;
        }
        tc_fence_after();
        uint8_t* st = ring + stage * stage_bytes;
        const uint64_t adesc = sw128_kmajor_desc(smem_u32(st));
        const uint64_t bdesc = sw128_kmajor_desc(smem_u32(st + a_bytes));
        const uint64_t bdesc2 = sw128_kmajor_desc(smem_u32(st + a_bytes + w_bytes));
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint32_t accum = (kb > kb0 || kk > 0) ? 1u : 0u;
          tc_mma_bf16(tmem_base, adesc + static_cast<uint64_t>(kk * 2), bdesc + static_cast<uint64_t>(kk * 2), idesc,
                      accum);
          if (split)
            tc_mma_bf16(tmem_base + static_cast<uint32_t>(lo_col), adesc + static_cast<uint64_t>(kk * 2),
                        bdesc2 + static_cast<uint64_t>(kk * 2), idesc, accum);
        }
        tc_commit(&empty[stage]);
        if (++stage == stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (mok) tc_commit(tfull);
      tc_commit(done);
      mbar_wait(done, 0, nullptr, status, limit_ns);
    }
    __syncwarp();
  } else {
    const int q = warp & 3;
    const int r = q * 32 + lane;
    // the leading CTA's bias, read while the UMMAs run (E <= kRegE: one
    // expert per thread of the first quarter)
    if (kE > 0 && rank == 0 && br && r < E) bias_pref = br[r];
    // ------------- RMSNorm: this token's sum of x^2 over this CTA's K slice --
    // Row r of a 128B-swizzled x tile holds its 16-byte chunk c at position
    // c ^ (r & 7); each stage is summed on its own, then added to the total.
    if (norm_form) {
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, s_abort, status, limit_ns))) break;
        const uint8_t* row = ring + stage * stage_bytes + r * 128;
        float part_s = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(row + ((c ^ (r & 7)) << 4));
          const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float lo = __uint_as_float(u[i] << 16), hi = __uint_as_float(u[i] & 0xffff0000u);
            part_s = fmaf(lo, lo, part_s);
            part_s = fmaf(hi, hi, part_s);
          }
        }
        ss += part_s;
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
        if (++stage == stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    // -------------------------- read this CTA's partial logits from TMEM --
    const bool ok = __all_sync(0xffffffffu, mbar_wait(tfull, 0, s_abort, status, limit_ns));
    tc_fence_after();
    const uint32_t trow = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const int nchunks = (E + 31) >> 5;
    float* s_p = reinterpret_cast<float*>(ring);  // [128][ldp] when E > kRegE (ring free after the MMAs)
    for (int c = 0; c < nchunks; ++c) {
      uint32_t v[32];
      __syncwarp();
      if (ok) {
        tmem_ld_x32(trow + c * 32, v);
        tmem_ld_wait();
        if (split) {
          uint32_t v2[32];
          __syncwarp();
          tmem_ld_x32(trow + static_cast<uint32_t>(lo_col) + c * 32, v2);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) + __uint_as_float(v2[i]));
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0u;
      }
      if (kE > 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
#pragma unroll
          for (int cc = 0; cc * 32 < kL; ++cc)
            if (c == cc && cc * 32 + i < kL) lg[cc * 32 + i] = __uint_as_float(v[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (c * 32 + i < E) s_p[r * ldp + c * 32 + i] = __uint_as_float(v[i]);
      }
    }
    if (S > 1 && rank > 0) {  // this CTA's share of the K loop goes to the leader
      float* dst = part + ((size_t)(rank - 1) * kRB + r) * E;
      if (kE > 0 && (E & 3) == 0) {  // rows of E floats start on 16-byte boundaries
#pragma unroll
        for (int e = 0; e < kL; e += 4)
          if (e < E) st_cluster_v4(dst + e, 0, lg[e], lg[e + 1], lg[e + 2], lg[e + 3]);
      } else if (kE > 0) {
#pragma unroll
        for (int e = 0; e < kL; ++e)
          if (e < E) st_cluster_f32(dst + e, 0, lg[e]);
      } else {
        for (int e = 0; e < E; ++e) st_cluster_f32(dst + e, 0, s_p[r * ldp + e]);
      }
      if (norm_form) st_cluster_f32(part_ss + (size_t)(rank - 1) * kRB + r, 0, ss);
    }
  }

  if (S > 1) cluster_sync_all();  // every partial has landed in the leading CTA

  if (kE > 0 && rank == 0 && warp >= 2) {
    // ------------------------- E <= kRegE: one thread per token, in registers --
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int t = tok0 + r;
    const bool valid = t < T;
    const int ld = E + 1;
    float* s_p = reinterpret_cast<float*>(ring);  // [128][E+1] probabilities
    float bv[kMaxTopK];
    int be[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      bv[j] = -INFINITY;
      be[j] = 0x7fffffff;
    }
    bool finite = true;
    if (br) {  // the bias once per block (read before the cluster barrier), then from shared memory
      if (r < E) s_bias[r] = bias_pref;
      epi_bar();
    }
    // RMSNorm scale of this token (1 without the norm)
    float rn = 1.0f;
    if (norm_form) {
      for (int s2 = 0; s2 < S - 1; ++s2) ss += part_ss[(size_t)s2 * kRB + r];
      const float ms = ss / (float)d;
      rn = norm_form == MOE_NORM_RMS ? 1.0f / sqrtf(ms + norm_eps) : 1.0f / (sqrtf(ms) + norm_eps);
      if (valid) rnorm[t] = rn;
    }
    float lse;  // log sum_e exp(logit)
    if (kE > 0) {
      // the other CTAs' partial logits in rank order, the norm scale, the
      // bias, the maximum
      for (int s2 = 0; s2 < S - 1; ++s2) {
        const float* src = part + ((size_t)s2 * kRB + r) * E;
        if ((E & 3) == 0) {
#pragma unroll
          for (int e = 0; e < kL; e += 4)
            if (e < E) {
              const float4 p4 = *reinterpret_cast<const float4*>(src + e);
              lg[e] += p4.x;
              lg[e + 1] += p4.y;
              lg[e + 2] += p4.z;
              lg[e + 3] += p4.w;
            }
        } else {
#pragma unroll
          for (int e = 0; e < kL; ++e)
            if (e < E) lg[e] += src[e];
        }
      }
      // four independent chains (experts e mod 4) for the maximum and the sum
      float mc[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int e = 0; e < kL; ++e)
        if (e < E) {
          if (norm_form) lg[e] *= rn;
          if (br) lg[e] += s_bias[e];
          finite = finite && isfinite(lg[e]);
          mc[e & 3] = fmaxf(mc[e & 3], lg[e]);
        }
      const float m = fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3]));
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int e = 0; e < kL; ++e)
        if (e < E) {
          lg[e] = __expf(lg[e] - m);
          sc[e & 3] += lg[e];
        }
      const float s = (sc[0] + sc[1]) + (sc[2] + sc[3]);
      lse = m + logf(s);
      const float inv_s = 1.0f / s;
#pragma unroll
      for (int e = 0; e < kL; ++e)
        if (e < E) {
          const float p = lg[e] * inv_s;
          s_p[r * ld + e] = valid ? p : 0.f;
          lg[e] = (p != p) ? -INFINITY : p;
        }
      // k passes of an arg-max over the (at most kE) probabilities: a strict
      // comparison in ascending expert order keeps the lower index on ties,
      // and the first candidate is always taken, so every token gets k
      // distinct experts even when some probabilities are -inf
      uint32_t taken = 0;
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j) {
        if (j < k) {
          float best = -INFINITY;
          int bi = -1;
#pragma unroll
          for (int e = 0; e < kL; ++e)
            if (e < E && !((taken >> e) & 1u) && (bi < 0 || lg[e] > best)) {
              best = lg[e];
              bi = e;
            }
          taken |= 1u << bi;
          bv[j] = best;
          be[j] = bi;
        }
      }
    }
    if (valid && !finite) atomicOr(status, MOE_DEV_NONFINITE);
    if (blk_z) {  // this warp's sum of logsumexp^2 (a fixed shuffle tree)
      float z = valid ? lse * lse : 0.f;
#pragma unroll
      for (int off = 16; off; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
      if (lane == 0) s_z[q] = z;
    }
    float psel = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j)
      if (j < k) psel += bv[j];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j < k) {
        float g;
        if (!renorm)
          g = bv[j];
        else if (psel > 0.f)
          g = bv[j] / psel;
        else
          g = 1.0f / (float)k;
        if (valid) {
          topk_idx[(size_t)t * k + j] = be[j];
          topk_gate[(size_t)t * k + j] = g;
        }
        s_idx[r * kMaxTopK + j] = valid ? be[j] : -1;
      }
    }
    __syncwarp();

    // per-warp histogram and in-warp rank of each assignment
    uint32_t myrank[kMaxTopK];
    int mine[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      myrank[j] = 0;
      mine[j] = j < k ? s_idx[r * kMaxTopK + j] : -1;
    }
#pragma unroll 4
    for (int e = 0; e < E; ++e) {
      int jhit = -1;
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j)
        if (mine[j] == e) jhit = j;
      const uint32_t mask = __ballot_sync(0xffffffffu, jhit >= 0);
      const uint32_t rk = __popc(mask & ((1u << lane) - 1u));
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j)
        if (j == jhit) myrank[j] = rk;
      if (lane == 0) s_wcnt[q * E + e] = __popc(mask);
    }
    epi_bar();
    // block totals and the exclusive prefix over the 4 row quarters
    int my_tot = 0;     // thread r < E: expert r's count in this block
    float my_ps = 0.f;  //                and its probability sum
    for (int e = r; e < E; e += kRB) {
      int run = 0;
      for (int qq = 0; qq < 4; ++qq) {
        const int c = s_wcnt[qq * E + e];
        s_wcnt[qq * E + e] = run;
        run += c;
      }
      blk_cnt[(size_t)blk * E + e] = run;
      float ps0 = 0.f, ps1 = 0.f, ps2 = 0.f, ps3 = 0.f;  // four chains over the block's tokens
      // rows past the batch hold probability 0: stop at the last group of
      // four that holds a token (the sums are the same)
      const int nr4 = (min(kRB, T - tok0) + 3) & ~3;
#pragma unroll 4
      for (int rr = 0; rr < nr4; rr += 4) {
        ps0 += s_p[rr * ld + e];
        ps1 += s_p[(rr + 1) * ld + e];
        ps2 += s_p[(rr + 2) * ld + e];
        ps3 += s_p[(rr + 3) * ld + e];
      }
      blk_psum[(size_t)blk * E + e] = (ps0 + ps1) + (ps2 + ps3);
      my_tot = run;
      my_ps = (ps0 + ps1) + (ps2 + ps3);
    }
    if (blk_z && r == 0) blk_z[blk] = ((s_z[0] + s_z[1]) + s_z[2]) + s_z[3];
    if (scan.offsets) {
      // the whole batch is this one block: the routing scan's results follow
      // from its counts directly (the same arithmetic and order as
      // route_scan_kernel for one block), and no scan kernel runs
      for (int i = r; i < scan.n_mt; i += kRB) scan.mt_done[i] = 0;
      if (q == 0) single_block_scan(scan, T, E, k, my_tot, my_ps,
                                    blk_z ? ((s_z[0] + s_z[1]) + s_z[2]) + s_z[3] : 0.f, blk_cnt, lane);
    }
    epi_bar();
    if (valid) {
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j)
        if (j < k) lrank[(size_t)t * k + j] = (int)myrank[j] + s_wcnt[q * E + be[j]];
    }
  }

  if (kE == 0 && rank == 0) {
    // ------------- E > kRegE: all six warps finish the block, four lanes a token --
    // Expert e of a token belongs to lane e mod 4 of its four: the softmax
    // reduces over the four lanes with two shuffles, each lane keeps a sorted
    // top-k list of its experts, and k rounds of a four-lane arg-max merge
    // them (ties to the lower index, as every list is). A warp takes eight
    // tokens four rows apart, so its 32 lanes read 32 different banks of the
    // odd-strided rows. The histogram is a bit mask per (expert, 32-token
    // chunk), from which the in-block ranks and the counts follow; one warp
    // per expert sums its probabilities in a fixed order.
    float* s_p = reinterpret_cast<float*>(ring);             // [128][ldp] logits, then probabilities
    uint32_t* s_mask = reinterpret_cast<uint32_t*>(s_wcnt);  // [E][4] tokens of a chunk choosing e
    if (warp >= 2) {
      const int r = (warp & 3) * 32 + lane;
      float rn = 1.0f;  // RMSNorm scale of this token (1 without the norm)
      if (norm_form) {
        for (int s2 = 0; s2 < S - 1; ++s2) ss += part_ss[(size_t)s2 * kRB + r];
        const float ms = ss / (float)d;
        rn = norm_form == MOE_NORM_RMS ? 1.0f / sqrtf(ms + norm_eps) : 1.0f / (sqrtf(ms) + norm_eps);
        if (tok0 + r < T) rnorm[tok0 + r] = rn;
      }
      s_rn[r] = rn;
    }
    if (br)
      for (int e = threadIdx.x; e < E; e += kGemmThreads) s_bias[e] = br[e];
    for (int i = threadIdx.x; i < 4 * E; i += kGemmThreads) s_mask[i] = 0u;
    __syncthreads();

    const int sub = lane & 3;
    for (int set = warp; set < kRB / 8; set += kGemmThreads / 32) {  // 16 sets of 8 tokens
      const int r = (set >> 2) * 32 + (set & 3) + 4 * (lane >> 2);
      const int t = tok0 + r;
      const bool valid = t < T;
      float* pr = s_p + r * ldp;
      const float rn = s_rn[r];
      float m = -INFINITY;
      bool finite = true;
      for (int e = sub; e < E; e += 4) {
        float l = pr[e];
        for (int s2 = 0; s2 < S - 1; ++s2) l += part[((size_t)s2 * kRB + r) * E + e];
        if (norm_form) l *= rn;
        if (br) l += s_bias[e];
        finite = finite && isfinite(l);
        pr[e] = l;
        m = fmaxf(m, l);
      }
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      float sum = 0.f;
      for (int e = sub; e < E; e += 4) {
        const float ex = __expf(pr[e] - m);
        pr[e] = ex;
        sum += ex;
      }
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      const float lse = m + logf(sum);
      const float inv_s = 1.0f / sum;
      float bv[kMaxTopK];
      int be[kMaxTopK];
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j) {
        bv[j] = -INFINITY;
        be[j] = 0x7fffffff;
      }
      for (int e = sub; e < E; e += 4) {
        const float p = pr[e] * inv_s;
        pr[e] = valid ? p : 0.f;
        topk_insert(bv, be, (p != p) ? -INFINITY : p, e);  // a NaN ranks last
      }
      // k rounds: the best head of the four lists wins and leaves its list
      float gv[kMaxTopK];
      int ge[kMaxTopK];
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j) {
        gv[j] = 0.f;
        ge[j] = 0;
        if (j < k) {
          float cv = bv[0];
          int ce = be[0];
#pragma unroll
          for (int off = 1; off <= 2; off <<= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, cv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, ce, off);
            if (ahead(ov, oe, cv, ce)) {
              cv = ov;
              ce = oe;
            }
          }
          gv[j] = cv;
          ge[j] = ce;
          const bool won = be[0] == ce;
#pragma unroll
          for (int i = 0; i + 1 < kMaxTopK; ++i) {
            bv[i] = won ? bv[i + 1] : bv[i];
            be[i] = won ? be[i + 1] : be[i];
          }
          if (won) {
            bv[kMaxTopK - 1] = -INFINITY;
            be[kMaxTopK - 1] = 0x7fffffff;
          }
        }
      }
      int fin = finite ? 1 : 0;
      fin &= __shfl_xor_sync(0xffffffffu, fin, 1);
      fin &= __shfl_xor_sync(0xffffffffu, fin, 2);
      float psel = 0.f;
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j)
        if (j < k) psel += gv[j];
      if (sub == 0) {
        if (valid && !fin) atomicOr(status, MOE_DEV_NONFINITE);
        s_lse2[r] = valid ? lse * lse : 0.f;
      }
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j) {
        if (j < k && (j & 3) == sub) {  // slot j is written by lane j mod 4
          float g;
          if (!renorm)
            g = gv[j];
          else if (psel > 0.f)
            g = gv[j] / psel;
          else
            g = 1.0f / (float)k;
          if (valid) {
            topk_idx[(size_t)t * k + j] = ge[j];
            topk_gate[(size_t)t * k + j] = g;
            atomicOr(&s_mask[ge[j] * 4 + (r >> 5)], 1u << (r & 31));
          }
          s_idx[r * kMaxTopK + j] = valid ? ge[j] : -1;
        }
      }
    }
    __syncthreads();

    // rank of each assignment among the block's tokens choosing its expert
    for (int i = threadIdx.x; i < kRB * k; i += kGemmThreads) {
      const int r = i / k, j = i - r * k;
      const int e = s_idx[r * kMaxTopK + j];
      if (e >= 0) {
        const int c = r >> 5;
        int rk = __popc(s_mask[e * 4 + c] & ((1u << (r & 31)) - 1u));
        for (int cc = 0; cc < c; ++cc) rk += __popc(s_mask[e * 4 + cc]);
        lrank[(size_t)(tok0 + r) * k + j] = rk;
      }
    }
    // per expert: the block's count and its probability sum (a fixed tree)
    for (int e = warp; e < E; e += kGemmThreads / 32) {
      float ps = ((s_p[lane * ldp + e] + s_p[(lane + 32) * ldp + e]) + s_p[(lane + 64) * ldp + e]) +
                 s_p[(lane + 96) * ldp + e];
#pragma unroll
      for (int off = 16; off; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      if (lane == 0) {
        blk_psum[(size_t)blk * E + e] = ps;
        blk_cnt[(size_t)blk * E + e] =
            __popc(s_mask[e * 4]) + __popc(s_mask[e * 4 + 1]) + __popc(s_mask[e * 4 + 2]) + __popc(s_mask[e * 4 + 3]);
      }
    }
    if (blk_z && warp == 0) {  // per 32-token quarter a shuffle tree, then the quarters in order
      float z = 0.f;
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        float zq = s_lse2[qq * 32 + lane];
#pragma unroll
        for (int off = 16; off; off >>= 1) zq += __shfl_xor_sync(0xffffffffu, zq, off);
        z = qq == 0 ? zq : z + zq;
      }
      if (lane == 0) blk_z[blk] = z;
    }
  }

  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

// SMs of the current device, queried once per device (host threads that race
// on the first query store the same value).
int sm_count() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  const int have = cache[dev].load(std::memory_order_acquire);
  if (have > 0) return have;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  cache[dev].store(n, std::memory_order_release);
  return n;
}

}  // namespace

cudaError_t launch_router_tc(const void* x, const void* w_router, const float* b_router, int T, int d, int E, int k,
                             int renorm, const RouterNorm& norm, int32_t* topk_idx, float* topk_gate, int32_t* lrank,
                             int32_t* blk_cnt, float* blk_psum, float* blk_z, const RouterScan& scan,
                             int32_t* status, cudaStream_t stream) {
  const bool split = norm.form != 0 && norm.w_hi != nullptr;
  const RouterCfg c = router_cfg(T, d, E, norm.form != 0, split, sm_count());
  CUtensorMap tmX, tmW, tmW2;
  if (!make_tmap_bf16_2d(&tmX, x, (uint64_t)T, (uint64_t)d, kRB) ||
      !make_tmap_bf16_2d(&tmW, split ? norm.w_hi : w_router, (uint64_t)E, (uint64_t)d, (uint32_t)c.npad) ||
      !make_tmap_bf16_2d(&tmW2, split ? norm.w_lo : w_router, (uint64_t)E, (uint64_t)d, (uint32_t)c.npad))
    return cudaErrorInvalidValue;
  // the register path unrolled for 8 or 16 experts: its code runs once per
  // block, so the shorter body of the common E <= 8 spends less on fetching it
  auto kern = E <= 8 ? router_tc_kernel<8> : E <= kRegE ? router_tc_kernel<kRegE> : router_tc_kernel<0>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, c.smem_bytes);
  if (err != cudaSuccess) return err;
  const int nb = (T + kRB - 1) / kRB;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nb * c.S);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = c.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  attrs[1].id = cudaLaunchAttributeClusterDimension;
  attrs[1].val.clusterDim.x = c.S;
  attrs[1].val.clusterDim.y = 1;
  attrs[1].val.clusterDim.z = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = c.S > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, tmX, tmW, tmW2, b_router, T, d, E, k, renorm, c.npad, c.lo_col, split ? 1 : 0,
                            c.S, c.stages, c.stage_bytes, c.part_bytes, c.tmem_cols, norm.form, norm.eps, norm.rnorm,
                            topk_idx, topk_gate, lrank, blk_cnt, blk_psum, blk_z,
                            router_does_scan(T, E, MOE_BF16) ? scan : RouterScan{}, status, kWaitLimitNs);
}

namespace {

// hi = bf16(w * W_r) (round to nearest even), lo = bf16(w * W_r - hi): the
// product of two bf16 values is exact in fp32, and hi + lo keeps about 16 of
// its bits.
__global__ void __launch_bounds__(256) split_router_weight_kernel(const uint4* __restrict__ wr,
                                                                 const uint4* __restrict__ w, int E, int dv,
                                                                 uint4* __restrict__ hi, uint4* __restrict__ lo) {
  pdl_wait();
  const int n = E * dv;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const uint4 a = wr[i], b = w[i % dv];
    const uint32_t ua[4] = {a.x, a.y, a.z, a.w}, ub[4] = {b.x, b.y, b.z, b.w};
    uint32_t h[4], l[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float p0 = __uint_as_float(ua[j] << 16) * __uint_as_float(ub[j] << 16);
      const float p1 = __uint_as_float(ua[j] & 0xffff0000u) * __uint_as_float(ub[j] & 0xffff0000u);
      const __nv_bfloat16 h0 = __float2bfloat16_rn(p0), h1 = __float2bfloat16_rn(p1);
      const __nv_bfloat16 l0 = __float2bfloat16_rn(p0 - __bfloat162float(h0));
      const __nv_bfloat16 l1 = __float2bfloat16_rn(p1 - __bfloat162float(h1));
      h[j] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
      l[j] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
    }
    hi[i] = make_uint4(h[0], h[1], h[2], h[3]);
    lo[i] = make_uint4(l[0], l[1], l[2], l[3]);
  }
  pdl_trigger();
}

}  // namespace

cudaError_t launch_split_router_weight(const void* w_router, const void* norm_w, int E, int d, void* hi, void* lo,
                                       cudaStream_t stream) {
  const int dv = d / 8;
  const int n = E * dv;
  int blocks = (n + 255) / 256;
  if (blocks > 4 * sm_count()) blocks = 4 * sm_count();
  return launch_pdl(split_router_weight_kernel, dim3(blocks), dim3(256), 0, stream,
                    static_cast<const uint4*>(w_router), static_cast<const uint4*>(norm_w), E, dv,
                    static_cast<uint4*>(hi), static_cast<uint4*>(lo));
}

}  // namespace moe
