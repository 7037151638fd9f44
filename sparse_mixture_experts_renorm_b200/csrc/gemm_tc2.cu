// gemm_tc2.cu — kernel (c): the two grouped expert GEMMs on tcgen05 with a
// pair of CTAs (cta_group::2) per 256 x 256 output tile.
//
//   mode 0 (gate/up):  H[r, :] = SiLU(Xp[r] . W_gate[e]^T) * (Xp[r] . W_up[e]^T)
//   mode 1 (down):     Y[r, :] = H[r] . W_down[e]^T
//
// for every dispatched row r of expert e (axonml-nn layers/moe.rs,
// Expert::forward: down(SiLU(gate(x)) * up(x)); Model Architecture Patterns,
// "SwiGLU FFN"). Rows are expert-contiguous, so expert e's rows form the M
// dimension of its own GEMM; 256-row tiles that run past the expert's last row
// compute on neighbouring rows (or TMA zero fill) and are masked at the store.
//
// A cluster of two CTAs on two SMs owns one tile at a time. Weight-major
// form: each CTA stages its own 128 weight rows as A (mode 0: the 64 gate rows
// and the 64 up rows of its 64 hidden units; mode 1: 128 W_down rows) and one
// half of the tile's token rows as B through a TMA ring (5 or 6 stages, 11
// for the stream configuration), both signalling the leading CTA's barrier. One
// thread of the leading CTA issues 256xNx16 UMMAs that read A and B from both
// CTAs' shared memory and write each CTA's 128 rows of the fp32 accumulator
// into that CTA's TMEM (double-buffered, 2 x 256 columns); commits are
// multicast to both CTAs. Each CTA's 8 epilogue warps, two per TMEM lane
// quarter taking alternate 32-token chunks, drain their TMEM lanes (SwiGLU +
// bf16 in mode 0, fp32 in mode 1) and release the accumulator to the leader.
// Per UMMA FLOP this moves a third fewer bytes from L2 to shared memory than
// one CTA per 128 x 256 tile.
//
// Token-major form (the wide configuration's gate/up GEMM, and a down GEMM
// whose grid has at most three tiles per CTA pair): the tile's 256 token rows
// are the UMMA M operand (128 per CTA) and its weight rows the N operand. For
// gate/up, CTA 0 stages the block's 128 gate rows and CTA 1 the same units'
// 128 up rows, so every TMEM lane holds one token's gate values in columns
// 0-127 and its up values in columns 128-255 and SwiGLU needs no exchange
// between warps: the epilogue goes from TMEM to registers to its token's H
// row and leaves shared memory to the TMA ring (6 stages) and the UMMAs. For
// down, each lane holds one token's 256 outputs. The operand bytes per tile
// are the same as in the weight-major form.
//
// Persistent: clusters walk a device-side tile list built from the routing
// counts (experts in order; n-tile outer, m-tile inner inside an expert, so
// clusters running together share weight tiles in L2). Shared experts
// ("moe_shared_experts", KempnerForge ModelConfig) are extra groups after the
// routed experts, each over all T tokens, with their own weight tensor maps.
// Every wait is bounded.
#include <atomic>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kHalfBytes = 128 * kBK * 2;          // 16 KB: 128 rows x 64 bf16
constexpr int kSmallRows = 16;                     // B box for tiles of <= 32 tokens

// Configurations of the kernel. "Wide" tiles (many tokens per expert): warps
// 2-9 drain the accumulator, two per TMEM lane quarter taking alternate
// 32-column chunks; token-major with a 6-stage ring and no epilogue staging
// (WideTM), or weight-major with a 5-stage ring (Wide, the down GEMM with the
// folded combine on longer grids).
// "Narrow" tiles (decode-sized batches that stream the weights from HBM): a
// deeper 6-stage ring keeps more bytes in flight and warps 2-5 drain it.
// "Stream" (at most 32 tokens in the whole batch, so every tile's token rows
// fit the 16-row box): the B slot shrinks to 2 KB and the ring to 11 stages
// of 18 KB, nearly twice the weight bytes in flight of the narrow ring.
// Epilogue staging: per group of four epilogue warps the gate and up rows of
// a 32-token chunk (mode 0, 2 x 64 x 33 fp32), or one 32 x 32 fp32 transpose
// tile per epilogue warp (mode 1, 32 x 36).
template <int kSt, int kEw, int kBRows, bool kTokMajor = false>
struct Gemm2Cfg {
  static constexpr bool kTokM = kTokMajor;  // token rows as the UMMA M operand (see the kernel)
  static constexpr int kStages = kSt;
  static constexpr int kEpiWarps = kEw;
  static constexpr int kBSlotRows = kBRows;            // token rows a stage holds per CTA
  static constexpr int kBSlotBytes = kBRows * kBK * 2;
  static constexpr int kThreads = 64 + 32 * kEw;
  static constexpr int kEpiBytesM0 = (kEw / 4) * (2 * 64 * 33 * 4);
  static constexpr int kEpiBytesM1 = kEw * 32 * 36 * 4;
  static constexpr int kEpiBytes = kTokMajor ? 0 : (kEpiBytesM1 > kEpiBytesM0 ? kEpiBytesM1 : kEpiBytesM0);
  static constexpr int kSmemBytes = kSt * (kHalfBytes + kBSlotBytes) + kEpiBytes + 1024 + 4096;
};
using Gemm2Wide = Gemm2Cfg<5, 8, 128>;
using Gemm2WideTM = Gemm2Cfg<6, 8, 128, true>;  // token-major: no epilogue staging, a sixth stage
using Gemm2Narrow = Gemm2Cfg<6, 4, 128>;
using Gemm2Stream = Gemm2Cfg<11, 4, kSmallRows>;
static_assert(Gemm2Wide::kSmemBytes <= 227 * 1024 && Gemm2WideTM::kSmemBytes <= 227 * 1024 &&
                  Gemm2Narrow::kSmemBytes <= 227 * 1024 &&
                  Gemm2Stream::kSmemBytes <= 227 * 1024,
              "shared memory");

// named barrier of one group of four epilogue warps (ids 1 and 2, 128 threads)
__device__ __forceinline__ void epi_bar(int half) { asm volatile("bar.sync %0, 128;" ::"r"(1 + half) : "memory"); }

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t num_clusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Shared::cluster address of the same shared variable in CTA `rank`.
__device__ __forceinline__ uint32_t map_to_cta(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA tile load into this CTA's shared memory whose completion is counted on
// the barrier at `bar_cluster` (the leading CTA's).
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint32_t bar_cluster, int x,
                                                 int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on the barrier at this offset in both CTAs of the pair once the
// pair's UMMAs issued so far have completed.
__device__ __forceinline__ void tc_commit_pair_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)0x3)
      : "memory");
}
__device__ __forceinline__ void tc_commit_pair_local(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

// 32 accumulator columns of this warp's lanes, summed over the tile's
// accumulators in order (a tile with one accumulator is a plain load).
__device__ __forceinline__ void ld_chunk_sum(uint32_t taddr, int nacc, int stride, uint32_t (&v)[32]) {
  __syncwarp();
  tmem_ld_x32(taddr, v);
  tmem_ld_wait();
  for (int a = 1; a < nacc; ++a) {
    uint32_t w[32];
    __syncwarp();
    tmem_ld_x32(taddr + a * stride, w);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) + __uint_as_float(w[i]));
  }
}

struct TileCoord {
  int e, m, n;  // group (routed expert, then shared experts), token tile, weight block
};

// Rows of group g: routed experts read and write their dispatched rows;
// shared expert s reads sh.rows rows at sh.in0 + s * sh.in_step and writes
// them at sh.out0 + s * sh.rows.
struct GroupRows {
  int in0, out0, cnt, widx;
  bool shared;
};

__device__ __forceinline__ GroupRows group_rows(int g, const int* s_off, int E, const SharedGroups& sh) {
  GroupRows r;
  if (g < E) {
    r.in0 = r.out0 = s_off[g];
    r.cnt = s_off[g + 1] - s_off[g];
    r.widx = g;
    r.shared = false;
  } else {
    const int s = g - E;
    r.in0 = sh.in0 + s * sh.in_step;
    r.out0 = sh.out0 + s * sh.rows;
    r.cnt = sh.rows;
    r.widx = s;
    r.shared = true;
  }
  return r;
}

__device__ __forceinline__ TileCoord decode_tile(int tile, int n_tiles, const int* s_mt, int E) {
  const int q = tile / n_tiles;
  int lo = 0, hi = E;  // s_mt[lo] <= q < s_mt[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_mt[mid] <= q)
      lo = mid;
    else
      hi = mid;
  }
  TileCoord c;
  c.e = lo;
  const int mt_e = s_mt[lo + 1] - s_mt[lo];
  const int local = tile - s_mt[lo] * n_tiles;
  c.n = local / mt_e;
  c.m = local - c.n * mt_e;
  return c;
}

__device__ __forceinline__ float silu_f32(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// One GEMM of the kernel: its shared-expert groups, output width N (hidden
// units for gate/up, features for down), reduction length K and output.
struct GemmPhase {
  SharedGroups sh;
  int N, K;
  void* out;
};

// Orders this thread's generic-proxy global accesses with its async-proxy
// (TMA) accesses.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Waits until *counter >= target (acquire at GPU scope), polling with a short
// sleep, for at most limit_ns; on time-out MOE_DEV_TIMEOUT is OR-ed into the
// status word and the CTA-wide abort flag raised. Returns false when giving up.
__device__ __forceinline__ bool wait_counter_geq(const int32_t* counter, int target, volatile int* abort_flag,
                                                 int32_t* status, uint64_t limit_ns) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
  if (v >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    __nanosleep(128);
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
    if (v >= target) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicOr(status, MOE_DEV_TIMEOUT);
      return false;
    }
  }
}

// kMode 0: gate/up only; 1: down only; 2: both in one persistent launch
// (every gate/up tile, then every down tile; a down tile's producers wait
// until all gate/up tiles of its token tile have stored their H rows, counted
// in mt_done, so one projection's last round overlaps the other's first).
// Maps: tmA0/tmA1 (W_gate/W_up, or W_down twice in mode 1), tmS0/tmS1 (the
// shared experts' counterparts), tmB/tmBs (the B operand in 128- and 16-row
// boxes); in mode 2 tmD/tmSD/tmH/tmHs are the down projection's.
template <int kMode, int kSt, int kEw, int kBRows, bool kTokM>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(64 + 32 * kEw, 1)
    grouped_gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                            const __grid_constant__ CUtensorMap tmS0, const __grid_constant__ CUtensorMap tmS1,
                            const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmBs,
                            const __grid_constant__ CUtensorMap tmD, const __grid_constant__ CUtensorMap tmSD,
                            const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmHs,
                            const int32_t* __restrict__ offsets, const int32_t* __restrict__ mtile256, int E,
                            const GemmPhase p0, const GemmPhase p1, const int32_t* __restrict__ perm_tok,
                            const float* __restrict__ rgate, float* __restrict__ comb_out,
                            int32_t* __restrict__ mt_done, int32_t* status, uint64_t limit_ns) {
  using Cfg = Gemm2Cfg<kSt, kEw, kBRows, kTokM>;
  // token-major tiles: the tile's 256 token rows are the UMMA M operand (128
  // per CTA) and its weight rows the N operand. Gate/up: the block's 128
  // hidden units, gate rows from CTA 0 and up rows from CTA 1, so each TMEM
  // lane holds one token's gate (columns 0-127) and up (128-255) values side
  // by side. Down: the block's 256 output features, 128 W_down rows per CTA,
  // so each lane holds one token's 256 outputs.
  constexpr bool kTM = kTokM && kMode != 2;
  constexpr int kBSlot = Cfg::kBSlotBytes;
  constexpr int kGroups = kEw / 4;  // groups of four epilogue warps (one per TMEM lane quarter each)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                           // [stages][128 weight rows x 64]
  uint8_t* sB = smem + kSt * kHalfBytes;   // [stages][<= kBRows token rows x 64]
  float* sEpi = reinterpret_cast<float*>(smem + kSt * (kHalfBytes + kBSlot));
  float* sY = sEpi;  // [8][32][36] (mode 1)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSt * (kHalfBytes + kBSlot) + Cfg::kEpiBytes);
  uint64_t* full = bars;                 // leader: A+B bytes of both CTAs
  uint64_t* empty = bars + kSt;     // both: stage consumed by the pair's UMMAs
  uint64_t* tfull = bars + 2 * kSt; // both: accumulator ready
  uint64_t* tempty = tfull + 2;          // leader: 256 epilogue arrivals
  uint64_t* done = tempty + 2;           // leader: every UMMA completed
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_off = reinterpret_cast<int*>(s_tmem + 4);  // [E+1]
  int* s_mt = s_off + (E + 1);                       // [G+1]
  const int G = E + p0.sh.n;                         // GEMM groups: routed, then shared experts

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cid = (int)cluster_id_x();
  const int ncl = (int)num_clusters_x();
  // weight blocks per expert: 128 hidden units (gate + up rows) or 256 output
  // features; phase 1 exists in mode 2 only
  const int n_wb0 = kMode == 1 ? (p0.N + 255) / 256 : (p0.N + 127) / 128;
  const int n_wb1 = kMode == 2 ? (p1.N + 255) / 256 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSt; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * 32 * kEw);
    }
    mbar_init(done, 1);
    *s_abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    if (kMode != 1) tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmBs);
    if (p0.sh.n > 0) {
      tma_prefetch_desc(&tmS0);
      if (kMode != 1) tma_prefetch_desc(&tmS1);
    }
    if (kMode == 2) {
      tma_prefetch_desc(&tmD);
      tma_prefetch_desc(&tmH);
      tma_prefetch_desc(&tmHs);
      if (p0.sh.n > 0) tma_prefetch_desc(&tmSD);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(s_tmem, 2 * kBN);
    tmem_relinquish_pair();
  }
  pdl_wait();  // the routing tables and the A/B operands come from the kernels before
  for (int i = threadIdx.x; i <= G; i += blockDim.x) {
    if (i <= E) s_off[i] = offsets[i];
    s_mt[i] = mtile256[i];
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers are initialised before any remote signal
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total0 = s_mt[G] * n_wb0;          // tiles of the first (or only) GEMM
  const int total = total0 + s_mt[G] * n_wb1;  // plus the down tiles in mode 2

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int tile = cid; ok && tile < total; tile += ncl) {
        const bool ph1 = kMode == 2 && tile >= total0;
        const int mode = kMode == 2 ? (ph1 ? 1 : 0) : kMode;
        const GemmPhase& P = ph1 ? p1 : p0;
        const int KB = P.K / kBK;
        const TileCoord tc = decode_tile(ph1 ? tile - total0 : tile, ph1 ? n_wb1 : n_wb0, s_mt, G);
        const GroupRows gr = group_rows(tc.e, s_off, E, P.sh);
        const int ntok = min(256, gr.cnt - tc.m * 256);
        const int half = kTM ? 128 : ((ntok + 15) & ~15) >> 1;  // token rows of the tile held by each CTA
        const bool small = !kTM && half <= kSmallRows;
        if (!small && kBRows < 128) {  // the launcher guarantees this cannot happen
          atomicOr(status, MOE_DEV_INTERNAL);
          *s_abort = 1;
          ok = false;
          break;
        }
        const int brow = gr.in0 + tc.m * 256 + (int)rank * half;
        const bool tm_gu = kTM && mode == 0;  // token-major gate/up
        const int arow = tm_gu       ? gr.widx * P.N + tc.n * 128
                         : mode == 0 ? gr.widx * P.N + tc.n * 128 + (int)rank * 64
                                     : gr.widx * P.N + tc.n * 256 + (int)rank * 128;
        const CUtensorMap* mA0 = tm_gu ? (rank == 0 ? (gr.shared ? &tmS0 : &tmA0) : (gr.shared ? &tmS1 : &tmA1))
                                       : (ph1 ? (gr.shared ? &tmSD : &tmD) : (gr.shared ? &tmS0 : &tmA0));
        const CUtensorMap* mA1 = tm_gu ? mA0 : (ph1 ? mA0 : (gr.shared ? &tmS1 : &tmA1));
        const CUtensorMap* mB = ph1 ? (small ? &tmHs : &tmH) : (small ? &tmBs : &tmB);
        const uint32_t bytes = 2u * (uint32_t)(kHalfBytes + (small ? kSmallRows * 128 : kHalfBytes));
        if (ph1) {
          // the H rows of this token tile are complete once every epilogue
          // warp of both CTAs of every gate/up tile over them has stored its
          // part (one count per warp and tile)
          if (!wait_counter_geq(mt_done + s_mt[tc.e] + tc.m, 2 * kEw * n_wb0, s_abort, status, limit_ns)) {
            ok = false;
            break;
          }
          fence_proxy_async_global();  // the TMA reads below see those generic-proxy stores
        }
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, s_abort, status, limit_ns)) {
            ok = false;
            break;
          }
          const uint32_t fbar = map_to_cta(&full[stage], 0);
          if (leader) mbar_arrive_expect_tx(&full[stage], bytes);
          if (tm_gu) {
            // this CTA's 128 weight rows: gate rows of the block's 128 units
            // in CTA 0, the same units' up rows in CTA 1
            tma_load_2d_pair(sA + stage * kHalfBytes, mA0, fbar, kb * kBK, arow);
            tma_load_2d_pair(sA + stage * kHalfBytes + kHalfBytes / 2, mA0, fbar, kb * kBK, arow + 64);
          } else if (mode == 0) {
            // rows 0-63: gate rows of this CTA's 64 hidden units, 64-127: up rows
            tma_load_2d_pair(sA + stage * kHalfBytes, mA0, fbar, kb * kBK, arow);
            tma_load_2d_pair(sA + stage * kHalfBytes + kHalfBytes / 2, mA1, fbar, kb * kBK, arow);
          } else {
            tma_load_2d_pair(sA + stage * kHalfBytes, mA0, fbar, kb * kBK, arow);
          }
          tma_load_2d_pair(sB + stage * kBSlot, mB, fbar, kb * kBK, brow);
          ++issued;
          if (++stage == kSt) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Loads land on the leader's barriers: the leader waits for the last
      // phase of each stage it armed (these cover both CTAs' bytes).
      if (leader) {
        const int n = issued < kSt ? issued : kSt;
        for (int i = 0; i < n; ++i) {
          if (stage == 0) {
            stage = kSt;
            phase ^= 1u;
          }
          --stage;
          mbar_wait(&full[stage], phase, nullptr, status, limit_ns);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------ MMA issuer (leader only) --
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = cid; ok && tile < total; tile += ncl) {
        const bool ph1 = kMode == 2 && tile >= total0;
        const GemmPhase& P = ph1 ? p1 : p0;
        const int KB = P.K / kBK;
        const TileCoord tc = decode_tile(ph1 ? tile - total0 : tile, ph1 ? n_wb1 : n_wb0, s_mt, G);
        const int ntok = min(256, group_rows(tc.e, s_off, E, P.sh).cnt - tc.m * 256);
        const int nt16 = kTM ? 256 : (ntok + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(256, nt16);
        // narrow tiles spread their K loop over independent accumulators
        const int nacc = kTM ? 1 : (nt16 <= 64 ? 4 : (nt16 <= 128 ? 2 : 1));
        const int acc_stride = kBN / nacc;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, s_abort, status, limit_ns)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full[stage], phase, s_abort, status, limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t wslot = smem_u32(sA + stage * kHalfBytes), tslot = smem_u32(sB + stage * kBSlot);
          const uint64_t adesc = sw128_kmajor_desc(kTM ? tslot : wslot);
          const uint64_t bdesc = sw128_kmajor_desc(kTM ? wslot : tslot);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const int a = kk % nacc;
            tc_mma_bf16_pair(d_tmem + static_cast<uint32_t>(a * acc_stride), adesc + static_cast<uint64_t>(kk * 2),
                             bdesc + static_cast<uint64_t>(kk * 2), idesc, (kb > 0 || kk >= nacc) ? 1u : 0u);
          }
          tc_commit_pair_both(&empty[stage]);
          if (++stage == kSt) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_both(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      tc_commit_pair_local(done);
      mbar_wait(done, 0, nullptr, status, limit_ns);
    }
    __syncwarp();
  } else {
    // --------------------------------------------------------- epilogue --
    // TMEM lane = weight row of this CTA, column = token of the tile.
    const int q = warp & 3;
    const uint32_t tempty_leader0 = map_to_cta(&tempty[0], 0);
    const uint32_t tempty_leader1 = map_to_cta(&tempty[1], 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = cid; tile < total; tile += ncl) {
      const bool ph1 = kMode == 2 && tile >= total0;
      const int mode = kMode == 2 ? (ph1 ? 1 : 0) : kMode;
      const GemmPhase& P = ph1 ? p1 : p0;
      const int N = P.N;
      const TileCoord tc = decode_tile(ph1 ? tile - total0 : tile, ph1 ? n_wb1 : n_wb0, s_mt, G);
      const GroupRows gr = group_rows(tc.e, s_off, E, P.sh);
      const int ntok = min(256, gr.cnt - tc.m * 256);
      const size_t row0 = static_cast<size_t>(gr.out0) + static_cast<size_t>(tc.m * 256);
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_phase, s_abort, status, limit_ns))) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * kBN);
      const int nchunks = (ntok + 31) >> 5;
      const int nt16 = (ntok + 15) & ~15;
      const int nacc = nt16 <= 64 ? 4 : (nt16 <= 128 ? 2 : 1);
      const int acc_stride = kBN / nacc;
      if (kTM && mode == 0) {
        // TMEM lane = one token of this CTA's half of the tile; columns 0-127
        // hold its gate and 128-255 its up values for the block's 128 hidden
        // units. SwiGLU stays in the thread, which writes 32 units (64 bytes)
        // of its token's H row per chunk; the two groups take alternate chunks.
        const int tok = (int)rank * 128 + q * 32 + lane;
        const bool live = tok < ntok;
        __nv_bfloat16* hrow = static_cast<__nv_bfloat16*>(P.out) + (row0 + (live ? tok : 0)) * static_cast<size_t>(N);
#pragma unroll 1
        for (int c = (warp - 2) >> 2; c < 4; c += kGroups) {
          uint32_t g[32], u[32];
          __syncwarp();
          tmem_ld_x32(tbase + c * 32, g);
          tmem_ld_x32(tbase + 128 + c * 32, u);
          tmem_ld_wait();
          const int unit0 = tc.n * 128 + c * 32;
          if (live && unit0 < N) {
            uint4* dst = reinterpret_cast<uint4*>(hrow + unit0);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint32_t pk[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int a = 8 * j + 2 * i;
                pk[i] = pack_bf16x2(silu_f32(__uint_as_float(g[a])) * __uint_as_float(u[a]),
                                    silu_f32(__uint_as_float(g[a + 1])) * __uint_as_float(u[a + 1]));
              }
              dst[j] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
          }
        }
      } else if (kTM) {
        // TMEM lane = one token of this CTA's half of the tile, columns =
        // the block's 256 output features. Each thread writes 32 features
        // (128 bytes) of its token per chunk: fp32 Y rows, or with the
        // combine folded in, gate * y added into the token's output row (two
        // adds per element into a zeroed row, so the order cannot matter).
        const int tok = (int)rank * 128 + q * 32 + lane;
        const bool live = tok < ntok;
        const size_t r = row0 + static_cast<size_t>(live ? tok : 0);
        const bool fold = comb_out != nullptr && !gr.shared;
        float* dst = fold ? comb_out + static_cast<size_t>(live ? perm_tok[r] : 0) * N
                          : static_cast<float*>(P.out) + r * N;
        const float gs = fold && live ? rgate[r] : 1.0f;
#pragma unroll 1
        for (int c = (warp - 2) >> 2; c < 8; c += kGroups) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld_x32(tbase + c * 32, v);
          tmem_ld_wait();
          const int o = tc.n * 256 + c * 32;
          if (live && o < N) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float a0 = __uint_as_float(v[4 * j]), a1 = __uint_as_float(v[4 * j + 1]);
              const float a2 = __uint_as_float(v[4 * j + 2]), a3 = __uint_as_float(v[4 * j + 3]);
              if (fold)
                red_add_v4(dst + o + 4 * j, gs * a0, gs * a1, gs * a2, gs * a3);
              else
                *reinterpret_cast<float4*>(dst + o + 4 * j) = make_float4(a0, a1, a2, a3);
            }
          }
        }
      } else if (mode == 0) {
        // TMEM lanes 0-63 hold the gate rows, 64-127 the up rows of this
        // CTA's 64 hidden units. Per 32-token chunk both halves go to shared
        // memory; then every thread finishes 16 (token, unit) pairs and
        // writes them as two 16-byte vectors of H.
        const int half = (warp - 2) >> 2;  // which group of epilogue warps
        float* sG = sEpi + half * (2 * 64 * 33);  // [64][33] gate chunk
        float* sU = sG + 64 * 33;                 // [64][33] up chunk
        const int j = (q & 1) * 32 + lane;
        float* sdst = (q < 2 ? sG : sU) + j * 33;
        const int et = ((warp - 2) & 3) * 32 + lane;  // 0..127 within the group
        const int tt = et >> 2;           // token of the chunk
        const int ug = (et & 3) * 16;     // first of its 16 units
        const int hid0 = tc.n * 128 + (int)rank * 64;
#pragma unroll 1
        for (int c = half; c < nchunks; c += kGroups) {
          uint32_t v[32];
          ld_chunk_sum(tbase + c * 32, nacc, acc_stride, v);
#pragma unroll
          for (int t = 0; t < 32; ++t) sdst[t] = __uint_as_float(v[t]);
          epi_bar(half);
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int u0 = ug + 2 * i;
            const float h0 = silu_f32(sG[u0 * 33 + tt]) * sU[u0 * 33 + tt];
            const float h1 = silu_f32(sG[(u0 + 1) * 33 + tt]) * sU[(u0 + 1) * 33 + tt];
            pk[i] = pack_bf16x2(h0, h1);
          }
          epi_bar(half);
          const int tok = c * 32 + tt;
          if (tok < ntok && hid0 < N) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(P.out) + (row0 + tok) * N + hid0 + ug);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      } else {
        // lane = output feature. Each warp turns its 32 features x 32 tokens
        // of a chunk around in shared memory and writes token rows of Y as
        // 16-byte vectors (8 lanes per 128-byte row, 4 rows per instruction).
        const int o0 = tc.n * 256 + (int)rank * 128 + q * 32;
        float* tw = sY + (warp - 2) * (32 * 36);
        const int vr = lane >> 3, vc = (lane & 7) * 4;
#pragma unroll 1
        for (int c = (warp - 2) >> 2; c < nchunks; c += kGroups) {
          uint32_t v[32];
          ld_chunk_sum(tbase + c * 32, nacc, acc_stride, v);
#pragma unroll
          for (int t = 0; t < 32; ++t) tw[t * 36 + lane] = __uint_as_float(v[t]);
          __syncwarp();
          if (o0 < N) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int t = vr + 4 * i;
              const int tok = c * 32 + t;
              if (tok < ntok) {
                const float4 val = *reinterpret_cast<const float4*>(tw + t * 36 + vc);
                if (comb_out && !gr.shared) {
                  // combine folded in: out[token] += gate * y (two adds per
                  // element into a zeroed row, so the order cannot matter)
                  const size_t r = row0 + tok;
                  const float g = rgate[r];
                  red_add_v4(comb_out + (size_t)perm_tok[r] * N + o0 + vc, g * val.x, g * val.y, g * val.z,
                             g * val.w);
                } else {
                  *reinterpret_cast<float4*>(static_cast<float*>(P.out) + (row0 + tok) * N + o0 + vc) = val;
                }
              }
            }
          }
        }
      }
      __syncwarp();
      tc_fence_before();
      mbar_arrive_cluster(acc == 0 ? tempty_leader0 : tempty_leader1);
      if (kMode == 2 && !ph1) {
        // this warp's H stores of the tile are done: count them for the down
        // tiles that read these rows (release at GPU scope after the warp's
        // stores; the readers acquire, then fence the async proxy)
        fence_proxy_async_global();
        __syncwarp();
        if (lane == 0) {
          asm volatile("fence.acq_rel.gpu;" ::: "memory");
          atomicAdd(mt_done + s_mt[tc.e] + tc.m, 1);
        }
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its peer may still touch its shared memory or TMEM
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 2 * kBN);
  }
}

// Resident CTA pairs per GPU for one configuration, queried once per device.
// Host threads may race on the first query of a device; each computes the
// same value and the atomic store publishes it.
template <class Cfg>
int max_active_pairs(const void* kern) {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  const int have = cache[dev].load(std::memory_order_acquire);
  if (have > 0) return have;
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(Cfg::kThreads, 1, 1);
    cfg.dynamicSmemBytes = Cfg::kSmemBytes;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) return 0;
    cache[dev].store(n, std::memory_order_release);
    return n;
  }
}

// Streaming multiprocessors of the current device, queried once per device.
int device_sm_count() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int n = cache[dev].load(std::memory_order_acquire);
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 0;
  cache[dev].store(n, std::memory_order_release);
  return n;
}

// The tensor maps of one launch (see the kernel; unused ones repeat others).
struct Tc2Maps {
  CUtensorMap a0, a1, s0, s1, b, bs, d, sd, h, hs;
};

template <int kMode, class Cfg>
cudaError_t launch_tc2_cfg(const Tc2Maps& m, const int32_t* offsets, const int32_t* mtile256, int R_rows, int E,
                           const GemmPhase& p0, const GemmPhase& p1, const int32_t* perm_tok, const float* rgate,
                           float* comb_out, int32_t* mt_done, int32_t* status, cudaStream_t stream) {
  auto kern = grouped_gemm_tc2_kernel<kMode, Cfg::kStages, Cfg::kEpiWarps, Cfg::kBSlotRows, Cfg::kTokM>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
  if (err != cudaSuccess) return err;
  const int pairs = max_active_pairs<Cfg>(reinterpret_cast<const void*>(kern));
  if (pairs <= 0) return cudaErrorInvalidConfiguration;
  const int n_wb0 = kMode == 1 ? (p0.N + 255) / 256 : (p0.N + 127) / 128;
  const int n_wb1 = kMode == 2 ? (p1.N + 255) / 256 : 0;
  const long long max_tiles = (long long)(R_rows / 256 + E + p0.sh.n) * (n_wb0 + n_wb1);
  // mode 2 needs every cluster resident at once (a down tile waits for gate/up
  // tiles of other clusters): never more clusters than fit on the GPU
  const int clusters = (int)(max_tiles < pairs ? max_tiles : pairs);
  if (clusters <= 0) return cudaSuccess;
  return launch_pdl(kern, dim3(2 * clusters), dim3(Cfg::kThreads), Cfg::kSmemBytes, stream, m.a0, m.a1, m.s0, m.s1,
                    m.b, m.bs, m.d, m.sd, m.h, m.hs, offsets, mtile256, E, p0, p1, perm_tok, rgate, comb_out, mt_done,
                    status, kWaitLimitNs);
}

// Batches whose every group has at most 32 rows (max_rows_per_group: T, the
// most a routed expert or a shared expert can receive) take the stream
// configuration; other decode-sized batches (fewer than 64 rows per group on
// average) the narrow one, everything else the wide one; the down projection
// only with the combine folded in (its fp32 Y stores run better with fewer
// epilogue warps and the deeper ring).
template <int kMode>
cudaError_t launch_tc2(const Tc2Maps& m, const int32_t* offsets, const int32_t* mtile256, int R_rows,
                       int max_rows_per_group, int E, const GemmPhase& p0, const int32_t* perm_tok,
                       const float* rgate, float* comb_out, int32_t* status, cudaStream_t stream) {
  const bool wide = (long long)R_rows >= 64ll * (E + p0.sh.n) && (kMode == 0 || comb_out != nullptr);
  if (max_rows_per_group <= 2 * kSmallRows)
    return launch_tc2_cfg<kMode, Gemm2Stream>(m, offsets, mtile256, R_rows, E, p0, p0, perm_tok, rgate, comb_out,
                                              nullptr, status, stream);
  if constexpr (kMode == 0) {
    if (wide)
      return launch_tc2_cfg<kMode, Gemm2WideTM>(m, offsets, mtile256, R_rows, E, p0, p0, perm_tok, rgate, comb_out,
                                                nullptr, status, stream);
  } else {
    if (wide) {
      // A grid of at most three down tiles per CTA pair exposes the last
      // tile's epilogue: the token-major form, whose epilogue adds straight
      // from TMEM into the output rows, finishes it sooner. On longer grids
      // it needs fewer cycles but ran at a lower power-capped clock than the
      // weight-major form, whose adds cover 128-byte output rows.
      const long long tiles = (long long)(R_rows / 256 + E + p0.sh.n) * ((p0.N + 255) / 256);
      if (tiles <= 3ll * (device_sm_count() / 2))
        return launch_tc2_cfg<kMode, Gemm2WideTM>(m, offsets, mtile256, R_rows, E, p0, p0, perm_tok, rgate,
                                                  comb_out, nullptr, status, stream);
      return launch_tc2_cfg<kMode, Gemm2Wide>(m, offsets, mtile256, R_rows, E, p0, p0, perm_tok, rgate, comb_out,
                                              nullptr, status, stream);
    }
  }
  return launch_tc2_cfg<kMode, Gemm2Narrow>(m, offsets, mtile256, R_rows, E, p0, p0, perm_tok, rgate, comb_out,
                                            nullptr, status, stream);
}

}  // namespace

cudaError_t launch_gemm_gateup_tc2(const CUtensorMap& tm_wg, const CUtensorMap& tm_wu, const CUtensorMap& tm_sg,
                                   const CUtensorMap& tm_su, const CUtensorMap& tm_xp, const CUtensorMap& tm_xp_small,
                                   const int32_t* offsets, const int32_t* mtile, int R_rows, int E,
                                   const SharedGroups& sh, int I, int d, void* h, int32_t* status,
                                   cudaStream_t stream) {
  const Tc2Maps m{tm_wg, tm_wu, tm_sg, tm_su, tm_xp, tm_xp_small, tm_wg, tm_sg, tm_xp, tm_xp_small};
  const GemmPhase p0{sh, I, d, h};
  return launch_tc2<0>(m, offsets, mtile, R_rows, sh.rows, E, p0, nullptr, nullptr, nullptr, status, stream);
}

cudaError_t launch_gemm_down_tc2(const CUtensorMap& tm_wd, const CUtensorMap& tm_sd, const CUtensorMap& tm_h,
                                 const CUtensorMap& tm_h_small, const int32_t* offsets, const int32_t* mtile,
                                 int R_rows, int E, const SharedGroups& sh, int I, int d, float* y,
                                 const int32_t* perm_tok, const float* rgate, float* comb_out, int32_t* status,
                                 cudaStream_t stream) {
  const Tc2Maps m{tm_wd, tm_wd, tm_sd, tm_sd, tm_h, tm_h_small, tm_wd, tm_sd, tm_h, tm_h_small};
  const GemmPhase p0{sh, d, I, y};
  return launch_tc2<1>(m, offsets, mtile, R_rows, sh.rows, E, p0, perm_tok, rgate, comb_out, status, stream);
}

bool gemms_fused(int T, moe_dtype dtype) { return dtype == MOE_BF16 && T > 0 && T <= 2 * kSmallRows; }

cudaError_t launch_gemm_fused_tc2(const CUtensorMap& tm_wg, const CUtensorMap& tm_wu, const CUtensorMap& tm_sg,
                                  const CUtensorMap& tm_su, const CUtensorMap& tm_xp_small, const CUtensorMap& tm_wd,
                                  const CUtensorMap& tm_sd, const CUtensorMap& tm_h_small, const int32_t* offsets,
                                  const int32_t* mtile, int R_rows, int E, const SharedGroups& sh_up,
                                  const SharedGroups& sh_down, int I, int d, void* h, float* y,
                                  const int32_t* perm_tok, const float* rgate, float* comb_out, int32_t* mt_done,
                                  int32_t* status, cudaStream_t stream) {
  // every group holds at most 32 rows, so the 16-row boxes serve every tile
  const Tc2Maps m{tm_wg, tm_wu, tm_sg, tm_su, tm_xp_small, tm_xp_small, tm_wd, tm_sd, tm_h_small, tm_h_small};
  const GemmPhase p0{sh_up, I, d, h};
  const GemmPhase p1{sh_down, d, I, y};
  return launch_tc2_cfg<2, Gemm2Stream>(m, offsets, mtile, R_rows, E, p0, p1, perm_tok, rgate, comb_out, mt_done,
                                        status, stream);
}

}  // namespace moe
