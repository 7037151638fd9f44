// gemm_tc.cu — kernel (c): the two grouped expert GEMMs on the 5th-generation
// tensor cores (tcgen05, accumulators in TMEM, operands staged by TMA).
//
//   mode 0 (gate/up):  H[r, :] = SiLU(Xp[r] . W_gate[e]^T) * (Xp[r] . W_up[e]^T)
//   mode 1 (down):     Y[r, :] = H[r] . W_down[e]^T
//
// for every dispatched row r of expert e (axonml-nn layers/moe.rs,
// Expert::forward: down(SiLU(gate(x)) * up(x)); Model Architecture Patterns,
// "SwiGLU FFN"). Rows are expert-contiguous, so expert e's rows form the
// M dimension of its own GEMM; tiles of 128 rows that run past the expert's
// last row compute on neighbouring rows (or TMA zero fill) and are masked at
// the store.
//
// Structure: persistent CTAs, one per SM, walk a device-side tile list built
// from the routing counts (no host synchronisation). Warp 0 issues TMA loads
// into a 4-stage shared-memory ring; warp 1 owns 512 TMEM columns and issues
// 128x256x16 UMMAs (one thread), committing each stage back to the loader;
// warps 2-5 drain the double-buffered accumulator with tcgen05.ld, apply the
// SwiGLU (mode 0) and store. In mode 0 the 256 accumulator columns of a tile
// are 128 gate columns followed by the 128 up columns of the same hidden
// units, so the SwiGLU is applied without another pass over H.
#include "common.cuh"

namespace moe {
namespace {

struct TileCoord {
  int e, m, n;
};

// Tile index -> (expert, m-tile, n-tile). Experts in order; inside an expert
// the n-tile is the outer index and the m-tile the inner one, so CTAs that run
// at the same time read the same weight tiles (one HBM read, L2 hits after).
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

__device__ __forceinline__ float silu_f32(float z) { return z / (1.0f + __expf(-z)); }

template <int kMode>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                           const __grid_constant__ CUtensorMap tmB1, const int32_t* __restrict__ offsets,
                           const int32_t* __restrict__ mtile128, int E, int N, int K, void* __restrict__ out,
                           int32_t* status, uint64_t limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kTileABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* tfull = bars + 2 * kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_off = reinterpret_cast<int*>(s_tmem + 4);  // [E+1]
  int* s_mt = s_off + (E + 1);                       // [E+1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = kMode == 0 ? (N + 127) / 128 : (N + kBN - 1) / kBN;
  const int KB = K / kBK;

  for (int i = threadIdx.x; i <= E; i += blockDim.x) {
    s_off[i] = offsets[i];
    s_mt[i] = mtile128[i];
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 128);
    }
    mbar_init(done, 1);
    *s_abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (kMode == 0) tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, 2 * kBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total = s_mt[E] * n_tiles;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const TileCoord tc = decode_tile(tile, n_tiles, s_mt, E);
        const int arow = s_off[tc.e] + tc.m * kBM;
        const int brow = kMode == 0 ? tc.e * N + tc.n * 128 : tc.e * N + tc.n * kBN;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, s_abort, status, limit_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], kStageBytes);
          tma_load_2d(sA + stage * kTileABytes, &tmA, &full[stage], kb * kBK, arow);
          if (kMode == 0) {
            tma_load_2d(sB + stage * kTileBBytes, &tmB0, &full[stage], kb * kBK, brow);
            tma_load_2d(sB + stage * kTileBBytes + kTileBBytes / 2, &tmB1, &full[stage], kb * kBK, brow);
          } else {
            tma_load_2d(sB + stage * kTileBBytes, &tmB0, &full[stage], kb * kBK, brow);
          }
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Every issued load must have landed before the CTA may exit: wait
      // (time-bounded, regardless of the abort flag) on the most recent load
      // of each stage.
      const int n = issued < kStages ? issued : kStages;
      for (int i = 0; i < n; ++i) {
        if (stage == 0) {
          stage = kStages;
          phase ^= 1u;
        }
        --stage;
        mbar_wait(&full[stage], phase, nullptr, status, limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, kBN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, s_abort, status, limit_ns)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full[stage], phase, s_abort, status, limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = sw128_kmajor_desc(smem_u32(sA + stage * kTileABytes));
          const uint64_t bdesc = sw128_kmajor_desc(smem_u32(sB + stage * kTileBBytes));
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            tc_mma_bf16(d_tmem, adesc + static_cast<uint64_t>(kk * 2), bdesc + static_cast<uint64_t>(kk * 2), idesc,
                        (kb | kk) != 0 ? 1u : 0u);
          tc_commit(&empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // All MMAs issued by this thread complete before TMEM is released.
      tc_commit(done);
      mbar_wait(done, 0, nullptr, status, limit_ns);
    }
    __syncwarp();
  } else {
    // --------------------------------------------------------- epilogue --
    const int q = warp & 3;  // this warp may access TMEM lanes 32q .. 32q+31
    const int r = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const TileCoord tc = decode_tile(tile, n_tiles, s_mt, E);
      if (!mbar_wait(&tfull[acc], acc_phase, s_abort, status, limit_ns)) break;
      tc_fence_after();
      const int cnt = s_off[tc.e + 1] - s_off[tc.e];
      const bool row_ok = tc.m * kBM + r < cnt;
      const size_t grow = static_cast<size_t>(s_off[tc.e]) + static_cast<size_t>(tc.m * kBM + r);
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * kBN);
      if (kMode == 0) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t g[32], u[32];
          __syncwarp();
          tmem_ld_x32(tbase + c * 32, g);
          tmem_ld_x32(tbase + 128 + c * 32, u);
          tmem_ld_wait();
          const int col0 = tc.n * 128 + c * 32;
          if (row_ok && col0 < N) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float h0 = silu_f32(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]);
              const float h1 = silu_f32(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
              pk[i] = pack_bf16x2(h0, h1);
            }
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + grow * N + col0);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld_x32(tbase + c * 32, v);
          tmem_ld_wait();
          const int col0 = tc.n * kBN + c * 32;
          if (row_ok && col0 < N) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + grow * N + col0);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                   __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
          }
        }
      }
      __syncwarp();
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * kBN);
  }
}

template <int kMode>
cudaError_t launch_tc(const CUtensorMap& tmA, const CUtensorMap& tmB0, const CUtensorMap& tmB1,
                      const int32_t* offsets, const int32_t* mtile128, int R, int E, int N, int K, void* out,
                      int32_t* status, int num_sms, cudaStream_t stream) {
  auto kern = grouped_gemm_tc_kernel<kMode>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes);
  if (err != cudaSuccess) return err;
  const int n_tiles = kMode == 0 ? (N + 127) / 128 : (N + kBN - 1) / kBN;
  const long long max_tiles = (long long)(R / kBM + E) * n_tiles;
  const int grid = (int)(max_tiles < num_sms ? max_tiles : num_sms);
  if (grid <= 0) return cudaSuccess;
  kern<<<grid, kGemmThreads, kGemmSmemBytes, stream>>>(tmA, tmB0, tmB1, offsets, mtile128, E, N, K, out, status,
                                                      kWaitLimitNs);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_gateup_tc(const CUtensorMap& tm_xp, const CUtensorMap& tm_wg, const CUtensorMap& tm_wu,
                                  const int32_t* offsets, const int32_t* mtile128, int R, int E, int I, int d, void* h,
                                  int32_t* status, int num_sms, cudaStream_t stream) {
  return launch_tc<0>(tm_xp, tm_wg, tm_wu, offsets, mtile128, R, E, I, d, h, status, num_sms, stream);
}

cudaError_t launch_gemm_down_tc(const CUtensorMap& tm_h, const CUtensorMap& tm_wd, const int32_t* offsets,
                                const int32_t* mtile128, int R, int E, int I, int d, float* y, int32_t* status,
                                int num_sms, cudaStream_t stream) {
  return launch_tc<1>(tm_h, tm_wd, tm_wd, offsets, mtile128, R, E, d, I, y, status, num_sms, stream);
}

}  // namespace moe
