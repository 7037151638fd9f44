// gemm_simt.cu — the fp32 grouped expert GEMMs (same two steps as gemm_tc2.cu:
// gate/up with the SwiGLU fused into the epilogue, then down) on the FFMA
// pipes. The fp32 workload's 1e-4 tolerance rules out TF32 tensor cores, and
// it is small, so a plain shared-memory-tiled kernel serves it.
//
// Each CTA computes one 64 x 64 output tile of one group (a routed expert,
// then the shared experts); blockIdx.y walks the groups' 64-row tiles in order
// (found from the device-side offsets), so no host synchronisation is needed.
// The K loop accumulates in index order.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kSK = 32;  // K columns per staged slice
static_assert(kSimtBM == kSimtBN, "the staging loop fills the A and B slices with one index");

template <int kMode>
__global__ void __launch_bounds__(256) grouped_gemm_simt_kernel(const float* __restrict__ A,
                                                                const float* __restrict__ B0,
                                                                const float* __restrict__ B1,
                                                                const float* __restrict__ S0,
                                                                const float* __restrict__ S1,
                                                                const int32_t* __restrict__ offsets, int E,
                                                                SharedGroups sh, int N, int K,
                                                                float* __restrict__ out) {
  __shared__ int s_info[4];  // group, first input row, first output row, rows in this tile
  pdl_wait();
  if (threadIdx.x == 0) {
    int mt = blockIdx.y, cum = 0, g = -1, in0 = 0, out0 = 0, rows = 0;
    for (int gg = 0; gg < E + sh.n; ++gg) {
      int c, gin, gout;
      if (gg < E) {
        c = offsets[gg + 1] - offsets[gg];
        gin = gout = offsets[gg];
      } else {
        c = sh.rows;
        gin = sh.in0 + (gg - E) * sh.in_step;
        gout = sh.out0 + (gg - E) * sh.rows;
      }
      const int tiles = (c + kSimtBM - 1) / kSimtBM;
      if (mt < cum + tiles) {
        g = gg;
        in0 = gin + (mt - cum) * kSimtBM;
        out0 = gout + (mt - cum) * kSimtBM;
        rows = min(kSimtBM, c - (mt - cum) * kSimtBM);
        break;
      }
      cum += tiles;
    }
    s_info[0] = g;
    s_info[1] = in0;
    s_info[2] = out0;
    s_info[3] = rows;
  }
  __syncthreads();
  const int g = s_info[0];
  if (g < 0) return;
  const int in0 = s_info[1], out0 = s_info[2], rows = s_info[3];
  const int n0 = blockIdx.x * kSimtBN;

  __shared__ float sA[kSK][kSimtBM + 4];
  __shared__ float sB0[kSK][kSimtBN + 4];
  __shared__ float sB1[kMode == 0 ? kSK : 1][kSimtBN + 4];

  const int tid = threadIdx.x;
  const int ty = tid / 16, tx = tid % 16;
  float acc0[4][4] = {}, acc1[4][4] = {};
  const bool shared = g >= E;
  const size_t widx = shared ? (size_t)(g - E) : (size_t)g;
  const float* Bexp0 = (shared ? S0 : B0) + widx * N * K;
  const float* Bexp1 = kMode == 0 ? (shared ? S1 : B1) + widx * N * K : nullptr;

  for (int k0 = 0; k0 < K; k0 += kSK) {
#pragma unroll 4  // the loads of half a slice in flight at once
    for (int i0 = 0; i0 < kSimtBM * kSK; i0 += 256) {
      const int i = i0 + tid;
      const int r = i / kSK, c = i % kSK;
      sA[c][r] = (r < rows && k0 + c < K) ? A[(size_t)(in0 + r) * K + k0 + c] : 0.f;
      const bool nok = n0 + r < N && k0 + c < K;
      sB0[c][r] = nok ? Bexp0[(size_t)(n0 + r) * K + k0 + c] : 0.f;
      if (kMode == 0) sB1[c][r] = nok ? Bexp1[(size_t)(n0 + r) * K + k0 + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < kSK; ++c) {
      float a[4], b0[4], b1[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = sA[c][ty * 4 + i];
        b0[i] = sB0[c][tx * 4 + i];
        if (kMode == 0) b1[i] = sB1[c][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc0[i][j] = fmaf(a[i], b0[j], acc0[i][j]);
          if (kMode == 0) acc1[i][j] = fmaf(a[i], b1[j], acc1[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i;
    if (r >= rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc0[i][j];
      if (kMode == 0) v = v / (1.0f + expf(-v)) * acc1[i][j];
      out[(size_t)(out0 + r) * N + n] = v;
    }
  }
}

template <int kMode>
cudaError_t launch_simt(const float* A, const float* B0, const float* B1, const float* S0, const float* S1,
                        const int32_t* offsets, int R_rows, int E, const SharedGroups& sh, int N, int K, float* out,
                        cudaStream_t stream) {
  const int max_mtiles = R_rows / kSimtBM + E + sh.n;
  dim3 grid((N + kSimtBN - 1) / kSimtBN, max_mtiles);
  return launch_pdl(grouped_gemm_simt_kernel<kMode>, grid, dim3(256), 0, stream, A, B0, B1, S0, S1, offsets, E, sh, N,
                    K, out);
}

}  // namespace

cudaError_t launch_gemm_gateup_simt(const float* xp, const float* wg, const float* wu, const float* swg,
                                    const float* swu, const int32_t* offsets, int R_rows, int E,
                                    const SharedGroups& sh, int I, int d, float* h, cudaStream_t stream) {
  return launch_simt<0>(xp, wg, wu, swg, swu, offsets, R_rows, E, sh, I, d, h, stream);
}

cudaError_t launch_gemm_down_simt(const float* h, const float* wd, const float* swd, const int32_t* offsets,
                                  int R_rows, int E, const SharedGroups& sh, int I, int d, float* y,
                                  cudaStream_t stream) {
  return launch_simt<1>(h, wd, nullptr, swd, nullptr, offsets, R_rows, E, sh, d, I, y, stream);
}

}  // namespace moe
