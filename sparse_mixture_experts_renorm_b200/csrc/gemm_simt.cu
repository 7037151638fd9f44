// gemm_simt.cu — the fp32 grouped expert GEMMs (same two steps as gemm_tc.cu:
// gate/up with the SwiGLU fused into the epilogue, then down) on the FFMA
// pipes. The fp32 workload's 1e-4 tolerance rules out TF32 tensor cores, and
// it is small, so a plain shared-memory-tiled kernel serves it.
//
// Each CTA computes one 64 x 64 output tile of one expert; blockIdx.y walks the
// experts' 64-row tiles in order (found from the device-side offsets), so no
// host synchronisation is needed. The K loop accumulates in index order.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kSK = 16;

template <int kMode>
__global__ void __launch_bounds__(256) grouped_gemm_simt_kernel(const float* __restrict__ A,
                                                                const float* __restrict__ B0,
                                                                const float* __restrict__ B1,
                                                                const int32_t* __restrict__ offsets, int E, int N,
                                                                int K, float* __restrict__ out) {
  __shared__ int s_info[3];  // expert, first row, rows in this tile
  pdl_wait();
  if (threadIdx.x == 0) {
    int mt = blockIdx.y, cum = 0, e = -1, row0 = 0, rows = 0;
    for (int ee = 0; ee < E; ++ee) {
      const int c = offsets[ee + 1] - offsets[ee];
      const int tiles = (c + kSimtBM - 1) / kSimtBM;
      if (mt < cum + tiles) {
        e = ee;
        row0 = offsets[ee] + (mt - cum) * kSimtBM;
        rows = min(kSimtBM, c - (mt - cum) * kSimtBM);
        break;
      }
      cum += tiles;
    }
    s_info[0] = e;
    s_info[1] = row0;
    s_info[2] = rows;
  }
  __syncthreads();
  const int e = s_info[0];
  if (e < 0) return;
  const int row0 = s_info[1], rows = s_info[2];
  const int n0 = blockIdx.x * kSimtBN;

  __shared__ float sA[kSK][kSimtBM + 4];
  __shared__ float sB0[kSK][kSimtBN + 4];
  __shared__ float sB1[kMode == 0 ? kSK : 1][kSimtBN + 4];

  const int tid = threadIdx.x;
  const int ty = tid / 16, tx = tid % 16;
  float acc0[4][4] = {}, acc1[4][4] = {};
  const float* Bexp0 = B0 + (size_t)e * N * K;
  const float* Bexp1 = kMode == 0 ? B1 + (size_t)e * N * K : nullptr;

  for (int k0 = 0; k0 < K; k0 += kSK) {
    for (int i = tid; i < kSimtBM * kSK; i += 256) {
      const int r = i / kSK, c = i % kSK;
      sA[c][r] = (r < rows && k0 + c < K) ? A[(size_t)(row0 + r) * K + k0 + c] : 0.f;
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
      out[(size_t)(row0 + r) * N + n] = v;
    }
  }
}

template <int kMode>
cudaError_t launch_simt(const float* A, const float* B0, const float* B1, const int32_t* offsets, int R, int E, int N,
                        int K, float* out, cudaStream_t stream) {
  const int max_mtiles = R / kSimtBM + E;
  dim3 grid((N + kSimtBN - 1) / kSimtBN, max_mtiles);
  return launch_pdl(grouped_gemm_simt_kernel<kMode>, grid, dim3(256), 0, stream, A, B0, B1, offsets, E, N, K, out);
}

}  // namespace

cudaError_t launch_gemm_gateup_simt(const float* xp, const float* wg, const float* wu, const int32_t* offsets, int R,
                                    int E, int I, int d, float* h, cudaStream_t stream) {
  return launch_simt<0>(xp, wg, wu, offsets, R, E, I, d, h, stream);
}

cudaError_t launch_gemm_down_simt(const float* h, const float* wd, const int32_t* offsets, int R, int E, int I, int d,
                                  float* y, cudaStream_t stream) {
  return launch_simt<1>(h, wd, nullptr, offsets, R, E, d, I, y, stream);
}

}  // namespace moe
