// moe_internal.h — constants, workspace layout and kernel launchers shared by
// the translation units of the library (host-side declarations only).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "moe.h"  // include/ is on the include path

namespace moe {

// Router: tokens per CTA. One CTA's routing partials form one block of the
// two-level scan that gives every dispatched row its position: 128 tokens
// (the UMMA M) for the bf16 tensor-core router, 32 for the fp32 SIMT router.
constexpr int kRouterTokensTc = 128;
constexpr int kRouterTokensSimt = 32;
constexpr int kRouterThreads = 128;
constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 8;

// tcgen05 grouped GEMM tiling.
constexpr int kTileM = 256;       // rows (dispatched tokens) per tile of the CTA pair
constexpr int kBM = 128;          // rows per CTA
constexpr int kBN = 256;          // UMMA N: 128 gate + 128 up columns, or 256 down columns
constexpr int kBK = 64;           // K per pipeline stage (one 128-byte swizzle row of bf16)
constexpr int kStages = 4;        // shared-memory pipeline depth
constexpr int kGemmThreads = 192; // warp 0 TMA, warp 1 MMA + TMEM owner, warps 2-5 epilogue
constexpr int kTileABytes = kBM * kBK * 2;
constexpr int kTileBBytes = kBN * kBK * 2;
constexpr int kStageBytes = kTileABytes + kTileBBytes;
constexpr int kGemmSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 4096 /*barriers, tables*/;

// fp32 SIMT grouped GEMM tiling.
constexpr int kSimtBM = 64;
constexpr int kSimtBN = 64;

// Bounded waits give up after this long (a healthy wait takes microseconds).
constexpr uint64_t kWaitLimitNs = 1000000000ull;

// Byte offsets of every scratch array inside the caller's workspace.
struct Workspace {
  size_t status;      // int32 [1]     device status word used when the caller passes none
  size_t offsets;     // int32 [E+1]   first dispatched row of each expert
  size_t counts;      // int32 [E]     assignments per expert (when the caller passes none)
  size_t mtile;       // int32 [E+1]   prefix of ceil(count/kTileM) (tcgen05 tile schedule)
  size_t aux;         // fp32  [1]     statistic (when the caller passes none)
  size_t blk_cnt;     // int32 [nb*E]  per-router-block counts, then per-block base rows
  size_t blk_psum;    // fp32  [nb*E]  per-router-block sums of probabilities
  size_t lrank;       // int32 [T*k]   rank of (t,j) among its block's tokens of that expert
  size_t perm_tok;    // int32 [T*k]
  size_t inv;         // int32 [T*k]
  size_t rgate;       // fp32  [T*k]   gate of every dispatched row
  size_t xp;          // dtype [T*k, d] expert-contiguous copy of x
  size_t h;           // dtype [T*k, I] SwiGLU hidden activations
  size_t y;           // fp32  [T*k, d] expert outputs
  size_t total;
};

Workspace workspace_layout(int T, int d, int E, int k, int I, moe_dtype dtype);

// Sets the calling thread's moe_last_error_detail() message (printf format).
void set_error_detail(const char* fmt, ...);

inline int router_block_tokens(moe_dtype dtype) { return dtype == MOE_BF16 ? kRouterTokensTc : kRouterTokensSimt; }
inline int router_blocks(int T, moe_dtype dtype) {
  const int rb = router_block_tokens(dtype);
  return (T + rb - 1) / rb;
}

// Encode a 2-D bf16 tensor map (rows x cols, row-major) with a box of
// box_rows x 64 columns and the 128-byte swizzle. Returns false on failure.
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);

// Launch with programmatic stream serialisation (see pdl_wait in common.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---- launchers (all asynchronous on `stream`) ----

cudaError_t launch_router(moe_dtype dtype, const void* x, const void* w_router, const float* b_router, int T,
                          int d, int E, int k, int renorm, int32_t* topk_idx, float* topk_gate, int32_t* lrank,
                          int32_t* blk_cnt, float* blk_psum, int32_t* status, cudaStream_t stream);

cudaError_t launch_router_tc(const void* x, const void* w_router, const float* b_router, int T, int d, int E, int k,
                             int renorm, int32_t* topk_idx, float* topk_gate, int32_t* lrank, int32_t* blk_cnt,
                             float* blk_psum, int32_t* status, cudaStream_t stream);

cudaError_t launch_route_scan(int nb, int T, int E, int k, int32_t* blk_cnt, const float* blk_psum, int32_t* counts,
                              int32_t* offsets, int32_t* mtile, float* aux, cudaStream_t stream);

// Also records the gate of every dispatched row (rgate) and, when zero_out is
// given, clears out[T, d] for a combine done by the down GEMM's epilogue.
cudaError_t launch_permute(moe_dtype dtype, const void* x, int T, int d, int E, int k, int rb, const int32_t* topk_idx,
                           const int32_t* lrank, const int32_t* blk_base, int32_t* perm_tok, int32_t* inv,
                           void* xp, const float* topk_gate, float* rgate, float* zero_out, int32_t* status,
                           cudaStream_t stream);

cudaError_t launch_combine(int T, int d, int k, const float* y, const int32_t* inv, const float* topk_gate,
                           float* out, int32_t* status, cudaStream_t stream);

// tcgen05 grouped GEMMs (bf16) on CTA pairs: 256 weight rows x up to 256
// dispatched tokens per tile. mode 0: H = SiLU(Xp Wg^T) * (Xp Wu^T) per
// expert; mode 1: Y = H Wd^T per expert.
cudaError_t launch_gemm_gateup_tc2(const CUtensorMap& tm_wg, const CUtensorMap& tm_wu, const CUtensorMap& tm_xp,
                                   const CUtensorMap& tm_xp_small, const int32_t* offsets, const int32_t* mtile,
                                   int R, int E, int I, int d, void* h, int32_t* status, cudaStream_t stream);
// comb_out != nullptr: instead of storing Y, add gate * y of every dispatched
// row into comb_out[token] (used when k = 2, where the two adds commute).
cudaError_t launch_gemm_down_tc2(const CUtensorMap& tm_wd, const CUtensorMap& tm_h, const CUtensorMap& tm_h_small,
                                 const int32_t* offsets, const int32_t* mtile, int R, int E, int I, int d, float* y,
                                 const int32_t* perm_tok, const float* rgate, float* comb_out, int32_t* status,
                                 cudaStream_t stream);

// fp32 SIMT grouped GEMMs.
cudaError_t launch_gemm_gateup_simt(const float* xp, const float* wg, const float* wu, const int32_t* offsets,
                                    int R, int E, int I, int d, float* h, cudaStream_t stream);
cudaError_t launch_gemm_down_simt(const float* h, const float* wd, const int32_t* offsets, int R, int E, int I,
                                  int d, float* y, cudaStream_t stream);

}  // namespace moe
