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
constexpr int kRouterThreads = 256;
constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 8;
constexpr int kRouterRegExperts = 16;  // up to this many experts the tensor-core router keeps logits in registers

// tcgen05 grouped GEMM tiling.
constexpr int kTileM = 256;       // dispatched tokens per tile of the CTA pair (UMMA N)
constexpr int kBN = 256;          // weight rows per tile of the CTA pair (UMMA M)
constexpr int kBK = 64;           // K per pipeline stage (one 128-byte swizzle row of bf16)
constexpr int kGemmThreads = 192; // warp 0 TMA, warp 1 MMA + TMEM owner, warps 2-5 epilogue

// fp32 SIMT grouped GEMM tiling.
constexpr int kSimtBM = 64;
constexpr int kSimtBN = 64;

// Bounded waits give up after this long (a healthy wait takes microseconds).
constexpr uint64_t kWaitLimitNs = 1000000000ull;

// Byte offsets of every scratch array inside the caller's workspace. The
// arrays up to and including `inv` sit at offsets that depend on the shape
// only (not on the options), so moe_get_permutation can find them.
struct Workspace {
  size_t status;      // int32 [1]     device status word used when the caller passes none
  size_t offsets;     // int32 [E+1]   first dispatched (kept) row of each expert
  size_t counts;      // int32 [E]     assignments per expert (when the caller passes none)
  size_t mtile;       // int32 [E+1+kMaxShared] prefix of 256-token tiles over the GEMM groups
  size_t aux;         // fp32  [1]     statistic (when the caller passes none)
  size_t blk_cnt;     // int32 [nb*E]  per-router-block counts, then per-block base rows
  size_t blk_psum;    // fp32  [nb*E]  per-router-block sums of probabilities
  size_t lrank;       // int32 [T*k]   rank of (t,j) among its block's tokens of that expert
  size_t perm_tok;    // int32 [T*k]
  size_t inv;         // int32 [T*k]   row of each (token, slot), -1 when dropped
  size_t rgate;       // fp32  [T*k]   gate of every dispatched row
  size_t xp;          // dtype [T*k (+T), d] expert-contiguous (normalised) x; then x_hat for shared experts
  size_t h;           // dtype [T*k + S*T, I] SwiGLU hidden activations (routed rows, then shared)
  size_t y;           // fp32  [T*k + S*T, d] expert outputs
  size_t blk_z;       // fp32  [nb]    per-router-block sums of logsumexp^2
  size_t zloss;       // fp32  [1]     z-loss (when the caller passes none)
  size_t dropped;     // int32 [1]     dropped assignments (when the caller passes none)
  size_t rnorm;       // fp32  [T]     RMSNorm scale of every token
  size_t wr_hi;       // bf16  [E, d]  high part of w * W_r (norm with a weight, bf16)
  size_t wr_lo;       // bf16  [E, d]  low part of w * W_r
  size_t mt_done;     // int32 [n_mt]  per token tile: gate/up epilogue warps done (fused GEMMs)
  size_t n_mt;        //               its length: an upper bound on the GEMMs' token tiles
  size_t total;
};

constexpr int kMaxShared = MOE_MAX_SHARED;

// The shared experts as extra groups of the grouped GEMMs: group E + s takes
// `rows` (= T) rows starting at in0 + s * in_step of the input and writes them
// at out0 + s * rows of the output.
struct SharedGroups {
  int n;        // number of shared experts (0: none)
  int rows;     // T
  int in0;      // first input row of shared expert 0
  int in_step;  // input rows between shared experts (0: they all read the same rows)
  int out0;     // first output row of shared expert 0
};

// Pre-MoE RMSNorm as the router applies it.
struct RouterNorm {
  int form;          // moe_norm_form (0: none)
  float eps;
  const void* w;     // fp32 path: the norm weight [d] (NULL: ones)
  const void* w_hi;  // bf16 path: high part of w * W_r (NULL: no weight, plain W_r)
  const void* w_lo;  // bf16 path: low part of w * W_r
  float* rnorm;      // [T] out: the per-token scale
};

Workspace workspace_layout(int T, int d, int E, int k, int I, moe_dtype dtype, int n_shared = 0, bool norm = false);

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

// The routing scan's outputs (see launch_route_scan), for a router that
// computes them itself.
struct RouterScan {
  int32_t* counts = nullptr;
  int32_t* offsets = nullptr;
  int32_t* mtile = nullptr;
  float* aux = nullptr;
  float* zloss = nullptr;
  int32_t* dropped = nullptr;
  int32_t* mt_done = nullptr;
  int n_mt = 0;
  int cap = -1;
  int n_shared = 0;
};

// A bf16 batch that fits one tensor-core router block (T <= 128) with at
// most kRouterRegExperts experts: the router also does the routing scan, and
// no scan kernel is launched.
inline bool router_does_scan(int T, int E, moe_dtype dtype) {
  return dtype == MOE_BF16 && T > 0 && T <= kRouterTokensTc && E <= kRouterRegExperts;
}

// blk_z (nullable): per-block sums of logsumexp(logits)^2 for the z-loss.
// scan: where the scan's outputs go when router_does_scan (ignored otherwise).
cudaError_t launch_router(moe_dtype dtype, const void* x, const void* w_router, const float* b_router, int T,
                          int d, int E, int k, int renorm, const RouterNorm& norm, int32_t* topk_idx,
                          float* topk_gate, int32_t* lrank, int32_t* blk_cnt, float* blk_psum, float* blk_z,
                          const RouterScan& scan, int32_t* status, cudaStream_t stream);

cudaError_t launch_router_tc(const void* x, const void* w_router, const float* b_router, int T, int d, int E, int k,
                             int renorm, const RouterNorm& norm, int32_t* topk_idx, float* topk_gate, int32_t* lrank,
                             int32_t* blk_cnt, float* blk_psum, float* blk_z, const RouterScan& scan,
                             int32_t* status, cudaStream_t stream);

// hi[e,c] + lo[e,c] = w[c] * W_r[e,c] (bf16 + bf16; the fp32 product is exact).
cudaError_t launch_split_router_weight(const void* w_router, const void* norm_w, int E, int d, void* hi, void* lo,
                                       cudaStream_t stream);

// cap < 0: no capacity. Writes counts (before dropping), offsets and the GEMM
// tile prefix over the kept rows and the shared groups, aux, and optionally
// the z-loss (from blk_z) and the dropped count.
// mt_done (nullable): the fused GEMMs' per-token-tile counters, n_mt of them,
// cleared here for the call.
cudaError_t launch_route_scan(int nb, int T, int E, int k, int cap, int n_shared, int32_t* blk_cnt,
                              const float* blk_psum, const float* blk_z, int32_t* counts, int32_t* offsets,
                              int32_t* mtile, float* aux, float* zloss, int32_t* dropped, int32_t* mt_done, int n_mt,
                              cudaStream_t stream);

// The routing scan's outputs for a permute that does the scan itself (see
// permute_does_scan); offsets == NULL: the scan kernel ran, and blk_base
// holds every router block's base rows.
struct PermuteScanArgs {
  int nb = 0, cap = -1, n_shared = 0, n_mt = 0;
  const float* blk_psum = nullptr;
  const float* blk_z = nullptr;
  int32_t* counts = nullptr;
  int32_t* offsets = nullptr;
  int32_t* mtile = nullptr;
  float* aux = nullptr;
  float* zloss = nullptr;
  int32_t* dropped = nullptr;
  int32_t* mt_done = nullptr;
};

// When the router did not do the scan and the batch has few router blocks
// (nb * E at most 4096 per-block counts, which every permute block sums
// again), the permute does the routing scan and no scan kernel runs.
inline bool permute_does_scan(int nb, int E) { return (long long)nb * E <= 4096; }

// Also records the gate of every dispatched row (rgate) and, when zero_out is
// given, clears out[T, d] for a combine done by the down GEMM's epilogue.
// rnorm != NULL: rows are x * rnorm[t] * norm_w (norm_w NULL: ones), rounded
// to the dtype. shared_row0 >= 0: the (normalised) row of token t is also
// written at row shared_row0 + t. has_cap: a row past its expert's kept count
// is a dropped slot (inv = -1), not an error. scan.offsets != NULL: blk_base
// holds the router's per-block counts and the permute does the routing scan.
cudaError_t launch_permute(moe_dtype dtype, const void* x, int T, int d, int E, int k, int rb, const int32_t* topk_idx,
                           const int32_t* lrank, const int32_t* blk_base, const int32_t* offsets, int has_cap,
                           int32_t* perm_tok, int32_t* inv, void* xp, const float* topk_gate, float* rgate,
                           float* zero_out, const float* rnorm, const void* norm_w, int shared_row0,
                           const PermuteScanArgs& scan, int32_t* status, cudaStream_t stream);

// out[t] = sum_j gate[t,j] * Y[inv[t,j]] (dropped slots skipped when has_cap)
//        + sum_s Y[shared_row0 + s*T + t].
cudaError_t launch_combine(int T, int d, int k, const float* y, const int32_t* inv, const float* topk_gate,
                           int has_cap, int n_shared, int shared_row0, float* out, int32_t* status,
                           cudaStream_t stream);

// tcgen05 grouped GEMMs (bf16) on CTA pairs: 256 weight rows x up to 256
// dispatched tokens per tile. mode 0: H = SiLU(Xp Wg^T) * (Xp Wu^T) per
// expert; mode 1: Y = H Wd^T per expert. Groups 0..E-1 are the routed experts
// (rows from `offsets`), groups E.. the shared experts (`sh`, weights from the
// tm_s* maps). R_rows: rows of the output scratch.
cudaError_t launch_gemm_gateup_tc2(const CUtensorMap& tm_wg, const CUtensorMap& tm_wu, const CUtensorMap& tm_sg,
                                   const CUtensorMap& tm_su, const CUtensorMap& tm_xp, const CUtensorMap& tm_xp_small,
                                   const int32_t* offsets, const int32_t* mtile, int R_rows, int E,
                                   const SharedGroups& sh, int I, int d, void* h, int32_t* status,
                                   cudaStream_t stream);
// comb_out != nullptr: instead of storing Y, add gate * y of every dispatched
// row into comb_out[token] (used when k = 2 without shared experts, where the
// two adds commute).
cudaError_t launch_gemm_down_tc2(const CUtensorMap& tm_wd, const CUtensorMap& tm_sd, const CUtensorMap& tm_h,
                                 const CUtensorMap& tm_h_small, const int32_t* offsets, const int32_t* mtile,
                                 int R_rows, int E, const SharedGroups& sh, int I, int d, float* y,
                                 const int32_t* perm_tok, const float* rgate, float* comb_out, int32_t* status,
                                 cudaStream_t stream);

// Both projections in one persistent launch (batches of at most 32 tokens,
// where the GEMMs stream the weights): every gate/up tile, then every down
// tile, a down tile starting once the gate/up tiles of its token tile are
// stored (counted in mt_done, cleared by the routing scan).
bool gemms_fused(int T, moe_dtype dtype);
cudaError_t launch_gemm_fused_tc2(const CUtensorMap& tm_wg, const CUtensorMap& tm_wu, const CUtensorMap& tm_sg,
                                  const CUtensorMap& tm_su, const CUtensorMap& tm_xp_small, const CUtensorMap& tm_wd,
                                  const CUtensorMap& tm_sd, const CUtensorMap& tm_h_small, const int32_t* offsets,
                                  const int32_t* mtile, int R_rows, int E, const SharedGroups& sh_up,
                                  const SharedGroups& sh_down, int I, int d, void* h, float* y,
                                  const int32_t* perm_tok, const float* rgate, float* comb_out, int32_t* mt_done,
                                  int32_t* status, cudaStream_t stream);

// fp32 SIMT grouped GEMMs (same groups as above; sw*: the shared weights).
cudaError_t launch_gemm_gateup_simt(const float* xp, const float* wg, const float* wu, const float* swg,
                                    const float* swu, const int32_t* offsets, int R_rows, int E,
                                    const SharedGroups& sh, int I, int d, float* h, cudaStream_t stream);
cudaError_t launch_gemm_down_simt(const float* h, const float* wd, const float* swd, const int32_t* offsets,
                                  int R_rows, int E, const SharedGroups& sh, int I, int d, float* y,
                                  cudaStream_t stream);

}  // namespace moe
