/*
 * moe.h — C ABI of the B200 (sm_100a) sparse top-k Mixture-of-Experts
 * forward pass.
 *
 * The layer (axonml-nn layers/moe.rs: MoERouter::route, Expert::forward,
 * MoELayer::forward, load_balancing_loss, expert_utilization; Mixtral MoE
 * Block, exported PyTorch _moe_forward; Model Architecture Patterns,
 * "Top-K Router" and "SwiGLU FFN"):
 *
 *   p[t,:]      = softmax_e( x[t,:] . W_r[e,:] + b[e] )
 *   idx[t,:]    = the k largest p[t,e], ordered by p descending and, among
 *                 equal p, by expert index ascending
 *   gate[t,j]   = p[t,idx[t,j]] / sum_j' p[t,idx[t,j']]   (renorm = 1)
 *               = p[t,idx[t,j]]                            (renorm = 0)
 *   y_e(x)      = W_down[e] ( SiLU(W_gate[e] x) * (W_up[e] x) ),
 *                 SiLU(z) = z / (1 + exp(-z))
 *   out[t,:]    = sum_j gate[t,j] * y_{idx[t,j]}(x[t,:])
 *   counts[e]   = #{(t,j) : idx[t,j] = e}
 *   aux         = E * sum_e (counts[e] / (T*k)) * (sum_t p[t,e] / T)
 *
 * Conventions for every entry point:
 *   - All tensors are row-major and contiguous. Weights use the nn.Linear
 *     [out, in] layout, stacked per expert (the layout that KempnerForge
 *     ModelConfig.moe_packed_experts selects): W_router [E, d], W_gate [E, I, d],
 *     W_up [E, I, d], W_down [E, d, I].
 *   - Pointers documented as "device" must be CUDA device (or managed)
 *     memory on the current device; the caller owns every buffer. The
 *     library allocates no device memory: all scratch lives in the caller's
 *     workspace.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Calls are
 *     asynchronous on it and never synchronise the host.
 *   - Argument errors are returned synchronously before anything is
 *     launched; moe_last_error_detail() then gives a one-line reason.
 *     Errors detected on the device (a bounded wait that gave up, a
 *     non-finite router logit) are OR-ed into the caller's device status word
 *     as MOE_DEV_* bits, to be read after the stream is synchronised.
 *   - Nothing aborts the process.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* NULL required pointer, T < 0, k < 1, k > E, d/I/E <= 0 */
  MOE_ERR_UNSUPPORTED = 2, /* valid layer, but outside what the kernels take (see below) */
  MOE_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  MOE_ERR_WORKSPACE = 6    /* workspace NULL or smaller than moe_workspace_size() */
} moe_status;

/* Bits of the device status word. */
#define MOE_DEV_TIMEOUT 0x1   /* a bounded wait inside a kernel gave up; outputs are invalid */
#define MOE_DEV_NONFINITE 0x2 /* a router logit was NaN or infinite; that token's outputs are undefined */
#define MOE_DEV_INTERNAL 0x4  /* an internal consistency check failed (a dispatched row out of range);
                                 the offending access was skipped and the outputs are invalid */

typedef enum {
  MOE_F32 = 0, /* x and all weights fp32; every product accumulated in fp32 (SIMT FFMA) */
  MOE_BF16 = 1 /* x and all weights bf16; fp32 accumulation; SwiGLU hidden stored as bf16 */
} moe_dtype;

/*
 * Limits (MOE_ERR_UNSUPPORTED beyond them):
 *   E <= 256, k <= 8, T*k < 2^31, d*I < 2^31 per expert;
 *   MOE_BF16: d % 64 == 0 and I % 64 == 0 (128-byte TMA rows);
 *   MOE_F32 : d % 4 == 0 (16-byte rows).
 */

/*
 * moe_workspace_size — bytes of device scratch moe_forward needs for this
 * shape. Returns 0 if the shape is invalid or unsupported (see
 * moe_last_error_detail). The workspace holds the per-block routing
 * partials, the dispatch order, the expert-contiguous copy of x, the SwiGLU
 * hidden activations [T*k, I] and the fp32 expert outputs [T*k, d].
 */
size_t moe_workspace_size(int T, int d, int E, int k, int I, moe_dtype dtype);

/*
 * moe_forward — the whole layer on one GPU.
 *
 *   x          device, [T, d], dtype
 *   w_router   device, [E, d], dtype (router Linear, no bias)
 *   b_router   device, [E] fp32, or NULL: per-expert logit bias added before
 *              the softmax (the skewed-load workload's bias)
 *   w_gate     device, [E, I, d], dtype
 *   w_up       device, [E, I, d], dtype
 *   w_down     device, [E, d, I], dtype
 *   renorm     1: gates renormalised over the k selected experts (1/k each
 *              if their sum is not positive); 0: raw top-k probabilities
 *   out        device, [T, d] fp32 — written, never read
 *   topk_idx   device, [T, k] int32 — selected experts, best first
 *   topk_gate  device, [T, k] fp32 — their gates
 *   counts     device, [E] int32, or NULL — assignments per expert
 *   aux        device, [1] fp32, or NULL — load-balancing statistic
 *   workspace  device, at least moe_workspace_size() bytes, 256-byte aligned
 *   status_dev device, [1] int32, or NULL — MOE_DEV_* bits are OR-ed in; the
 *              caller clears it. NULL: the library keeps its own word in the
 *              workspace (cleared each call).
 *
 * T = 0 is valid: counts are zeroed and aux is set to 0 (axonml-nn moe.rs,
 * load_balancing_loss returns zero when there are no tokens).
 * Results are deterministic: the same inputs give bit-identical outputs.
 */
moe_status moe_forward(const void* x, const void* w_router, const float* b_router,
                       const void* w_gate, const void* w_up, const void* w_down,
                       int T, int d, int E, int k, int I, int renorm, moe_dtype dtype,
                       float* out, int32_t* topk_idx, float* topk_gate, int32_t* counts,
                       float* aux, void* workspace, size_t workspace_bytes, int32_t* status_dev,
                       void* stream);

/*
 * Kernels of one moe_forward, in launch order (both dtypes):
 *   0 router_topk, 1 route_scan, 2 permute, 3 grouped_gemm_gateup_swiglu,
 *   4 grouped_gemm_down, 5 combine.
 * moe_kernel_name(i) returns the name (a static string; NULL out of range).
 * Some shapes merge kernels (moe_launch_plan says which); a merged kernel's
 * slot is then empty.
 */
#define MOE_NUM_KERNELS 6
const char* moe_kernel_name(int i);

/*
 * moe_forward_events — moe_forward, plus per-kernel timing marks: events[i]
 * (a cudaEvent_t created by the caller) is recorded on `stream` just before
 * kernel i is launched and events[MOE_NUM_KERNELS] after the last one, so
 * cudaEventElapsedTime(events[i], events[i+1]) is kernel i's device time.
 * n_events must be at least MOE_NUM_KERNELS + 1. With T = 0 no kernel runs
 * and no event is recorded. Same results as moe_forward.
 */
moe_status moe_forward_events(const void* x, const void* w_router, const float* b_router,
                              const void* w_gate, const void* w_up, const void* w_down,
                              int T, int d, int E, int k, int I, int renorm, moe_dtype dtype,
                              float* out, int32_t* topk_idx, float* topk_gate, int32_t* counts,
                              float* aux, void* workspace, size_t workspace_bytes,
                              int32_t* status_dev, void* stream, void* const* events, int n_events);

/*
 * moe_get_permutation — copy out the dispatch order that the last
 * moe_forward on this workspace (same shape arguments) produced
 * (axonml-nn moe.rs, MoELayer::forward: rows grouped by expert in ascending
 * expert order, tokens ascending within an expert):
 *   offsets  device, [E+1] int32 — first dispatched row of each expert
 *   perm_tok device, [T*k] int32 — token of each dispatched row
 *   inv      device, [T, k] int32 — dispatched row of each (token, slot)
 * Any of the three may be NULL. Enqueued on `stream`.
 */
moe_status moe_get_permutation(const void* workspace, size_t workspace_bytes, int T, int d, int E,
                               int k, int I, moe_dtype dtype, int32_t* offsets, int32_t* perm_tok,
                               int32_t* inv, void* stream);

/*
 * Options of the layer that the pages name as configuration knobs. A zeroed
 * struct (with struct_bytes set) is the plain layer of moe_forward.
 *
 * Pre-MoE RMSNorm (the block normalises x before this layer: Mixtral MoE
 * Block, "post_attn_norm", nn.RMSNorm; Model Architecture Patterns,
 * "RMSNorm (no bias, no mean centering)"):
 *   MOE_NORM_RMS              x_hat = x / sqrt(mean_c x^2 + eps) * w
 *   MOE_NORM_RMS_EPS_OUTSIDE  x_hat = w * x / (sqrt(mean_c x^2) + eps)
 * The router and every expert then see x_hat instead of x. The router folds
 * the per-token scale into its logits (exact x, w * W_r split into two bf16
 * terms), and the experts read x_hat rounded once to the layer dtype.
 *
 * Shared experts (KempnerForge ModelConfig, moe_shared_experts: experts
 * that every token passes through): n_shared SwiGLU MLPs of the routed
 * experts' shape, applied to every token and added with weight 1:
 *   out[t] += sum_s W_sdown[s] (SiLU(W_sgate[s] x_t) * (W_sup[s] x_t))
 *
 * Capacity (KempnerForge ModelConfig, moe_capacity_factor: zero keeps
 * every assignment, a positive factor limits the tokens an expert takes): every expert keeps at most C = ceil(cf * T * k / E) assignments,
 * its first C in dispatch order (tokens ascending); a dropped slot adds
 * nothing to out. topk_idx, topk_gate, counts and aux are those before
 * dropping; moe_get_permutation reports the kept rows and inv = -1 for a
 * dropped slot.
 *
 * Router z-loss (the ST-MoE statistic of "moe_router_z_loss_weight"):
 *   z = (1/T) sum_t ( log sum_e exp(logit[t,e]) )^2, logits with their bias.
 *
 * Folded combine (no counterpart on the pages): on the bf16 path with k = 2
 * and no shared experts the down GEMM's epilogue adds gate * y of every
 * expert row into the zeroed fp32 output with atomic adds instead of storing
 * Y for a combine kernel; two additions into zero commute, so that result is
 * bit-identical from run to run. fold_combine != 0 does the same for every
 * k (still bf16, no shared experts): no Y rows are written or read back, but
 * with k > 2 the order of a token's additions varies between runs, so the
 * output equals the combine kernel's up to fp32 rounding and is not
 * bit-reproducible. Off by default.
 */
typedef enum {
  MOE_NORM_NONE = 0,
  MOE_NORM_RMS = 1,
  MOE_NORM_RMS_EPS_OUTSIDE = 2
} moe_norm_form;

#define MOE_MAX_SHARED 8

typedef struct moe_options {
  size_t struct_bytes;       /* sizeof(moe_options) */
  int norm_form;             /* moe_norm_form */
  float norm_eps;            /* >= 0 and finite */
  const void* norm_weight;   /* device, [d] in the layer dtype, or NULL for ones */
  int n_shared;              /* 0 .. MOE_MAX_SHARED */
  const void* shared_gate;   /* device, [n_shared, I, d], dtype */
  const void* shared_up;     /* device, [n_shared, I, d], dtype */
  const void* shared_down;   /* device, [n_shared, d, I], dtype */
  double capacity_factor;    /* 0: no dropping; > 0 and finite: the cap above */
  int32_t* dropped;          /* device, [1] int32, or NULL: assignments dropped */
  float* z_loss;             /* device, [1] fp32, or NULL: the z-loss statistic */
  int fold_combine;          /* nonzero: fold the combine into the down GEMM for every k (above) */
} moe_options;

/*
 * moe_workspace_size_ex — moe_workspace_size for a layer with options (opt
 * may be NULL: the plain layer). Shared experts add T rows to the dispatched
 * input and n_shared * T rows to the hidden and output scratch. Returns 0 for
 * an invalid shape or invalid options.
 */
size_t moe_workspace_size_ex(int T, int d, int E, int k, int I, moe_dtype dtype, const moe_options* opt);

/*
 * moe_forward_ex — moe_forward with options (opt may be NULL) and optional
 * per-kernel timing events (events may be NULL with n_events = 0; otherwise
 * as moe_forward_events). The workspace must hold moe_workspace_size_ex()
 * bytes for the same options. Invalid options (unknown norm form, negative
 * or non-finite eps or capacity factor, n_shared outside 0..MOE_MAX_SHARED,
 * a NULL or misaligned shared weight, struct_bytes smaller than the struct)
 * give MOE_ERR_INVALID_ARG before anything is launched. With the norm and
 * a weight on the bf16 path, an extra small kernel that splits w * W_r runs
 * before the router and is timed with it.
 */
moe_status moe_forward_ex(const void* x, const void* w_router, const float* b_router,
                          const void* w_gate, const void* w_up, const void* w_down,
                          int T, int d, int E, int k, int I, int renorm, moe_dtype dtype,
                          const moe_options* opt, float* out, int32_t* topk_idx, float* topk_gate,
                          int32_t* counts, float* aux, void* workspace, size_t workspace_bytes,
                          int32_t* status_dev, void* stream, void* const* events, int n_events);

/*
 * moe_launch_plan — which kernels a call with this shape and these options
 * (NULL: none) launches, as a bit set; -1 if the arguments are invalid (see
 * moe_last_error_detail). Host only; launches nothing.
 *   MOE_PLAN_FUSED_COMBINE: the combine runs in the down GEMM's epilogue
 *     (bf16, no shared experts, k = 2 or fold_combine set): kernel 5 is not
 *     launched.
 *   MOE_PLAN_FUSED_GEMMS: both projections run in one persistent kernel
 *     (bf16, 1 <= T <= 32, where the GEMMs stream the weights from HBM):
 *     slot 3 times both, slot 4 is empty.
 *   MOE_PLAN_ROUTER_WEIGHT_SPLIT: a small kernel splits w * W_r into two
 *     bf16 terms before the router (bf16 RMSNorm with a weight); its time
 *     falls in slot 0.
 *   MOE_PLAN_FUSED_SCAN: the router does the routing scan itself (bf16,
 *     1 <= T <= 128 tokens, one router block, E <= 16): slot 1 is empty.
 *   MOE_PLAN_PERMUTE_SCAN: otherwise, when the batch has few router blocks
 *     (blocks of 128 tokens for bf16, 32 for fp32; blocks x E <= 4096), every
 *     permute block redoes the scan's sums for its own rows and the permute
 *     writes the scan's results: slot 1 is empty, slot 2 times both.
 */
#define MOE_PLAN_FUSED_COMBINE 1
#define MOE_PLAN_FUSED_GEMMS 2
#define MOE_PLAN_ROUTER_WEIGHT_SPLIT 4
#define MOE_PLAN_FUSED_SCAN 8
#define MOE_PLAN_PERMUTE_SCAN 16
int moe_launch_plan(int T, int d, int E, int k, int I, moe_dtype dtype, const moe_options* opt);

/*
 * moe_forward_noalloc — moe_forward for callers that cannot allocate device
 * memory: the same layer, arguments and results, but the scratch lives in a
 * static array of MOE_NOALLOC_SCRATCH_BYTES inside the library's device image
 * instead of a caller workspace. The pages have no counterpart; it exists for
 * callers that run inside an engine or plugin whose host framework owns every
 * device allocation, or a serving loop that forbids allocation after warm-up.
 *
 *   - Shapes whose moe_workspace_size() exceeds MOE_NOALLOC_SCRATCH_BYTES are
 *     rejected with MOE_ERR_WORKSPACE and a message (nothing is launched);
 *     16 MiB covers, for example, a 32-token decode batch of the Mixtral
 *     shape (d=4096, E=8, k=2, I=14336), which needs about 3.3 MB.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it with
 *     the id of the current CUDA context; a call in another context (after
 *     cudaDeviceReset, or in a context the caller made current) looks it up
 *     again. Make the first call on a device, and the first in a new
 *     context, before any stream capture. The call allocates nothing: no
 *     cudaMalloc, no cudaFree.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind; the library rewrites everything it reads on each call, and
 *     clears its own status word when status_dev is NULL. Calls that overlap
 *     on the GPU (concurrent streams, or other threads) race on the array:
 *     serialise them.
 *   - Every GPU that loads the library holds the array until the process
 *     exits.
 */
#define MOE_NOALLOC_SCRATCH_BYTES (16u << 20)
moe_status moe_forward_noalloc(const void* x, const void* w_router, const float* b_router,
                               const void* w_gate, const void* w_up, const void* w_down,
                               int T, int d, int E, int k, int I, int renorm, moe_dtype dtype,
                               float* out, int32_t* topk_idx, float* topk_gate, int32_t* counts,
                               float* aux, int32_t* status_dev, void* stream);

/*
 * moe_pipeline — the layer called repeatedly on batches that live in host
 * memory, the end-to-end path of a serving loop: the pipeline copies batch
 * i+1 in and batch i-1 out while batch i computes, on three streams (its own
 * copy-in and copy-out streams, and the caller's compute stream). The pages
 * have no counterpart (their layers take tensors already in place).
 *
 * moe_layer_desc describes the layer once: device weights as for
 * moe_forward_ex, the shape and dtype, options (copied at create; NULL for
 * none), the caller's workspace (moe_workspace_size[_ex] bytes), device
 * buffers shared by every batch (topk_idx [T,k], topk_gate [T,k], counts [E]
 * or NULL, status_dev [1] or NULL) and two device staging slots per batch
 * tensor: x_dev[b] [T,d] in the dtype, out_dev[b] [T,d] fp32, aux_dev[b] [1]
 * fp32. The library allocates no device memory; create makes two streams
 * and six events, which destroy releases.
 *
 * moe_pipeline_submit(p, x_host, out_host, aux_host) enqueues one batch and
 * returns without waiting: x_host [T,d] in the dtype, out_host [T,d] fp32,
 * aux_host [1] fp32 or NULL, in host memory (pinned memory lets the copies
 * overlap the compute; pageable memory works but serialises). The host
 * buffers must stay untouched until moe_pipeline_synchronize returns; the
 * topk_idx/topk_gate/counts buffers hold the last computed batch's values.
 * moe_pipeline_stream(p, MOE_PIPELINE_COPY_IN | _COMPUTE | _COPY_OUT) gives
 * the streams, for callers that order their own work or timing events
 * against them. moe_pipeline_destroy synchronises, then frees.
 */
typedef struct moe_layer_desc {
  size_t struct_bytes;          /* sizeof(moe_layer_desc) */
  const void* w_router;         /* device [E, d] */
  const float* b_router;        /* device [E] or NULL */
  const void* w_gate;           /* device [E, I, d] */
  const void* w_up;             /* device [E, I, d] */
  const void* w_down;           /* device [E, d, I] */
  int T, d, E, k, I, renorm;
  moe_dtype dtype;
  const moe_options* opt;       /* NULL: the plain layer */
  void* workspace;
  size_t workspace_bytes;
  int32_t* topk_idx;            /* device [T, k] */
  float* topk_gate;             /* device [T, k] */
  int32_t* counts;              /* device [E] or NULL */
  int32_t* status_dev;          /* device [1] or NULL */
  void* x_dev[2];               /* device [T, d] dtype, one per slot */
  float* out_dev[2];            /* device [T, d] fp32 */
  float* aux_dev[2];            /* device [1] fp32 */
} moe_layer_desc;

typedef struct moe_pipeline moe_pipeline;
#define MOE_PIPELINE_COPY_IN 0
#define MOE_PIPELINE_COMPUTE 1
#define MOE_PIPELINE_COPY_OUT 2
moe_status moe_pipeline_create(const moe_layer_desc* desc, void* compute_stream, moe_pipeline** out);
moe_status moe_pipeline_submit(moe_pipeline* p, const void* x_host, float* out_host, float* aux_host);
moe_status moe_pipeline_synchronize(moe_pipeline* p);
void* moe_pipeline_stream(const moe_pipeline* p, int which);
moe_status moe_pipeline_destroy(moe_pipeline* p);

/*
 * moe_selftest_wait_timeout — a diagnostic of the failure handling every
 * kernel of the library shares: it launches one warp on `stream` that waits
 * on a shared-memory barrier phase nothing will complete, through the same
 * bounded wait the kernels use, with a limit of limit_ns nanoseconds
 * (1e6 .. 5e9). The wait gives up, OR-s MOE_DEV_TIMEOUT into *status_dev
 * (device int32, not cleared here) and the kernel returns; the context stays
 * usable. The pages have no counterpart (their Rust layer panics instead).
 */
moe_status moe_selftest_wait_timeout(int32_t* status_dev, long long limit_ns, void* stream);

/*
 * moe_last_error_detail — the reason for the calling thread's last non-OK
 * status, NUL-terminated into buf (truncated to n bytes). Returns the full
 * length of the message.
 */
size_t moe_last_error_detail(char* buf, size_t n);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
