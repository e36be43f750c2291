/*
 * moe.h -- C ABI of the B200 (sm_100a) sparse Mixture-of-Experts FFN layer.
 *
 * The layer (forward pass only), per token t with row x_t = x[t, 0:H]:
 *   router   l = x_t . Wgate^T (+ optional per-expert bias)        [E]
 *            p = softmax(l); S = top_k(p); w_j = scale * p_Sj / sum_S p
 *   experts  y_e = down_e( silu(clamp(gate_e(x_t))) * clamp(up_e(x_t)) )
 *   combine  out_t = sum_j w_j * y_{S_j}(x_t) + shared(x_t)
 * Sources: page "腾讯混元Hy4 Preview深度技术解析" (MoERouter and MoELayer
 * sketches: bias-free gate, softmax, top-k, routed plus always-on shared
 * expert); page "腾讯混元Hy3正式版深度解析" (SparseMoERouter: top-k weights
 * renormalised to sum to one; MoEFeedForward: bias-free SwiGLU FFN with
 * gate/up/down projections); page "Hy4 preview config.json 终极深度解读",
 * section "MoE 路由专家256 选 8" (256 routed experts, top-8, 1 shared expert,
 * moe_intermediate_size 2048, norm_topk_prob, routed_scaling_factor 2.827
 * applied to the routed experts only, swiglu_limit 10.0 clamping the SwiGLU
 * inputs to +-10).
 *
 * Conventions shared by every entry point
 *  - Pointers named as device pointers must be device memory owned by the
 *    caller; the library never allocates or frees device memory on a call.
 *    Tensors are dense, row-major, and 16-byte aligned.
 *  - Scratch memory comes from the caller's `workspace` (device, 256-byte
 *    aligned) of at least moe_workspace_size(problem, call) bytes.  Its first
 *    4 bytes hold the DEVICE ERROR WORD (int32): kernels set it to a nonzero
 *    moe_status (MOE_ERR_TIMEOUT, MOE_ERR_BAD_INDEX) when a bounded wait
 *    expires or an index input is out of range.  The library never clears
 *    it; read it with moe_read_device_status and clear it with
 *    moe_clear_device_status.  Calls that share a workspace must be ordered
 *    on one stream.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy stream).  Every
 *    call only enqueues work and returns; MOE_OK means the arguments were
 *    valid and all launches were accepted.  No call synchronises the host
 *    except moe_read_device_status.
 *  - Errors are returned, never thrown; on any error nothing is enqueued.
 *  - dtype: MOE_BF16 - x, weights, outputs bf16; all sums in fp32 on tensor
 *    cores.  MOE_F32 - x, weights, outputs fp32; the router runs in fp32 on
 *    CUDA cores, the expert GEMMs on tensor cores reading the fp32 operands
 *    as TF32 (10-bit mantissa; tcgen05 kind::tf32), with fp32 sums, and h and
 *    the expert output rows stay fp32.
 *  - Shapes supported: T >= 0 (T == 0 is a no-op), H and I multiples of 64,
 *    1 <= top_k <= min(E, 32), E <= 256, num_shared in {0,1},
 *    T*top_k < 2^31.  Anything else returns MOE_ERR_UNSUPPORTED.
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
    MOE_ERR_INVALID_ARG = 1, /* null pointer, bad alignment, NaN scale, ... */
    MOE_ERR_UNSUPPORTED = 2, /* shape or dtype outside the supported set */
    MOE_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required */
    MOE_ERR_CUDA = 4,        /* a CUDA launch or runtime call failed */
    MOE_ERR_TIMEOUT = 5,     /* (device error word) a bounded wait expired */
    MOE_ERR_BAD_INDEX = 6    /* (device error word) an index input was out of range */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Which entry point a workspace is sized for. */
typedef enum {
    MOE_CALL_ROUTE = 0,
    MOE_CALL_ROUTER_LOGITS = 1,
    MOE_CALL_PERMUTE = 2,
    MOE_CALL_FFN = 3,
    MOE_CALL_COMBINE = 4,
    MOE_CALL_FORWARD = 5,
    MOE_CALL_ROUTER_STATS = 6,
    MOE_CALL_FORWARD_FP8 = 7
} moe_call;

typedef struct {
    int64_t T;            /* tokens */
    int32_t H;            /* hidden size */
    int32_t E;            /* routed experts */
    int32_t I;            /* expert (and shared expert) intermediate size */
    int32_t top_k;        /* experts per token */
    int32_t num_shared;   /* 0 or 1 always-on shared expert of width I */
    float routed_scale;   /* routed_scaling_factor (2.827 for Hy4) */
    float clip_limit;     /* swiglu_limit; > 0 clamps gate and up to [-L, L]; <= 0 or inf: off */
    int32_t dtype;        /* moe_dtype */
} moe_problem;

/* Bytes of workspace the given entry point needs for this problem. 0 on a
 * problem that fails validation.  For MOE_CALL_FFN the size covers
 * max(T*top_k, T) rows in E groups. */
size_t moe_workspace_size(const moe_problem* problem, int32_t call);

/* Static description of a status code. */
const char* moe_status_string(int32_t status);

/*
 * moe_expert_tile_rows -- the token-row tile widths moe_forward and
 * moe_forward_fp8 use for this problem (host only, no CUDA call): each
 * expert's rows (and the shared expert's T rows) are cut into
 * c = ceil(rows / width) chunks of ceil16(ceil(rows / c)) rows, the last one
 * shorter, and every chunk is one token tile of the gate/up (*gate_up_rows)
 * or the down GEMM (*down_rows).  Useful to test or profile every tile of a
 * schedule.  Both outputs are host pointers.
 */
int32_t moe_expert_tile_rows(const moe_problem* problem, int32_t* gate_up_rows,
                             int32_t* down_rows);

/*
 * moe_router_logits -- the router's gate GEMM:
 *   logits[t, e] = sum_h x[t, h] * gate_w[e, h]      (fp32 [T, E], device, out)
 * x: [T, H] device; gate_w: [E, H] device (nn.Linear weight layout).
 * (page "腾讯混元Hy4 Preview深度技术解析", MoERouter: gate = Linear(hidden,
 * num_experts, bias=False).)
 */
int32_t moe_router_logits(const moe_problem* problem, const void* x, const void* gate_w,
                          float* logits, void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_route -- router: gate GEMM, softmax over experts, top-k, renormalise,
 * scale (page "腾讯混元Hy3正式版深度解析", SparseMoERouter.forward; page
 * "Hy4 preview config.json 终极深度解读", norm_topk_prob and
 * routed_scaling_factor).
 *   x          [T, H] device
 *   gate_w     [E, H] device
 *   logit_bias [E] fp32 device or NULL (added to the logits; synthetic skew)
 *   topk_idx   [T, top_k] int32 device, out: experts by descending
 *              probability, exact ties to the lower index
 *   topk_w     [T, top_k] fp32 device, out: scale * p_j / sum_sel p
 */
int32_t moe_route(const moe_problem* problem, const void* x, const void* gate_w,
                  const float* logit_bias, int32_t* topk_idx, float* topk_w, void* workspace,
                  size_t ws_bytes, void* stream);

/*
 * moe_permute -- dispatch: group the (token, slot) assignments by expert
 * (page tqpw.cn/news/149001, section 2.1 "MoE 的基本工作原理": per-expert
 * mask dispatch x[expert_mask]).  Permuted rows are ordered by expert, then
 * token, then slot.  Each token's top_k experts must be distinct.
 *   topk_idx  [T, top_k] int32 device (values in [0, E))
 *   x         [T, H] device
 *   offsets   [E+1] int32 device, out: expert e owns rows offsets[e]..offsets[e+1]-1
 *   pos       [T, top_k] int32 device, out: permuted row of assignment (t, j)
 *   src_token [T*top_k] int32 device, out: token of each permuted row
 *   x_perm    [T*top_k, H] device (problem dtype), out: x_perm[pos[t,j]] = x[t]
 */
int32_t moe_permute(const moe_problem* problem, const int32_t* topk_idx, const void* x,
                    int32_t* offsets, int32_t* pos, int32_t* src_token, void* x_perm,
                    void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_grouped_swiglu_ffn -- one SwiGLU FFN per group of rows (page
 * "腾讯混元Hy3正式版深度解析", MoEFeedForward; clamp from swiglu_limit):
 *   for g in [0, n_groups), rows r in [offsets[g], offsets[g+1]):
 *     y_perm[r] = down_g( silu(clamp(gate_g(x_perm[r]))) * clamp(up_g(x_perm[r])) )
 *   x_perm   [rows, H] device (problem dtype)
 *   offsets  [n_groups+1] int32 device, non-decreasing, offsets[n_groups] <= rows
 *   expert_w [n_groups, 3, I, H] device: gate_proj, up_proj ([I,H], nn.Linear
 *            layout) and down_proj stored transposed as [I,H]
 *            (y[h] = sum_i a[i] * W[g,2,i,h])
 *   y_perm   [rows, H] device (problem dtype), out; rows outside every group
 *            are left untouched
 * n_groups in [1, 256]; top_k, E, T and routed_scale of `problem` are unused
 * (the shared expert is run as n_groups = 1 over x itself).
 */
int32_t moe_grouped_swiglu_ffn(const moe_problem* problem, const void* x_perm, int64_t rows,
                               const int32_t* offsets, int32_t n_groups, const void* expert_w,
                               void* y_perm, void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_combine -- weighted sum back into token order, plus the shared expert
 * (page "腾讯混元Hy4 Preview深度技术解析", MoELayer.forward: routed output
 * accumulated with the routing weights, then plus the shared output):
 *   out[t] = sum_j topk_w[t,j] * y_perm[pos[t,j]]  (+ shared_y[t])
 * summed in slot order in fp32 (deterministic).
 *   y_perm   [T*top_k, H] device (problem dtype)
 *   pos      [T, top_k] int32 device
 *   topk_w   [T, top_k] fp32 device
 *   shared_y [T, H] device or NULL
 *   out      [T, H] device (problem dtype), out
 */
int32_t moe_combine(const moe_problem* problem, const void* y_perm, const int32_t* pos,
                    const float* topk_w, const void* shared_y, void* out, void* workspace,
                    size_t ws_bytes, void* stream);

/*
 * moe_forward -- the whole layer in one call: route, dispatch, grouped
 * gate/up GEMM with the clamp + SwiGLU fused into its epilogue, grouped down
 * GEMM whose epilogue multiplies each row by its routing weight (the shared
 * expert is one more group, with weight 1) and stores the weighted rows, then
 * a combine kernel that adds each token's top_k rows and its shared-expert
 * row in slot order, in fp32, and writes the output dtype.  Every sum is
 * taken in a fixed order, so the output is bitwise reproducible from run to
 * run.  (Setting MOE_COMBINE=atomic in the environment selects the other
 * form: the down epilogue scatter-adds into an fp32 token accumulator, whose
 * result bits then depend on the order of the atomic additions, within the
 * stated tolerance.)
 *   x            [T, H] device
 *   gate_w       [E, H] device
 *   logit_bias   [E] fp32 device or NULL
 *   expert_w     [E, 3, I, H] device (layout as in moe_grouped_swiglu_ffn)
 *   shared_w     [3, I, H] device, or NULL when num_shared == 0
 *   out          [T, H] device (problem dtype), out
 *   topk_idx_out [T, top_k] int32 device or NULL, out
 *   topk_w_out   [T, top_k] fp32 device or NULL, out
 */
int32_t moe_forward(const moe_problem* problem, const void* x, const void* gate_w,
                    const float* logit_bias, const void* expert_w, const void* shared_w,
                    void* out, int32_t* topk_idx_out, float* topk_w_out, void* workspace,
                    size_t ws_bytes, void* stream);

/*
 * moe_route_noalloc -- moe_route for callers that cannot allocate device
 * memory: no workspace argument, and no allocation of any kind inside.
 * There is no counterpart on the pages: it is a deployment convenience.
 * Some callers cannot hand the library a workspace: code that runs while a
 * CUDA stream is being captured (where cudaMalloc is not allowed), serving
 * loops whose framework allocator already owns all device memory, and
 * latency-critical paths that must not call cudaMalloc/cudaFree because those
 * can synchronise the device.  This entry point keeps its scratch (the fp32
 * router logits, T*E floats) in a fixed 1 MiB device array built into the
 * library, which every GPU that loads the library holds until the process
 * exits.  Arguments and outputs are those of moe_route.
 *  - Capacity: 256 + 4*T*E bytes must fit in MOE_ROUTE_NOALLOC_SCRATCH_BYTES
 *    (e.g. T <= 1023 tokens at E = 256); larger problems return
 *    MOE_ERR_WORKSPACE and enqueue nothing.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current, and keeps it for the
 *    life of the process; make that first call before any stream capture.
 *    A device reset (cudaDeviceReset, or anything else that destroys the
 *    primary context) invalidates the kept address: do not call this entry
 *    point again in a process that has reset the device.
 *  - All calls share the one array and it keeps the last call's contents:
 *    calls that overlap on the GPU (different streams, or different host
 *    threads, on one device) race and corrupt each other's logits.  Order
 *    them on one stream.  The device error word in the array is cleared at
 *    each call and is not reported to the caller.
 */
#define MOE_ROUTE_NOALLOC_SCRATCH_BYTES (1u << 20)
int32_t moe_route_noalloc(const moe_problem* problem, const void* x, const void* gate_w,
                          const float* logit_bias, int32_t* topk_idx, float* topk_w,
                          void* stream);

/*
 * moe_router_stats -- the router's load-balancing statistics over the T
 * tokens (page "腾讯混元Hy3正式版深度解析", SparseMoERouter: the auxiliary
 * load-balancing loss and the running expert counts):
 *   P_out[e]  = (1/T) sum_t softmax(logits[t] + bias)[e]   mean probability  [E] fp32
 *   f_out[e]  = #{(t,j): topk_idx[t,j] == e} / (T*top_k)   selection share   [E] fp32
 *   aux_out[0] = E * sum_e P_out[e] * f_out[e]             auxiliary loss    [1] fp32
 *   ema_counts[e] <- m*ema_counts[e] + (1-m)*count[e]      [E] fp32 in/out, or NULL
 *   ema_total[0]  <- m*ema_total[0] + (1-m)*T              [1] fp32 in/out, or NULL
 * with m = momentum in [0,1] (the sketch uses 0.9); all pointers are device
 * memory.  The routing (logits, top-k) is the one moe_route computes.  Sums
 * are taken in a fixed order, so the results are reproducible.  T must be >= 1.
 */
int32_t moe_router_stats(const moe_problem* problem, const void* x, const void* gate_w,
                         const float* logit_bias, float* P_out, float* f_out, float* aux_out,
                         float* ema_counts, float* ema_total, float momentum, void* workspace,
                         size_t ws_bytes, void* stream);

/*
 * FP8 expert weights (page "1M上下文实战：Hy4 preview如何从容处理百万token级长
 * 文档", section "最快部署 1M 上下文": the official deployment uses FP8
 * weights).  The pages give no number format; this library uses OCP E4M3
 * codes with power-of-two scales s = 2^n, n the smallest integer with
 * 448 * 2^n >= the channel's largest magnitude, so that every encoding
 * decision is exact:
 *   gate/up weights: one scale per output row i of each matrix,
 *   down weights:    one scale per output column h,
 *   token rows x_t:  one scale per token (computed inside moe_forward_fp8),
 *   SwiGLU output h: one fixed scale from the clamp bound silu(L) * L.
 * The expert GEMMs run on tcgen05 kind::f8f6f4 (E4M3 x E4M3, fp32 sums); the
 * router stays in bf16.
 *
 * moe_quantize_weights_fp8 -- encode [n_experts, 3, I, H] weights (problem
 * dtype; device) into E4M3 codes q (same shape, uint8, device) with scales
 * scale_gu [n_experts, 2, I] (gate rows, then up rows) and scale_d
 * [n_experts, H] (fp32, device).  H and I must be multiples of 128; w and q
 * must be 16-byte aligned (else MOE_ERR_INVALID_ARG).
 * Run once per weight set (e.g. at load time); nothing is allocated.
 */
int32_t moe_quantize_weights_fp8(const moe_problem* problem, int32_t n_experts, const void* w,
                                 uint8_t* q, float* scale_gu, float* scale_d, void* stream);

/*
 * moe_forward_fp8 -- moe_forward with FP8 expert (and shared-expert) weights
 * from moe_quantize_weights_fp8 (shared_*: n_experts = 1, or NULL without a
 * shared expert).  x, gate_w, out: bf16.  Requires dtype MOE_BF16, H and I
 * multiples of 128, and clip_limit > 0 (it bounds h).  The combine is the
 * fixed-order gather (deterministic).  Workspace: MOE_CALL_FORWARD_FP8.
 */
int32_t moe_forward_fp8(const moe_problem* problem, const void* x, const void* gate_w,
                        const float* logit_bias, const uint8_t* expert_q,
                        const float* expert_scale_gu, const float* expert_scale_d,
                        const uint8_t* shared_q, const float* shared_scale_gu,
                        const float* shared_scale_d, void* out, int32_t* topk_idx_out,
                        float* topk_w_out, void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_check_wait_timeout -- self-check of the bounded waits every kernel uses
 * (mbarrier phase waits, and the global-counter wait of the fused routing
 * step).  Launches one thread that waits on an mbarrier nobody arrives on and
 * on a counter nobody increments, each with a limit of about 0.1 s; both give
 * up, and MOE_ERR_TIMEOUT is written to the workspace's error word.
 * *waits_timed_out (host) receives one bit per wait that gave up (3 = both).
 * The workspace needs 256 bytes (any workspace from moe_workspace_size has
 * them); the call waits for the stream.  Nothing faults or hangs, and the
 * context stays usable: clear the error word with moe_clear_device_status.
 */
int32_t moe_check_wait_timeout(void* workspace, size_t ws_bytes, int32_t* waits_timed_out,
                               void* stream);

/* Copy the device error word of `workspace` to *status_out (host), waiting
 * for the stream.  Returns MOE_OK or MOE_ERR_CUDA / MOE_ERR_INVALID_ARG. */
int32_t moe_read_device_status(const void* workspace, int32_t* status_out, void* stream);

/* Enqueue a reset of the device error word to 0. */
int32_t moe_clear_device_status(void* workspace, void* stream);

/* Number of kernels this library has launched since it was loaded. */
int64_t moe_launch_count(void);

/*
 * Per-kernel timing.  moe_profile_start(max_launches) creates up to
 * 2*max_launches CUDA events (on the current device) and from then on records
 * one before and one after every kernel the library launches, on that
 * launch's stream.  moe_profile_stop waits for the events, fills up to
 * `max_entries` records of (kernel name, launches, total milliseconds), sets
 * *n_entries, releases the events and turns recording off.
 */
typedef struct {
    const char* name;
    int32_t launches;
    double total_ms;
} moe_kernel_time;

int32_t moe_profile_start(int32_t max_launches);
int32_t moe_profile_stop(moe_kernel_time* entries, int32_t max_entries, int32_t* n_entries);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
