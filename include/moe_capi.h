/*
 * moe_capi.h — C ABI of the B200 (sm_100a) DeepSeekMoE layer: the forward,
 * the bias controller, node-limited routing, the sequence-wise balance
 * statistics, the FP8 backward of the expert path, and the layer with its
 * routed experts sharded over several GPUs (expert parallelism).
 *
 * The layer (sources: "DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing,
 * Multi-Token Prediction, and FP8 Training at 671B Scale", trishampatil.com,
 * section III "The mechanism" and "How the bias is set", section V "Four
 * details"; "DeepSeek-V3, explained", vibeengines.com, recipe steps 3, 4, 5
 * and 7; "DeepSeek-V3 Technical Report", deepforge.srivtx.xyz, "Per-tile FP8
 * scaling"):
 *
 *   s[t,i]  = sigmoid(x_t . e_i)                          sigmoid affinity
 *   ids_t   = TopK_i(s[t,i] + b_i, K)                     bias only selects
 *   g[t,k]  = s[t,ids_k] / sum_k s[t,ids_k]               unbiased gates
 *   y_t     = FFN_shared(x_t) + sum_k g[t,k] FFN_{ids_k}(x_t)
 *   FFN(u)  = W_down (silu(W_gate u) * (W_up u))          SwiGLU, FP8 E4M3:
 *             u and h in 1x128 tiles, weights in 128x128 blocks, fp32 sums
 *   b_i    <- b_i + gamma * sign(T*K/N - c_i)             per step, c_i = load
 *
 * and, for training, the gradients of y with respect to x (through the
 * experts), the gates and the expert weights, with the Dgrad and Wgrad GEMMs
 * in FP8 as well ("DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing, ...",
 * section V, Figure 6).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers, row-major, owned by the caller;
 *     the library never allocates or frees device memory.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Work is
 *     enqueued asynchronously; no call synchronises except moe_get_status.
 *   - Return value: MOE_OK or a negative moe_status. Argument errors are
 *     detected on the host before anything is enqueued. A launch failure
 *     returns MOE_ERR_CUDA. Errors found on the device (a count or index
 *     that fails its check, a bounded wait that gave up) are recorded in the
 *     status word at the start of the workspace, read by moe_get_status;
 *     device code never traps.
 *   - bf16 tensors are passed as `const void*` holding IEEE bfloat16.
 *   - E4M3 tensors hold OCP E4M3FN bytes (bias 7, max 448, NaN 0x7F).
 *   - Scales are the multipliers 448 / amax (dequantised = code / scale).
 *   - NaN or Inf in the layer input is outside the contract.
 */
#ifndef MOE_CAPI_H
#define MOE_CAPI_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_SHAPE = -1,      /* a size outside the supported range */
  MOE_ERR_NULL = -2,       /* a required pointer is NULL */
  MOE_ERR_CUDA = -3,       /* a CUDA call or kernel launch failed */
  MOE_ERR_TIMEOUT = -4,    /* device status: a bounded wait gave up */
  MOE_ERR_BOUNDS = -5,     /* device status: a count or index check failed */
  MOE_ERR_WORKSPACE = -6,  /* workspace too small */
  MOE_ERR_ALIGN = -7       /* a pointer is not aligned as required */
} moe_status;

/*
 * Layer sizes. T tokens, H hidden, N routed experts, K routed experts per
 * token, I intermediate size of every expert (routed and shared: the shared
 * expert has the routed experts' shape, "DeepSeek-V3, explained", step 3).
 * Supported: T >= 0 (T = 0 is an empty batch: the calls do no work, clear
 * the counts they output and accept NULL token-sized buffers); H a multiple
 * of 256; I a multiple of 128; N a multiple of 16 with 16 <= N <= 1024;
 * 1 <= K <= min(N, 16).
 *
 * G, M: node-limited routing ("DeepSeek-V3, explained", recipe step 5;
 * "DeepSeek-V3 Technical Report" (deepforge.srivtx.xyz), "Balancing without
 * a balance loss"). The routed experts form G contiguous groups of N/G (the
 * nodes holding them); a token's group score is the sum of its K/M highest
 * biased scores s_i + b_i inside the group, and its K experts are chosen only
 * from its M best groups (ties to the lower group id). G = 0 (or G = M)
 * routes over all N experts. Otherwise: 1 <= M <= G <= 32, N % G == 0,
 * K % M == 0 and K/M <= N/G.
 */
typedef struct {
  int32_t T, H, N, K, I;
  int32_t G, M;
} moe_shape;

/*
 * Layer weights (device, caller-owned). Group N (the last) is the shared
 * expert; groups 0..N-1 are the routed experts.
 *   gate_w [N, H]              float32 centroids e_i (gating stays in high
 *                              precision: "DeepSeek-V3, explained", step 7)
 *   w13    [N+1, 2I, H]        E4M3: for each 128-channel block c of the
 *                              intermediate size, 128 rows of W_gate
 *                              (channels 128c..128c+127) then the 128 rows
 *                              of W_up for the same channels
 *   s13    [N+1, 2I/128, H/128] float32 block scales of w13 (same row order)
 *   w2     [N+1, H, I]         E4M3 W_down
 *   s2     [N+1, H/128, I/128] float32 block scales of w2
 *   gate_split  optional (NULL: made on every call): bf16 [3, N, H], gate_w
 *               split exactly into three bf16 terms by moe_split_gate. The
 *               tensor-core router multiplies these; with them given,
 *               moe_forward skips the split. The caller re-splits whenever
 *               gate_w changes (after every optimiser step, in training).
 * w13 and w2 must be 16-byte aligned; gate_split 16-byte aligned.
 */
typedef struct {
  const float* gate_w;
  const uint8_t* w13;
  const float* s13;
  const uint8_t* w2;
  const float* s2;
  const void* gate_split;
} moe_weights;

/*
 * Byte offsets of the intermediates inside the forward workspace, for
 * inspection by tests and tools after moe_forward has completed. Rows of the
 * expert GEMMs ("GEMM rows") are laid out expert-major: routed expert e owns
 * rows [row_start[e], row_start[e] + counts[e]), row_start 128-aligned and
 * increasing in e; the shared expert owns rows [routed_cap, routed_cap + T)
 * in token order. Rows between segments are padding and hold no data.
 */
typedef struct {
  int64_t routed_cap;   /* first GEMM row of the shared expert (multiple of 128) */
  int64_t rows_total;   /* GEMM rows allocated (routed_cap + T rounded to 128) */
  size_t status;        /* uint32 status word (also at offset 0) */
  size_t counts;        /* int32 [N]: tokens routed to each expert (c_i) */
  size_t offsets;       /* int32 [N+1]: exclusive scan of counts */
  size_t group_rows;    /* int32 [N+1]: rows of each GEMM group (counts, then T) */
  size_t row_start;     /* int32 [N+1]: first GEMM row of each group */
  size_t row_token;     /* int32 [routed_cap]: token of each routed row, -1 on padding */
  size_t token_row;     /* int32 [T, K]: GEMM row of (token t, slot k) */
  size_t topk_ids;      /* int32 [T, K] (used when the caller passes none) */
  size_t topk_gates;    /* float [T, K] (used when the caller passes none) */
  size_t logits;        /* float [T, N] gate logits x . e_i */
  size_t a_q;           /* E4M3 [rows_total, H]: GEMM1 input rows; x_q in the shared rows
                           (before the rows are written, the router's partial
                           logits when it splits the gate GEMM's reduction) */
  size_t a_s;           /* float [rows_total, H/128] */
  size_t h_q;           /* E4M3 [rows_total, I]: SwiGLU output, 1x128 re-quantised */
  size_t h_s;           /* float [rows_total, I/128] */
  size_t y_rows;        /* bf16 [rows_total, H]: expert outputs before the combine */
  size_t gate_split;    /* bf16 [3, N, H]: the fp32 centroids as three bf16 terms */
  size_t bal_scratch;   /* moe_balance_stats scratch: float [T] token sums, then
                           float and int32 [T + ceil(T/128), N] chunk partials */
  size_t perm_scratch;  /* int32 [ceil(T/128), N]: the permutation's per-chunk
                           expert counts, then first rows */
  size_t total;         /* workspace bytes required */
} moe_ws_layout;

/*
 * Online 1x128 activation quantisation ("DeepSeek-V3 Technical Report",
 * deepforge.srivtx.xyz, "Per-tile FP8 scaling"; "DeepSeek-V3, explained",
 * step 7). For each row r and 128-column tile j:
 *   amax = max |x[r, 128j .. 128j+127]|,  scale = fp32(448 / amax) (1 if 0),
 *   q[r, c] = e4m3_rne_satfinite(fp32(x[r, c] * scale)).
 * x: bf16 [rows, cols]; q: uint8 [rows, cols]; scales: float [rows, cols/128].
 * cols must be a positive multiple of 128; x and q 16-byte aligned. rows = 0
 * is a no-op (the pointers may then be NULL).
 */
int moe_quantize_1x128(const void* x, int64_t rows, int64_t cols, uint8_t* q, float* scales,
                       void* stream);

/*
 * 128x128 weight block quantisation (same pages, same rule per block), for
 * preparing w13/w2 once at set-up. w: float [rows, cols]; q: uint8 [rows,
 * cols]; scales: float [rows/128, cols/128]. rows and cols positive multiples
 * of 128; w and q 16-byte aligned.
 */
int moe_quantize_128x128(const float* w, int64_t rows, int64_t cols, uint8_t* q, float* scales,
                         void* stream);

/*
 * The fp32 centroids as three bf16 terms, hi + mid + lo == gate_w exactly
 * (each term the bf16 rounding of what the previous ones leave), for
 * moe_weights.gate_split: gate_w float [N, H] -> gate_split bf16 [3, N, H]
 * (term-major). Done once at set-up, or after every change of gate_w.
 * Both 16-byte aligned; N >= 1, H >= 1.
 */
int moe_split_gate(const float* gate_w, int32_t N, int32_t H, void* gate_split, void* stream);

/* Workspace bytes needed by moe_route / moe_forward for `sh` (0 if invalid). */
size_t moe_workspace_size(moe_shape sh);

/* Fills *out with the workspace layout for `sh`. */
int moe_workspace_layout(moe_shape sh, moe_ws_layout* out);

/*
 * Routing ("DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing, ...",
 * section III equations for s, g' and g). Computes the fp32 gate logits,
 * sigmoid affinities, top-K of s + b (ties to the lower expert id; output
 * order biased score descending), the gates normalised from the unbiased
 * affinities, and the per-expert counts.
 *   gate_w: float [N, H]; x: bf16 [T, H]; bias: float [N]
 *   topk_ids: int32 [T, K]; topk_gates: float [T, K]; counts: int32 [N]
 *   ws: workspace of at least moe_workspace_size(sh) bytes, 256-byte aligned.
 */
int moe_route(moe_shape sh, const float* gate_w, const void* x, const float* bias,
              int32_t* topk_ids, float* topk_gates, int32_t* counts, void* ws, size_t ws_bytes,
              void* stream);

/*
 * Routing without a workspace. The pages have no counterpart to this entry
 * point: it exists for callers that cannot hand the library scratch memory,
 * such as a host application that owns every device allocation through its
 * own pool and does not let plug-in libraries allocate, or a latency-critical
 * loop where a cudaMalloc (which may synchronise the device) is not allowed.
 *
 * The same routing as moe_route, with two differences. The gate logits come
 * from an fp32 SIMT kernel rather than moe_route's split-bf16 tensor-core
 * kernel: both are fp32-accurate, so the ids, counts and gates agree with
 * moe_route's except on tokens whose K-th and (K+1)-th biased scores are
 * within about 1e-5 relative (near ties), and the gates within about 1e-6.
 * And the T x N gate logits live in a fixed array inside the library's
 * device memory: 4 MiB,
 * MOE_ROUTE_NOALLOC_MAX_LOGITS floats, present on every GPU that loads the
 * library until the process exits. Nothing is allocated; the caller passes
 * only inputs and outputs, as for moe_route. Returns MOE_ERR_WORKSPACE, before
 * enqueuing anything, when T * N exceeds MOE_ROUTE_NOALLOC_MAX_LOGITS.
 *
 * Every call looks up the array's device address on the current device
 * (cudaGetSymbolAddress, no allocation); the first call on a device also
 * loads the library's kernels there, so make it before any stream capture.
 * Every call uses the same array: calls whose work overlaps on the GPU (other
 * streams, other host threads on the same device) race on it, so the caller
 * must serialise them. The logits are fully rewritten by each call and
 * `counts` is zeroed by the call, so no earlier contents leak into a result.
 * Device status is not recorded (routing has no device-side checks).
 */
#define MOE_ROUTE_NOALLOC_MAX_LOGITS 1048576
int moe_route_noalloc(moe_shape sh, const float* gate_w, const void* x, const float* bias,
                      int32_t* topk_ids, float* topk_gates, int32_t* counts, void* stream);

/*
 * Backward of the expert path in FP8 ("DeepSeek-V3: Auxiliary-Loss-Free MoE
 * Load Balancing, Multi-Token Prediction, and FP8 Training at 671B Scale",
 * section V, Figure 6: Dgrad GEMMs in E4M3 with 1x128 activation tiles,
 * 128x128 weight blocks and fp32 accumulation). Gating stays in high
 * precision, so the router's backward is the caller's: it gets the gate
 * gradients.
 *
 * moe_transpose_weights: set-up for the backward. Writes each expert's W13
 * [2I, H] and W2 [H, I] codes transposed, and their 128x128 block scales
 * transposed with them (a block keeps its own scale, so these are the
 * quantised transposed weights):
 *   w13t E4M3 [N+1, H, 2I], s13t float [N+1, H/128, 2I/128]
 *   w2t  E4M3 [N+1, I, H],  s2t  float [N+1, I/128, H/128]
 * Caller-owned device buffers, 16-byte aligned.
 */
int moe_transpose_weights(moe_shape sh, const moe_weights* w, uint8_t* w13t, float* s13t,
                          uint8_t* w2t, float* s2t, void* stream);

/*
 * Bytes of the backward's own workspace (bws); 0 for a shape the backward
 * does not support (it needs I to be a multiple of 256 besides the forward's
 * rules).
 */
size_t moe_backward_workspace_size(moe_shape sh);

/*
 * Backward of the last moe_forward on `ws` (same x, weights and shape) for
 * the upstream gradient dy of its output, with the routing held fixed:
 *   dY rows    g[t,k] dy[t] for the routed slots, dy[t] for the shared expert,
 *              quantised 1x128 along H
 *   dh         = dY . W2 per expert (FP8 grouped GEMM on w2t), fp32
 *   [G | U]    recomputed from the forward's quantised x rows (w13), fp32
 *   dG, dU     = dh U silu'(G), dh silu(G), quantised 1x128
 *   dX rows    = dG . W_gate + dU . W_up per expert (FP8 grouped GEMM on w13t)
 *   dx[t]      = the sum of the token's K + 1 row gradients (shared first,
 *                then slots by ascending expert id), rounded once to bf16
 *   dgates[t,k] = dy[t] . Y_k[t] with the forward's bf16 expert output row
 *   dw2 [N+1, H, I] = per expert, dY^T . h over its rows (Wgrad), fp32
 *   dw13 [N+1, 2I, H] = per expert, [dG | dU]^T . x over its rows, in w13's
 *                row order (gate block c, then up block c), fp32
 * Wgrad operands are quantised in tiles of 128 GEMM rows x 1 channel (the
 * tiles run along the reduction, which is over tokens here), h and dG/dU
 * from the recomputed [G | U] and dh, x from the bf16 input.
 *   w: the forward's weights; wt: moe_transpose_weights' output in a
 *   moe_weights (w13 = w13t, s13 = s13t, w2 = w2t, s2 = s2t; gate_w unused)
 *   topk_ids, topk_gates: the forward's [T, K] outputs; x: its bf16 input
 *   (only read for the weight gradients; may be NULL without them)
 *   dy, dx: bf16 [T, H], 16-byte aligned; dgates: float [T, K]
 *   dw13, dw2: the weight gradients, or both NULL to skip them
 *   ws: the forward's workspace (read only, apart from its status word);
 *   bws: moe_backward_workspace_size(sh) bytes, 256-byte aligned.
 * Errors: MOE_ERR_SHAPE, MOE_ERR_NULL, MOE_ERR_ALIGN, MOE_ERR_WORKSPACE; device
 * checks in ws's status word (moe_get_status).
 */
int moe_backward(moe_shape sh, const moe_weights* w, const moe_weights* wt,
                 const int32_t* topk_ids, const float* topk_gates, const void* x, const void* dy,
                 void* ws, size_t ws_bytes, void* bws, size_t bws_bytes, void* dx, float* dgates,
                 float* dw13, float* dw2, void* stream);

/*
 * Complementary sequence-wise balance statistics ("DeepSeek-V3:
 * Auxiliary-Loss-Free MoE Load Balancing, Multi-Token Prediction, and FP8
 * Training at 671B Scale", section III; "DeepSeek-V3, explained", step 4),
 * for the routing that the last moe_route or moe_forward call on `ws` made.
 * The T tokens form S = ceil(T / seq_len) sequences of seq_len consecutive
 * tokens (the last may be shorter, T_s tokens). For sequence s and expert i:
 *   f[s, i] = N / (K * T_s) * #{(t, k) in s : topk_ids[t, k] = i}
 *   P[s, i] = (1 / T_s) * sum_{t in s} s_ti / sum_j s_tj   (all N affinities)
 *   loss[s] = alpha * sum_i f[s, i] * P[s, i]
 * with s_ti the router's sigmoid affinities (recomputed from the logits the
 * router left in ws; the call writes only the bal_scratch region of ws). Sums
 * run in a fixed order: results are reproducible.
 *   topk_ids: int32 [T, K] of that call; f, P: float [S, N]; loss: float [S]
 * Errors: MOE_ERR_SHAPE for a bad shape or seq_len < 1; MOE_ERR_NULL;
 * MOE_ERR_WORKSPACE if ws_bytes < moe_workspace_size(sh).
 */
int moe_balance_stats(moe_shape sh, int32_t seq_len, float alpha, void* ws, size_t ws_bytes,
                      const int32_t* topk_ids, float* f, float* P, float* loss, void* stream);

/*
 * The whole layer forward: quantise x (1x128), route, permute token rows by
 * expert (expert ascending, token ascending; no token dropped), grouped FP8
 * SwiGLU expert FFNs for the routed experts and the shared expert, and the
 * weighted combine y_t = Y_shared[t] + sum_k g[t,k] Y[row(t,k)] accumulated in
 * fp32 (shared first, then slots by ascending expert id) and rounded once to
 * bf16. No residual is added.
 *   w: weights (see moe_weights); x: bf16 [T, H]; bias: float [N]
 *   y: bf16 [T, H], 16-byte aligned
 *   topk_ids_opt, topk_gates_opt, counts_opt: optional outputs (may be NULL),
 *   shapes as in moe_route; counts_opt feeds moe_update_bias.
 *   ws: workspace of at least moe_workspace_size(sh) bytes, 256-byte aligned;
 *   its contents are valid until the next call that uses it.
 */
int moe_forward(moe_shape sh, const moe_weights* w, const void* x, const float* bias, void* y,
                int32_t* topk_ids_opt, float* topk_gates_opt, int32_t* counts_opt, void* ws,
                size_t ws_bytes, void* stream);

/*
 * moe_forward with stage timing: identical work and results, and in addition
 * records events[i] on `stream` before stage i and events[6] after the last:
 *   0 route, 1 permute (scan, scatter), 2 quantise x into the token's
 *   shared-expert and routed GEMM rows, 3 up/gate GEMM + SwiGLU +
 *   re-quantisation, 4 down GEMM, 5 combine.
 * events: MOE_TRACE_EVENTS cudaEvent_t handles created by the caller
 * (n_events >= MOE_TRACE_EVENTS, none NULL, else MOE_ERR_NULL).
 */
#define MOE_TRACE_EVENTS 7
int moe_forward_traced(moe_shape sh, const moe_weights* w, const void* x, const float* bias,
                       void* y, int32_t* topk_ids_opt, float* topk_gates_opt, int32_t* counts_opt,
                       void* ws, size_t ws_bytes, void* stream, void* const* events,
                       int32_t n_events);

/*
 * Aux-loss-free bias controller ("DeepSeek-V3: Auxiliary-Loss-Free MoE Load
 * Balancing, ...", section III "How the bias is set"; "DeepSeek-V3,
 * explained", step 4): b_i <- fp32(b_i + gamma * sign(T*K - N*c_i)), i.e. an
 * overloaded expert loses gamma, an underloaded one gains gamma, one exactly
 * at the mean load T*K/N keeps its bias. bias: float [N], updated in place;
 * counts: int32 [N]. gamma = 0 leaves the bias unchanged.
 */
int moe_update_bias(float* bias, const int32_t* counts, int32_t N, int32_t T, int32_t K,
                    float gamma, void* stream);

/*
 * Stage entry points: the grouped FP8 expert GEMMs alone, on caller-laid-out
 * rows ("DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing, ...", section
 * V "Four details", items 1-2: E4M3 operands, one scale per 1x128 activation
 * tile and 128x128 weight block, partial sums promoted to fp32 every 128
 * products). Group g (0 <= g < n_groups) uses weight set g and owns GEMM rows
 * [group_start[g], group_start[g] + group_rows[g]); group_start must be
 * multiples of 128, the segments must not overlap and must lie inside
 * [0, rows). group_rows and group_start are DEVICE int32 arrays [n_groups].
 * status_ws: a device uint32 status word (may be the forward workspace).
 *
 * moe_expert_up: per group, G = A_hat W_gate^T, U = A_hat W_up^T in fp32,
 *   h = silu(G) * U, h re-quantised 1x128.
 *   a_q [rows, H] E4M3, a_s [rows, H/128]; w13/s13 as in moe_weights with
 *   n_groups sets; h_q [rows, I] E4M3, h_s [rows, I/128].
 * moe_expert_down: per group, Y = h_hat W_down^T, written as the fp32
 *   totals (the accumulator before any output rounding; the backward's
 *   GEMMs use this form). h_q/h_s as above; w2/s2 as in moe_weights;
 *   y_rows float [rows, H].
 * moe_expert_down_bf16: the same GEMM as the layer runs it, each fp32 total
 *   rounded once to bf16 (round to nearest even): the FP8 GEMMs give BF16
 *   outputs ("DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing, ...",
 *   section V, Figure 6). Bit for bit the bf16 rounding of moe_expert_down's
 *   output. y_rows bf16 [rows, H].
 * Rows outside every segment are not written.
 */
int moe_expert_up(int32_t H, int32_t I, int32_t n_groups, const int32_t* group_rows,
                  const int32_t* group_start, int64_t rows, const uint8_t* a_q, const float* a_s,
                  const uint8_t* w13, const float* s13, uint8_t* h_q, float* h_s,
                  uint32_t* status_ws, void* stream);

int moe_expert_down(int32_t H, int32_t I, int32_t n_groups, const int32_t* group_rows,
                    const int32_t* group_start, int64_t rows, const uint8_t* h_q,
                    const float* h_s, const uint8_t* w2, const float* s2, void* y_rows,
                    uint32_t* status_ws, void* stream);

int moe_expert_down_bf16(int32_t H, int32_t I, int32_t n_groups, const int32_t* group_rows,
                         const int32_t* group_start, int64_t rows, const uint8_t* h_q,
                         const float* h_s, const uint8_t* w2, const float* s2, void* y_rows,
                         uint32_t* status_ws, void* stream);

/*
 * Expert parallelism ("DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing,
 * Multi-Token Prediction, and FP8 Training at 671B Scale", section V,
 * "Training at Scale" and "Custom all-to-all kernels"; "DeepSeek-V3,
 * explained", recipe step 8). The layer runs on W ranks (1 <= W <= 16, one GPU
 * each, N % W == 0, N/W a multiple of 16 and >= 16). Rank d holds routed
 * experts [d N/W, (d+1) N/W) plus the shared expert, as a moe_weights with
 * El + 1 = N/W + 1 weight sets (its El experts in order, then the shared
 * expert), and the whole gate gate_w [N, H]. Every rank routes its own T
 * tokens. A token travels once to each rank that holds one of its experts,
 * as one packed FP8 row:
 *   [codes: H bytes][scales: H/128 float][local ids: K int32][gates: K float]
 * padded to moe_ep_row_bytes(sh) (a multiple of 16). Local id k is the
 * expert's index on the destination (-1: slot k's expert is elsewhere; its
 * gate is then 0). A step, on every rank:
 *   1. moe_ep_dispatch: route, then fill `send` with this rank's rows,
 *      destination-major (rank 0's rows first), tokens ascending within each
 *      destination; send_counts[2d] = rows for rank d, send_counts[2d+1] =
 *      (token, slot) pairs for rank d.
 *   2. the caller exchanges send_counts (an all-to-all of 2 int32 per pair of
 *      ranks) and then the rows (an all-to-all with those row counts); the
 *      received rows are source-major. moe_ep_shared may run meanwhile.
 *   3. moe_ep_experts on the received rows: out[j] = sum over row j's local
 *      slots, by ascending expert id, of gate * expert(x_j), fp32 [R, H].
 *   4. the caller sends each `out` row back to its source (the reverse
 *      all-to-all), which then holds them in its send order.
 *   5. moe_ep_combine: y_t = shared_t + sum over the token's destination
 *      ranks, ascending, of the returned rows (fp32), rounded once to bf16.
 * The quantisation, GEMMs and gates are the single-GPU layer's, so each
 * expert output matches moe_forward's; only the order of the fp32 additions
 * in the combine differs. Device checks go to the status word at the start
 * of the workspace used (moe_get_status).
 */

/* Bytes of one packed dispatch row (0 for an invalid shape). */
int64_t moe_ep_row_bytes(moe_shape sh);

/* Workspace of moe_ep_dispatch / moe_ep_shared / moe_ep_combine (0 if the
 * shape or W is not supported). */
size_t moe_ep_dispatch_workspace_size(moe_shape sh, int32_t W);

/*
 * Step 1. gate_w: float [N, H]; gate_split_opt: NULL, or gate_w's three bf16
 * terms [3, N, H] made by moe_split_gate (16-byte aligned; NULL: they are made
 * on every call); x: bf16 [T, H]; bias: float [N]. Optional outputs as in
 * moe_forward (topk_ids and topk_gates [T, K] with global expert
 * ids; counts [N] of this rank's tokens, for moe_update_bias after a sum over
 * ranks). send: uint8 [send_cap, moe_ep_row_bytes], 16-byte aligned
 * (T * min(W, K) rows always suffice; a row beyond send_cap is dropped and
 * flagged). send_counts: int32 [W, 2] device. ws: the source workspace,
 * 256-byte aligned; it keeps the send slots and the shared-expert rows for
 * steps 1b and 5. T = 0 clears send_counts and counts only.
 */
int moe_ep_dispatch(moe_shape sh, int32_t W, const float* gate_w, const void* gate_split_opt,
                    const void* x, const float* bias,
                    int32_t* topk_ids_opt, float* topk_gates_opt, int32_t* counts_opt,
                    uint8_t* send, int64_t send_cap, int32_t* send_counts, void* ws,
                    size_t ws_bytes, void* stream);

/* Step 1b: the shared expert on this rank's tokens (after moe_ep_dispatch on
 * the same ws), fp32 rows kept in ws for moe_ep_combine. w_local: this rank's
 * weights (El + 1 sets); gate_w is not read. */
int moe_ep_shared(moe_shape sh, int32_t W, const moe_weights* w_local, void* ws, size_t ws_bytes,
                  void* stream);

/* Workspace of moe_ep_experts for R received rows holding `pairs` slots with
 * a local expert (0 if unsupported, or pairs > R K). */
size_t moe_ep_expert_workspace_size(moe_shape sh, int32_t W, int64_t R, int64_t pairs);

/*
 * Step 3. recv: R packed rows, 16-byte aligned; pairs: the sum of the
 * received send_counts[2d+1] (checked on the device against the rows). out:
 * float [R, H], 16-byte aligned. w_local: this rank's weights; gate_w is not
 * read. ws: moe_ep_expert_workspace_size(sh, W, R, pairs) bytes, 256-byte
 * aligned. R = 0 does nothing.
 */
int moe_ep_experts(moe_shape sh, int32_t W, const moe_weights* w_local, const uint8_t* recv,
                   int64_t R, int64_t pairs, float* out, void* ws, size_t ws_bytes, void* stream);

/* Step 5. ret: float [ret_rows, H], the returned rows in this rank's send
 * order (ret_rows = its total send rows); ws: the workspace of its
 * moe_ep_dispatch and moe_ep_shared; y: bf16 [T, H], 16-byte aligned. */
int moe_ep_combine(moe_shape sh, int32_t W, const float* ret, int64_t ret_rows, void* ws,
                   size_t ws_bytes, void* y, void* stream);

/*
 * Peer mode: the same steps without the two row all-to-alls and without any
 * host synchronisation. The kernels move the rows themselves, with plain
 * stores to the other ranks' buffers over NVLink/NVSwitch, so
 * moving the data overlaps computing it. Every rank owns, in its own memory:
 *   recv   uint8 [W * T_cap, row_bytes]  receive buffer: segment s (rows
 *          s*T_cap ..) holds the rows source s sends to this rank;
 *   counts int32 [W]  counts[s] = rows source s wrote into its segment;
 *   ret    float [W * T_cap, H]  return buffer: segment d holds the partial
 *          sums rank d sends back for this rank's rows.
 * The calls take DEVICE arrays of W pointers to those buffers on every rank
 * (peer_recv[d], peer_counts[d], peer_ret[s]), mapped into this process
 * (CUDA IPC or symmetric memory); index `rank` is the caller's own. T_cap
 * (>= every rank's T) is the same on all ranks. Order of a step, every rank:
 *   moe_ep_dispatch_peer  (writes rows, ids, gates and its count into peers)
 *   barrier               (e.g. a stream-ordered all-reduce of one int)
 *   moe_ep_shared, moe_ep_experts_peer (writes partials into the sources)
 *   barrier
 *   moe_ep_combine_peer
 * The kernels end their remote writes with a system-scope fence; the
 * barriers order every rank's writes before any rank reads them, and the
 * next step's writes after this step's reads. No kernel waits on another
 * rank.
 */
size_t moe_ep_peer_expert_workspace_size(moe_shape sh, int32_t W, int32_t T_cap);

int moe_ep_dispatch_peer(moe_shape sh, int32_t W, int32_t rank, int32_t T_cap,
                         const float* gate_w, const void* gate_split_opt, const void* x,
                         const float* bias, int32_t* topk_ids_opt, float* topk_gates_opt,
                         int32_t* counts_opt, uint8_t* const* peer_recv,
                         int32_t* const* peer_counts, int32_t* send_counts_opt, void* ws,
                         size_t ws_bytes, void* stream);

/* recv, recv_counts: this rank's own buffers; peer_ret: device array [W] of
 * the ranks' return buffers; ws: moe_ep_peer_expert_workspace_size bytes. */
int moe_ep_experts_peer(moe_shape sh, int32_t W, int32_t rank, int32_t T_cap,
                        const moe_weights* w_local, const uint8_t* recv,
                        const int32_t* recv_counts, float* const* peer_ret, void* ws,
                        size_t ws_bytes, void* stream);

/* ret: this rank's own return buffer; ws: its dispatch workspace. */
int moe_ep_combine_peer(moe_shape sh, int32_t W, int32_t T_cap, const float* ret, void* ws,
                        size_t ws_bytes, void* y, void* stream);

/*
 * Synchronises `stream`, reads and clears the device status word at the
 * start of `ws` (a forward workspace or a bare uint32 status word). Returns
 * MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_BOUNDS (timeout reported first), or
 * MOE_ERR_CUDA if the stream reports an error.
 */
int moe_get_status(void* ws, void* stream);

/* Number of streaming multiprocessors of the current device (0 on error). */
int moe_device_sm_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_CAPI_H */
