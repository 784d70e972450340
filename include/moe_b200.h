/*
 * moe_b200.h — C ABI of the B200 (sm_100a) forward pass of one Mixture-of-Experts layer.
 *
 * The layer (router -> permute -> grouped expert FFN -> combine) is the one the
 * following pages describe; each entry point cites the passage that defines it:
 *   [P2] "MoE模型高效推理：CANN算子库优化实践" (intelliparadigm.com)
 *   [P3] "ops-transformer 仓库 - MoE 算子优化实战" (gitcode.csdn.net)
 *   [P4] lshu.cn/news/82007: calling the MoE fused operators through torch_npu
 *   [P1] hnwysp.cn/news/132341: ops-transformer MoE operator optimisation
 *   [P5] "ops-transformer 算子精讲：昇腾 NPU 上的注意力机制与融合算子实现" (mhpn.cn)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Ownership: the caller allocates and frees every buffer.  The library never
 *   allocates device memory; scratch comes from a caller-provided workspace
 *   `ws` of at least moe_workspace_bytes(...) bytes (256-byte aligned).  The
 *   one exception is moe_permute_noalloc: it takes no workspace, keeps its
 *   scratch in library-owned device memory and reports kernel-found errors
 *   only through its status_out argument.
 * Pointers: device pointers unless stated otherwise, 16-byte aligned.
 * Layouts: dense row-major.  x[T,H]; w_gate[H,E]; w1,w3[E,H,F]; w2[E,F,H];
 *   topk_idx / topk_gate / row_map [T,top_k]; x_perm, y [rows,H]; h [rows,F].
 *   T tokens, H hidden, F expert intermediate size, E experts.
 * Element type: MOE_BF16 (bf16 storage, fp32 accumulation, tensor cores) or
 *   MOE_F32 (fp32 storage and arithmetic on CUDA cores, no TF32).
 * Asynchrony: every call is enqueued on `stream` and returns at once.
 *   Argument errors are detected on the host and returned before any launch.
 *   Errors found by kernels (an expert id outside [0,E), a pipeline wait that
 *   timed out) are written to a status word at the start of `ws`; read it with
 *   moe_get_device_status().
 * Limits: 1 <= top_k <= 8, top_k <= E <= 256, H and F multiples of 8,
 *   T*top_k*max(H,F) < 2^31.  Violations return MOE_ERR_INVALID_ARG or
 *   MOE_ERR_UNSUPPORTED.
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
  MOE_ERR_INVALID_ARG = 1,         /* null/misaligned pointer, bad size or enum          */
  MOE_ERR_INDEX_OUT_OF_RANGE = 2,  /* an expert id outside [0,E) ([P4] §5.2, §7)          */
  MOE_ERR_WORKSPACE = 3,           /* ws smaller than moe_workspace_bytes()               */
  MOE_ERR_UNSUPPORTED = 4,         /* sizes outside the limits above                      */
  MOE_ERR_CUDA = 5,                /* a CUDA runtime or driver call failed                */
  MOE_ERR_TIMEOUT = 6,             /* a kernel's bounded pipeline wait ran out            */
  MOE_ERR_BOUNDS = 7               /* debug build only: an internal index fell outside its
                                      buffer; the access was skipped (see below)           */
} moe_status;

/* Debug build.  libmoe_b200_debug.so is the same library compiled with
 * MOE_DEBUG: before the accesses they guard, kernels check internal indices
 * (scatter destination rows, router expert ids, combine rows against the
 * T x k rows of y, grouped-GEMM tiles against the output and the K-split
 * areas); a failed check records MOE_ERR_BOUNDS in the status word and skips
 * the access instead of trapping.  Results are otherwise identical.
 * Logging.  With MOE_LOG=1 in the environment when the library loads, every
 * call prints its launch plan (kernel, grid, tiles, splits) to stderr.      */

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

typedef enum {
  MOE_ACT_SWIGLU = 0,   /* h = silu(x W1) * (x W3)                                        */
  MOE_ACT_GELU = 1,     /* h = gelu(x W1), exact erf form; w3 unused                      */
  MOE_ACT_IDENTITY = 2  /* test experts: y = x (weights unused)                           */
} moe_act;

typedef void* moe_stream_t;  /* a cudaStream_t; NULL = the legacy default stream */

/* Bytes of workspace that every entry point below needs for these sizes
 * (the fused moe_forward needs the most; one size serves every call).  For
 * bf16 layers it includes 40 MiB of fp32 partial sums and 16 KiB of tickets
 * with which the SwiGLU expert GEMM cuts its last partial wave of tiles in
 * two along K (results deterministic; see moe_forward).                    */
size_t moe_workspace_bytes(int T, int H, int F, int E, int top_k, moe_act act, moe_dtype dt);

/* Router.  [P2] §2.1 (gates = softmax(x @ W_gate), top_k(gates, k=2)), §3.2.1
 * (renormalise the kept experts); [P5] ch.8 (normalize_scores=True).
 *   logits[t,e] = sum_h x[t,h] W_gate[h,e] + gate_bias[e]   (fp32 accumulate)
 *   topk_idx[t,0..k-1]: the k largest logits, slot 0 the largest; ties go to the
 *     lower expert id; NaN ranks below -inf.
 *   topk_gate[t,s] = exp(l_s - l_0) / sum_j exp(l_j - l_0) over the k selected
 *     (softmax over all E renormalised over the top-k).
 * gate_bias (fp32 [E]) and logits_out (fp32 [T,E]) may be NULL.           */
moe_status moe_route(const void* x, const void* w_gate, const float* gate_bias,
                     int T, int H, int E, int top_k, moe_dtype dt,
                     int32_t* topk_idx, float* topk_gate, float* logits_out,
                     moe_stream_t stream);

/* Selection and gates only, from caller-given fp32 logits [T,E]; same rules as
 * moe_route.  Lets a caller check selection on identical logits.           */
moe_status moe_route_from_logits(const float* logits, int T, int E, int top_k,
                                 int32_t* topk_idx, float* topk_gate, moe_stream_t stream);

/* Permute / dispatch.  [P4] §4 (npu_moe_token_preprocess: token rearrangement),
 * §5.2 (int32 expert ids in [0,E)), §5.3 (fixed per-expert buffer); [P1] §3.2
 * (capacity_factor); [P3] SparseGather.
 *   expert_counts[e]  (pre-drop) = #{(t,s): token_expert_idx[t,s] = e}
 *   C = ceil(capacity_factor * T * top_k / E); no limit when capacity_factor <= 0
 *   Pairs (t,s) are walked in token order, then slot order; a pair is kept when
 *   fewer than C pairs of its expert were kept before it.
 *   expert_offsets[E+1]: exclusive prefix sum of kept counts; R = offsets[E].
 *   Kept pair (t,s) of expert e goes to row offsets[e] + (its arrival rank):
 *     row_token[row] = t, row_map[t,s] = row; dropped pairs get row_map = -1.
 *   x_perm (optional, [T*top_k,H]): x_perm[row] = x[row_token[row]].
 * Out-of-range ids are not clamped: they count as dropped and the device
 * status becomes MOE_ERR_INDEX_OUT_OF_RANGE.  x may be NULL when x_perm is.
 * row_token must hold T*top_k entries (only the first R are written).      */
moe_status moe_permute(const void* x, const int32_t* token_expert_idx,
                       int T, int H, int E, int top_k, float capacity_factor, moe_dtype dt,
                       void* x_perm, int32_t* expert_counts, int32_t* expert_offsets,
                       int32_t* row_token, int32_t* row_map,
                       void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_permute for callers that cannot allocate device memory (no counterpart on
 * the pages: it exists for hosts such as an engine plugin that must run on
 * memory planned before the model starts, or a serving process that reserved
 * its whole device budget up front, where neither cudaMalloc nor a caller
 * workspace is available).  Same inputs, outputs and results as moe_permute,
 * but its scratch (status word + per-tile expert histogram) lives in a 1 MiB
 * array of device memory owned by the library, held by every GPU that loads
 * the library until exit.  Limit: ceil(T/128) * E <= 262080, else
 * MOE_ERR_UNSUPPORTED before any launch.  status_out (device int32, nullable)
 * receives MOE_OK or the first kernel-detected error (MOE_ERR_INDEX_OUT_OF_RANGE);
 * when NULL such errors are not reported (the pairs are still dropped).  All
 * calls on a device share the array: calls whose kernels overlap on the GPU
 * (e.g. two unordered streams) race.  The first call on a device looks up the
 * array's device address with that device current; make it before any stream
 * capture.  Allocates nothing (no cudaMalloc/cudaFree).                     */
moe_status moe_permute_noalloc(const void* x, const int32_t* token_expert_idx,
                               int T, int H, int E, int top_k, float capacity_factor,
                               moe_dtype dt, void* x_perm, int32_t* expert_counts,
                               int32_t* expert_offsets, int32_t* row_token, int32_t* row_map,
                               int32_t* status_out, moe_stream_t stream);

/* Grouped expert FFN.  [P4] §3 (x times expert_weight[num_experts, hidden,
 * intermediate], then activation and down-projection), §4 (npu_moe_matmul);
 * [P1] §2.2 (one batched GEMM instead of one launch per expert).
 * For every expert e and row r in [offsets[e], offsets[e+1]):
 *   a_r = x_perm[r]            when row_token == NULL
 *       = x[row_token[r]]      otherwise (rows gathered on the fly; x_perm unused)
 *   h_r = act(a_r W1[e] [, a_r W3[e]])  rounded to dt
 *   y_r = h_r W2[e]                     rounded to dt
 * T is the row count of x (for the gathered form).  y has R_max >= R rows;
 * rows >= R are not written.  R is read on the device from expert_offsets[E]
 * (no host synchronisation).  h lives in ws, after a 256-byte status block:
 * the call needs 256 + R_max * F * sizeof(dt) bytes (MOE_ERR_WORKSPACE
 * below that; 256 for MOE_ACT_IDENTITY).  moe_grouped_ffn_workspace_bytes
 * returns a size with room for two optional parts, used when ws_bytes covers
 * them: (1) with row_token, bf16 and gathered != 0, the rows copied into
 * expert order, after which the dense kernel runs (faster than gathering
 * four rows per TMA request inside the GEMM); a row_token entry outside
 * [0, T) is then reported as MOE_ERR_INVALID_ARG through the device status
 * and its row skipped; (2) for bf16, fp32 partial sums (40 MiB) and tickets
 * that let the GEMMs cut their last partial wave of tiles along K.         */
size_t moe_grouped_ffn_workspace_bytes(int R_max, int H, int F, moe_act act, moe_dtype dt,
                                       int gathered);
moe_status moe_grouped_ffn(const void* x_perm, const int32_t* row_token, const void* x,
                           const void* w1, const void* w3, const void* w2,
                           const int32_t* expert_offsets, int R_max, int T, int H, int F,
                           int E, moe_act act, moe_dtype dt, void* y,
                           void* ws, size_t ws_bytes, moe_stream_t stream);

/* Deterministic weighted combine.  [P2] §2.1 (sum of gate-weighted expert
 * outputs); [P3] SparseScatterAdd; [P4] §4 (npu_moe_token_postprocess).
 *   out[t] = sum_{s=0..k-1, row_map[t,s] >= 0} topk_gate[t,s] * y[row_map[t,s]]
 * summed in slot order in fp32 and rounded once to dt; no atomics, so the
 * result is bit-identical from run to run.  topk_gate may be NULL: every
 * weight is 1, and with top_k = 1 the call is a plain row gather
 * out[t] = y[row_map[t,0]] (exact; zero where row_map is -1).  Every
 * row_map entry must be -1 or a row of y: the call does not know y's row
 * count and does not check (the debug build checks entries against T x k,
 * the row count moe_permute produces, and skips the others).               */
moe_status moe_unpermute_combine(const void* y, const float* topk_gate, const int32_t* row_map,
                                 int T, int H, int top_k, moe_dtype dt, void* out,
                                 moe_stream_t stream);

/* The whole layer: route -> permute -> grouped FFN -> combine, enqueued on one
 * stream with no host synchronisation.  [P3] MoEOperator::Forward; [P5] ch.8
 * moe_router(x, router_weight, expert_weights, top_k, normalize_scores=True,
 * capacity_factor); [P4] §1 (fusing permute, matmul, softmax, experts, combine).
 * topk_idx_out [T,k] and expert_counts_out [E] (pre-drop) may be NULL.
 * Results are the same bit for bit on every run of the same inputs on the
 * same GPU model.  The SwiGLU GEMM may add the two K halves of its last
 * partial wave of tiles in fp32 (which tiles depends on the expert counts and
 * the SM count), so two layers whose routing differs may round a token's
 * output differently in the last bit; the tolerance against exact arithmetic
 * is unchanged.                                                            */
moe_status moe_forward(const void* x, const void* w_gate, const float* gate_bias,
                       const void* w1, const void* w3, const void* w2,
                       int T, int H, int F, int E, int top_k, float capacity_factor,
                       moe_act act, moe_dtype dt, void* out,
                       int32_t* topk_idx_out, int32_t* expert_counts_out,
                       void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_forward that also records CUDA events at its stage boundaries, for
 * measuring each kernel of the fused path on the stream it runs on.
 * events: n_events (>= 7) cudaEvent_t handles; events[i] is recorded before
 * stage i and events[6] after the last: route (0-1), offsets scan (1-2;
 * empty: the scan runs inside the scatter kernel), scatter (2-3), expert
 * GEMM-1 (3-4), expert GEMM-2 (4-5), combine (5-6).  A NULL entry is not
 * recorded; an event between two kernels ends their programmatic-launch
 * overlap, so recording fewer boundaries perturbs the timing less.          */
moe_status moe_forward_timed(const void* x, const void* w_gate, const float* gate_bias,
                             const void* w1, const void* w3, const void* w2,
                             int T, int H, int F, int E, int top_k, float capacity_factor,
                             moe_act act, moe_dtype dt, void* out,
                             void* ws, size_t ws_bytes, moe_stream_t stream,
                             void* const* events, int n_events);

/* moe_forward with x and out in HOST memory (page-locked for asynchronous
 * copies): copies x into the workspace, runs the layer, copies out back, all on
 * `stream`.  The caller synchronises the stream before reading out_host.
 * ws must hold moe_forward_host_workspace_bytes(...) bytes.                 */
size_t moe_forward_host_workspace_bytes(int T, int H, int F, int E, int top_k, moe_act act,
                                        moe_dtype dt);
moe_status moe_forward_host(const void* x_host, const void* w_gate, const float* gate_bias,
                            const void* w1, const void* w3, const void* w2,
                            int T, int H, int F, int E, int top_k, float capacity_factor,
                            moe_act act, moe_dtype dt, void* out_host,
                            void* ws, size_t ws_bytes, moe_stream_t stream);

/* A run of n_batches independent layer forwards, batch i reading x_host[i]
 * [T, H] and writing out_host[i] [T, H] (both in HOST memory, page-locked for
 * the copies to overlap; the pointers may repeat, e.g. a ring of buffers).
 * Each batch is one moe_forward of its own T tokens (its own capacity, its
 * own drops); the weights are shared.  Batch i's host-to-device copy runs on
 * copy_in, its layer on stream and its device-to-host copy on copy_out, over
 * two device stages of x and two of out used in turn, so the copy-in of batch
 * i+1 and the copy-out of batch i-1 overlap the layer of batch i.  Null
 * copy streams mean `stream` (no overlap; the same results).  All work is
 * ordered after what is already queued on `stream`, and `stream` is ordered
 * after all of it on return: synchronise `stream` before reading out_host.
 * ws must hold
 * moe_forward_host_batches_workspace_bytes(...) bytes (the moe_forward
 * workspace plus four T x H stages).  Errors as moe_forward, all detected
 * before anything is queued; creates and destroys seven CUDA events (no
 * device allocation).                       */
size_t moe_forward_host_batches_workspace_bytes(int T, int H, int F, int E, int top_k,
                                                moe_act act, moe_dtype dt);
moe_status moe_forward_host_batches(const void* const* x_host, void* const* out_host,
                                    int n_batches, const void* w_gate, const float* gate_bias,
                                    const void* w1, const void* w3, const void* w2,
                                    int T, int H, int F, int E, int top_k,
                                    float capacity_factor, moe_act act, moe_dtype dt,
                                    void* ws, size_t ws_bytes, moe_stream_t stream,
                                    moe_stream_t copy_in, moe_stream_t copy_out);

/* Router load statistics.  [P3] "实战中的坑与解法" (track each expert's load)
 * and [P4] §5.3 name an auxiliary load-balancing loss (--moe-aux-loss-coeff)
 * but not its formula, so the
 * router's two per-expert statistics are returned instead of a loss:
 *   expert_counts[e] (int32, pre-drop) = #{(t,s): topk_idx[t,s] = e}
 *   prob_mean[e]     (fp32)            = (1/T) sum_t softmax_e(logits[t])
 * with the softmax over all E experts of the fp32 logits moe_route computes
 * (bias included).  Also writes topk_idx / topk_gate exactly as moe_route.
 * Both sums run in a fixed order: bit-identical from run to run.  Runs the
 * router without splitting H across CTAs.  ws: device scratch of at least
 * moe_route_stats_workspace_bytes(T, E) bytes (256-byte aligned); errors as
 * moe_route, plus MOE_ERR_WORKSPACE.                                        */
size_t moe_route_stats_workspace_bytes(int T, int E);
moe_status moe_route_stats(const void* x, const void* w_gate, const float* gate_bias,
                           int T, int H, int E, int top_k, moe_dtype dt,
                           int32_t* topk_idx, float* topk_gate,
                           int32_t* expert_counts, float* prob_mean,
                           void* ws, size_t ws_bytes, moe_stream_t stream);

/* Per-token expert matmul with one expert per token (top_k = 1, up-projection
 * only, no activation).  [P4] §3: x[tokens, hidden], expert_weight[num_experts,
 * hidden, intermediate] and int32 token_expert_idx[tokens] in, [tokens,
 * intermediate] out; §5.2: ids outside [0, E) are errors, not clamped.
 *   out[t] = x[t] @ expert_weight[token_expert_idx[t]]   rounded once to dt
 * out is [T, I] (I = intermediate size, a multiple of 8).  The tokens are
 * rearranged by expert (the permute step, no capacity limit), multiplied by
 * the grouped GEMM and put back in token order.  A token whose id is outside
 * [0, E) gets a zero row in out and the device status becomes
 * MOE_ERR_INDEX_OUT_OF_RANGE.  ws: device scratch of at least
 * moe_expert_matmul_workspace_bytes(T, H, I, E, dt) bytes.                   */
size_t moe_expert_matmul_workspace_bytes(int T, int H, int I, int E, moe_dtype dt);
moe_status moe_expert_matmul(const void* x, const void* expert_weight,
                             const int32_t* token_expert_idx, int T, int H, int I, int E,
                             moe_dtype dt, void* out, void* ws, size_t ws_bytes,
                             moe_stream_t stream);

/* Threshold gating (a variable number of experts per token).  [P2] §3.2.1:
 * compute every expert's gate score (softmax over all E of the logits, §2.1),
 * keep only the experts whose score exceeds delta (default 1/E), renormalise
 * the kept ones.  Readings where the page is silent: kept experts are ordered
 * largest first (ties to the lower id); at most k_max are kept (1 <= k_max <=
 * min(8, E), the caller's slot count); when none exceeds delta the largest
 * alone is kept.  delta <= 0 selects the default 1/E.
 *   topk_idx [T,k_max]: kept ids, then -1;  topk_gate [T,k_max]: renormalised
 *   gates exp(l_s - l_0) / sum_kept exp(l_j - l_0), then 0;
 *   n_selected [T]: number kept;  token_offsets [T+1] (nullable): exclusive
 *   prefix sum of n_selected, the CSR row offsets of the selection.
 * moe_threshold_select starts from caller-given fp32 logits [T,E] (parity
 * hook, like moe_route_from_logits).                                        */
moe_status moe_threshold_select(const float* logits, int T, int E, int k_max, float delta,
                                int32_t* topk_idx, float* topk_gate, int32_t* n_selected,
                                int32_t* token_offsets, moe_stream_t stream);

/* The whole layer with threshold gating: router logits -> threshold selection
 * (as above) -> permute (slots with id -1 are unused, not errors; capacity
 * C = ceil(capacity_factor * T * k_max / E)) -> grouped FFN -> combine over
 * each token's kept slots.  topk_idx_out [T,k_max] and n_selected_out [T] may
 * be NULL.  ws: at least moe_forward_threshold_workspace_bytes(...) bytes.   */
size_t moe_forward_threshold_workspace_bytes(int T, int H, int F, int E, int k_max, moe_act act,
                                             moe_dtype dt);
moe_status moe_forward_threshold(const void* x, const void* w_gate, const float* gate_bias,
                                 const void* w1, const void* w3, const void* w2,
                                 int T, int H, int F, int E, int k_max, float delta,
                                 float capacity_factor, moe_act act, moe_dtype dt, void* out,
                                 int32_t* topk_idx_out, int32_t* n_selected_out,
                                 void* ws, size_t ws_bytes, moe_stream_t stream);

/* Self-test hook (no counterpart on the pages): applies, elementwise to fp32
 * z[n] on the device, the activations the bf16 expert-GEMM epilogue uses
 * before rounding h to bf16 — GELU z Phi(z) with Phi(z) = erfc(-z/sqrt 2)/2
 * and erfc from the Numerical Recipes (2nd ed., section 6.2) Chebyshev fit
 * (fractional error below 1.2e-7), and SiLU z / (1 + e^-z) with the hardware
 * exponential and reciprocal — so tests can bound their error against exact
 * values.  The fp32 path uses erfcf / expf.                                  */
moe_status moe_selftest_epilogue_activations(const float* z, int n, float* gelu_out,
                                             float* silu_out, moe_stream_t stream);

/* Self-test hook (no counterpart on the pages): one kernel whose bounded
 * pipeline wait can never be satisfied.  The wait gives up after its limit
 * (1 s) and records MOE_ERR_TIMEOUT in the status word at the start of ws (at
 * least 256 bytes) — the path every tcgen05 kernel takes when a TMA or MMA
 * completion never arrives — and the kernel returns, leaving the context
 * usable.  Read the result with moe_get_device_status().                    */
moe_status moe_selftest_bounded_wait(void* ws, moe_stream_t stream);

/* Where the fused forward (moe_forward, moe_forward_timed,
 * moe_forward_threshold) leaves its intermediates inside ws, for tests and
 * tools that read them after the call has completed (no counterpart on the
 * pages).  For the given sizes, writes the byte offset of section `which`
 * from the start of ws and its size in bytes.  Contents once the forward has
 * completed, valid until ws is reused:
 *   MOE_WS_TOPK_IDX   int32 [T,k]   (only when topk_idx_out was NULL)
 *   MOE_WS_TOPK_GATE  fp32  [T,k]
 *   MOE_WS_COUNTS     int32 [E]     pre-drop (only when expert_counts_out was NULL)
 *   MOE_WS_OFFSETS    int32 [E+1]   post-drop exclusive prefix, R = offsets[E]
 *   MOE_WS_ROW_TOKEN  int32 [T*k]   first R entries written
 *   MOE_WS_ROW_MAP    int32 [T,k]   -1 = dropped
 *   MOE_WS_X_PERM     dt    [T*k,H] first R rows written (bf16 only)
 *   MOE_WS_H          dt    [T*k,F] first R rows written
 *   MOE_WS_Y          dt    [T*k,H] first R rows written
 * Returns MOE_ERR_INVALID_ARG for bad sizes, enums or null outputs.          */
typedef enum {
  MOE_WS_TOPK_IDX = 0,
  MOE_WS_TOPK_GATE = 1,
  MOE_WS_COUNTS = 2,
  MOE_WS_OFFSETS = 3,
  MOE_WS_ROW_TOKEN = 4,
  MOE_WS_ROW_MAP = 5,
  MOE_WS_X_PERM = 6,
  MOE_WS_H = 7,
  MOE_WS_Y = 8
} moe_ws_section;
moe_status moe_workspace_section(int T, int H, int F, int E, int top_k, moe_act act,
                                 moe_dtype dt, moe_ws_section which, size_t* offset,
                                 size_t* bytes);

/* Tuning hook (no counterpart on the pages): selects the bf16 grouped-GEMM
 * kernel for the calls that follow, process-wide, so tests and benchmarks can
 * run each one.  0 = automatic (the default, or MOE_GEMM_VARIANT read once
 * when the library loads); 1 = row tiles of 128 rows, one CTA each; 2 = row
 * tiles of 256 rows on CTA pairs; 3 = token-as-N tiles on CTA pairs (the
 * tokens of an expert as the MMA's N; dense A rows only, gathered rows use
 * the automatic choice); 4 = the same without cutting the last partial
 * wave of tiles along K.  Returns MOE_ERR_INVALID_ARG for other values.
 * Not synchronised with calls running on other host threads.               */
moe_status moe_set_gemm_variant(int variant);

/* Synchronises `stream`, then returns the status the kernels of the last
 * call(s) on this workspace recorded (MOE_OK when none), and clears it.      */
moe_status moe_get_device_status(void* ws, moe_stream_t stream);

/* A constant string naming the status code. */
const char* moe_status_string(moe_status s);

/* Library build tag (architecture and version). */
const char* moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
