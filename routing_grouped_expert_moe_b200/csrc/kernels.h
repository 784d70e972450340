// Internal launch interfaces between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

constexpr int kMaxE = 256;
constexpr int kMaxTopK = 8;

// ---------------------------------------------------------------- tuning
// Measurement aids, read from the environment once when the library is loaded
// (never on a launch path).  The defaults are the product configuration.
struct Tuning {
  bool pdl = true;              // MOE_PDL=0: launch without programmatic dependent launch
  int gemm_variant = 0;         // MOE_GEMM_VARIANT=1|2|3: the initial grouped-GEMM choice
  int gemm_ctas = 0;            // MOE_GEMM_CTAS=n: cap the persistent GEMM grid at n CTAs
  int epi_sleep_ns = 1000;      // MOE_EPI_SLEEP=ns: epilogue warps' sleep between polls
  int route_split_cap = 0;      // MOE_ROUTE_SPLIT=1..16: cap the router's split of H
  bool route_shallow = false;   // MOE_ROUTE_DEEP=0: keep the router's shallow ring
  int tokn_nacc = 0;            // MOE_TOKN_NACC=1|2: force the accumulators per tile (GELU, down)
  int tokn_bk = 0;              // MOE_TOKN_BK=64|128: force the K per pipeline stage
  int tokn_split = 2;           // MOE_TOKN_SPLIT=1: no K-split of the last partial wave
  bool log = false;             // MOE_LOG=1: print launch plans to stderr
  bool tokn_stash = true;       // MOE_TOKN_STASH=0: SwiGLU epilogue holds TMEM while storing
};
const Tuning& tuning();
// Grouped-GEMM kernel choice: 0 automatic, 1 | 2 | 3 forced (moe_set_gemm_variant;
// starts as Tuning::gemm_variant).
int gemm_variant();

// ---------------------------------------------------------------- launches
// Programmatic dependent launch: with it on, a kernel's CTAs may be scheduled
// while its predecessor in the stream is finishing, and run their prologue;
// every kernel of this library executes griddepcontrol.wait (pdl_wait) before
// it touches global memory, which returns once the predecessor grid has
// completed and its writes are visible.
inline bool pdl_enabled() { return tuning().pdl; }

// MOE_LOG=1 (read when the library loads): launch plans on stderr, one line
// per launch (kernel, grid, block, shared memory, cluster) and one per plan
// decision (router split, GEMM variant and tile shape, scatter/combine split).
inline bool log_enabled() { return tuning().log; }
void log_line(const char* fmt, ...) __attribute__((format(printf, 1, 2)));
void log_launch(const void* kern, dim3 grid, dim3 block, size_t smem, int cluster_x);

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t s, int cluster_x, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  if (log_enabled()) log_launch(reinterpret_cast<const void*>(kern), grid, block, smem, cluster_x);
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// ---------------------------------------------------------------- router
struct RouteArgs {
  const void* x;        // [T,H] bf16 or fp32
  const void* wg;       // [H,E]
  const float* bias;    // [E] or null
  int T, H, E, top_k, dt_bf16;
  int32_t* topk_idx;    // [T,k]
  float* topk_gate;     // [T,k]
  float* logits_out;    // [T,E] or null
  int* tile_counts;     // [tiles,E] or null: per-tile expert histogram
  int* status;          // device status word or null (pipeline-wait timeouts)
  float* partials;      // split-H partial logits [tiles, S, 128, E] (tcgen05 path, S > 1)
  int* tickets;         // [tiles] arrival counters, zero between calls (S > 1)
};

struct RoutePlan {
  int kind;   // 0 = CUDA cores (fp32, or E not a multiple of 8), 2 = tcgen05
  int NPAD;   // tcgen05 path: experts padded to the MMA N (64, 128 or 256)
  int BT;     // tokens per CTA tile
  int tiles;  // CTA tiles along T
  int ck;     // CTAs splitting H per token tile (tcgen05 path)
};

RoutePlan route_plan(int T, int H, int E, int dt_bf16, int num_sms, bool can_split);
cudaError_t launch_route(const RouteArgs& a, const RoutePlan& p, cudaStream_t s);
cudaError_t launch_route_tc(const RouteArgs& a, const RoutePlan& p, cudaStream_t s);
constexpr int kRouteMaxCtas = 600;  // cap on tiles * split (sizes the partial-logit buffer)
cudaError_t launch_route_from_logits(const RouteArgs& a, const float* logits, cudaStream_t s);

// ---------------------------------------------------------------- permute
struct PermuteArgs {
  const int32_t* idx;   // [T,k] expert ids
  int T, k, E;
  int BT;               // tokens per tile (must match the histogram's tiling)
  int tiles;
  int split;            // CTAs per tile in the scatter (share the x_perm row copies)
  int cap;              // per-expert capacity (INT32_MAX when unlimited)
  int* tile_counts;     // [tiles,E] per-tile expert histogram (read by the scatter)
  int32_t* counts;      // [E]   pre-drop counts
  int32_t* offsets;     // [E+1] post-drop exclusive prefix
  int32_t* row_token;   // [T*k]
  int32_t* row_map;     // [T*k]
  const void* x;        // [T,H] (for x_perm) or null
  void* x_perm;         // [T*k,H] or null
  int H, elem_bytes;
  int* status;
  int empty_slots;      // 1: id -1 marks an unused slot (threshold gating), not an error
};

constexpr int kPermuteBT = 128;
cudaError_t launch_hist(const PermuteArgs& a, cudaStream_t s);
cudaError_t launch_scatter(const PermuteArgs& a, cudaStream_t s);

// ---------------------------------------------------------------- grouped GEMM
// MODE 0: out = gelu(A B1); MODE 1: out = silu(A B1) * (A B3); MODE 2: out = A B1.
struct GemmArgs {
  const int32_t* offsets;    // [E+1] row segments per expert
  const int32_t* row_token;  // gathered A rows (GATHER) or null
  int E, N, K;               // output columns, reduction length
  int R_max;                 // rows available in the output / row_token
  int T;                     // rows of the gathered source
  void* out;                 // [R_max, N]
  int* status;
  int* sched;                // tile counter of the dynamic schedule (zero before the launch)
  int epi_sleep_ns;          // epilogue warps' sleep between polls of the accumulator barrier
  // K-split of the last partial wave of tiles (token-as-N kernel; null: off)
  float* split_ws;           // split_units x kSplitUnitFloats fp32 partial sums
  int* split_tickets;        // split_tiles x kSplitTileTickets tickets, zero before the launch
  int split_units, split_tiles;
  int split_max;             // 2: cut the last partial wave of tiles in two along K; 1: no
};

// One K-split part's partial sums: 2 CTAs x 8 epilogue warps x 4 chunks of 32
// tokens x 2 accumulators x 32 tokens x 32 columns.
constexpr int kSplitUnitFloats = 2 * 8 * 4 * 2 * 32 * 32;
constexpr int kSplitTileTickets = 16;  // one per epilogue warp of the pair
constexpr int kSplitTiles = 128;       // split tiles per GEMM (at most the CTA pairs - 1)
constexpr int kSplitUnits = 80;        // split parts per GEMM (at most the CTA pairs)

// bf16 tensor-core (tcgen05) path. a_src: x_perm/h rows (dense) or x (gather).
cudaError_t launch_gemm_tc(int mode, bool gather, const void* a_src, int a_rows, const void* b1,
                           const void* b3, const GemmArgs& g, int num_sms, cudaStream_t s);
// Token-as-N variant on CTA pairs (dense A rows only; needs g.sched).
cudaError_t launch_gemm_tokn(int mode, const void* a_src, int a_rows, const void* b1,
                             const void* b3, const GemmArgs& g, int num_sms, cudaStream_t s);
// CTA-pair variant (cta_group::2), tensor maps prepared by launch_gemm_tc.
cudaError_t launch_gemm_tc_pair(int mode, bool gather, const CUtensorMap& ma,
                                const CUtensorMap& mb1, const CUtensorMap& mb3,
                                const CUtensorMap& mo, const GemmArgs& g, int num_sms,
                                cudaStream_t s);
// The bf16 epilogue's activations applied elementwise (self-test hook).
cudaError_t launch_epilogue_activations(const float* z, int n, float* gelu, float* silu,
                                        cudaStream_t s);
// fp32 CUDA-core path (no TF32).
cudaError_t launch_gemm_simt(int mode, const void* a_src, const void* b1, const void* b3,
                             const GemmArgs& g, int num_sms, cudaStream_t s);
// Identity experts: out[r] = a[r] or x[row_token[r]].
cudaError_t launch_copy_rows(const void* a_src, const GemmArgs& g, int elem_bytes,
                             cudaStream_t s);

// ---------------------------------------------------------------- combine
// status (nullable): where a debug build records a row_map entry outside y.
cudaError_t launch_combine(const void* y, const float* gate, const int32_t* row_map, int T,
                           int H, int k, int dt_bf16, void* out, int num_sms, cudaStream_t s,
                           int* status);

// ---------------------------------------------------------------- router statistics
// Per-expert pre-drop counts (summed from the router's per-tile histogram) and
// the mean over tokens of the full softmax, from fp32 logits [T,E].
constexpr int kStatsBT = 128;  // tokens per CTA of the probability pass
cudaError_t launch_route_stats(const float* logits, const int* tile_counts, int count_tiles, int T,
                               int E, float* tile_prob, int32_t* counts, float* prob_mean,
                               cudaStream_t s);

// ---------------------------------------------------------------- threshold gating
// Per token: experts with softmax probability > delta, largest first, at most
// k_max (the largest always kept); idx/gate [T,k_max] padded with -1 / 0;
// n_sel [T]; token_offsets [T+1] (exclusive prefix of n_sel) when non-null.
cudaError_t launch_route_threshold(const float* logits, int T, int E, int k_max, float delta,
                                   int32_t* idx, float* gate, int32_t* n_sel,
                                   int32_t* token_offsets, cudaStream_t s);

// ---------------------------------------------------------------- self-tests
// One bounded wait that can never be satisfied (records the timeout status).
cudaError_t launch_selftest_bounded_wait(int* status, cudaStream_t s);

// ---------------------------------------------------------------- misc
// Clears the status word and n counters (the router's tickets).
cudaError_t launch_clear_status(int* status, cudaStream_t s, int* counters = nullptr, int n = 0,
                                int* counters2 = nullptr, int n2 = 0);

}  // namespace moe
