// C ABI of the MoE layer (declared in include/moe_b200.h): argument checks,
// workspace layout and the launch sequence of each entry point.  No entry
// point allocates device memory or synchronises the stream (except
// moe_get_device_status, whose job is to synchronise).
#include <cxxabi.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "kernels.h"
#include "moe_b200.h"

using namespace moe;

namespace moe {
namespace {
int env_int(const char* name, int dflt) {
  const char* e = getenv(name);
  return (e && e[0]) ? atoi(e) : dflt;
}
Tuning read_tuning() {
  Tuning t;
  t.pdl = env_int("MOE_PDL", 1) != 0;
  const int v = env_int("MOE_GEMM_VARIANT", 0);
  t.gemm_variant = (v >= 1 && v <= 4) ? v : 0;
  t.gemm_ctas = env_int("MOE_GEMM_CTAS", 0);
  t.epi_sleep_ns = env_int("MOE_EPI_SLEEP", t.epi_sleep_ns);
  if (t.epi_sleep_ns < 0) t.epi_sleep_ns = 0;
  t.route_split_cap = env_int("MOE_ROUTE_SPLIT", 0);
  t.route_shallow = env_int("MOE_ROUTE_DEEP", 1) == 0;
  t.tokn_nacc = env_int("MOE_TOKN_NACC", 0);
  t.tokn_bk = env_int("MOE_TOKN_BK", 0);
  t.tokn_split = env_int("MOE_TOKN_SPLIT", 2);
  t.log = env_int("MOE_LOG", 0) != 0;
  t.tokn_stash = env_int("MOE_TOKN_STASH", 1) != 0;
  return t;
}
// Initialised when the library is loaded.
const Tuning g_tuning = read_tuning();
std::atomic<int> g_gemm_variant{g_tuning.gemm_variant};
}  // namespace
const Tuning& tuning() { return g_tuning; }
int gemm_variant() { return g_gemm_variant.load(std::memory_order_relaxed); }

void log_line(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  std::fputs("[moe] ", stderr);
  std::vfprintf(stderr, fmt, ap);
  std::fputc('\n', stderr);
  va_end(ap);
}

void log_launch(const void* kern, dim3 grid, dim3 block, size_t smem, int cluster_x) {
  const char* name = nullptr;
  if (cudaFuncGetName(&name, kern) != cudaSuccess || name == nullptr) name = "?";
  int dm = 0;
  char* readable = abi::__cxa_demangle(name, nullptr, nullptr, &dm);
  const char* shown = (readable != nullptr && dm == 0) ? readable : name;
  if (std::strncmp(shown, "void ", 5) == 0) shown += 5;  // a template's return type
  const char* paren = std::strchr(shown, '(');  // drop the parameter list
  const int len = paren ? static_cast<int>(paren - shown) : static_cast<int>(std::strlen(shown));
  log_line("launch %.*s grid=%u block=%u smem=%zu cluster=%d pdl=%d", len, shown, grid.x, block.x,
           smem, cluster_x, tuning().pdl ? 1 : 0);
  std::free(readable);
}
}  // namespace moe

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

int elem_bytes(moe_dtype dt) { return dt == MOE_BF16 ? 2 : 4; }

int num_sms_current() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Workspace: [status | topk_idx | topk_gate | tile_counts | sched + tickets + split tickets |
//             partials | counts | offsets | row_token | row_map | x_perm | h | y | split sums |
//             x_stage | out_stage]
// sched: the grouped GEMMs' tile counters (kSchedCounters ints), directly
// followed by the router's tickets and the two GEMMs' K-split tickets, so one
// clear covers all three.
constexpr int kSchedCounters = 4;
constexpr int kSplitTicketInts = kSplitTiles * kSplitTileTickets;  // per GEMM
constexpr size_t kSplitSumBytes = static_cast<size_t>(kSplitUnits) * kSplitUnitFloats * 4;
struct WsLayout {
  size_t status, topk_idx, topk_gate, tile_counts, sched, tickets, split_tickets, partials,
      counts, offsets, row_token, row_map, x_perm, h, y, split_sums, x_stage, out_stage, logits,
      n_sel, total;
  int clear_ints;  // ints zeroed from sched on
};

// Workspaces that begin with the status word's 256-byte block keep the GEMMs'
// tile counters in that block, 16 bytes in.
constexpr size_t kSchedInStatusBlock = 16;

WsLayout ws_layout(int T, int H, int F, int E, int k, moe_act act, moe_dtype dt, bool host_stage,
                   bool threshold = false) {
  WsLayout L{};
  const size_t eb = elem_bytes(dt);
  const size_t R = static_cast<size_t>(T) * k;
  const size_t tiles = static_cast<size_t>(T) / 16 + 1;  // finest token tiling used
  size_t o = 0;
  L.status = o;      o = align_up(o + 4);
  L.topk_idx = o;    o = align_up(o + R * 4);
  L.topk_gate = o;   o = align_up(o + R * 4);
  L.tile_counts = o; o = align_up(o + tiles * E * 4);
  L.sched = o;
  L.tickets = o + kSchedCounters * 4;
  L.split_tickets = L.tickets + (static_cast<size_t>(T) / 128 + 1) * 4;
  L.clear_ints = kSchedCounters + T / 128 + 1 + 2 * kSplitTicketInts;
  o = align_up(L.split_tickets + 2 * kSplitTicketInts * 4);
  L.partials = o;    o = align_up(o + static_cast<size_t>(kRouteMaxCtas) * 128 * E * 4);
  L.counts = o;      o = align_up(o + static_cast<size_t>(E) * 4);
  L.offsets = o;     o = align_up(o + static_cast<size_t>(E + 1) * 4);
  L.row_token = o;   o = align_up(o + R * 4);
  L.row_map = o;     o = align_up(o + R * 4);
  L.x_perm = o;      o = align_up(o + R * H * eb);
  L.h = o;           o = align_up(o + (act == MOE_ACT_IDENTITY ? 0 : R * F * eb));
  L.y = o;           o = align_up(o + R * H * eb);
  const bool tc = dt == MOE_BF16 && act != MOE_ACT_IDENTITY;  // tensor-core experts
  L.split_sums = o;  o = align_up(o + (tc ? kSplitSumBytes : 0));
  if (host_stage) {
    L.x_stage = o;   o = align_up(o + static_cast<size_t>(T) * H * eb);
    L.out_stage = o; o = align_up(o + static_cast<size_t>(T) * H * eb);
  }
  if (threshold) {
    L.logits = o;    o = align_up(o + static_cast<size_t>(T) * E * 4);
    L.n_sel = o;     o = align_up(o + (static_cast<size_t>(T) + 1) * 4);
  }
  L.total = o;
  return L;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

moe_status check_common(int T, int H, int E, int k, moe_dtype dt) {
  if (dt != MOE_F32 && dt != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (T < 0 || H <= 0 || E <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
  if (k > E) return MOE_ERR_INVALID_ARG;
  if (H % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (E > kMaxE || k > kMaxTopK) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

bool index_range_ok(int T, int k, int width) {
  return static_cast<long long>(T) * k * width < (1LL << 31);
}

int capacity_of(float cf, int T, int k, int E) {
  if (!(cf > 0.f)) return INT32_MAX;
  const double c = std::ceil(static_cast<double>(cf) * static_cast<double>(T) * k / E);
  if (c >= static_cast<double>(INT32_MAX)) return INT32_MAX;
  return c < 1.0 ? 1 : static_cast<int>(c);
}

cudaStream_t as_stream(moe_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// Grouped FFN on prepared buffers (shared by moe_grouped_ffn and moe_forward).
// sched: two zeroed tile counters (GEMM-1, GEMM-2).  split_sums (kSplitSumBytes)
// and split_tickets (2 x kSplitTicketInts zeroed ints), or nulls: room for the
// GEMMs' K-split tail.
moe_status run_ffn(const void* x_perm, const int32_t* row_token, const void* x, const void* w1,
                   const void* w3, const void* w2, const int32_t* offsets, int R_max, int T,
                   int H, int F, int E, moe_act act, moe_dtype dt, void* y, void* h, int* status,
                   int* sched, float* split_sums, int* split_tickets, cudaStream_t s,
                   cudaEvent_t mid_event = nullptr) {
  const int nsm = num_sms_current();
  const bool gather = row_token != nullptr;
  const void* a_src = gather ? x : x_perm;
  const int a_rows = gather ? T : R_max;
  GemmArgs g{};
  g.offsets = offsets;
  g.E = E;
  g.R_max = R_max;
  g.T = T;
  g.status = status;
  if (split_sums != nullptr && split_tickets != nullptr) {
    g.split_ws = split_sums;
    g.split_units = kSplitUnits;
    g.split_tiles = kSplitTiles;
  }
  if (act == MOE_ACT_IDENTITY) {
    g.row_token = row_token;
    g.N = H;
    g.K = H;
    g.out = y;
    if (launch_copy_rows(a_src, g, elem_bytes(dt), s) != cudaSuccess) return MOE_ERR_CUDA;
    return cuda_status(mid_event ? cudaEventRecord(mid_event, s) : cudaSuccess);
  }
  const int mode1 = act == MOE_ACT_SWIGLU ? 1 : 0;
  // GEMM-1: h = act(A W1 [, A W3])
  g.row_token = row_token;
  g.N = F;
  g.K = H;
  g.out = h;
  g.sched = sched;
  g.split_tickets = g.split_ws ? split_tickets : nullptr;
  cudaError_t err;
  if (dt == MOE_BF16)
    err = launch_gemm_tc(mode1, gather, a_src, a_rows, w1, w3, g, nsm, s);
  else
    err = launch_gemm_simt(mode1, a_src, w1, w3, g, nsm, s);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  if (mid_event && cudaEventRecord(mid_event, s) != cudaSuccess) return MOE_ERR_CUDA;
  // GEMM-2: y = h W2 (rows already in expert order)
  g.row_token = nullptr;
  g.N = H;
  g.K = F;
  g.out = y;
  g.sched = sched + 1;
  g.split_tickets = g.split_ws ? split_tickets + kSplitTicketInts : nullptr;
  if (dt == MOE_BF16)
    err = launch_gemm_tc(2, false, h, R_max, w2, nullptr, g, nsm, s);
  else
    err = launch_gemm_simt(2, h, w2, nullptr, g, nsm, s);
  return cuda_status(err);
}

}  // namespace

extern "C" {

size_t moe_workspace_bytes(int T, int H, int F, int E, int top_k, moe_act act, moe_dtype dt) {
  if (T < 0 || H <= 0 || F <= 0 || E <= 0 || top_k <= 0) return 0;
  return ws_layout(T, H, F, E, top_k, act, dt, false).total;
}

size_t moe_forward_host_workspace_bytes(int T, int H, int F, int E, int top_k, moe_act act,
                                        moe_dtype dt) {
  if (T < 0 || H <= 0 || F <= 0 || E <= 0 || top_k <= 0) return 0;
  return ws_layout(T, H, F, E, top_k, act, dt, true).total;
}

size_t moe_grouped_ffn_workspace_bytes(int R_max, int H, int F, moe_act act, moe_dtype dt,
                                       int gathered) {
  if (R_max < 0 || H <= 0 || F <= 0) return 0;
  if (dt != MOE_F32 && dt != MOE_BF16) return 0;
  const size_t eb = elem_bytes(dt);
  const bool tc = dt == MOE_BF16 && act != MOE_ACT_IDENTITY;
  size_t n = align_up(4) + (act == MOE_ACT_IDENTITY ? 0 : static_cast<size_t>(R_max) * F * eb);
  if (gathered && tc) n = align_up(n) + static_cast<size_t>(R_max) * H * eb;
  if (tc) n = align_up(n) + align_up(2 * kSplitTicketInts * 4) + kSplitSumBytes;
  return n;
}

moe_status moe_route(const void* x, const void* w_gate, const float* gate_bias, int T, int H,
                     int E, int top_k, moe_dtype dt, int32_t* topk_idx, float* topk_gate,
                     float* logits_out, moe_stream_t stream) {
  moe_status st = check_common(T, H, E, top_k, dt);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!x || !w_gate || !topk_idx || !topk_gate) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_gate)) return MOE_ERR_INVALID_ARG;
  if (!index_range_ok(T, 1, H) || !index_range_ok(T, 1, E)) return MOE_ERR_UNSUPPORTED;
  RouteArgs a{};
  a.x = x; a.wg = w_gate; a.bias = gate_bias;
  a.T = T; a.H = H; a.E = E; a.top_k = top_k; a.dt_bf16 = dt == MOE_BF16;
  a.topk_idx = topk_idx; a.topk_gate = topk_gate; a.logits_out = logits_out;
  a.tile_counts = nullptr;
  const RoutePlan p = route_plan(T, H, E, a.dt_bf16, num_sms_current(), false);
  return cuda_status(launch_route(a, p, as_stream(stream)));
}

moe_status moe_route_from_logits(const float* logits, int T, int E, int top_k, int32_t* topk_idx,
                                 float* topk_gate, moe_stream_t stream) {
  if (T < 0 || E <= 0 || top_k <= 0 || top_k > E) return MOE_ERR_INVALID_ARG;
  if (E > kMaxE || top_k > kMaxTopK) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!logits || !topk_idx || !topk_gate) return MOE_ERR_INVALID_ARG;
  if (!index_range_ok(T, 1, E)) return MOE_ERR_UNSUPPORTED;
  RouteArgs a{};
  a.T = T; a.E = E; a.top_k = top_k;
  a.topk_idx = topk_idx; a.topk_gate = topk_gate;
  return cuda_status(launch_route_from_logits(a, logits, as_stream(stream)));
}

moe_status moe_permute(const void* x, const int32_t* token_expert_idx, int T, int H, int E,
                       int top_k, float capacity_factor, moe_dtype dt, void* x_perm,
                       int32_t* expert_counts, int32_t* expert_offsets, int32_t* row_token,
                       int32_t* row_map, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_common(T, H, E, top_k, dt);
  if (st != MOE_OK) return st;
  if (!token_expert_idx || !expert_counts || !expert_offsets || !row_token || !row_map || !ws)
    return MOE_ERR_INVALID_ARG;
  if (x_perm && (!x || !aligned16(x) || !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
  if (!index_range_ok(T, top_k, H)) return MOE_ERR_UNSUPPORTED;
  const WsLayout L = ws_layout(T, H, 8, E, top_k, MOE_ACT_IDENTITY, dt, false);
  if (ws_bytes < L.tile_counts + (static_cast<size_t>(T) / 16 + 1) * E * 4)
    return MOE_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  int* status = at<int>(ws, L.status);
  if (launch_clear_status(status, s) != cudaSuccess) return MOE_ERR_CUDA;
  PermuteArgs p{};
  p.idx = token_expert_idx;
  p.T = T; p.k = top_k; p.E = E;
  p.BT = kPermuteBT;
  p.tiles = (T + kPermuteBT - 1) / kPermuteBT;
  p.split = 1;
  if (x_perm)
    while (p.split < 16 && p.tiles * p.split < 2 * num_sms_current()) p.split *= 2;
  p.cap = capacity_of(capacity_factor, T, top_k, E);
  p.tile_counts = at<int>(ws, L.tile_counts);
  p.counts = expert_counts; p.offsets = expert_offsets;
  p.row_token = row_token; p.row_map = row_map;
  p.x = x; p.x_perm = x_perm; p.H = H; p.elem_bytes = elem_bytes(dt);
  p.status = status;
  if (T == 0) {
    // no pairs: counts are zero, every offset is zero
    if (cudaMemsetAsync(expert_counts, 0, E * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
    return cuda_status(cudaMemsetAsync(expert_offsets, 0, (E + 1) * 4, s));
  }
  if (launch_hist(p, s) != cudaSuccess) return MOE_ERR_CUDA;
  return cuda_status(launch_scatter(p, s));
}

moe_status moe_grouped_ffn(const void* x_perm, const int32_t* row_token, const void* x,
                           const void* w1, const void* w3, const void* w2,
                           const int32_t* expert_offsets, int R_max, int T, int H, int F, int E,
                           moe_act act, moe_dtype dt, void* y, void* ws, size_t ws_bytes,
                           moe_stream_t stream) {
  if (dt != MOE_F32 && dt != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (act != MOE_ACT_SWIGLU && act != MOE_ACT_GELU && act != MOE_ACT_IDENTITY)
    return MOE_ERR_INVALID_ARG;
  if (R_max < 0 || T < 0 || H <= 0 || F <= 0 || E <= 0) return MOE_ERR_INVALID_ARG;
  if (H % 8 != 0 || F % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (E > kMaxE) return MOE_ERR_UNSUPPORTED;
  if (!expert_offsets || !y || !ws) return MOE_ERR_INVALID_ARG;
  const bool gather = row_token != nullptr;
  const void* a_src = gather ? x : x_perm;
  if (!a_src || !aligned16(a_src) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  if (act != MOE_ACT_IDENTITY) {
    if (!w1 || !w2 || !aligned16(w1) || !aligned16(w2)) return MOE_ERR_INVALID_ARG;
    if (act == MOE_ACT_SWIGLU && (!w3 || !aligned16(w3))) return MOE_ERR_INVALID_ARG;
  }
  if (gather && T <= 0) return MOE_ERR_INVALID_ARG;
  if (!index_range_ok(R_max, 1, H > F ? H : F)) return MOE_ERR_UNSUPPORTED;
  if (R_max == 0) return MOE_OK;
  // [status block | h: R_max x F | gathered rows: R_max x H (optional) |
  //  K-split tickets + sums (optional)]; the optional parts are used when ws has room
  const size_t h_off = align_up(4);
  const size_t need = h_off + static_cast<size_t>(R_max) * F * elem_bytes(dt);
  if (act != MOE_ACT_IDENTITY && ws_bytes < need) return MOE_ERR_WORKSPACE;
  if (ws_bytes < h_off) return MOE_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  int* status = at<int>(ws, 0);
  int* sched = at<int>(ws, kSchedInStatusBlock);
  const bool tc = dt == MOE_BF16 && act != MOE_ACT_IDENTITY;
  const size_t xg_off = align_up(need);
  const size_t xg_bytes = static_cast<size_t>(R_max) * H * elem_bytes(dt);
  const bool gather_dense = gather && tc && ws_bytes >= xg_off + xg_bytes;
  const size_t sp_off = gather_dense ? align_up(xg_off + xg_bytes) : xg_off;
  const size_t sp_tickets_bytes = align_up(2 * kSplitTicketInts * 4);
  const bool split = tc && ws_bytes >= sp_off + sp_tickets_bytes + kSplitSumBytes;
  int* sp_tickets = split ? at<int>(ws, sp_off) : nullptr;
  float* sp_sums = split ? at<float>(ws, sp_off + sp_tickets_bytes) : nullptr;
  if (launch_clear_status(status, s, sched, 2, sp_tickets, split ? 2 * kSplitTicketInts : 0) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  // Gathered bf16 rows with room in ws: copy them into expert order once and
  // run the dense kernel (a gathering TMA moves four rows per request).
  if (gather_dense) {
    GemmArgs g{};
    g.offsets = expert_offsets;
    g.row_token = row_token;
    g.E = E;
    g.N = H;
    g.R_max = R_max;
    g.T = T;
    g.out = at<void>(ws, xg_off);
    g.status = status;
    if (launch_copy_rows(x, g, elem_bytes(dt), s) != cudaSuccess) return MOE_ERR_CUDA;
    return run_ffn(at<void>(ws, xg_off), nullptr, x, w1, w3, w2, expert_offsets, R_max, T, H, F,
                   E, act, dt, y, at<void>(ws, h_off), status, sched, sp_sums, sp_tickets, s);
  }
  return run_ffn(x_perm, row_token, x, w1, w3, w2, expert_offsets, R_max, T, H, F, E, act, dt, y,
                 at<void>(ws, h_off), status, sched, sp_sums, sp_tickets, s);
}

moe_status moe_unpermute_combine(const void* y, const float* topk_gate, const int32_t* row_map,
                                 int T, int H, int top_k, moe_dtype dt, void* out,
                                 moe_stream_t stream) {
  if (dt != MOE_F32 && dt != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (T < 0 || H <= 0 || top_k <= 0 || H % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (top_k > kMaxTopK) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!y || !row_map || !out || !aligned16(y) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if (!index_range_ok(T, top_k, H)) return MOE_ERR_UNSUPPORTED;
  return cuda_status(launch_combine(y, topk_gate, row_map, T, H, top_k, dt == MOE_BF16, out,
                                    num_sms_current(), as_stream(stream), nullptr));
}

// ---------------------------------------------------------------- router statistics
// Workspace: [status | logits [T,E] | per-tile counts | per-tile probability sums]
size_t moe_route_stats_workspace_bytes(int T, int E) {
  if (T < 0 || E <= 0) return 0;
  size_t o = align_up(4);
  o = align_up(o + static_cast<size_t>(T) * E * 4);
  o = align_up(o + (static_cast<size_t>(T) / 16 + 1) * E * 4);
  o = align_up(o + (static_cast<size_t>(T) / kStatsBT + 1) * E * 4);
  return o;
}

moe_status moe_route_stats(const void* x, const void* w_gate, const float* gate_bias, int T, int H,
                           int E, int top_k, moe_dtype dt, int32_t* topk_idx, float* topk_gate,
                           int32_t* expert_counts, float* prob_mean, void* ws, size_t ws_bytes,
                           moe_stream_t stream) {
  moe_status st = check_common(T, H, E, top_k, dt);
  if (st != MOE_OK) return st;
  if (!x || !w_gate || !topk_idx || !topk_gate || !expert_counts || !prob_mean || !ws)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_gate)) return MOE_ERR_INVALID_ARG;
  if (!index_range_ok(T, 1, H) || !index_range_ok(T, 1, E)) return MOE_ERR_UNSUPPORTED;
  if (ws_bytes < moe_route_stats_workspace_bytes(T, E)) return MOE_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  if (T == 0) {
    if (cudaMemsetAsync(expert_counts, 0, E * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
    return cuda_status(cudaMemsetAsync(prob_mean, 0, E * 4, s));
  }
  const size_t o_logits = align_up(4);
  const size_t o_counts = align_up(o_logits + static_cast<size_t>(T) * E * 4);
  const size_t o_prob = align_up(o_counts + (static_cast<size_t>(T) / 16 + 1) * E * 4);
  RouteArgs a{};
  a.x = x; a.wg = w_gate; a.bias = gate_bias;
  a.T = T; a.H = H; a.E = E; a.top_k = top_k; a.dt_bf16 = dt == MOE_BF16;
  a.topk_idx = topk_idx; a.topk_gate = topk_gate;
  a.logits_out = at<float>(ws, o_logits);
  a.tile_counts = at<int>(ws, o_counts);
  a.status = at<int>(ws, 0);
  if (launch_clear_status(a.status, s) != cudaSuccess) return MOE_ERR_CUDA;
  const RoutePlan p = route_plan(T, H, E, a.dt_bf16, num_sms_current(), false);
  if (launch_route(a, p, s) != cudaSuccess) return MOE_ERR_CUDA;
  return cuda_status(launch_route_stats(a.logits_out, a.tile_counts, p.tiles, T, E,
                                        at<float>(ws, o_prob), expert_counts, prob_mean, s));
}

// ---------------------------------------------------------------- k = 1 expert matmul
// Workspace: [status | tile_counts | counts | offsets | row_token | row_map | x_perm | y]
namespace {
struct MatmulWs {
  size_t tile_counts, counts, offsets, row_token, row_map, x_perm, y, total;
};
MatmulWs matmul_ws(int T, int H, int I, int E, moe_dtype dt) {
  MatmulWs L{};
  const size_t eb = elem_bytes(dt);
  size_t o = align_up(4);
  L.tile_counts = o; o = align_up(o + (static_cast<size_t>(T) / kPermuteBT + 1) * E * 4);
  L.counts = o;      o = align_up(o + static_cast<size_t>(E) * 4);
  L.offsets = o;     o = align_up(o + static_cast<size_t>(E + 1) * 4);
  L.row_token = o;   o = align_up(o + static_cast<size_t>(T) * 4);
  L.row_map = o;     o = align_up(o + static_cast<size_t>(T) * 4);
  L.x_perm = o;      o = align_up(o + static_cast<size_t>(T) * H * eb);
  L.y = o;           o = align_up(o + static_cast<size_t>(T) * I * eb);
  L.total = o;
  return L;
}
}  // namespace

moe_status moe_selftest_epilogue_activations(const float* z, int n, float* gelu_out,
                                             float* silu_out, moe_stream_t stream) {
  if (n < 0 || (n > 0 && (!z || !gelu_out || !silu_out))) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_epilogue_activations(z, n, gelu_out, silu_out, as_stream(stream)));
}

moe_status moe_selftest_bounded_wait(void* ws, moe_stream_t stream) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  int* status = at<int>(ws, 0);
  if (launch_clear_status(status, s) != cudaSuccess) return MOE_ERR_CUDA;
  return cuda_status(launch_selftest_bounded_wait(status, s));
}

size_t moe_expert_matmul_workspace_bytes(int T, int H, int I, int E, moe_dtype dt) {
  if (T < 0 || H <= 0 || I <= 0 || E <= 0) return 0;
  return matmul_ws(T, H, I, E, dt).total;
}

moe_status moe_expert_matmul(const void* x, const void* expert_weight,
                             const int32_t* token_expert_idx, int T, int H, int I, int E,
                             moe_dtype dt, void* out, void* ws, size_t ws_bytes,
                             moe_stream_t stream) {
  moe_status st = check_common(T, H, E, 1, dt);
  if (st != MOE_OK) return st;
  if (I <= 0 || I % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !expert_weight || !token_expert_idx || !out || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(expert_weight) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if (!index_range_ok(T, 1, H) || !index_range_ok(T, 1, I)) return MOE_ERR_UNSUPPORTED;
  const MatmulWs L = matmul_ws(T, H, I, E, dt);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  int* status = at<int>(ws, 0);
  int* sched = at<int>(ws, kSchedInStatusBlock);
  if (launch_clear_status(status, s, sched, 1) != cudaSuccess) return MOE_ERR_CUDA;
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* row_map = at<int32_t>(ws, L.row_map);
  void* x_perm = at<void>(ws, L.x_perm);
  void* y = at<void>(ws, L.y);
  // token rearrangement by expert (no capacity limit)
  PermuteArgs p{};
  p.idx = token_expert_idx;
  p.T = T; p.k = 1; p.E = E;
  p.BT = kPermuteBT;
  p.tiles = (T + kPermuteBT - 1) / kPermuteBT;
  p.split = 1;
  while (p.split < 16 && p.tiles * p.split < 2 * num_sms_current()) p.split *= 2;
  p.cap = INT32_MAX;
  p.tile_counts = at<int>(ws, L.tile_counts);
  p.counts = at<int32_t>(ws, L.counts); p.offsets = offsets;
  p.row_token = at<int32_t>(ws, L.row_token); p.row_map = row_map;
  p.x = x; p.x_perm = x_perm; p.H = H; p.elem_bytes = elem_bytes(dt);
  p.status = status;
  if (launch_hist(p, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_scatter(p, s) != cudaSuccess) return MOE_ERR_CUDA;
  // per-expert matmul of the expert-major rows: y = x_perm W[e]
  GemmArgs g{};
  g.offsets = offsets;
  g.E = E; g.R_max = T; g.T = T; g.status = status;
  g.N = I; g.K = H; g.out = y; g.sched = sched;
  const cudaError_t err =
      dt == MOE_BF16 ? launch_gemm_tc(2, false, x_perm, T, expert_weight, nullptr, g,
                                      num_sms_current(), s)
                     : launch_gemm_simt(2, x_perm, expert_weight, nullptr, g, num_sms_current(), s);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  // back to token order: out[t] = y[row_map[t]] (weight 1)
  return cuda_status(launch_combine(y, nullptr, row_map, T, I, 1, dt == MOE_BF16, out,
                                    num_sms_current(), s, status));
}

}  // extern "C"

namespace {

// Threshold gating instead of top-k (moe_forward_threshold): top_k is then the
// slot count k_max and delta the probability threshold.
struct Gating {
  bool threshold = false;
  float delta = 0.f;
  int32_t* n_sel_out = nullptr;
};

// Every host-side check of a layer forward, in order.  MOE_OK with T == 0
// means there is nothing to launch.
moe_status check_forward(const void* x, const void* w_gate, const void* w1, const void* w3,
                         const void* w2, int T, int H, int F, int E, int top_k, moe_act act,
                         moe_dtype dt, const void* out, const void* ws, size_t ws_bytes,
                         bool threshold) {
  moe_status st = check_common(T, H, E, top_k, dt);
  if (st != MOE_OK) return st;
  if (act != MOE_ACT_SWIGLU && act != MOE_ACT_GELU && act != MOE_ACT_IDENTITY)
    return MOE_ERR_INVALID_ARG;
  if (F <= 0 || F % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !w_gate || !out || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_gate) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if (act != MOE_ACT_IDENTITY) {
    if (!w1 || !w2 || !aligned16(w1) || !aligned16(w2)) return MOE_ERR_INVALID_ARG;
    if (act == MOE_ACT_SWIGLU && (!w3 || !aligned16(w3))) return MOE_ERR_INVALID_ARG;
  }
  if (!index_range_ok(T, top_k, H > F ? H : F) || !index_range_ok(T, 1, E))
    return MOE_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(ws) % kAlign != 0) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < ws_layout(T, H, F, E, top_k, act, dt, false, threshold).total)
    return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

moe_status forward_impl(const void* x, const void* w_gate, const float* gate_bias, const void* w1,
                        const void* w3, const void* w2, int T, int H, int F, int E, int top_k,
                        float capacity_factor, moe_act act, moe_dtype dt, void* out,
                        int32_t* topk_idx_out, int32_t* expert_counts_out, void* ws,
                        size_t ws_bytes, moe_stream_t stream, cudaEvent_t const* ev,
                        const Gating& gating = Gating()) {
  moe_status st = check_forward(x, w_gate, w1, w3, w2, T, H, F, E, top_k, act, dt, out, ws,
                                ws_bytes, gating.threshold);
  if (st != MOE_OK || T == 0) return st;
  const WsLayout L = ws_layout(T, H, F, E, top_k, act, dt, false, gating.threshold);

  cudaStream_t s = as_stream(stream);
  const int nsm = num_sms_current();
  int* status = at<int>(ws, L.status);
  int32_t* topk_idx = topk_idx_out ? topk_idx_out : at<int32_t>(ws, L.topk_idx);
  float* topk_gate = at<float>(ws, L.topk_gate);
  int32_t* counts = expert_counts_out ? expert_counts_out : at<int32_t>(ws, L.counts);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* row_token = at<int32_t>(ws, L.row_token);
  int32_t* row_map = at<int32_t>(ws, L.row_map);
  const bool bf16 = dt == MOE_BF16;
  // bf16 experts stream their A rows densely (2-D TMA) from x_perm, which the
  // scatter kernel gathers once; gathering inside the GEMM (TMA gather4, one
  // 4-row request per lane per k-block) measured 2.9x slower on GEMM-1.  The
  // fp32 CUDA-core experts gather through row_token directly.
  void* x_perm = bf16 ? at<void>(ws, L.x_perm) : nullptr;

  auto mark = [&](int i) { return ev && ev[i] ? cudaEventRecord(ev[i], s) : cudaSuccess; };
  int* sched = at<int>(ws, L.sched);
  int* tickets = at<int>(ws, L.tickets);
  if (launch_clear_status(status, s, sched, L.clear_ints) != cudaSuccess) return MOE_ERR_CUDA;
  // 1. route (+ per-tile histogram)
  if (mark(0) != cudaSuccess) return MOE_ERR_CUDA;
  RouteArgs ra{};
  ra.x = x; ra.wg = w_gate; ra.bias = gate_bias;
  ra.T = T; ra.H = H; ra.E = E; ra.top_k = top_k; ra.dt_bf16 = bf16;
  ra.topk_idx = topk_idx; ra.topk_gate = topk_gate; ra.logits_out = nullptr;
  ra.tile_counts = at<int>(ws, L.tile_counts);
  ra.status = status;
  ra.partials = at<float>(ws, L.partials);
  ra.tickets = tickets;
  if (gating.threshold) {  // the router's logits feed the threshold selection
    ra.logits_out = at<float>(ws, L.logits);
    ra.tile_counts = nullptr;
  }
  const RoutePlan rp = route_plan(T, H, E, bf16, nsm, true);
  if (launch_route(ra, rp, s) != cudaSuccess) return MOE_ERR_CUDA;
  PermuteArgs pa{};
  pa.idx = topk_idx;
  pa.T = T; pa.k = top_k; pa.E = E;
  pa.BT = rp.BT; pa.tiles = rp.tiles;
  pa.tile_counts = at<int>(ws, L.tile_counts);
  pa.status = status;
  if (gating.threshold) {
    int32_t* n_sel = gating.n_sel_out ? gating.n_sel_out : at<int32_t>(ws, L.n_sel);
    if (launch_route_threshold(ra.logits_out, T, E, top_k, gating.delta, topk_idx, topk_gate,
                               n_sel, nullptr, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    pa.BT = kPermuteBT;
    pa.tiles = (T + kPermuteBT - 1) / kPermuteBT;
    pa.empty_slots = 1;
    if (launch_hist(pa, s) != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (mark(1) != cudaSuccess) return MOE_ERR_CUDA;
  // 2. scatter (the per-expert scan over tiles runs in its prologue) over the
  // router's (or the histogram's) token tiles; the "scan" stage events stay
  // for the callers that time stages, with nothing between them
  // enough scatter CTAs to keep the x_perm row copies near HBM bandwidth
  pa.split = 1;
  if (x_perm)
    while (pa.split < 16 && pa.tiles * pa.split < 2 * nsm) pa.split *= 2;
  pa.cap = capacity_of(capacity_factor, T, top_k, E);
  pa.counts = counts; pa.offsets = offsets; pa.row_token = row_token; pa.row_map = row_map;
  pa.x = x; pa.x_perm = x_perm; pa.H = H; pa.elem_bytes = elem_bytes(dt);
  if (mark(2) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_scatter(pa, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (mark(3) != cudaSuccess) return MOE_ERR_CUDA;
  // 3. experts
  const int R_max = T * top_k;
  void* y = at<void>(ws, L.y);
  const bool tc = bf16 && act != MOE_ACT_IDENTITY;
  st = run_ffn(x_perm, bf16 ? nullptr : row_token, x, w1, w3, w2, offsets, R_max, T, H, F, E, act,
               dt, y, at<void>(ws, L.h), status, sched,
               tc ? at<float>(ws, L.split_sums) : nullptr,
               tc ? at<int>(ws, L.split_tickets) : nullptr, s, ev ? ev[4] : nullptr);
  if (st != MOE_OK) return st;
  if (mark(5) != cudaSuccess) return MOE_ERR_CUDA;
  // 4. combine
  if (launch_combine(y, topk_gate, row_map, T, H, top_k, bf16, out, nsm, s, status) != cudaSuccess)
    return MOE_ERR_CUDA;
  return cuda_status(mark(6));
}

}  // namespace

extern "C" {

moe_status moe_forward(const void* x, const void* w_gate, const float* gate_bias, const void* w1,
                       const void* w3, const void* w2, int T, int H, int F, int E, int top_k,
                       float capacity_factor, moe_act act, moe_dtype dt, void* out,
                       int32_t* topk_idx_out, int32_t* expert_counts_out, void* ws,
                       size_t ws_bytes, moe_stream_t stream) {
  return forward_impl(x, w_gate, gate_bias, w1, w3, w2, T, H, F, E, top_k, capacity_factor, act,
                      dt, out, topk_idx_out, expert_counts_out, ws, ws_bytes, stream, nullptr);
}

moe_status moe_threshold_select(const float* logits, int T, int E, int k_max, float delta,
                                int32_t* topk_idx, float* topk_gate, int32_t* n_selected,
                                int32_t* token_offsets, moe_stream_t stream) {
  if (T < 0 || E <= 0 || k_max <= 0 || k_max > E) return MOE_ERR_INVALID_ARG;
  if (E > kMaxE || k_max > kMaxTopK) return MOE_ERR_UNSUPPORTED;
  if (!(delta == delta)) return MOE_ERR_INVALID_ARG;  // NaN
  if (!logits || !topk_idx || !topk_gate || !n_selected) return MOE_ERR_INVALID_ARG;
  if (!index_range_ok(T, 1, E)) return MOE_ERR_UNSUPPORTED;
  cudaStream_t s = as_stream(stream);
  if (T == 0)
    return cuda_status(token_offsets ? cudaMemsetAsync(token_offsets, 0, 4, s) : cudaSuccess);
  const float d = delta > 0.f ? delta : 1.f / static_cast<float>(E);
  return cuda_status(launch_route_threshold(logits, T, E, k_max, d, topk_idx, topk_gate,
                                            n_selected, token_offsets, s));
}

size_t moe_forward_threshold_workspace_bytes(int T, int H, int F, int E, int k_max, moe_act act,
                                             moe_dtype dt) {
  if (T < 0 || H <= 0 || F <= 0 || E <= 0 || k_max <= 0) return 0;
  return ws_layout(T, H, F, E, k_max, act, dt, false, true).total;
}

moe_status moe_forward_threshold(const void* x, const void* w_gate, const float* gate_bias,
                                 const void* w1, const void* w3, const void* w2, int T, int H,
                                 int F, int E, int k_max, float delta, float capacity_factor,
                                 moe_act act, moe_dtype dt, void* out, int32_t* topk_idx_out,
                                 int32_t* n_selected_out, void* ws, size_t ws_bytes,
                                 moe_stream_t stream) {
  if (!(delta == delta)) return MOE_ERR_INVALID_ARG;
  Gating g;
  g.threshold = true;
  g.delta = delta > 0.f ? delta : (E > 0 ? 1.f / static_cast<float>(E) : 0.f);
  g.n_sel_out = n_selected_out;
  return forward_impl(x, w_gate, gate_bias, w1, w3, w2, T, H, F, E, k_max, capacity_factor, act,
                      dt, out, topk_idx_out, nullptr, ws, ws_bytes, stream, nullptr, g);
}

moe_status moe_forward_timed(const void* x, const void* w_gate, const float* gate_bias,
                             const void* w1, const void* w3, const void* w2, int T, int H, int F,
                             int E, int top_k, float capacity_factor, moe_act act, moe_dtype dt,
                             void* out, void* ws, size_t ws_bytes, moe_stream_t stream,
                             void* const* events, int n_events) {
  if (!events || n_events < 7) return MOE_ERR_INVALID_ARG;
  return forward_impl(x, w_gate, gate_bias, w1, w3, w2, T, H, F, E, top_k, capacity_factor, act,
                      dt, out, nullptr, nullptr, ws, ws_bytes, stream,
                      reinterpret_cast<cudaEvent_t const*>(events));
}

moe_status moe_forward_host(const void* x_host, const void* w_gate, const float* gate_bias,
                            const void* w1, const void* w3, const void* w2, int T, int H, int F,
                            int E, int top_k, float capacity_factor, moe_act act, moe_dtype dt,
                            void* out_host, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_common(T, H, E, top_k, dt);
  if (st != MOE_OK) return st;
  if (F <= 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x_host || !out_host || !ws) return MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(T, H, F, E, top_k, act, dt, true);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  const size_t bytes = static_cast<size_t>(T) * H * elem_bytes(dt);
  void* xd = at<void>(ws, L.x_stage);
  void* od = at<void>(ws, L.out_stage);
  if (cudaMemcpyAsync(xd, x_host, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  st = moe_forward(xd, w_gate, gate_bias, w1, w3, w2, T, H, F, E, top_k, capacity_factor, act, dt,
                   od, nullptr, nullptr, ws, L.x_stage, stream);
  if (st != MOE_OK) return st;
  return cuda_status(cudaMemcpyAsync(out_host, od, bytes, cudaMemcpyDeviceToHost, s));
}

// A run of independent batches with host x / out.  Device memory: the
// forward's own workspace, then two x stages and two out stages used in turn,
// so batch i's copy-in, batch i-1's layer and batch i-2's copy-out can run at
// the same time on three streams.  Seven events (created and destroyed here):
// `start` orders the copy streams after earlier work on `stream`; six order
// the reuse of each stage:
//   loaded[b]  copy-in of the batch in stage b done    -> its layer may start
//   done[b]    layer of the batch in stage b done       -> its copy-out may start,
//                                                          and stage b's x is free
//   drained[b] copy-out of the batch in stage b done    -> stage b's out is free
// cudaStreamWaitEvent binds to the event's latest record at the time of the
// call, and the host issues batch i's three steps in order, so each wait
// refers to the batch two steps earlier.
size_t moe_forward_host_batches_workspace_bytes(int T, int H, int F, int E, int top_k,
                                                moe_act act, moe_dtype dt) {
  if (T < 0 || H <= 0 || F <= 0 || E <= 0 || top_k <= 0) return 0;
  const size_t stage = align_up(static_cast<size_t>(T) * H * elem_bytes(dt));
  return ws_layout(T, H, F, E, top_k, act, dt, false).total + 4 * stage;
}

moe_status moe_forward_host_batches(const void* const* x_host, void* const* out_host,
                                    int n_batches, const void* w_gate, const float* gate_bias,
                                    const void* w1, const void* w3, const void* w2, int T, int H,
                                    int F, int E, int top_k, float capacity_factor, moe_act act,
                                    moe_dtype dt, void* ws, size_t ws_bytes,
                                    moe_stream_t stream, moe_stream_t copy_in,
                                    moe_stream_t copy_out) {
  moe_status st = check_common(T, H, E, top_k, dt);
  if (st != MOE_OK) return st;
  if (n_batches < 0 || F <= 0 || F % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (T == 0 || n_batches == 0) return MOE_OK;
  if (!x_host || !out_host || !ws) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n_batches; ++i)
    if (!x_host[i] || !out_host[i]) return MOE_ERR_INVALID_ARG;
  const size_t fwd = ws_layout(T, H, F, E, top_k, act, dt, false).total;
  const size_t bytes = static_cast<size_t>(T) * H * elem_bytes(dt);
  const size_t stage = align_up(bytes);
  void* xs[2] = {at<void>(ws, fwd), at<void>(ws, fwd + stage)};
  void* os[2] = {at<void>(ws, fwd + 2 * stage), at<void>(ws, fwd + 3 * stage)};
  // every check the batches' forwards will make, before anything is queued
  st = check_forward(xs[0], w_gate, w1, w3, w2, T, H, F, E, top_k, act, dt, os[0], ws, fwd, false);
  if (st != MOE_OK) return st;
  if (ws_bytes < fwd + 4 * stage) return MOE_ERR_WORKSPACE;
  cudaStream_t sc = as_stream(stream);
  cudaStream_t si = copy_in ? as_stream(copy_in) : sc;
  cudaStream_t so = copy_out ? as_stream(copy_out) : sc;

  cudaEvent_t ev[7] = {};  // start, loaded[2], done[2], drained[2]
  for (int i = 0; i < 7; ++i) {
    if (cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(ev[j]);
      return MOE_ERR_CUDA;
    }
  }
  cudaEvent_t start = ev[0], *loaded = ev + 1, *done = ev + 3, *drained = ev + 5;
  auto run = [&]() -> moe_status {
    // the copy streams start after everything already queued on `stream`
    if (cudaEventRecord(start, sc) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamWaitEvent(si, start, 0) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamWaitEvent(so, start, 0) != cudaSuccess) return MOE_ERR_CUDA;
    for (int i = 0; i < n_batches; ++i) {
      const int b = i & 1;
      if (i >= 2 && cudaStreamWaitEvent(si, done[b], 0) != cudaSuccess) return MOE_ERR_CUDA;
      if (cudaMemcpyAsync(xs[b], x_host[i], bytes, cudaMemcpyHostToDevice, si) != cudaSuccess)
        return MOE_ERR_CUDA;
      if (cudaEventRecord(loaded[b], si) != cudaSuccess) return MOE_ERR_CUDA;
      if (cudaStreamWaitEvent(sc, loaded[b], 0) != cudaSuccess) return MOE_ERR_CUDA;
      if (i >= 2 && cudaStreamWaitEvent(sc, drained[b], 0) != cudaSuccess) return MOE_ERR_CUDA;
      const moe_status s = moe_forward(xs[b], w_gate, gate_bias, w1, w3, w2, T, H, F, E, top_k,
                                       capacity_factor, act, dt, os[b], nullptr, nullptr, ws, fwd,
                                       stream);
      if (s != MOE_OK) return s;
      if (cudaEventRecord(done[b], sc) != cudaSuccess) return MOE_ERR_CUDA;
      if (cudaStreamWaitEvent(so, done[b], 0) != cudaSuccess) return MOE_ERR_CUDA;
      if (cudaMemcpyAsync(out_host[i], os[b], bytes, cudaMemcpyDeviceToHost, so) != cudaSuccess)
        return MOE_ERR_CUDA;
      if (cudaEventRecord(drained[b], so) != cudaSuccess) return MOE_ERR_CUDA;
    }
    return MOE_OK;
  };
  st = run();
  // `stream` ends after everything issued on the copy streams, also when a
  // step above failed part-way
  if (cudaEventRecord(loaded[0], si) != cudaSuccess ||
      cudaStreamWaitEvent(sc, loaded[0], 0) != cudaSuccess ||
      cudaEventRecord(drained[0], so) != cudaSuccess ||
      cudaStreamWaitEvent(sc, drained[0], 0) != cudaSuccess)
    st = st == MOE_OK ? MOE_ERR_CUDA : st;
  for (int i = 0; i < 7; ++i) cudaEventDestroy(ev[i]);  // released once their work completes
  return st;
}

moe_status moe_workspace_section(int T, int H, int F, int E, int top_k, moe_act act,
                                 moe_dtype dt, moe_ws_section which, size_t* offset,
                                 size_t* bytes) {
  if (dt != MOE_F32 && dt != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (act != MOE_ACT_SWIGLU && act != MOE_ACT_GELU && act != MOE_ACT_IDENTITY)
    return MOE_ERR_INVALID_ARG;
  if (T < 0 || H <= 0 || F <= 0 || E <= 0 || top_k <= 0 || !offset || !bytes)
    return MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(T, H, F, E, top_k, act, dt, false);
  const size_t R = static_cast<size_t>(T) * top_k;
  const size_t eb = elem_bytes(dt);
  switch (which) {
    case MOE_WS_TOPK_IDX: *offset = L.topk_idx; *bytes = R * 4; break;
    case MOE_WS_TOPK_GATE: *offset = L.topk_gate; *bytes = R * 4; break;
    case MOE_WS_COUNTS: *offset = L.counts; *bytes = static_cast<size_t>(E) * 4; break;
    case MOE_WS_OFFSETS: *offset = L.offsets; *bytes = static_cast<size_t>(E + 1) * 4; break;
    case MOE_WS_ROW_TOKEN: *offset = L.row_token; *bytes = R * 4; break;
    case MOE_WS_ROW_MAP: *offset = L.row_map; *bytes = R * 4; break;
    case MOE_WS_X_PERM: *offset = L.x_perm; *bytes = R * H * eb; break;
    case MOE_WS_H: *offset = L.h; *bytes = act == MOE_ACT_IDENTITY ? 0 : R * F * eb; break;
    case MOE_WS_Y: *offset = L.y; *bytes = R * H * eb; break;
    default: return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

moe_status moe_set_gemm_variant(int variant) {
  if (variant < 0 || variant > 4) return MOE_ERR_INVALID_ARG;
  moe::g_gemm_variant.store(variant, std::memory_order_relaxed);
  return MOE_OK;
}

moe_status moe_get_device_status(void* ws, moe_stream_t stream) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (v != 0 && cudaMemset(ws, 0, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  switch (v) {
    case 0: return MOE_OK;
    case MOE_ERR_INVALID_ARG: return MOE_ERR_INVALID_ARG;
    case MOE_ERR_INDEX_OUT_OF_RANGE: return MOE_ERR_INDEX_OUT_OF_RANGE;
    case MOE_ERR_TIMEOUT: return MOE_ERR_TIMEOUT;
    default: return MOE_ERR_CUDA;
  }
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_INDEX_OUT_OF_RANGE: return "MOE_ERR_INDEX_OUT_OF_RANGE";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_BOUNDS: return "MOE_ERR_BOUNDS";
  }
  return "MOE_ERR_UNKNOWN";
}

const char* moe_version(void) { return "moe_b200 0.1 sm_100a"; }

}  // extern "C"
