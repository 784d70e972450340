// moe_permute_noalloc: the permute/dispatch step for callers that cannot
// allocate device memory.
//
// Some hosts of this library are not allowed to call cudaMalloc or to hand out
// a workspace: an inference-engine plugin whose enqueue step must run on
// memory the engine planned before the model started, a serving process that
// reserved its whole device budget up front, or a real-time loop where
// cudaMalloc's implicit device-wide synchronisation is not acceptable.  For
// them this entry point keeps its scratch (the status word and the per-tile
// expert histogram that the scan turns into tile bases) in a fixed array in
// device global memory that the library owns.  The caller still passes every
// input and output buffer.
//
// Cost and limits:
//  * the array (kScratchBytes = 1 MiB) is part of the library image, so every
//    GPU that loads the library holds it until the process exits;
//  * ceil(T / 128) * E must not exceed kScratchInts - kTileCountsAt (262080):
//    e.g. T <= 4,193,280 tokens with 8 experts, T <= 130,944 with 256 experts.
//    Larger calls are rejected with MOE_ERR_UNSUPPORTED before any launch;
//  * the array is shared by every call on a device and keeps the last call's
//    contents: each call clears the status word it uses and rewrites every
//    histogram entry it reads, but two calls whose kernels overlap on the GPU
//    (for example on two streams without an ordering between them) race on it.
//
// The device address of the array is looked up once per device, with that
// device current, by the first call on it (cudaGetSymbolAddress); make that
// first call before any stream capture.  The address belongs to the device's
// current context: a call that finds another context current (after
// cudaDeviceReset, or once the primary context was released and created
// again) looks it up again, so make the first call after such a reset before
// any stream capture too.
#include <cuda.h>

#include <cmath>
#include <mutex>

#include "kernels.h"
#include "moe_b200.h"

using namespace moe;

namespace {

constexpr size_t kScratchBytes = size_t(1) << 20;
constexpr int kScratchInts = static_cast<int>(kScratchBytes / sizeof(int));
constexpr int kTileCountsAt = 64;  // ints; element 0 is the status word

static __device__ __align__(256) int g_permute_scratch[kScratchInts];

constexpr int kMaxDevices = 64;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The context current on this thread (driver entry point; null if unavailable).
CUcontext current_context() {
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrentFn>(p);
    return static_cast<CtxGetCurrentFn>(nullptr);
  }();
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of g_permute_scratch on the current device, looked up on the
// first call with the device's current context (and again if that context
// changed since).
int* scratch_on_current_device(cudaError_t* err) {
  static std::mutex mu;
  static int* addr[kMaxDevices] = {};
  static CUcontext ctx_of[kMaxDevices] = {};
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  const CUcontext ctx = current_context();
  if (addr[dev] == nullptr || ctx != ctx_of[dev]) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_permute_scratch);
    if (*err != cudaSuccess) return nullptr;
    addr[dev] = static_cast<int*>(p);
    ctx_of[dev] = current_context();  // the runtime call made the primary context current
  }
  return addr[dev];
}

}  // namespace

extern "C" moe_status moe_permute_noalloc(const void* x, const int32_t* token_expert_idx, int T,
                                          int H, int E, int top_k, float capacity_factor,
                                          moe_dtype dt, void* x_perm, int32_t* expert_counts,
                                          int32_t* expert_offsets, int32_t* row_token,
                                          int32_t* row_map, int32_t* status_out,
                                          moe_stream_t stream) {
  if (dt != MOE_F32 && dt != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (T < 0 || H <= 0 || E <= 0 || top_k <= 0 || top_k > E || H % 8 != 0)
    return MOE_ERR_INVALID_ARG;
  if (E > kMaxE || top_k > kMaxTopK) return MOE_ERR_UNSUPPORTED;
  if (!token_expert_idx || !expert_counts || !expert_offsets || !row_token || !row_map)
    return MOE_ERR_INVALID_ARG;
  const int eb = dt == MOE_BF16 ? 2 : 4;
  if (x_perm && (!x || (reinterpret_cast<uintptr_t>(x) & 15u) ||
                 (reinterpret_cast<uintptr_t>(x_perm) & 15u)))
    return MOE_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * top_k * H >= (1LL << 31)) return MOE_ERR_UNSUPPORTED;
  const int tiles = (T + kPermuteBT - 1) / kPermuteBT;
  if (static_cast<long long>(tiles) * E > kScratchInts - kTileCountsAt) return MOE_ERR_UNSUPPORTED;

  cudaError_t err;
  int* scratch = scratch_on_current_device(&err);
  if (scratch == nullptr) return MOE_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* status = status_out ? status_out : scratch;
  if (launch_clear_status(status, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (T == 0) {
    if (cudaMemsetAsync(expert_counts, 0, static_cast<size_t>(E) * 4, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    return cudaMemsetAsync(expert_offsets, 0, static_cast<size_t>(E + 1) * 4, s) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
  }
  PermuteArgs p{};
  p.idx = token_expert_idx;
  p.T = T;
  p.k = top_k;
  p.E = E;
  p.BT = kPermuteBT;
  p.tiles = tiles;
  // as moe_permute: enough CTAs per tile to spread the x_perm copies (only the
  // grid changes; the scratch holds one histogram row per tile either way)
  p.split = 1;
  if (x_perm) {
    int nsm = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      nsm = 148;
    while (p.split < 16 && tiles * p.split < 2 * nsm) p.split *= 2;
  }
  if (capacity_factor > 0.f) {  // C = ceil(cf * T * k / E), at least 1
    const double c =
        std::ceil(static_cast<double>(capacity_factor) * static_cast<double>(T) * top_k / E);
    p.cap = c >= 2147483647.0 ? INT32_MAX : (c < 1.0 ? 1 : static_cast<int>(c));
  } else {
    p.cap = INT32_MAX;
  }
  p.tile_counts = scratch + kTileCountsAt;  // every entry read below is written by k_hist first
  p.counts = expert_counts;
  p.offsets = expert_offsets;
  p.row_token = row_token;
  p.row_map = row_map;
  p.x = x;
  p.x_perm = x_perm;
  p.H = H;
  p.elem_bytes = eb;
  p.status = status;
  if (launch_hist(p, s) != cudaSuccess) return MOE_ERR_CUDA;
  return launch_scatter(p, s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
