// Router: logits = x @ W_gate (+ bias), top-k selection, renormalised gates,
// and the per-tile expert histogram that the permute step scans.
//
// "MoE模型高效推理：CANN算子库优化实践" §2.1 (gates = softmax(x @ W_gate); top-2),
// §3.2.1 (renormalise the kept gates); "ops-transformer 算子精讲" ch.8
// (normalize_scores=True).  The gates use the identity
//   softmax_s / sum_{kept} softmax = exp(l_s - l_0) / sum_j exp(l_j - l_0),
// so the full softmax over E is never formed.
//
// This file holds the selection epilogue shared with logits given by the
// caller, and the CUDA-core router used for fp32 storage or expert counts that
// are not a multiple of 8; bf16 routing runs on the tensor cores (route_tc.cu).
#include <cstdlib>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kRouteThreads = 256;

// ----------------------------------------------------------------------------
// Shared epilogue: top-k + gates for the CTA's tokens, then a warp-aggregated
// histogram of the chosen experts into tile_counts[tile][E].
// logits_s: [BT][ls_stride] fp32 (bias not yet added).
// ----------------------------------------------------------------------------
__device__ void route_select_and_count(const float* logits_s, int ls_stride, int BT, int token0,
                                       const RouteArgs& a, int tile, int* sel_s, int* cnt_s) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int k = a.top_k, E = a.E;
  const int per_lane = (E + 31) >> 5;  // <= 8

  for (int i = threadIdx.x; i < E; i += blockDim.x) cnt_s[i] = 0;

  for (int lt = warp; lt < BT; lt += nwarps) {
    const int t = token0 + lt;
    if (t >= a.T) {
      if (lane < k) sel_s[lt * k + lane] = -1;
      continue;
    }
    float v[8];
    int taken = 0;  // bit j: value j of this lane already selected
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      float x = 0.f;
      if (j < per_lane && e < E) {
        x = logits_s[lt * ls_stride + e];
        if (a.bias) x += a.bias[e];
        if (a.logits_out) a.logits_out[static_cast<size_t>(t) * E + e] = x;
      }
      v[j] = x;
    }
    float sv[8];
    int si[8];
    for (int s = 0; s < k; ++s) {
      // best not-yet-taken value of this lane
      float bv = 0.f;
      int bi = -1;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int e = lane + 32 * j;
        if (j < per_lane && e < E && !(taken & (1 << j))) {
          if (bi < 0 || ranks_before(v[j], e, bv, bi)) { bv = v[j]; bi = e; }
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        if (oi >= 0 && (bi < 0 || ranks_before(ov, oi, bv, bi))) { bv = ov; bi = oi; }
      }
      if (bi >= 0 && (bi & 31) == lane) taken |= 1 << (bi >> 5);
      sv[s] = bv;
      si[s] = bi;
    }
    if (lane == 0) {
      float z[8], sum = 0.f;
      for (int s = 0; s < k; ++s) { z[s] = expf(sv[s] - sv[0]); sum += z[s]; }
      for (int s = 0; s < k; ++s) {
        a.topk_idx[static_cast<size_t>(t) * k + s] = si[s];
        a.topk_gate[static_cast<size_t>(t) * k + s] = z[s] / sum;
        sel_s[lt * k + s] = si[s];
      }
    }
  }
  __syncthreads();
  if (a.tile_counts == nullptr) return;
  // Warp-aggregated histogram: one shared atomic per distinct expert per warp.
  const int n = BT * k;
  for (int base = warp * 32; base < n; base += nwarps * 32) {
    const int i = base + lane;
    int e = i < n ? sel_s[i] : -1;
    if (e >= 0 && !MOE_DCHECK(e < E, a.status)) e = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) atomicAdd(&cnt_s[e], __popc(peers));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += blockDim.x)
    a.tile_counts[static_cast<size_t>(tile) * E + i] = cnt_s[i];
}

// ----------------------------------------------------------------------------
// SIMT router (fp32 storage, or bf16 with an expert count that is not a
// multiple of 8).  One warp per token; lane l takes h = l, l + 32, ... (x read
// coalesced), experts in chunks of 8 accumulated per lane, then a warp
// butterfly per chunk (fixed order: deterministic).
// ----------------------------------------------------------------------------
constexpr int kSimtBT = 32;

template <typename Tin>
__device__ __forceinline__ float to_f(Tin v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

template <typename Tin>
__global__ void __launch_bounds__(kRouteThreads) k_route_simt(RouteArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int E_STR = a.E;
  float* lg = reinterpret_cast<float*>(smem);                       // [BT][E]
  int* sel_s = reinterpret_cast<int*>(lg + kSimtBT * E_STR);        // [BT][8]
  int* cnt_s = sel_s + kSimtBT * 8;                                 // [256]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int token0 = blockIdx.x * kSimtBT;
  pdl_wait_and_trigger();
  const Tin* x = static_cast<const Tin*>(a.x);
  const Tin* wg = static_cast<const Tin*>(a.wg);
  for (int lt = warp; lt < kSimtBT; lt += kRouteThreads / 32) {
    const int t = token0 + lt;
    if (t >= a.T) continue;
    const Tin* xr = x + static_cast<size_t>(t) * a.H;
    for (int e0 = 0; e0 < a.E; e0 += 8) {
      float acc[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = 0.f;
      for (int h = lane; h < a.H; h += 32) {
        const float xv = to_f<Tin>(xr[h]);
        const Tin* wr = wg + static_cast<size_t>(h) * a.E + e0;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (e0 + j < a.E) acc[j] = fmaf(xv, to_f<Tin>(wr[j]), acc[j]);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float v = acc[j];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == j && e0 + j < a.E) lg[lt * E_STR + e0 + j] = v;
      }
    }
  }
  __syncthreads();
  route_select_and_count(lg, E_STR, kSimtBT, token0, a, blockIdx.x, sel_s, cnt_s);
}

// Selection from caller-given fp32 logits.
__global__ void __launch_bounds__(kRouteThreads) k_route_from_logits(RouteArgs a,
                                                                     const float* logits) {
  extern __shared__ __align__(16) uint8_t smem[];
  float* lg = reinterpret_cast<float*>(smem);
  int* sel_s = reinterpret_cast<int*>(lg + kSimtBT * a.E);
  int* cnt_s = sel_s + kSimtBT * 8;
  const int token0 = blockIdx.x * kSimtBT;
  pdl_wait_and_trigger();
  for (int i = threadIdx.x; i < kSimtBT * a.E; i += kRouteThreads) {
    const int t = token0 + i / a.E;
    lg[i] = t < a.T ? logits[static_cast<size_t>(token0) * a.E + i] : 0.f;
  }
  __syncthreads();
  route_select_and_count(lg, a.E, kSimtBT, token0, a, blockIdx.x, sel_s, cnt_s);
}

// ----------------------------------------------------------------------------
// Host side: plan and launch
// ----------------------------------------------------------------------------
RoutePlan route_plan(int T, int H, int E, int dt_bf16, int num_sms, bool can_split) {
  RoutePlan p{};
  if (!dt_bf16 || (E % 8) != 0) {
    p.kind = 0;
    p.BT = kSimtBT;
    p.tiles = (T + kSimtBT - 1) / kSimtBT;
    p.ck = 1;
    return p;
  }
  p.kind = 2;
  p.NPAD = E <= 64 ? 64 : (E <= 128 ? 128 : 256);
  p.BT = 128;
  p.tiles = (T + 127) / 128;
  // split H over more CTAs while the token tiles leave SMs idle (needs workspace)
  const int num_kb = (H + 63) / 64;
  p.ck = 1;
  if (can_split)
    while (p.ck < 16 && p.tiles * p.ck * 2 <= kRouteMaxCtas && p.tiles * p.ck * 2 <= num_sms &&
           num_kb >= 4 * p.ck)
      p.ck *= 2;
  // a cap on the split (measurement aid)
  const int cap = tuning().route_split_cap;
  while (cap >= 1 && p.ck > cap) p.ck >>= 1;
  return p;
}

cudaError_t launch_route(const RouteArgs& a, const RoutePlan& p, cudaStream_t s) {
  if (log_enabled())
    log_line("router T=%d H=%d E=%d k=%d: %s, %d token tiles of %d, H split over %d CTAs%s", a.T,
             a.H, a.E, a.top_k, p.kind == 2 ? "tensor cores" : "CUDA cores", p.tiles, p.BT,
             p.kind == 2 ? p.ck : 1, p.kind == 2 ? ", experts padded to the MMA's N" : "");
  if (p.kind == 2) return launch_route_tc(a, p, s);
  const size_t smem = (kSimtBT * a.E + kSimtBT * 8 + 256) * 4;
  if (a.dt_bf16)
    return launch_kernel(k_route_simt<__nv_bfloat16>, dim3(p.tiles), dim3(kRouteThreads), smem, s,
                         1, a);
  return launch_kernel(k_route_simt<float>, dim3(p.tiles), dim3(kRouteThreads), smem, s, 1, a);
}

cudaError_t launch_route_from_logits(const RouteArgs& a, const float* logits, cudaStream_t s) {
  const int tiles = (a.T + kSimtBT - 1) / kSimtBT;
  const size_t smem = (kSimtBT * a.E + kSimtBT * 8 + 256) * 4;
  return launch_kernel(k_route_from_logits, dim3(tiles), dim3(kRouteThreads), smem, s, 1, a, logits);
}

}  // namespace moe
