// Router load statistics: per-expert assignment counts and the mean router
// probability over tokens, the two per-expert quantities a load-balancing
// auxiliary loss is built from.
//
// "ops-transformer 仓库 - MoE 算子优化实战", "实战中的坑与解法" (collect each
// expert's utilisation periodically against overloaded experts) and lshu.cn
// torch_npu fused-operator article §5.3 (--moe-aux-loss-coeff 0.01 against
// expert overload) name the per-expert load and an auxiliary load-balancing
// loss but not its formula, so only the statistics are produced:
//   count[e]     = #{(t,s): topk_idx[t,s] = e}            (pre-drop)
//   prob_mean[e] = (1/T) sum_t softmax(logits[t])[e]     (softmax over all E)
// Both reductions run in a fixed order (tokens within a tile, then tiles), so
// the result is the same bit for bit on every run.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kStatsThreads = 256;
constexpr int kStatsWarps = kStatsThreads / 32;

// One CTA per kStatsBT tokens: warp w takes tokens w, w+8, ... in order; lane j
// holds experts j, j+32, ...; a warp butterfly gives each token's max and
// denominator; each warp accumulates its tokens' probabilities in registers;
// the 8 warp partials are summed in warp order into tile_prob[tile][e].
__global__ void __launch_bounds__(kStatsThreads)
    k_route_prob_tiles(const float* __restrict__ logits, int T, int E, float* __restrict__ tile_prob) {
  __shared__ float part[kStatsWarps][kMaxE];
  pdl_wait_and_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kStatsBT;
  float acc[kMaxE / 32];
#pragma unroll
  for (int j = 0; j < kMaxE / 32; ++j) acc[j] = 0.f;
  for (int lt = warp; lt < kStatsBT; lt += kStatsWarps) {
    const int t = t0 + lt;
    if (t >= T) break;
    const float* l = logits + static_cast<size_t>(t) * E;
    float v[kMaxE / 32];
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < kMaxE / 32; ++j) {
      const int e = lane + 32 * j;
      v[j] = e < E ? l[e] : -INFINITY;
      mx = fmaxf(mx, v[j]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxE / 32; ++j) {
      const int e = lane + 32 * j;
      v[j] = e < E ? expf(v[j] - mx) : 0.f;
      sum += v[j];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    const float inv = 1.f / sum;
#pragma unroll
    for (int j = 0; j < kMaxE / 32; ++j) acc[j] += v[j] * inv;
  }
#pragma unroll
  for (int j = 0; j < kMaxE / 32; ++j) {
    const int e = lane + 32 * j;
    if (e < E) part[warp][e] = acc[j];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kStatsThreads) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kStatsWarps; ++w) s += part[w][e];
    tile_prob[static_cast<size_t>(blockIdx.x) * E + e] = s;
  }
}

// One CTA per expert: thread i sums tiles i, i + 256, ... in order, then a
// fixed tree over the 256 partial sums (the same order on every run).
__global__ void __launch_bounds__(kStatsThreads)
    k_route_stats_reduce(const int* __restrict__ tile_counts, int count_tiles,
                         const float* __restrict__ tile_prob, int prob_tiles, int T, int E,
                         int32_t* __restrict__ counts, float* __restrict__ prob_mean) {
  __shared__ int cs[kStatsThreads];
  __shared__ float ps[kStatsThreads];
  pdl_wait_and_trigger();
  const int e = blockIdx.x;
  int c = 0;
  float p = 0.f;
  for (int j = threadIdx.x; j < count_tiles; j += kStatsThreads)
    c += tile_counts[static_cast<size_t>(j) * E + e];
  for (int j = threadIdx.x; j < prob_tiles; j += kStatsThreads)
    p += tile_prob[static_cast<size_t>(j) * E + e];
  cs[threadIdx.x] = c;
  ps[threadIdx.x] = p;
  __syncthreads();
  for (int w = kStatsThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) {
      cs[threadIdx.x] += cs[threadIdx.x + w];
      ps[threadIdx.x] += ps[threadIdx.x + w];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    if (counts) counts[e] = cs[0];
    if (prob_mean) prob_mean[e] = ps[0] / static_cast<float>(T);
  }
}

cudaError_t launch_route_stats(const float* logits, const int* tile_counts, int count_tiles, int T,
                               int E, float* tile_prob, int32_t* counts, float* prob_mean,
                               cudaStream_t s) {
  const int prob_tiles = (T + kStatsBT - 1) / kStatsBT;
  cudaError_t err = launch_kernel(k_route_prob_tiles, dim3(prob_tiles), dim3(kStatsThreads), 0, s,
                                  1, logits, T, E, tile_prob);
  if (err != cudaSuccess) return err;
  return launch_kernel(k_route_stats_reduce, dim3(E), dim3(kStatsThreads), 0, s, 1, tile_counts,
                       count_tiles,
                       static_cast<const float*>(tile_prob), prob_tiles, T, E, counts, prob_mean);
}

}  // namespace moe
