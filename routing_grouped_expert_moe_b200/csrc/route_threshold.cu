// Threshold gating: a variable number of experts per token.
//
// "MoE模型高效推理：CANN算子库优化实践" §3.2.1 (sparse gate computation): compute
// every expert's gate score, keep only the experts whose score exceeds delta
// (by default delta = 1 / number of experts), and renormalise the kept ones.
// The scores are the softmax over all E experts of the fp32 router logits
// (§2.1).  Readings where the page is silent: the kept experts are ordered
// largest first (ties to the lower id), at most k_max of them are kept (the
// slot count the caller sizes its buffers for), and when no expert exceeds
// delta the largest one alone is kept, so the renormalisation is defined.
// Gates: g_s = exp(l_s - l_0) / sum_{kept j} exp(l_j - l_0), which equals
// p_s / sum_{kept} p.  Unused slots hold id -1 and gate 0.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kThrThreads = 256;
constexpr int kThrWarps = kThrThreads / 32;

// One warp per token; lane j holds experts j, j+32, ...
__global__ void __launch_bounds__(kThrThreads)
    k_route_threshold(const float* __restrict__ logits, int T, int E, int k_max, float delta,
                      int32_t* __restrict__ idx, float* __restrict__ gate,
                      int32_t* __restrict__ n_sel) {
  pdl_wait_and_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kThrWarps + warp;
  if (t >= T) return;
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
  for (int j = 0; j < kMaxE / 32; ++j)  // a NaN logit has no probability mass
    if (lane + 32 * j < E && !isnan(v[j])) sum += expf(v[j] - mx);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);

  int taken = 0;  // bit j: this lane's expert lane + 32 j already kept
  int n = 0;
  int sel[kMaxTopK];
  float sl[kMaxTopK];
  for (int s = 0; s < k_max; ++s) {
    float bv = 0.f;
    int bi = -1;
#pragma unroll
    for (int j = 0; j < kMaxE / 32; ++j) {
      const int e = lane + 32 * j;
      if (e < E && !(taken & (1 << j)) && (bi < 0 || ranks_before(v[j], e, bv, bi))) {
        bv = v[j];
        bi = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (oi >= 0 && (bi < 0 || ranks_before(ov, oi, bv, bi))) { bv = ov; bi = oi; }
    }
    if (bi < 0) break;
    const float p = expf(bv - mx) / sum;
    if (s > 0 && !(p > delta)) break;  // the largest is always kept
    if ((bi & 31) == lane) taken |= 1 << (bi >> 5);
    sel[n] = bi;
    sl[n] = bv;
    ++n;
  }
  if (lane == 0) {
    float z[kMaxTopK], zs = 0.f;
    for (int s = 0; s < n; ++s) { z[s] = expf(sl[s] - sl[0]); zs += z[s]; }
    for (int s = 0; s < k_max; ++s) {
      idx[static_cast<size_t>(t) * k_max + s] = s < n ? sel[s] : -1;
      gate[static_cast<size_t>(t) * k_max + s] = s < n ? z[s] / zs : 0.f;
    }
    if (n_sel) n_sel[t] = n;
  }
}

// Exclusive prefix sum of n[0..T) into out[0..T] (out[T] = total), one CTA:
// thread i sums a contiguous run, a block scan over the runs, then the runs
// are written.  Integer arithmetic: order does not matter.
constexpr int kScanT = 1024;
__global__ void __launch_bounds__(kScanT)
    k_token_offsets(const int32_t* __restrict__ n, int T, int32_t* __restrict__ out) {
  __shared__ int part[kScanT];
  pdl_wait_and_trigger();
  const int per = (T + kScanT - 1) / kScanT;
  const int b = threadIdx.x * per, e = min(T, b + per);
  int s = 0;
  for (int i = b; i < e; ++i) s += n[i];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int off = 1; off < kScanT; off <<= 1) {  // Hillis-Steele inclusive scan
    const int add = threadIdx.x >= off ? part[threadIdx.x - off] : 0;
    __syncthreads();
    part[threadIdx.x] += add;
    __syncthreads();
  }
  int run = part[threadIdx.x] - s;  // exclusive base of this run
  for (int i = b; i < e; ++i) {
    out[i] = run;
    run += n[i];
  }
  if (threadIdx.x == kScanT - 1) out[T] = part[kScanT - 1];
}

cudaError_t launch_route_threshold(const float* logits, int T, int E, int k_max, float delta,
                                   int32_t* idx, float* gate, int32_t* n_sel,
                                   int32_t* token_offsets, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  cudaError_t err = launch_kernel(k_route_threshold, dim3((T + kThrWarps - 1) / kThrWarps),
                                  dim3(kThrThreads), 0, s, 1, logits, T, E, k_max, delta, idx,
                                  gate, n_sel);
  if (err != cudaSuccess || token_offsets == nullptr) return err;
  if (n_sel == nullptr) return cudaErrorInvalidValue;
  return launch_kernel(k_token_offsets, dim3(1), dim3(kScanT), 0, s, 1,
                       static_cast<const int32_t*>(n_sel), T, token_offsets);
}

}  // namespace moe
