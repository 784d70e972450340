// Permute / dispatch: expert histogram, capacity clamp + offsets, and the
// stable scatter that gives every kept (token, slot) pair its expert-major row.
//
// lshu.cn torch_npu fused-operator article §4 (npu_moe_token_preprocess: token
// rearrangement), §5.2 (expert ids are int32 in [0, num_experts) — out-of-range
// ids are errors, never clamped), §5.3 (a fixed-size buffer per expert, which a
// skewed router overflows); hnwysp.cn ops-transformer MoE article §3.2
// (capacity_factor); "ops-transformer 仓库 - MoE 算子优化实战" (SparseGather,
// CSR storage of the sparse assignment).
//
// Pairs are ordered by a = t*k + s.  The tokens are cut into tiles of BT; the
// histogram gives per-tile counts; each scatter CTA scans them per expert for
// its own tile base (plus pre-drop counts, capacity clamp and offsets) and
// recomputes each pair's rank inside its tile with warp match/popc, so rank =
// tile base + rank in tile is the pair's arrival order among all pairs of
// that expert.
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kPermThreads = 256;

// Per-tile expert histogram of caller-given ids (the fused path gets it from
// the router).  Out-of-range ids are reported and not counted; with
// empty_slots, id -1 is an unused slot and is skipped silently.
__global__ void __launch_bounds__(kPermThreads) k_hist(PermuteArgs a) {
  __shared__ int cnt_s[kMaxE];
  pdl_wait_and_trigger();
  const int lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < a.E; i += kPermThreads) cnt_s[i] = 0;
  __syncthreads();
  const int a0 = blockIdx.x * a.BT * a.k;
  const int a1 = min(a.T, (blockIdx.x + 1) * a.BT) * a.k;
  for (int base = a0; base < a1; base += kPermThreads) {
    const int i = base + threadIdx.x;
    int e = -1;
    if (i < a1) {
      e = a.idx[i];
      if (e < 0 || e >= a.E) {
        if (!(a.empty_slots && e == -1)) record_status(a.status, kStatusIndexOutOfRange);
        e = -1;
      }
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) atomicAdd(&cnt_s[e], __popc(peers));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < a.E; i += kPermThreads)
    a.tile_counts[static_cast<size_t>(blockIdx.x) * a.E + i] = cnt_s[i];
}

// Stable scatter with the scan folded in.  CTA j handles pairs
// [j*BT*k, min(T,(j+1)*BT)*k) in rounds of 256.
//
// Prologue (every CTA, from the per-tile histogram): for each expert, the
// pairs routed to it in tiles before j (this tile's base), the total over all
// tiles (the pre-drop count), kept = min(count, C) and offsets = exclusive
// scan of kept over experts.  Thread (p, e) sums a contiguous run of tiles of
// expert e (consecutive threads read consecutive experts of a tile), then the
// runs are added in order; CTA 0 also writes counts and offsets.  Integer
// sums: every CTA gets the same values.
//
// Main loop: inside a round a pair's rank among same-expert pairs comes from
// __match_any_sync (rank in warp) plus an exclusive scan over warps, so
// rank = tile base + rank in tile is the pair's arrival order among all pairs
// of its expert.
constexpr int kScatterMaxPairs = 128 * kMaxTopK;

__global__ void __launch_bounds__(kPermThreads) k_scatter(PermuteArgs a) {
  __shared__ int wcnt[kPermThreads / 32][kMaxE];
  __shared__ int running[kMaxE];
  __shared__ int rows_s[kScatterMaxPairs];
  __shared__ int part_all[kPermThreads], part_before[kPermThreads];
  __shared__ int base_s[kMaxE], total_s[kMaxE], off_s[kMaxE];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = a.split > 0 ? a.split : 1;
  const int j = blockIdx.x / split, part = blockIdx.x % split;  // tile, share of its copies
  const int a0 = j * a.BT * a.k;
  const int a1 = min(a.T, (j + 1) * a.BT) * a.k;
  pdl_wait_and_trigger();

  {  // ---- scan prologue
    int Ep = 1;
    while (Ep < a.E) Ep <<= 1;
    const int P = kPermThreads / Ep;  // runs per expert (E <= 256)
    const int e = threadIdx.x % Ep, p = threadIdx.x / Ep;
    const int run = (a.tiles + P - 1) / P;
    const int j0 = p * run, j1 = min(a.tiles, j0 + run);
    int s_all = 0, s_before = 0;
    if (e < a.E)
      for (int jj = j0; jj < j1; ++jj) {
        const int v = a.tile_counts[static_cast<size_t>(jj) * a.E + e];
        s_all += v;
        if (jj < j) s_before += v;
      }
    part_all[threadIdx.x] = s_all;
    part_before[threadIdx.x] = s_before;
    __syncthreads();
    for (int ee = threadIdx.x; ee < a.E; ee += kPermThreads) {
      int tot = 0, bef = 0;
      for (int q = 0; q < P; ++q) {
        tot += part_all[q * Ep + ee];
        bef += part_before[q * Ep + ee];
      }
      total_s[ee] = tot;
      base_s[ee] = bef;
    }
    __syncthreads();
    if (warp == 0) {
      int acc = 0;
      for (int b = 0; b < a.E; b += 32) {
        const int ee = b + lane;
        const int kept = ee < a.E ? min(total_s[ee], a.cap) : 0;
        int incl = kept;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += u;
        }
        if (ee < a.E) {
          off_s[ee] = acc + incl - kept;
          if (blockIdx.x == 0) {
            a.counts[ee] = total_s[ee];
            a.offsets[ee] = acc + incl - kept;
          }
        }
        acc += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (blockIdx.x == 0 && lane == 0) a.offsets[a.E] = acc;
    }
  }
  for (int i = threadIdx.x; i < a.E; i += kPermThreads) running[i] = 0;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = a0; base < a1; base += kPermThreads) {
    for (int i = threadIdx.x; i < (kPermThreads / 32) * a.E; i += kPermThreads)
      wcnt[i / a.E][i % a.E] = 0;
    __syncthreads();
    const int i = base + threadIdx.x;
    int e = -1;
    if (i < a1) {
      e = a.idx[i];
      if (e < 0 || e >= a.E) e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank_w = __popc(peers & lt_mask);
    if (e >= 0 && lane == __ffs(peers) - 1) wcnt[warp][e] = __popc(peers);
    __syncthreads();
    for (int ee = threadIdx.x; ee < a.E; ee += kPermThreads) {
      int s = running[ee];
#pragma unroll
      for (int w = 0; w < kPermThreads / 32; ++w) {
        const int c = wcnt[w][ee];
        wcnt[w][ee] = s;
        s += c;
      }
      running[ee] = s;
    }
    __syncthreads();
    if (i < a1) {
      int row = -1;
      if (e >= 0) {
        const int rank = base_s[e] + wcnt[warp][e] + rank_w;
        if (rank < a.cap && MOE_DCHECK(off_s[e] + rank < a.T * a.k, a.status)) {
          row = off_s[e] + rank;
          if (part == 0) a.row_token[row] = i / a.k;
        }
      }
      if (part == 0) a.row_map[i] = row;
      rows_s[i - a0] = row;
    }
    __syncthreads();
  }
  if (a.x_perm == nullptr) return;
  // Gather the kept rows of x into x_perm: this CTA's share of the tile's
  // pairs, one warp per pair, 16-byte vectors.
  const int row_bytes = a.H * a.elem_bytes;
  const int vecs = row_bytes / 16;
  const int share = (a1 - a0 + split - 1) / split;
  const int p0 = a0 + part * share, p1 = min(a1, p0 + share);
  for (int p = p0 + warp; p < p1; p += kPermThreads / 32) {
    const int row = rows_s[p - a0];
    if (row < 0) continue;
    const int t = p / a.k;
    const int4* src = reinterpret_cast<const int4*>(static_cast<const uint8_t*>(a.x) +
                                                    static_cast<size_t>(t) * row_bytes);
    int4* dst = reinterpret_cast<int4*>(static_cast<uint8_t*>(a.x_perm) +
                                        static_cast<size_t>(row) * row_bytes);
    for (int v = lane; v < vecs; v += 32) dst[v] = __ldg(src + v);
  }
}

cudaError_t launch_hist(const PermuteArgs& a, cudaStream_t s) {
  return launch_kernel(k_hist, dim3(a.tiles), dim3(kPermThreads), 0, s, 1, a);
}

cudaError_t launch_scatter(const PermuteArgs& a, cudaStream_t s) {
  if (a.BT * a.k > kScatterMaxPairs) return cudaErrorInvalidValue;
  if (log_enabled())
    log_line("scatter T=%d k=%d E=%d: %d token tiles of %d, %d CTAs per tile, capacity %d%s", a.T,
             a.k, a.E, a.tiles, a.BT, a.split > 0 ? a.split : 1, a.cap,
             a.x_perm ? ", rows copied to x_perm" : "");
  return launch_kernel(k_scatter, dim3(a.tiles * (a.split > 0 ? a.split : 1)), dim3(kPermThreads),
                       0, s, 1, a);
}

__global__ void k_clear_status(int* status, int* counters, int n, int* counters2, int n2) {
  pdl_wait_and_trigger();
  if (blockIdx.x == 0 && threadIdx.x == 0) *status = 0;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    counters[i] = 0;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n2; i += gridDim.x * blockDim.x)
    counters2[i] = 0;
}

cudaError_t launch_clear_status(int* status, cudaStream_t s, int* counters, int n, int* counters2,
                                int n2) {
  return launch_kernel(k_clear_status, dim3(1), dim3(512), 0, s, 1, status, counters,
                       counters ? n : 0, counters2, counters2 ? n2 : 0);
}

}  // namespace moe
