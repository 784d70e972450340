// Deterministic weighted combine back to token order.
//
// "MoE模型高效推理：CANN算子库优化实践" §2.1 (the layer output is the sum of the
// gate-weighted expert outputs); "ops-transformer 仓库 - MoE 算子优化实战"
// (SparseScatterAdd); lshu.cn torch_npu article §4 (npu_moe_token_postprocess
// restores token order).  The pages aggregate with atomic adds (hnwysp.cn
// article §2.2, stage 3); here each token reads its own k rows and sums them in
// slot order, so the result is the same bit for bit on every run.
//
// One warp per token (or per part of a token's row when there are few tokens),
// 16-byte vector loads of each kept row, fp32 accumulation by FMA in slot
// order, one rounding to the storage type.  A null gate array
// means every weight is 1 (the unpermute of a k = 1 matmul: out[t] = y[row]).
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kCombineThreads = 256;

// One output vector: the kept slots' rows weighted by their gates, summed by
// FMA in slot order in fp32, rounded once to the storage type.
template <bool BF16>
__device__ __forceinline__ void combine_store(const int4 (&q)[kMaxTopK],
                                              const int (&rows)[kMaxTopK],
                                              const float (&g)[kMaxTopK], uint8_t* dst) {
  constexpr int EPV = BF16 ? 8 : 4;
  float acc[EPV];
#pragma unroll
  for (int i = 0; i < EPV; ++i) acc[i] = 0.f;
#pragma unroll
  for (int s = 0; s < kMaxTopK; ++s) {
    if (rows[s] < 0) continue;
    if constexpr (BF16) {
      const uint32_t w[4] = {static_cast<uint32_t>(q[s].x), static_cast<uint32_t>(q[s].y),
                             static_cast<uint32_t>(q[s].z), static_cast<uint32_t>(q[s].w)};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = fmaf(g[s], bf16_lo(w[i]), acc[2 * i]);
        acc[2 * i + 1] = fmaf(g[s], bf16_hi(w[i]), acc[2 * i + 1]);
      }
    } else {
      acc[0] = fmaf(g[s], __int_as_float(q[s].x), acc[0]);
      acc[1] = fmaf(g[s], __int_as_float(q[s].y), acc[1]);
      acc[2] = fmaf(g[s], __int_as_float(q[s].z), acc[2]);
      acc[3] = fmaf(g[s], __int_as_float(q[s].w), acc[3]);
    }
  }
  int4 o;
  if constexpr (BF16) {
    o.x = static_cast<int>(pack_bf16x2(acc[0], acc[1]));
    o.y = static_cast<int>(pack_bf16x2(acc[2], acc[3]));
    o.z = static_cast<int>(pack_bf16x2(acc[4], acc[5]));
    o.w = static_cast<int>(pack_bf16x2(acc[6], acc[7]));
  } else {
    o.x = __float_as_int(acc[0]);
    o.y = __float_as_int(acc[1]);
    o.z = __float_as_int(acc[2]);
    o.w = __float_as_int(acc[3]);
  }
  *reinterpret_cast<int4*>(dst) = o;
}

// Work item w (one warp): token w / split, and every split-th chunk of 64
// vectors of its row starting at chunk w % split (split > 1 when there are too
// few tokens to fill the GPU with warps).
template <bool BF16>
__global__ void __launch_bounds__(kCombineThreads)
    k_combine(const uint8_t* __restrict__ y, const float* __restrict__ gate,
              const int32_t* __restrict__ row_map, int T, int H, int k, int split,
              uint8_t* __restrict__ out, int* status) {
  pdl_wait_and_trigger();
  constexpr int EPV = BF16 ? 8 : 4;  // elements per 16-byte vector
  constexpr int EB = BF16 ? 2 : 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nvec = H / EPV;
  const long long items = static_cast<long long>(T) * split;
  for (long long w = static_cast<long long>(blockIdx.x) * (kCombineThreads / 32) + warp;
       w < items; w += static_cast<long long>(gridDim.x) * (kCombineThreads / 32)) {
    const int t = static_cast<int>(w / split);
    const int part = static_cast<int>(w % split);
    int rows[kMaxTopK];
    float g[kMaxTopK];
#pragma unroll
    for (int s = 0; s < kMaxTopK; ++s) {
      rows[s] = s < k ? __ldg(row_map + static_cast<size_t>(t) * k + s) : -1;
      // y has the T x k rows of the permute's layout
      if (rows[s] >= 0 && !MOE_DCHECK(rows[s] < T * k, status)) rows[s] = -1;
      g[s] = s < k ? (gate ? __ldg(gate + static_cast<size_t>(t) * k + s) : 1.f) : 0.f;
    }
    // two 16-byte vectors per lane and round: every load of both is in flight
    // before the first FMA
    for (int v0 = part * 64 + lane; v0 < nvec; v0 += 64 * split) {
      const int v1 = v0 + 32;
      const bool two = v1 < nvec;
      int4 qa[kMaxTopK], qb[kMaxTopK];
#pragma unroll
      for (int s = 0; s < kMaxTopK; ++s) {
        qa[s] = make_int4(0, 0, 0, 0);
        qb[s] = make_int4(0, 0, 0, 0);
        if (rows[s] < 0) continue;
        const uint8_t* yr = y + static_cast<size_t>(rows[s]) * H * EB;
        qa[s] = __ldg(reinterpret_cast<const int4*>(yr + static_cast<size_t>(v0) * EPV * EB));
        if (two)
          qb[s] = __ldg(reinterpret_cast<const int4*>(yr + static_cast<size_t>(v1) * EPV * EB));
      }
      combine_store<BF16>(qa, rows, g,
                          out + (static_cast<size_t>(t) * H + static_cast<size_t>(v0) * EPV) * EB);
      if (two)
        combine_store<BF16>(qb, rows, g,
                            out + (static_cast<size_t>(t) * H + static_cast<size_t>(v1) * EPV) * EB);
    }
  }
}

cudaError_t launch_combine(const void* y, const float* gate, const int32_t* row_map, int T,
                           int H, int k, int dt_bf16, void* out, int num_sms, cudaStream_t s,
                           int* status) {
  const int warps_per_cta = kCombineThreads / 32;
  // split a row over several warps when the tokens alone leave the GPU short
  // of warps (about 32 per SM keep enough loads in flight)
  const int chunks = (H / (dt_bf16 ? 8 : 4) + 63) / 64;
  int split = (num_sms * 32) / (T > 0 ? T : 1);
  if (split > chunks) split = chunks;
  if (split < 1) split = 1;
  const long long items = static_cast<long long>(T) * split;
  long long grid = (items + warps_per_cta - 1) / warps_per_cta;
  const long long cap = static_cast<long long>(num_sms) * 8;  // resident CTAs; more loop inside
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  if (log_enabled())
    log_line("combine T=%d H=%d k=%d: %d warp(s) per token row, %lld CTAs", T, H, k, split, grid);
  if (dt_bf16)
    return launch_kernel(k_combine<true>, dim3(static_cast<unsigned>(grid)), dim3(kCombineThreads),
                         0, s, 1, static_cast<const uint8_t*>(y), gate, row_map, T, H, k, split,
                         static_cast<uint8_t*>(out), status);
  return launch_kernel(k_combine<false>, dim3(static_cast<unsigned>(grid)), dim3(kCombineThreads),
                       0, s, 1, static_cast<const uint8_t*>(y), gate, row_map, T, H, k, split,
                       static_cast<uint8_t*>(out), status);
}

}  // namespace moe
