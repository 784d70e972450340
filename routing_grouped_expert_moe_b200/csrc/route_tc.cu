// Router on the tensor cores: logits = x @ W_gate (+ bias) with tcgen05, then
// top-k, renormalised gates and the per-tile expert histogram.
//
// "MoE模型高效推理：CANN算子库优化实践" §2.1 (gates = softmax(x @ W_gate), pick the
// top-2) and §3.2.1 (renormalise the kept gates); "ops-transformer 算子精讲" ch.8
// (normalize_scores=True).  Gates use softmax_s / sum_kept softmax =
// exp(l_s - l_0) / sum_j exp(l_j - l_0), so the full softmax is never formed.
//
// One CTA owns 128 tokens.  A = x rows (K-major, 128-byte swizzle, 2-D TMA
// boxes of 128 x 64); B = W_gate [H, E] read as-is, MN-major: TMA boxes of 64
// experts x 64 rows of H, experts beyond E zero-filled, so the MMA has
// N = NPAD = 64, 128 or 256.  The fp32 logits land in TMEM with one token per
// lane, so each epilogue thread owns one token's logit row and selects its
// top-k by insertion (larger logit first, NaN last, ties to the lower expert
// id) with a branch-free insertion over 64-bit order keys.  Reading x is the
// cost (H*2 bytes per token); the MMA work, even padded, stays well below it.
// When there are fewer token tiles than SMs, H is split over S independent
// CTAs: each writes its partial logits to the workspace, and the last CTA of
// the tile to finish (an atomic ticket) sums all S partials in rank order —
// deterministic whichever CTA is last — then selects.
#include <climits>
#include <cstdlib>

#include "gemm_common.cuh"

namespace moe {

constexpr int R_BT = 128;          // tokens per CTA
constexpr int R_THREADS = 192;     // producer, MMA, 4 epilogue warps
constexpr int R_A_BYTES = R_BT * 64 * 2;

// DEEP: one CTA per SM (token tiles x H splits fit on the SMs), so the ring
// takes ~192 KB and keeps twice the bytes in flight; otherwise ~96 KB so two
// CTAs share an SM.
template <int NPAD, bool DEEP>
struct RouteTcCfg {
  static constexpr int B_BYTES = NPAD * 64 * 2;
  static constexpr int STAGE_BYTES = R_A_BYTES + B_BYTES;
  static constexpr int STAGES = (NPAD == 64 ? 4 : (NPAD == 128 ? 3 : 2)) * (DEEP ? 2 : 1);
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = NPAD;
};

// Total-order selection key: larger logit first, NaN below everything (even
// -inf), equal logits to the lower expert id.  High word: the float's bits
// mapped to an order-preserving unsigned integer (-0 folded onto +0, NaN to 0);
// low word: ~e.  A larger key ranks first.
__device__ __forceinline__ unsigned long long select_key(float v, int e) {
  v = v + 0.0f;  // -0 -> +0
  const int b = __float_as_int(v);
  int o = b >= 0 ? b : (b ^ 0x7FFFFFFF);
  if (isnan(v)) o = INT_MIN;
  return (static_cast<unsigned long long>(static_cast<uint32_t>(o) ^ 0x80000000u) << 32) |
         static_cast<uint32_t>(0xFFFFFFFFu - static_cast<uint32_t>(e));
}

__device__ __forceinline__ float key_value(unsigned long long key) {
  const int o = static_cast<int>(static_cast<uint32_t>(key >> 32) ^ 0x80000000u);
  return __int_as_float(o >= 0 ? o : (o ^ 0x7FFFFFFF));
}

__device__ __forceinline__ int key_expert(unsigned long long key) {
  return static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(key));
}

// Keep the K largest keys, sorted (branch-free insertion).
template <int K>
__device__ __forceinline__ void topk_push(unsigned long long (&best)[K], unsigned long long key) {
#pragma unroll
  for (int j = 0; j < K; ++j) {
    const unsigned long long hi = best[j] > key ? best[j] : key;
    key = best[j] > key ? key : best[j];
    best[j] = hi;
  }
}

__device__ __forceinline__ void epi_bar() {  // the 4 epilogue warps only
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

// Gates, outputs and the tile histogram for one token (one epilogue thread).
template <int K>
__device__ __forceinline__ void route_tc_finish(const RouteArgs& a, int tile, int t, int lane,
                                                int et, const unsigned long long (&best)[K],
                                                int* cnt_s) {
  const bool valid = t < a.T;
  if (valid) {
    const float l0 = key_value(best[0]);
    float z[K], sum = 0.f;
#pragma unroll
    for (int s = 0; s < K; ++s)
      if (s < a.top_k) { z[s] = expf(key_value(best[s]) - l0); sum += z[s]; }
#pragma unroll
    for (int s = 0; s < K; ++s)
      if (s < a.top_k && MOE_DCHECK(key_expert(best[s]) < a.E, a.status)) {
        a.topk_idx[static_cast<size_t>(t) * a.top_k + s] = key_expert(best[s]);
        a.topk_gate[static_cast<size_t>(t) * a.top_k + s] = z[s] / sum;
      }
  }
  if (a.tile_counts == nullptr) return;
  // warp-aggregated histogram: one shared atomic per distinct expert per warp and slot
#pragma unroll
  for (int s = 0; s < K; ++s) {
    if (s >= a.top_k) break;
    const int e = valid ? key_expert(best[s]) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) atomicAdd(&cnt_s[e], __popc(peers));
  }
  epi_bar();
  for (int i = et; i < a.E; i += 128)
    a.tile_counts[static_cast<size_t>(tile) * a.E + i] = cnt_s[i];
}

template <int NPAD, int K, bool DEEP>
__global__ void __launch_bounds__(R_THREADS)
    k_route_tc(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
               const RouteArgs a, int S) {
  using C = RouteTcCfg<NPAD, DEEP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t full_bar[C::STAGES];
  __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
  __shared__ __align__(8) uint64_t tfull_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int last_s;
  __shared__ float bias_s[kMaxE];
  __shared__ int cnt_s[kMaxE];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, krank = blockIdx.y;
  const int token0 = tile * R_BT;
  const int num_kb = (a.H + 63) / 64;
  const int per = (num_kb + S - 1) / S;
  const int kb0 = krank * per;
  const int kb1 = min(num_kb, kb0 + per);
  const int my_kb = max(0, kb1 - kb0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    mbar_init(&tfull_bar, 1);
    abort_s = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_s, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait_and_trigger();
  const uint32_t tmem_base = tmem_base_s;
  volatile int* abort_flag = &abort_s;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, a.status)) break;
        uint8_t* sA = smem + stage * C::STAGE_BYTES;
        uint8_t* sB = sA + R_A_BYTES;
        mbar_arrive_expect_tx(&full_bar[stage], C::STAGE_BYTES);
        tma_load_2d(sA, &tmX, &full_bar[stage], kb * 64, token0);
#pragma unroll
        for (int j = 0; j < NPAD / 64; ++j)
          tma_load_2d(sB + j * G_BCHUNK, &tmW, &full_bar[stage], 64 * j, kb * 64);
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && my_kb > 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(R_BT, NPAD, false, true);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&full_bar[stage], phase, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + stage * C::STAGE_BYTES);
        const uint32_t b_base = a_base + R_A_BYTES;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t adesc = smem_desc(a_base + kk * 32, 16, 1024);
          const uint64_t bdesc = smem_desc(b_base + kk * 2048, G_BCHUNK, 1024);
          umma_f16(tmem_base, adesc, bdesc, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&empty_bar[stage]);
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
      if (ok) umma_commit(&tfull_bar);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int et = threadIdx.x - 64;  // 0..127
    const int q = warp & 3;
    const int row = q * 32 + lane;    // TMEM lane = token within the tile
    const int t = token0 + row;
    for (int i = et; i < a.E; i += 128) {
      bias_s[i] = a.bias ? a.bias[i] : 0.f;
      cnt_s[i] = 0;
    }
    bool have = false;
    if (my_kb > 0) {
      int w = 1;
      if (lane == 0) w = mbar_wait(&tfull_bar, 0, abort_flag, a.status);
      have = __shfl_sync(0xffffffffu, w, 0) != 0;
      tc_fence_after();
    }
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    epi_bar();  // bias_s and cnt_s ready
    if (S == 1) {
      unsigned long long best[K];
#pragma unroll
      for (int j = 0; j < K; ++j) best[j] = 0ull;
#pragma unroll 1
      for (int c = 0; c < NPAD / 32; ++c) {
        if (c * 32 >= a.E) break;  // uniform across the warp
        float v[32];
        if (have) {
          tmem_ld32(t_row + c * 32, v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int e = c * 32 + j;
          if (e < a.E) {
            const float l = v[j] + bias_s[e];
            if (a.logits_out && t < a.T) a.logits_out[static_cast<size_t>(t) * a.E + e] = l;
            topk_push<K>(best, select_key(l, e));
          }
        }
      }
      route_tc_finish<K>(a, tile, t, lane, et, best, cnt_s);
    } else {
      // Split over S CTAs: write this CTA's partial logits, then the last CTA
      // of the tile (atomic ticket) sums every partial in rank order.
      float* mine = a.partials + (static_cast<size_t>(tile) * S + krank) * R_BT * a.E +
                    static_cast<size_t>(row) * a.E;
#pragma unroll 1
      for (int c = 0; c < NPAD / 32; ++c) {
        if (c * 32 >= a.E) break;
        float v[32];
        if (have) {
          tmem_ld32(t_row + c * 32, v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          if (c * 32 + j < a.E)
            *reinterpret_cast<float4*>(mine + c * 32 + j) = make_float4(v[j], v[j + 1], v[j + 2],
                                                                        v[j + 3]);
      }
      __threadfence();
      epi_bar();
      if (et == 0) last_s = atomicAdd(&a.tickets[tile], 1) == S - 1;
      epi_bar();
      if (last_s) {
        __threadfence();
        unsigned long long best[K];
#pragma unroll
        for (int j = 0; j < K; ++j) best[j] = 0ull;
        const float* base = a.partials + static_cast<size_t>(tile) * S * R_BT * a.E +
                            static_cast<size_t>(row) * a.E;
        for (int e0 = 0; e0 < a.E; e0 += 4) {
          float4 acc = __ldcg(reinterpret_cast<const float4*>(base + e0));
          for (int r = 1; r < S; ++r) {  // rank order: deterministic
            const float4 p =
                __ldcg(reinterpret_cast<const float4*>(base + static_cast<size_t>(r) * R_BT * a.E +
                                                       e0));
            acc.x += p.x; acc.y += p.y; acc.z += p.z; acc.w += p.w;
          }
          const float l4[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int e = e0 + j;
            const float l = l4[j] + bias_s[e];
            if (a.logits_out && t < a.T) a.logits_out[static_cast<size_t>(t) * a.E + e] = l;
            topk_push<K>(best, select_key(l, e));
          }
        }
        route_tc_finish<K>(a, tile, t, lane, et, best, cnt_s);
        if (et == 0) a.tickets[tile] = 0;  // ready for the next call
      }
    }
  }

  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

static int num_sms_for_route() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}


// W_gate [H, E] as a 2-D map (E contiguous), 64 x 64 boxes, 128-byte swizzle;
// experts beyond E read as zeros.
static bool make_map_wgate(CUtensorMap* m, const void* base, uint64_t H, uint64_t E) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {E, H};
  cuuint64_t strides[1] = {E * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NPAD, int K, bool DEEP>
static cudaError_t launch_route_tc_nkd(const CUtensorMap& mx, const CUtensorMap& mw,
                                       const RouteArgs& a, int tiles, int S, cudaStream_t s) {
  using C = RouteTcCfg<NPAD, DEEP>;
  auto kern = k_route_tc<NPAD, K, DEEP>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (err != cudaSuccess) return err;
  return launch_kernel(kern, dim3(tiles, S, 1), dim3(R_THREADS), C::SMEM, s, 1, mx, mw, a, S);
}

template <int NPAD, int K>
static cudaError_t launch_route_tc_nk(const CUtensorMap& mx, const CUtensorMap& mw,
                                      const RouteArgs& a, int tiles, int S, cudaStream_t s) {
  if (tiles * S <= num_sms_for_route() && !tuning().route_shallow)
    return launch_route_tc_nkd<NPAD, K, true>(mx, mw, a, tiles, S, s);
  return launch_route_tc_nkd<NPAD, K, false>(mx, mw, a, tiles, S, s);
}

template <int NPAD>
static cudaError_t launch_route_tc_n(const CUtensorMap& mx, const CUtensorMap& mw,
                                     const RouteArgs& a, int tiles, int S, cudaStream_t s) {
  if (a.top_k <= 1) return launch_route_tc_nk<NPAD, 1>(mx, mw, a, tiles, S, s);
  if (a.top_k <= 2) return launch_route_tc_nk<NPAD, 2>(mx, mw, a, tiles, S, s);
  if (a.top_k <= 4) return launch_route_tc_nk<NPAD, 4>(mx, mw, a, tiles, S, s);
  return launch_route_tc_nk<NPAD, 8>(mx, mw, a, tiles, S, s);
}

cudaError_t launch_route_tc(const RouteArgs& a, const RoutePlan& p, cudaStream_t s) {
  CUtensorMap mx, mw;
  if (!make_map_2d(&mx, a.x, static_cast<uint64_t>(a.T), static_cast<uint64_t>(a.H), R_BT))
    return cudaErrorInvalidValue;
  if (!make_map_wgate(&mw, a.wg, static_cast<uint64_t>(a.H), static_cast<uint64_t>(a.E)))
    return cudaErrorInvalidValue;
  if (p.ck > 1 && (a.partials == nullptr || a.tickets == nullptr)) return cudaErrorInvalidValue;
  switch (p.NPAD) {
    case 64: return launch_route_tc_n<64>(mx, mw, a, p.tiles, p.ck, s);
    case 128: return launch_route_tc_n<128>(mx, mw, a, p.tiles, p.ck, s);
    case 256: return launch_route_tc_n<256>(mx, mw, a, p.tiles, p.ck, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
