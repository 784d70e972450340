// Router: logits = x @ W_gate (+ bias), top-k selection, renormalised gates,
// and the per-tile expert histogram that the permute step scans.
//
// "MoE模型高效推理：CANN算子库优化实践" §2.1 (gates = softmax(x @ W_gate); top-2),
// §3.2.1 (renormalise the kept gates); "ops-transformer 算子精讲" ch.8
// (normalize_scores=True).  The gates use the identity
//   softmax_s / sum_{kept} softmax = exp(l_s - l_0) / sum_j exp(l_j - l_0),
// so the full softmax over E is never formed.
//
// bf16 path: each CTA owns BT = 16*MT tokens.  x and W_gate chunks of 128 along
// H stream through a cp.async ring in shared memory; warps run mma.sync
// m16n8k16 (bf16 in, fp32 accumulate), split over expert tiles and H.  When T
// is small the H range is also split across the CTAs of a thread-block cluster
// and the partial logits are summed through distributed shared memory, so the
// x read is spread over enough SMs to reach HBM bandwidth.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace cg = cooperative_groups;

constexpr int kRouteThreads = 256;
constexpr int kRouteBK = 128;  // H elements per pipeline chunk

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
    const int e = i < n ? sel_s[i] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) atomicAdd(&cnt_s[e], __popc(peers));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += blockDim.x)
    a.tile_counts[static_cast<size_t>(tile) * E + i] = cnt_s[i];
}

// ----------------------------------------------------------------------------
// bf16 tensor-core router
// ----------------------------------------------------------------------------
template <int MT, int NTP>
struct RouteCfg {
  static constexpr int BT = 16 * MT;
  static constexpr int WN = NTP < 8 ? NTP : 8;  // warps along experts
  static constexpr int NW = NTP / WN;           // n-tiles per warp
  static constexpr int WK = 8 / WN;             // warps along H
  static constexpr int E_PAD = 8 * NTP;
  static constexpr int XS = kRouteBK + 8;                            // x row stride (elems)
  static constexpr int WSC = (NTP % 2 == 0) ? NTP + 1 : NTP;         // W row stride (16B units)
  static constexpr int WS = 8 * WSC;                                 // W row stride (elems)
  static constexpr int X_BYTES = BT * XS * 2;
  static constexpr int W_BYTES = kRouteBK * WS * 2;
  static constexpr int STAGE_BYTES = X_BYTES + W_BYTES;
  static constexpr int STAGES_RAW = (200 * 1024) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : (STAGES_RAW < 2 ? 2 : STAGES_RAW);
  static constexpr int RED_BYTES = WK * BT * E_PAD * 4;
  static constexpr int PIPE_BYTES = STAGES * STAGE_BYTES;
  static constexpr int SMEM = (PIPE_BYTES > RED_BYTES ? PIPE_BYTES : RED_BYTES) +
                              BT * E_PAD * 4 /*part*/ + BT * 8 * 4 /*sel*/ + 256 * 4 /*cnt*/;
  static_assert(MT * NW <= 8, "accumulator budget");
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const int sz = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(sz)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldmatrix_x2_trans(uint32_t (&r)[2], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4],
                                               const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

template <int MT, int NTP>
__global__ void __launch_bounds__(kRouteThreads) k_route_bf16(RouteArgs a, int ck) {
  using C = RouteCfg<MT, NTP>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* pipe = smem;
  const int pipe_region = C::PIPE_BYTES > C::RED_BYTES ? C::PIPE_BYTES : C::RED_BYTES;
  float* part = reinterpret_cast<float*>(smem + pipe_region);
  int* sel_s = reinterpret_cast<int*>(part + C::BT * C::E_PAD);
  int* cnt_s = sel_s + C::BT * 8;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wn = warp % C::WN, wk = warp / C::WN;
  const int tile = blockIdx.x, krank = blockIdx.y;
  const int token0 = tile * C::BT;
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(a.x);
  const __nv_bfloat16* wg = static_cast<const __nv_bfloat16*>(a.wg);

  const int nchunks = (a.H + kRouteBK - 1) / kRouteBK;
  const int per = (nchunks + ck - 1) / ck;
  const int c_begin = krank * per;
  const int c_end = min(nchunks, c_begin + per);
  const int my_chunks = max(0, c_end - c_begin);

  auto issue = [&](int ci, int slot) {
    uint8_t* xs = pipe + slot * C::STAGE_BYTES;
    uint8_t* ws = xs + C::X_BYTES;
    const int h0 = (c_begin + ci) * kRouteBK;
    // x chunk: BT rows x 16 pieces of 16 bytes
    for (int i = threadIdx.x; i < C::BT * 16; i += kRouteThreads) {
      const int r = i >> 4, p = i & 15;
      const int t = token0 + r, h = h0 + p * 8;
      const bool ok = (t < a.T) && (h < a.H);
      const __nv_bfloat16* src = ok ? x + static_cast<size_t>(t) * a.H + h : x;
      cp_async16(xs + (r * C::XS + p * 8) * 2, src, ok);
    }
    // W_gate chunk: 128 rows x (E/8) pieces; padded experts are zero-filled
    const int pieces = C::E_PAD / 8;
    for (int i = threadIdx.x; i < kRouteBK * pieces; i += kRouteThreads) {
      const int r = i / pieces, p = i % pieces;
      const int h = h0 + r, e = p * 8;
      const bool ok = (h < a.H) && (e < a.E);
      const __nv_bfloat16* src = ok ? wg + static_cast<size_t>(h) * a.E + e : wg;
      cp_async16(ws + (r * C::WS + p * 8) * 2, src, ok);
    }
  };

  float acc[MT][C::NW][4];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int n = 0; n < C::NW; ++n)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[m][n][j] = 0.f;

  // prologue: fill STAGES-1 slots
#pragma unroll 1
  for (int s = 0; s < C::STAGES - 1; ++s) {
    if (s < my_chunks) issue(s, s);
    cp_async_commit();
  }
#pragma unroll 1
  for (int ci = 0; ci < my_chunks; ++ci) {
    cp_async_wait<C::STAGES - 2>();
    __syncthreads();
    {
      const int nxt = ci + C::STAGES - 1;
      if (nxt < my_chunks) issue(nxt, nxt % C::STAGES);
      cp_async_commit();
    }
    const uint8_t* xs = pipe + (ci % C::STAGES) * C::STAGE_BYTES;
    const uint8_t* ws = xs + C::X_BYTES;
#pragma unroll
    for (int ks = wk; ks < kRouteBK / 16; ks += C::WK) {
      uint32_t bf[C::NW][2];
#pragma unroll
      for (int n = 0; n < C::NW; ++n) {
        const int nt = wn * C::NW + n;
        const int krow = ks * 16 + (lane & 15);
        ldmatrix_x2_trans(bf[n], ws + (krow * C::WS + nt * 8) * 2);
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        uint32_t af[4];
        const int row = m * 16 + (lane & 15);
        const int col = ks * 16 + (lane >> 4) * 8;
        ldmatrix_x4(af, xs + (row * C::XS + col) * 2);
#pragma unroll
        for (int n = 0; n < C::NW; ++n) mma_bf16_16816(acc[m][n], af, bf[n]);
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // reduce over the warps that split H inside the CTA (fixed order)
  float* red = reinterpret_cast<float*>(pipe);
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int n = 0; n < C::NW; ++n) {
      const int nt = wn * C::NW + n;
      const int r0 = m * 16 + (lane >> 2), c0 = nt * 8 + (lane & 3) * 2;
      float* base = red + static_cast<size_t>(wk) * C::BT * C::E_PAD;
      base[r0 * C::E_PAD + c0] = acc[m][n][0];
      base[r0 * C::E_PAD + c0 + 1] = acc[m][n][1];
      base[(r0 + 8) * C::E_PAD + c0] = acc[m][n][2];
      base[(r0 + 8) * C::E_PAD + c0 + 1] = acc[m][n][3];
    }
  __syncthreads();
  for (int i = threadIdx.x; i < C::BT * C::E_PAD; i += kRouteThreads) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < C::WK; ++w) s += red[w * C::BT * C::E_PAD + i];
    part[i] = s;
  }

  if (ck > 1) {
    // sum the partial logits of the cluster's CTAs in rank order on rank 0
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (krank == 0) {
      for (int i = threadIdx.x; i < C::BT * C::E_PAD; i += kRouteThreads) {
        float s = part[i];
        for (int r = 1; r < ck; ++r) s += cluster.map_shared_rank(part, r)[i];
        red[i] = s;
      }
    }
    cluster.sync();
    if (krank != 0) return;
    __syncthreads();
    for (int i = threadIdx.x; i < C::BT * C::E_PAD; i += kRouteThreads) part[i] = red[i];
  }
  __syncthreads();
  route_select_and_count(part, C::E_PAD, C::BT, token0, a, tile, sel_s, cnt_s);
}

// ----------------------------------------------------------------------------
// SIMT router (fp32 storage, or bf16 with an expert count that is not a
// multiple of 8).  One warp per token, lanes over experts, H in order.
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
  const Tin* x = static_cast<const Tin*>(a.x);
  const Tin* wg = static_cast<const Tin*>(a.wg);
  for (int lt = warp; lt < kSimtBT; lt += kRouteThreads / 32) {
    const int t = token0 + lt;
    if (t >= a.T) continue;
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    for (int h = 0; h < a.H; ++h) {
      const float xv = to_f<Tin>(x[static_cast<size_t>(t) * a.H + h]);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int e = lane + 32 * j;
        if (e < a.E) acc[j] = fmaf(xv, to_f<Tin>(wg[static_cast<size_t>(h) * a.E + e]), acc[j]);
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      if (e < a.E) lg[lt * E_STR + e] = acc[j];
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
static int next_pow2(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

RoutePlan route_plan(int T, int H, int E, int dt_bf16, int num_sms) {
  RoutePlan p{};
  if (!dt_bf16 || (E % 8) != 0) {
    p.kind = 0;
    p.BT = kSimtBT;
    p.tiles = (T + kSimtBT - 1) / kSimtBT;
    p.ck = 1;
    return p;
  }
  p.kind = 1;
  p.NTP = next_pow2((E + 7) / 8);
  const int WN = p.NTP < 8 ? p.NTP : 8;
  const int NW = p.NTP / WN;
  const int mt_max = 8 / NW;
  // largest token tile that still gives at least one wave of CTAs
  int MT = 1;
  for (int m = 2; m <= mt_max && m <= 8; m <<= 1)
    if ((T + 16 * m - 1) / (16 * m) >= num_sms) MT = m;
  p.MT = MT;
  p.BT = 16 * MT;
  p.tiles = (T + p.BT - 1) / p.BT;
  // split H across a cluster when there are too few token tiles
  const int nchunks = (H + kRouteBK - 1) / kRouteBK;
  p.ck = 1;
  while (p.ck < 8 && p.tiles * p.ck < num_sms && nchunks >= 2 * p.ck * 2) p.ck *= 2;
  return p;
}

template <int MT, int NTP>
static cudaError_t launch_bf16(const RouteArgs& a, const RoutePlan& p, cudaStream_t s) {
  using C = RouteCfg<MT, NTP>;
  auto kern = k_route_bf16<MT, NTP>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(p.tiles, p.ck, 1);
  cfg.blockDim = dim3(kRouteThreads, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = p.ck;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, p.ck);
}

template <int MT>
static cudaError_t dispatch_ntp(const RouteArgs& a, const RoutePlan& p, cudaStream_t s) {
  switch (p.NTP) {
    case 1: return launch_bf16<MT, 1>(a, p, s);
    case 2: return launch_bf16<MT, 2>(a, p, s);
    case 4: return launch_bf16<MT, 4>(a, p, s);
    case 8: return launch_bf16<MT, 8>(a, p, s);
    case 16: if constexpr (MT <= 4) return launch_bf16<MT, 16>(a, p, s); break;
    case 32: if constexpr (MT <= 2) return launch_bf16<MT, 32>(a, p, s); break;
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_route(const RouteArgs& a, const RoutePlan& p, cudaStream_t s) {
  if (p.kind == 0) {
    const size_t smem = (kSimtBT * a.E + kSimtBT * 8 + 256) * 4;
    if (a.dt_bf16)
      k_route_simt<__nv_bfloat16><<<p.tiles, kRouteThreads, smem, s>>>(a);
    else
      k_route_simt<float><<<p.tiles, kRouteThreads, smem, s>>>(a);
    return cudaGetLastError();
  }
  switch (p.MT) {
    case 1: return dispatch_ntp<1>(a, p, s);
    case 2: return dispatch_ntp<2>(a, p, s);
    case 4: return dispatch_ntp<4>(a, p, s);
    case 8: return dispatch_ntp<8>(a, p, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_route_from_logits(const RouteArgs& a, const float* logits, cudaStream_t s) {
  const int tiles = (a.T + kSimtBT - 1) / kSimtBT;
  const size_t smem = (kSimtBT * a.E + kSimtBT * 8 + 256) * 4;
  k_route_from_logits<<<tiles, kRouteThreads, smem, s>>>(a, logits);
  return cudaGetLastError();
}

}  // namespace moe
