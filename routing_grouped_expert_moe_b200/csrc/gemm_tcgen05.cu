// Grouped expert GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// lshu.cn torch_npu fused-operator article §3 (x[tokens, hidden] times
// expert_weight[num_experts, hidden, intermediate], then the activation and the
// down-projection) and §4 (npu_moe_matmul); hnwysp.cn ops-transformer MoE
// article §2.2 (the expert stage as one batched GEMM, fed by a prefetch stage,
// aggregated by a reduce stage — here TMA producer, tcgen05 MMA and a TMEM
// epilogue that runs concurrently with the next tile's main loop).
//
// One persistent CTA per SM walks a flat list of tiles (expert, n-tile, m-tile)
// built on the device from expert_offsets, so the number of kept rows never
// needs to reach the host.  m-tiles vary fastest, so the CTAs that share an
// expert's weight tile run at the same time and the second read hits L2.
//
// Tile: 128 rows x 256 accumulator columns x 64 K per stage, 4 stages.
//   A  (rows, K-major)       : 128 x 64 bf16, 128-byte swizzle, from a dense
//                              row-major source (2-D TMA) or gathered row by row
//                              through row_token (TMA tile::gather4).
//   B  (weights, N-major)    : W[e] is [K, N] with N contiguous, so B is fed
//                              MN-major: four 64-column TMA boxes, 128-byte swizzle.
//   D  (TMEM, fp32)          : 2 x 256 columns (double-buffered accumulator).
// Modes: 0 = gelu(A W1), 1 = silu(A W1) * (A W3) with W1 and W3 side by side in
// one N=256 MMA (128 output columns), 2 = A W (down-projection).
//
// Warp roles (320 threads): warp 0 TMA producer, warp 1 MMA issuer (and TMEM
// owner), warps 2-9 epilogue (TMEM lane quarter = warp % 4; two warps per
// quarter split the tile's columns, so the activation epilogue of one tile
// finishes within the next tile's main loop).
#include <cmath>

#include "gemm_common.cuh"

namespace moe {

template <int MODE, bool GATHER>
__global__ void __launch_bounds__(G_THREADS, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB1,
              const __grid_constant__ CUtensorMap tmB3, const __grid_constant__ CUtensorMap tmO,
              const GemmArgs args) {
  constexpr int BN_OUT = ModeCfg<MODE>::BN_OUT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t full_bar[G_STAGES];
  __shared__ __align__(8) uint64_t empty_bar[G_STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int s_prefix[kMaxE + 1];
  __shared__ int s_seg_start[kMaxE];
  __shared__ int s_seg_rows[kMaxE];
  __shared__ int s_mtiles[kMaxE];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = args.E;
  const int n_tiles_n = (args.N + BN_OUT - 1) / BN_OUT;
  const int num_kb = (args.K + G_BK - 1) / G_BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < G_STAGES; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull_bar[i], 1);
      mbar_init(&tempty_bar[i], 256);
    }
    abort_s = 0;
    fence_mbar_init();
  }
  pdl_wait_and_trigger();  // expert offsets and A rows come from the previous kernel
  if (warp == 0) {
    // Tile schedule from the expert segments: tiles(e) = ceil(rows_e/128) * n_tiles.
    int carry = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int rows = 0, s0 = 0;
      if (e < E) {
        s0 = args.offsets[e];
        rows = args.offsets[e + 1] - s0;
        if (rows < 0 || s0 < 0 || s0 + rows > args.R_max) {  // malformed segment: skip it
          record_status(args.status, 1);
          rows = 0;
        }
        s_seg_start[e] = s0;
        s_seg_rows[e] = rows;
      }
      const int mt = (rows + G_BM - 1) / G_BM;
      if (e < E) s_mtiles[e] = mt;
      int v = mt * n_tiles_n;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += u;
      }
      if (e < E) s_prefix[e + 1] = carry + v;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) {
      s_prefix[0] = 0;
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB1);
      if (MODE == 1) tma_prefetch_desc(&tmB3);
    }
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_s, G_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;
  const int total = s_prefix[E];
  volatile int* abort_flag = &abort_s;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    for (int tau = blockIdx.x; tau < total; tau += gridDim.x) {
      const TileInfo ti = decode_tile(tau, s_prefix, s_seg_start, s_seg_rows, s_mtiles, E, BN_OUT);
      int r4[4] = {0, 0, 0, 0};
      if (GATHER) {
        const int first = args.row_token[ti.m0];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int i = lane * 4 + j;
          r4[j] = i < ti.rows ? args.row_token[ti.m0 + i] : first;
        }
      }
      bool ok = true;
      for (int kb = 0; kb < num_kb; ++kb) {
        int w = 1;
        if (lane == 0) w = mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, args.status);
        if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
        uint8_t* sA = smem + stage * G_STAGE_BYTES;
        uint8_t* sB = sA + G_A_BYTES;
        const int k0 = kb * G_BK;
        if (lane == 0) mbar_arrive_expect_tx(&full_bar[stage], G_STAGE_BYTES);
        __syncwarp();
        if (GATHER) {
          tma_gather4(sA + lane * 512, &tmA, &full_bar[stage], k0, r4[0], r4[1], r4[2], r4[3]);
        } else if (lane == 0) {
          tma_load_2d(sA, &tmA, &full_bar[stage], k0, ti.m0);
        }
        if (lane == 0) {
          if (MODE == 1) {
            tma_load_3d(sB, &tmB1, &full_bar[stage], ti.n0, k0, ti.e);
            tma_load_3d(sB + G_BCHUNK, &tmB1, &full_bar[stage], ti.n0 + 64, k0, ti.e);
            tma_load_3d(sB + 2 * G_BCHUNK, &tmB3, &full_bar[stage], ti.n0, k0, ti.e);
            tma_load_3d(sB + 3 * G_BCHUNK, &tmB3, &full_bar[stage], ti.n0 + 64, k0, ti.e);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tma_load_3d(sB + j * G_BCHUNK, &tmB1, &full_bar[stage], ti.n0 + 64 * j, k0, ti.e);
          }
        }
        if (++stage == G_STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(G_BM, G_ACC_N, false, true);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int tau = blockIdx.x; tau < total; tau += gridDim.x) {
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, abort_flag, args.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * G_ACC_N);
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, abort_flag, args.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + stage * G_STAGE_BYTES);
          const uint32_t b_base = a_base + G_A_BYTES;
#pragma unroll
          for (int kk = 0; kk < G_BK / 16; ++kk) {
            // A: K-major, rows of 128 B, 8-row groups 1024 B apart; K step = 32 B.
            const uint64_t adesc = smem_desc(a_base + kk * 32, 16, 1024);
            // B: MN-major, 64-column boxes 8 KB apart (LBO), 8 K-rows 1024 B apart (SBO);
            //    K step of 16 rows = 2048 B.
            const uint64_t bdesc = smem_desc(b_base + kk * 2048, G_BCHUNK, 1024);
            umma_f16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty_bar[stage]);
          if (++stage == G_STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull_bar[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;             // TMEM lanes 32q .. 32q+31
    const int half = (warp - 2) >> 2;   // which half of the tile's columns
    const int row = q * 32 + lane;
    // this warp's staging box
    uint8_t* stg = smem + G_STAGES * G_STAGE_BYTES + (warp - 2) * G_STG_BYTES;
    int last_box = -1;  // box of the last committed bulk store
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.out);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tau = blockIdx.x; tau < total; tau += gridDim.x) {
      const TileInfo ti = decode_tile(tau, s_prefix, s_seg_start, s_seg_rows, s_mtiles, E, BN_OUT);
      int w = 1;
      if (lane == 0)
        w = mbar_wait_polite<false>(&tfull_bar[acc], acc_phase, abort_flag, args.status,
                                    args.epi_sleep_ns);
      if (!__shfl_sync(0xffffffffu, w, 0)) break;
      tc_fence_after();
      const uint32_t t_row =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * G_ACC_N);
      const bool row_ok = row < ti.rows && MOE_DCHECK(ti.m0 + row < args.R_max, args.status);
      const bool box_full = q * 32 + 32 <= ti.rows;  // all 32 rows of this warp in the tile
      __nv_bfloat16* orow =
          row_ok ? out + static_cast<size_t>(ti.m0 + row) * args.N + ti.n0 : nullptr;
      epilogue_tile<MODE, 1>(t_row, half, &tmO, stg, last_box, lane, box_full, row_ok,
                                 ti.m0 + q * 32, ti.n0, args.N, orow);
      tc_fence_before();
      mbar_arrive(&tempty_bar[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) bulk_wait0();  // this warp's bulk stores are complete
    __syncwarp();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, G_TMEM_COLS);
  }
}

// The activations the bf16 epilogue applies, elementwise (self-test hook).
__global__ void k_epilogue_activations(const float* __restrict__ z, int n, float* __restrict__ gelu,
                                       float* __restrict__ silu) {
  pdl_wait_and_trigger();
  // in pairs, with the same packed code the epilogue runs
  for (int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x); i < n; i += 2 * gridDim.x * blockDim.x) {
    const float2 zz = make_float2(z[i], i + 1 < n ? z[i + 1] : 0.f);
    const float2 g = gelu_epi2(zz), s = silu_epi2(zz);
    gelu[i] = g.x;
    silu[i] = s.x;
    if (i + 1 < n) {
      gelu[i + 1] = g.y;
      silu[i + 1] = s.y;
    }
  }
}

cudaError_t launch_epilogue_activations(const float* z, int n, float* gelu, float* silu,
                                        cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  return launch_kernel(k_epilogue_activations, dim3((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024),
                       dim3(256), 0, s, 1, z, n, gelu, silu);
}

// ----------------------------------------------------------------------------
// Host: launch
// ----------------------------------------------------------------------------
template <int MODE, bool GATHER>
static cudaError_t launch_tc(const CUtensorMap& a, const CUtensorMap& b1, const CUtensorMap& b3,
                             const CUtensorMap& o, const GemmArgs& g, int num_sms, cudaStream_t s) {
  auto kern = k_gemm_tc<MODE, GATHER>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G_SMEM);
  if (err != cudaSuccess) return err;
  return launch_kernel(kern, dim3(num_sms), dim3(G_THREADS), G_SMEM, s, 1, a, b1, b3, o, g);
}

// Kernel variant for dense A rows: the token-as-N pair kernel (gemm_tokn.cu:
// weights as the MMA's M, an expert's tokens as N, rounded up to 16 instead of
// to a 128- or 256-row tile, and fewer operand bytes per MMA clock), or the
// row-tiled kernels, one CTA per 128-row tile (1) or CTA pairs sharing 256-row
// tiles (2).  Gathered A rows (row_token) use the row-tiled kernels: the pair
// when the expected wave count for balanced experts of a = R_max / E rows
// (a / BM + 1/2 row tiles per expert; a pair tile counted at 0.92 of a one-CTA
// tile, as measured) is lower.  The tuning variant forces one.
static int choose_variant(int mode, bool gather, const GemmArgs& g, int num_sms) {
  const int forced = gemm_variant();
  if (forced >= 3 && !gather) return 3;  // 4: token-as-N without the K-split tail
  if (forced == 1 || forced == 2) return forced;
  if (!gather) return 3;
  const double a = static_cast<double>(g.R_max) / g.E;
  const double n_tiles = std::ceil(static_cast<double>(g.N) / (mode == 1 ? 128 : 256));
  const double t1 = g.E * (a / G_BM + 0.5) * n_tiles;
  const double t2 = g.E * (a / (2 * G_BM) + 0.5) * n_tiles;
  const double waves1 = std::ceil(t1 / num_sms);
  const double waves2 = std::ceil(t2 / (num_sms / 2));
  return 0.92 * waves2 < waves1 ? 2 : 1;
}

cudaError_t launch_gemm_tc(int mode, bool gather, const void* a_src, int a_rows, const void* b1,
                           const void* b3, const GemmArgs& g, int num_sms, cudaStream_t s) {
  GemmArgs ga = g;
  ga.epi_sleep_ns = tuning().epi_sleep_ns;
  // a cap on the persistent grid (measurement aid: how the GEMM scales with SMs)
  const int cap = tuning().gemm_ctas;
  if (cap >= 2 && cap < num_sms) num_sms = cap;
  const int variant = choose_variant(mode, gather, g, num_sms);
  if (log_enabled())
    log_line("grouped GEMM mode=%d (%s) gather=%d rows<=%d N=%d K=%d E=%d: %s", mode,
             mode == 1 ? "SwiGLU" : (mode == 0 ? "GELU" : "down"), gather ? 1 : 0, g.R_max, g.N,
             g.K, g.E,
             variant == 3 ? "token-as-N pair tiles"
                          : (variant == 2 ? "256-row pair tiles" : "128-row tiles"));
  if (variant == 3 && g.sched != nullptr)
    return launch_gemm_tokn(mode, a_src, a_rows, b1, b3, ga, num_sms, s);
  CUtensorMap ma, mb1, mb3, mo;
  // A: [a_rows, K]; dense source uses 128-row boxes, the gathered source 1-row boxes.
  if (!make_map_2d(&ma, a_src, static_cast<uint64_t>(a_rows), static_cast<uint64_t>(g.K),
                   gather ? 1u : static_cast<uint32_t>(G_BM)))
    return cudaErrorInvalidValue;
  if (!make_map_w(&mb1, b1, g.E, g.K, g.N)) return cudaErrorInvalidValue;
  if (mode == 1) {
    if (!make_map_w(&mb3, b3, g.E, g.K, g.N)) return cudaErrorInvalidValue;
  } else {
    mb3 = mb1;
  }
  if (!make_map_out(&mo, g.out, static_cast<uint64_t>(g.R_max), static_cast<uint64_t>(g.N)))
    return cudaErrorInvalidValue;
  if (variant == 2) return launch_gemm_tc_pair(mode, gather, ma, mb1, mb3, mo, ga, num_sms, s);
  switch (mode * 2 + (gather ? 1 : 0)) {
    case 0: return launch_tc<0, false>(ma, mb1, mb3, mo, ga, num_sms, s);
    case 1: return launch_tc<0, true>(ma, mb1, mb3, mo, ga, num_sms, s);
    case 2: return launch_tc<1, false>(ma, mb1, mb3, mo, ga, num_sms, s);
    case 3: return launch_tc<1, true>(ma, mb1, mb3, mo, ga, num_sms, s);
    case 4: return launch_tc<2, false>(ma, mb1, mb3, mo, ga, num_sms, s);
    case 5: return launch_tc<2, true>(ma, mb1, mb3, mo, ga, num_sms, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
