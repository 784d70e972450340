// Grouped expert GEMM on CTA pairs (tcgen05 cta_group::2).
//
// Same contract and tile list as the one-CTA kernel in gemm_tcgen05.cu
// (lshu.cn torch_npu fused-operator article §3-§4: per-expert x W1 [, x W3],
// activation, and the down-projection), but two CTAs of a cluster share one
// 256 x 256 x 64 MMA: each CTA stages its own 128 A rows and one half of the
// 256 B columns, so every SM moves 32 KB per k-block instead of 48 KB; the
// ring has 5 stages and each epilogue warp two staging boxes.  The pair's rows
// are two consecutive 128-row m-tiles of the same expert (an odd last m-tile
// leaves the second CTA's rows empty: computed, never stored).
//
// Roles per CTA (320 threads): warp 0 TMA producer (both CTAs; completion is
// counted on the first CTA's full barrier), warp 1 MMA issuer (first CTA only)
// and TMEM owner (both: the pair allocates together), warps 2-9 epilogue of the
// CTA's own 128 TMEM lanes (two warps per lane quarter, half the columns
// each).  The first CTA's commits arrive on both CTAs' "stage free" and
// "accumulator full" barriers; both CTAs' epilogues arrive on the first CTA's
// "accumulator free" barrier.
#include "gemm_common.cuh"

namespace moe {

constexpr int P_STAGES = 5;
constexpr int P_A_BYTES = G_BM * G_BK * 2;            // 16 KB: this CTA's 128 rows
constexpr int P_B_BYTES = (G_ACC_N / 2) * G_BK * 2;   // 16 KB: half of the 256 columns
constexpr int P_STAGE_BYTES = P_A_BYTES + P_B_BYTES;  // 32 KB
constexpr int P_SMEM = P_STAGES * P_STAGE_BYTES + G_EPI_WARPS * 2 * G_STG_BYTES + 1024;

struct PairTile {
  int e, n0, m0, rows, seg_start;
};

// Pair tile tau -> (expert, n-tile, this CTA's m-tile).  tiles(e) = ceil(mt_e/2) * n_tiles.
__device__ __forceinline__ PairTile decode_pair(int tau, const int* prefix, const int* seg_start,
                                                const int* seg_rows, const int* mtiles, int E,
                                                int bn_out, int rank) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= tau) lo = mid; else hi = mid;
  }
  PairTile t;
  t.e = lo;
  const int local = tau - prefix[lo];
  const int mp_count = (mtiles[lo] + 1) >> 1;
  const int n_tile = local / mp_count;
  const int mp = local - n_tile * mp_count;
  const int m_tile = 2 * mp + rank;
  t.seg_start = seg_start[lo];
  t.m0 = seg_start[lo] + m_tile * G_BM;
  t.rows = min(G_BM, seg_rows[lo] - m_tile * G_BM);  // <= 0: no rows for this CTA
  t.n0 = n_tile * bn_out;
  return t;
}

template <int MODE, bool GATHER>
__global__ void __launch_bounds__(G_THREADS, 1)
    k_gemm_tc_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB1,
                   const __grid_constant__ CUtensorMap tmB3, const __grid_constant__ CUtensorMap tmO,
              const GemmArgs args) {
  constexpr int BN_OUT = ModeCfg<MODE>::BN_OUT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t full_bar[P_STAGES];
  __shared__ __align__(8) uint64_t empty_bar[P_STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int s_prefix[kMaxE + 1];
  __shared__ int s_seg_start[kMaxE];
  __shared__ int s_seg_rows[kMaxE];
  __shared__ int s_mtiles[kMaxE];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs, 1: peer
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int E = args.E;
  const int n_tiles_n = (args.N + BN_OUT - 1) / BN_OUT;
  const int num_kb = (args.K + G_BK - 1) / G_BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < P_STAGES; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull_bar[i], 1);
      mbar_init(&tempty_bar[i], 16);  // one arrival per epilogue warp of both CTAs
    }
    abort_s = 0;
    fence_mbar_init();
  }
  pdl_wait_and_trigger();  // expert offsets and A rows come from the previous kernel
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int rows = 0, s0 = 0;
      if (e < E) {
        s0 = args.offsets[e];
        rows = args.offsets[e + 1] - s0;
        if (rows < 0 || s0 < 0 || s0 + rows > args.R_max) {
          record_status(args.status, 1);
          rows = 0;
        }
        s_seg_start[e] = s0;
        s_seg_rows[e] = rows;
      }
      const int mt = (rows + G_BM - 1) / G_BM;
      if (e < E) s_mtiles[e] = mt;
      int v = ((mt + 1) >> 1) * n_tiles_n;
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
    tmem_alloc_pair(&tmem_base_s, G_TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;
  const int total = s_prefix[E];
  volatile int* abort_flag = &abort_s;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    for (int tau = pair; tau < total; tau += npairs) {
      const PairTile ti = decode_pair(tau, s_prefix, s_seg_start, s_seg_rows, s_mtiles, E, BN_OUT,
                                      static_cast<int>(rank));
      int r4[4] = {0, 0, 0, 0};
      if (GATHER) {
        const int first = args.row_token[ti.seg_start];
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
        uint8_t* sA = smem + stage * P_STAGE_BYTES;
        uint8_t* sB = sA + P_A_BYTES;
        const uint32_t bar = mapa_shared(smem_u32(&full_bar[stage]), 0);
        const int k0 = kb * G_BK;
        if (rank == 0 && lane == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * P_STAGE_BYTES);
        __syncwarp();
        if (GATHER) {
          tma_gather4_pair(sA + lane * 512, &tmA, bar, k0, r4[0], r4[1], r4[2], r4[3]);
        } else if (lane == 0) {
          tma_load_2d_pair(sA, &tmA, bar, k0, ti.rows > 0 ? ti.m0 : ti.seg_start);
        }
        if (lane == 0) {
          if (MODE == 1) {  // CTA 0 holds the W1 half, CTA 1 the W3 half
            const CUtensorMap* mb = rank == 0 ? &tmB1 : &tmB3;
            tma_load_3d_pair(sB, mb, bar, ti.n0, k0, ti.e);
            tma_load_3d_pair(sB + G_BCHUNK, mb, bar, ti.n0 + 64, k0, ti.e);
          } else {          // CTA r holds columns n0 + 128 r .. + 127
            const int nb = ti.n0 + 128 * static_cast<int>(rank);
            tma_load_3d_pair(sB, &tmB1, bar, nb, k0, ti.e);
            tma_load_3d_pair(sB + G_BCHUNK, &tmB1, bar, nb + 64, k0, ti.e);
          }
        }
        if (++stage == P_STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (CTA 0)
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(2 * G_BM, G_ACC_N, false, true);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int tau = pair; tau < total; tau += npairs) {
        if (!mbar_wait_cluster(&tempty_bar[acc], acc_phase ^ 1u, abort_flag, args.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * G_ACC_N);
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, abort_flag, args.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + stage * P_STAGE_BYTES);
          const uint32_t b_base = a_base + P_A_BYTES;
#pragma unroll
          for (int kk = 0; kk < G_BK / 16; ++kk) {
            const uint64_t adesc = smem_desc(a_base + kk * 32, 16, 1024);
            const uint64_t bdesc = smem_desc(b_base + kk * 2048, G_BCHUNK, 1024);
            umma_f16_pair(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit_pair_both(&empty_bar[stage]);
          if (++stage == P_STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit_pair_both(&tfull_bar[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;             // TMEM lanes 32q .. 32q+31
    const int half = (warp - 2) >> 2;   // which half of the tile's columns
    const int row = q * 32 + lane;
    // this warp's two staging boxes
    uint8_t* stg = smem + P_STAGES * P_STAGE_BYTES + (warp - 2) * 2 * G_STG_BYTES;
    int last_box = -1;  // box of the last committed bulk store
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.out);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tau = pair; tau < total; tau += npairs) {
      const PairTile ti = decode_pair(tau, s_prefix, s_seg_start, s_seg_rows, s_mtiles, E, BN_OUT,
                                      static_cast<int>(rank));
      int w = 1;
      if (lane == 0)
        w = mbar_wait_polite<true>(&tfull_bar[acc], acc_phase, abort_flag, args.status,
                                   args.epi_sleep_ns);
      if (!__shfl_sync(0xffffffffu, w, 0)) break;
      tc_fence_after();
      const uint32_t t_row =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * G_ACC_N);
      const bool row_ok = row < ti.rows && MOE_DCHECK(ti.m0 + row < args.R_max, args.status);
      const bool box_full = q * 32 + 32 <= ti.rows;  // all 32 rows of this warp in the tile
      __nv_bfloat16* orow =
          row_ok ? out + static_cast<size_t>(ti.m0 + row) * args.N + ti.n0 : nullptr;
      epilogue_tile<MODE, 2>(t_row, half, &tmO, stg, last_box, lane, box_full, row_ok,
                                 ti.m0 + q * 32, ti.n0, args.N, orow);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&tempty_bar[acc]), 0));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) bulk_wait0();  // this warp's bulk stores are complete
    __syncwarp();
  }
  tc_fence_before();
  cluster_sync_all();  // neither CTA leaves while the pair's MMAs or arrivals may touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, G_TMEM_COLS);
  }
}

template <int MODE, bool GATHER>
static cudaError_t launch_pair(const CUtensorMap& a, const CUtensorMap& b1, const CUtensorMap& b3,
                               const CUtensorMap& o, const GemmArgs& g, int num_sms,
                               cudaStream_t s) {
  auto kern = k_gemm_tc_pair<MODE, GATHER>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM);
  if (err != cudaSuccess) return err;
  return launch_kernel(kern, dim3((num_sms / 2) * 2), dim3(G_THREADS), P_SMEM, s, 2, a, b1, b3, o,
                       g);
}

cudaError_t launch_gemm_tc_pair(int mode, bool gather, const CUtensorMap& ma,
                                const CUtensorMap& mb1, const CUtensorMap& mb3,
                                const CUtensorMap& mo, const GemmArgs& g, int num_sms,
                                cudaStream_t s) {
  switch (mode * 2 + (gather ? 1 : 0)) {
    case 0: return launch_pair<0, false>(ma, mb1, mb3, mo, g, num_sms, s);
    case 1: return launch_pair<0, true>(ma, mb1, mb3, mo, g, num_sms, s);
    case 2: return launch_pair<1, false>(ma, mb1, mb3, mo, g, num_sms, s);
    case 3: return launch_pair<1, true>(ma, mb1, mb3, mo, g, num_sms, s);
    case 4: return launch_pair<2, false>(ma, mb1, mb3, mo, g, num_sms, s);
    case 5: return launch_pair<2, true>(ma, mb1, mb3, mo, g, num_sms, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
