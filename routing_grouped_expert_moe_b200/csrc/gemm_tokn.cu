// Grouped expert GEMM with the tokens as the MMA's N dimension (CTA pairs,
// tcgen05 cta_group::2).
//
// Same contract as the row-tiled kernels (lshu.cn torch_npu fused-operator
// article §3-§4: per expert x W1 [, x W3], the activation, and the
// down-projection), computed transposed: for the tokens of one expert segment,
// D^T[f, t] = sum_k W[e][k, f] x[t, k].  The weight tile is the M = 256 operand
// (128 output columns per CTA, fed MN-major straight from W[e] = [K, N]) and
// the expert's tokens are the N operand, so an expert of n rows costs
// ceil(n / 16) * 16 token columns instead of a whole 128- or 256-row tile; a
// segment of more than 256 rows is split into equal groups of at most 256.
//
// The operand stream into each SM paces this kernel.  A pair tile of 256
// weight columns x 256 tokens x 64 K moves 16 KB of weights and 16 KB of
// tokens into each SM per 512 MMA clocks (64 B/clk); the SwiGLU form keeps two
// accumulators (W1 and W3) over the same token tile, 48 KB per 1024 clocks
// (48 B/clk).  Measured with every SM streaming, a pipeline stage takes about
// the same time whatever the tile's token count (a fixed cost per stage plus
// what one SM can bring in, ~47 B/clk), so a full 256-token SwiGLU tile keeps
// the tensor pipe ~91% busy over its main loop and a smaller token group
// leaves the rest idle.
//
// NACC accumulators per tile: NACC = 1 double-buffers one 256-column
// accumulator so the epilogue of a tile overlaps the next tile's main loop;
// NACC = 2 (SwiGLU: W1 and W3) fills the 512 TMEM columns with one tile.
//
// K-split tail: a tile's time is set by its number of pipeline stages (the
// loads' latency under load, not their bytes, paces a stage), so tiles of
// one launch take about the same time and the last wave, total mod the CTA
// pairs, runs on a fraction of the GPU.  When at most half the pairs are
// left for it (and the host asks for it: the SwiGLU GEMM-1), those last
// tiles are cut along K into two parts.  Each part writes its fp32
// accumulators to the workspace, then counts itself in on a ticket per
// epilogue warp; the part that comes second adds the other's sums to its own
// (fp32 addition of two terms is commutative, so the result does not depend
// on which part finished first) and runs the activation and the stores.  No
// part waits for another.
//
// Tiles are taken from a global counter (dynamic schedule: token groups of
// different sizes take different times).  The first CTA's producer takes the
// next tile and passes its index to the other CTA's producer through a mailbox
// in that CTA's shared memory; each producer passes it on to its own MMA and
// epilogue warps through a small ring.
//
// Roles: warp 0 (and warps 10, 11, ...) TMA producers, warp 1 MMA issuer
// (first CTA) and TMEM owner (both), warps 2-9 epilogue (two warps per TMEM
// lane quarter, alternate 32-token chunks).  The SwiGLU epilogue (STASH)
// drains, activates and packs all of its chunks into registers and hands TMEM
// back to the MMA before it stores them, so its stores overlap the next
// tile's main loop (measured 1.5-3% off the SwiGLU GEMM-1 on the Mixtral-
// shaped, 128-expert and 32-expert layers); it runs with two producer warps
// so that 352 threads leave it the registers.
#include "gemm_common.cuh"

namespace moe {

namespace {

constexpr int T_MAXN = 256;                 // tokens per tile
constexpr int T_XCHUNK = 128 * 64 * 2;      // tokens' smem per 64-wide K chunk: 128 rows, 16 KB
constexpr int T_SD = 4;                     // depth of the tile-index ring

// Per-SM TMA throughput grows with the bytes each pipeline stage moves and
// with the size of its boxes (measured: one 8 KB box per stage streams at
// ~12 B/clk, eight per stage at ~55, two 32 KB boxes at ~85), so a stage
// covers BK = 64 or 128 of K: weight boxes of 64 columns x BK rows, token
// boxes of 64 K x (32, 64 or 128) rows per 64-wide chunk of K.
template <int MODE, int NACC, int BK, bool STASH = false>
struct TokCfg {
  static constexpr int W_BOX = 64 * BK * 2;            // one 64-column weight box
  static constexpr int W_BYTES = 2 * W_BOX;            // 128 weight columns (one accumulator)
  static constexpr int A_BYTES = NACC * W_BYTES;
  static constexpr int X_BYTES = (BK / 64) * T_XCHUNK;
  static constexpr int STAGE_BYTES = A_BYTES + X_BYTES;
  static constexpr int NBOX = 1;                       // staging boxes per epilogue warp
  static constexpr int STAGES = (192 * 1024) / STAGE_BYTES;
  static constexpr int COLS_PER_TILE = MODE == 1 ? 256 : 256 * NACC;  // output columns per tile
  static constexpr int SMEM = STAGES * STAGE_BYTES + G_EPI_WARPS * NBOX * G_STG_BYTES + 1024;
  static_assert(STAGES >= 2, "pipeline needs two stages");
  // TMA producer warps.  One issuing thread streams at about half the rate an
  // SM can take (measured: 31 B/clk with one warp, 60 with two, 64 with four,
  // same boxes and stages), so PROD warps (warp 0, then warps 10, 11, ...)
  // each own the stages s = p mod PROD.  PROD divides STAGES: a stage always
  // has the same producer, which never gets more than one lap ahead of the
  // MMA on it (the empty barrier's parity tells only one lap from the next).
  // (STASH: two producers, so that 352 threads leave the epilogue the
  // registers for its packed outputs)
  static constexpr int PROD =
      STASH ? 2 : (STAGES <= 4 ? STAGES : (STAGES % 3 == 0 ? 3 : 2));
  static_assert(STAGES % PROD == 0, "every stage needs a single producer");
  static constexpr int THREADS = G_THREADS + 32 * (PROD - 1);
};

// Token rows one CTA loads per 64-wide K chunk for half_n needed rows
// (8 <= half_n <= 128, a multiple of 8): a first box of 32, 64 or 128 rows and,
// for 65-96 rows, a second box of 32 rows placed after it.
struct TokRows {
  int first, second;
};
__host__ __device__ constexpr TokRows tok_rows(int half_n) {
  return half_n <= 32 ? TokRows{32, 0}
                      : (half_n <= 64 ? TokRows{64, 0}
                                      : (half_n <= 96 ? TokRows{64, 32} : TokRows{128, 0}));
}

struct TokTile {
  int e, row0, rows, n, col0;
  int kb0, kb1;     // k-blocks of this part
  int unit;         // K-split part index over the split tiles (-1: a whole tile)
  int part, stile;  // part within its tile, split tile index
};

// Launch-wide schedule: tiles [0, t0) whole, tiles [t0, total) in S parts each.
struct TokSplit {
  int t0, S, units;
};

// Tile tau -> (expert, token group, output-column block); groups vary fastest,
// so the groups that share a weight tile run at the same time and the second
// read of the weights hits L2.
__device__ __forceinline__ TokTile decode_tok(int tau, const int* prefix, const int* seg_start,
                                             const int* seg_rows, const int* grp_rows,
                                             const int* ngrp, int E, int cols_per_tile,
                                             const TokSplit& sp, int num_kb) {
  int unit = -1, part = 0, stile = -1;
  if (tau >= sp.t0) {  // a K-split part
    unit = tau - sp.t0;
    stile = unit / sp.S;
    part = unit - stile * sp.S;
    tau = sp.t0 + stile;
  }
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= tau) lo = mid; else hi = mid;
  }
  const int local = tau - prefix[lo];
  const int ng = ngrp[lo];
  const int mb = local / ng;
  const int g = local - mb * ng;
  const int q = grp_rows[lo];
  TokTile t;
  t.e = lo;
  t.row0 = seg_start[lo] + g * q;
  t.rows = min(q, seg_rows[lo] - g * q);
  t.n = (t.rows + 15) & ~15;
  t.col0 = mb * cols_per_tile;
  t.unit = unit;
  t.part = part;
  t.stile = stile;
  t.kb0 = unit < 0 ? 0 : (part * num_kb) / sp.S;
  t.kb1 = unit < 0 ? num_kb : ((part + 1) * num_kb) / sp.S;
  return t;
}

__device__ __forceinline__ void st_shared_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Writes one warp's 32 tokens x 32 output columns (this lane's column, one
// value per token) to out: pairs of adjacent columns are formed with one
// shuffle per token pair and packed to bf16x2 (tok_pack), then staged as a
// [32 token][32 col] box for a TMA store, or (a ragged chunk: fewer than 32
// tokens left in the group) stored directly, masked by token (tok_store_packed).
__device__ __forceinline__ void tok_pack(const float (&v)[32], int lane, uint32_t (&w)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float send = (lane & 1) ? v[2 * i] : v[2 * i + 1];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
    w[i] = (lane & 1) ? pack_bf16x2(recv, v[2 * i + 1]) : pack_bf16x2(v[2 * i], recv);
  }
}

__device__ __forceinline__ void tok_store_packed(const uint32_t (&w)[16], const CUtensorMap* tmO,
                                                 uint8_t* stg, int lane, int vt, int row, int col,
                                                 int N, __nv_bfloat16* out) {
  const int tsub = lane & 1;          // token parity this lane writes
  const int wcol = lane >> 1;         // bf16x2 word within the 32 columns
  if (vt == 32) {
    uint32_t* sw = reinterpret_cast<uint32_t*>(stg);
#pragma unroll
    for (int i = 0; i < 16; ++i) sw[(2 * i + tsub) * 16 + wcol] = w[i];
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tmO, stg, col, row);
      bulk_commit();
    }
  } else {
    const int c = col + 2 * wcol;
    if (c < N) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int t = 2 * i + tsub;
        if (t < vt)
          *reinterpret_cast<uint32_t*>(out + static_cast<size_t>(row + t) * N + c) = w[i];
      }
    }
  }
}

__device__ __forceinline__ void tok_store_chunk(const float (&v)[32], const CUtensorMap* tmO,
                                                uint8_t* stg, int lane, int vt, int row,
                                                int col, int N, __nv_bfloat16* out) {
  uint32_t w[16];
  tok_pack(v, lane, w);
  tok_store_packed(w, tmO, stg, lane, vt, row, col, N, out);
}

template <int MODE>
__device__ __forceinline__ void tok_activate(float (&v)[32], const float (&u)[32]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float2 a = make_float2(v[2 * i], v[2 * i + 1]);
    if (MODE == 0) a = gelu_epi2(a);
    if (MODE == 1) a = fmul2(silu_epi2(a), make_float2(u[2 * i], u[2 * i + 1]));
    v[2 * i] = a.x;
    v[2 * i + 1] = a.y;
  }
}

}  // namespace

template <int MODE, int NACC, int BK, bool STASH>
__global__ void __launch_bounds__(TokCfg<MODE, NACC, BK, STASH>::THREADS, 1)
    k_gemm_tokn(const __grid_constant__ CUtensorMap tmX32, const __grid_constant__ CUtensorMap tmX64,
                const __grid_constant__ CUtensorMap tmX128, const __grid_constant__ CUtensorMap tmW1,
                const __grid_constant__ CUtensorMap tmW3, const __grid_constant__ CUtensorMap tmO,
                const GemmArgs args) {
  static_assert(!STASH || (MODE == 1 && NACC == 2), "the stash drains SwiGLU's two accumulators");
  using C = TokCfg<MODE, NACC, BK, STASH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t full_bar[C::STAGES];
  __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t sched_full[T_SD];
  __shared__ __align__(8) uint64_t sched_empty[T_SD];
  __shared__ __align__(8) uint64_t mb_full[T_SD];    // second CTA: a tile index has arrived
  __shared__ __align__(8) uint64_t mb_empty[T_SD];   // first CTA: the peer has read the slot
  __shared__ int s_tile[T_SD];
  __shared__ int mb_tile[T_SD];
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int s_prefix[kMaxE + 1];
  __shared__ int s_seg_start[kMaxE];
  __shared__ int s_seg_rows[kMaxE];
  __shared__ int s_grp_rows[kMaxE];
  __shared__ int s_ngrp[kMaxE];
  __shared__ TokSplit s_split;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int E = args.E;
  const int mblocks = (args.N + C::COLS_PER_TILE - 1) / C::COLS_PER_TILE;
  const int num_kb = (args.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull_bar[i], 1);
      mbar_init(&tempty_bar[i], 2 * G_EPI_WARPS);  // every epilogue warp of both CTAs
    }
    for (int i = 0; i < T_SD; ++i) {
      mbar_init(&sched_full[i], 1);
      // consumers: the epilogue warps, the other producers, the MMA warp (first CTA)
      mbar_init(&sched_empty[i], G_EPI_WARPS + (C::PROD - 1) + (rank == 0 ? 1 : 0));
      mbar_init(&mb_full[i], 1);
      mbar_init(&mb_empty[i], 1);
    }
    abort_s = 0;
    fence_mbar_init();
  }
  pdl_wait_and_trigger();  // expert offsets and token rows come from the previous kernel
  if (warp == 0) {
    // Per expert: rows n, token groups ceil(n / 256) of q = round16(ceil(n / groups)) rows
    // (the last may be shorter), tiles = groups x output-column blocks.
    int carry = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int rows = 0, s0 = 0, q = 16, ng = 0;
      if (e < E) {
        s0 = args.offsets[e];
        rows = args.offsets[e + 1] - s0;
        if (rows < 0 || s0 < 0 || s0 + rows > args.R_max) {  // malformed segment: skip it
          record_status(args.status, 1);
          rows = 0;
        }
        if (rows > 0) {
          const int g0 = (rows + T_MAXN - 1) / T_MAXN;
          q = (((rows + g0 - 1) / g0) + 15) & ~15;
          ng = (rows + q - 1) / q;
        }
        s_seg_start[e] = s0;
        s_seg_rows[e] = rows;
        s_grp_rows[e] = q;
        s_ngrp[e] = ng;
      }
      int v = ng * mblocks;
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
      // the last partial wave (total mod pairs tiles) in two parts along K, each
      // part at least 2 k-blocks, within the workspace's capacity
      const int total = carry;
      const int pairs = static_cast<int>(gridDim.x) >> 1;
      const int rem = pairs > 0 ? total % pairs : 0;
      int S = 1;
      if (args.split_max >= 2 && args.split_ws != nullptr && args.split_tickets != nullptr &&
          rem > 0 && 2 * rem <= pairs && rem <= args.split_tiles && 2 * rem <= args.split_units &&
          num_kb >= 4)
        S = 2;
      s_split.S = S > 1 ? S : 1;
      s_split.t0 = S > 1 ? total - rem : total;
      s_split.units = S > 1 ? total - rem + rem * S : total;
      tma_prefetch_desc(&tmX32);
      tma_prefetch_desc(&tmX64);
      tma_prefetch_desc(&tmX128);
      tma_prefetch_desc(&tmW1);
      if (MODE == 1) tma_prefetch_desc(&tmW3);
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
  const TokSplit sp = s_split;
  const int total = sp.units;  // whole tiles and K-split parts
  volatile int* abort_flag = &abort_s;
  volatile int* vs_tile = s_tile;
  volatile int* vmb_tile = mb_tile;

  // Consumers' side of the tile-index ring: the next tile (or -1 at the end).
  auto next_tile = [&](int i, bool& ok) -> int {
    const int slot = i % T_SD;
    const uint32_t ph = static_cast<uint32_t>(i / T_SD) & 1u;
    int tau = -1, w = 1;
    if (lane == 0) {
      w = mbar_wait(&sched_full[slot], ph, abort_flag, args.status);
      if (w) {
        tau = vs_tile[slot];
        mbar_arrive(&sched_empty[slot]);
      }
    }
    ok = __shfl_sync(0xffffffffu, w, 0) != 0;
    return __shfl_sync(0xffffffffu, tau, 0);
  };

  if (warp == 0 || warp >= 2 + G_EPI_WARPS) {
    // ------------------------------------------------------------ tile fetch + TMA producers
    // Producer p issues the stages whose running index g (over all tiles and
    // k-blocks) is p mod PROD, i.e. ring stages p, p + PROD, ...; producer 0
    // also fetches the tiles.
    const int p = warp == 0 ? 0 : warp - (1 + G_EPI_WARPS);
    if (lane == 0) {
      uint32_t g = 0;
      for (int i = 0;; ++i) {
        const int slot = i % T_SD;
        const uint32_t ph = static_cast<uint32_t>(i / T_SD) & 1u;
        int tau;
        if (p != 0) {
          if (!mbar_wait(&sched_full[slot], ph, abort_flag, args.status)) break;
          tau = vs_tile[slot];
          mbar_arrive(&sched_empty[slot]);
        } else if (rank == 0) {
          if (!mbar_wait(&sched_empty[slot], ph ^ 1u, abort_flag, args.status)) break;
          if (!mbar_wait(&mb_empty[slot], ph ^ 1u, abort_flag, args.status)) break;
          tau = atomicAdd(args.sched, 1);
          if (tau >= total) tau = -1;
          vs_tile[slot] = tau;
          mbar_arrive(&sched_full[slot]);
          st_shared_cluster_u32(mapa_shared(smem_u32(&mb_tile[slot]), 1), static_cast<uint32_t>(tau));
          mbar_arrive_remote(mapa_shared(smem_u32(&mb_full[slot]), 1));
        } else {
          if (!mbar_wait_cluster(&mb_full[slot], ph, abort_flag, args.status)) break;
          tau = vmb_tile[slot];
          mbar_arrive_remote(mapa_shared(smem_u32(&mb_empty[slot]), 0));
          if (!mbar_wait(&sched_empty[slot], ph ^ 1u, abort_flag, args.status)) break;
          vs_tile[slot] = tau;
          mbar_arrive(&sched_full[slot]);
        }
        if (tau < 0) break;
        const TokTile ti = decode_tok(tau, s_prefix, s_seg_start, s_seg_rows, s_grp_rows, s_ngrp, E,
                                      C::COLS_PER_TILE, sp, num_kb);
        const int half_n = ti.n >> 1;
        // this CTA's token rows: one box of 32, 64 or 128 rows, or 64 + 32
        const TokRows xr = tok_rows(half_n);
        const int rows_ld = xr.first + xr.second;
        const CUtensorMap* xa = xr.first == 32 ? &tmX32 : (xr.first == 64 ? &tmX64 : &tmX128);
        const bool x_second = xr.second != 0;  // a 32-row box after a 64-row one
        const int xrow = ti.row0 + static_cast<int>(rank) * half_n;
        const uint32_t tx = 2u * static_cast<uint32_t>(C::A_BYTES + (BK / 64) * rows_ld * 128);
        const int wcol = ti.col0 + 128 * static_cast<int>(rank);
        bool ok = true;
        for (int kb = ti.kb0; kb < ti.kb1; ++kb, ++g) {
          if (g % C::PROD != static_cast<uint32_t>(p)) continue;
          const int stage = static_cast<int>(g % C::STAGES);
          const uint32_t phase = (g / C::STAGES) & 1u;
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, args.status)) { ok = false; break; }
          uint8_t* sA = smem + stage * C::STAGE_BYTES;
          uint8_t* sX = sA + C::A_BYTES;
          const uint32_t bar = mapa_shared(smem_u32(&full_bar[stage]), 0);
          const int k0 = kb * BK;
          if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], tx);
          if (MODE == 1) {  // accumulator 0: W1, accumulator 1: W3, same 128 columns
            tma_load_3d_pair(sA, &tmW1, bar, wcol, k0, ti.e);
            tma_load_3d_pair(sA + C::W_BOX, &tmW1, bar, wcol + 64, k0, ti.e);
            tma_load_3d_pair(sA + C::W_BYTES, &tmW3, bar, wcol, k0, ti.e);
            tma_load_3d_pair(sA + C::W_BYTES + C::W_BOX, &tmW3, bar, wcol + 64, k0, ti.e);
          } else {
#pragma unroll
            for (int j = 0; j < NACC; ++j) {
              tma_load_3d_pair(sA + j * C::W_BYTES, &tmW1, bar, wcol + 256 * j, k0, ti.e);
              tma_load_3d_pair(sA + j * C::W_BYTES + C::W_BOX, &tmW1, bar, wcol + 256 * j + 64,
                               k0, ti.e);
            }
          }
#pragma unroll
          for (int c = 0; c < BK / 64; ++c) {
            tma_load_2d_pair(sX + c * T_XCHUNK, xa, bar, k0 + 64 * c, xrow);
            if (x_second)
              tma_load_2d_pair(sX + c * T_XCHUNK + 64 * 128, &tmX32, bar, k0 + 64 * c, xrow + 64);
          }
        }
        if (!ok) break;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (first CTA)
    if (rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int i = 0;; ++i) {
        bool ok;
        const int tau = next_tile(i, ok);
        if (!ok || tau < 0) break;
        if (lane == 0) {
          const TokTile ti = decode_tok(tau, s_prefix, s_seg_start, s_seg_rows, s_grp_rows,
                                        s_ngrp, E, C::COLS_PER_TILE, sp, num_kb);
          const uint32_t idesc = idesc_bf16_f32(256, ti.n, true, false);
          if (!mbar_wait_cluster(&tempty_bar[acc], acc_phase ^ 1u, abort_flag, args.status)) {
            ok = false;
          } else {
            tc_fence_after();
            const uint32_t d0 = tmem_base + static_cast<uint32_t>(NACC == 2 ? 0 : acc * 256);
            for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
              if (!mbar_wait(&full_bar[stage], phase, abort_flag, args.status)) { ok = false; break; }
              tc_fence_after();
              const uint32_t a_base = smem_u32(smem + stage * C::STAGE_BYTES);
              const uint32_t x_base = a_base + C::A_BYTES;
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk) {
                // tokens: K-major, one 16 KB chunk per 64 of K; rows of 128 B, 8-row
                // groups 1024 B apart, K step 32 B
                const uint64_t xdesc =
                    smem_desc(x_base + (kk >> 2) * T_XCHUNK + (kk & 3) * 32, 16, 1024);
#pragma unroll
                for (int j = 0; j < NACC; ++j) {
                  // weights: MN-major, 64-column boxes W_BOX apart, K step of 16 rows = 2 KB
                  const uint64_t wdesc =
                      smem_desc(a_base + j * C::W_BYTES + kk * 2048, C::W_BOX, 1024);
                  umma_f16_pair(d0 + j * 256, wdesc, xdesc, idesc,
                                (kb != ti.kb0 || kk != 0) ? 1u : 0u);
                }
              }
              umma_commit_pair_both(&empty_bar[stage]);
              if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
            }
            if (ok) umma_commit_pair_both(&tfull_bar[acc]);
          }
        }
        if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
        if (NACC == 1) {
          if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        } else {
          acc_phase ^= 1u;
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;            // TMEM lanes 32q .. 32q+31
    const int half = (warp - 2) >> 2;  // alternate 32-token chunks
    uint8_t* stg = smem + C::STAGES * C::STAGE_BYTES + (warp - 2) * G_STG_BYTES;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.out);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int i = 0;; ++i) {
      bool ok;
      const int tau = next_tile(i, ok);
      if (!ok || tau < 0) break;
      const TokTile ti = decode_tok(tau, s_prefix, s_seg_start, s_seg_rows, s_grp_rows, s_ngrp, E,
                                    C::COLS_PER_TILE, sp, num_kb);
      int w = 1;
      if (lane == 0)
        w = mbar_wait_polite<true>(&tfull_bar[acc], acc_phase, abort_flag, args.status,
                                   args.epi_sleep_ns);
      if (!__shfl_sync(0xffffffffu, w, 0)) break;
      tc_fence_after();
      const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                              static_cast<uint32_t>(NACC == 2 ? 0 : acc * 256);
      const int nch = (ti.n + 31) >> 5;
      const int colw = ti.col0 + 128 * static_cast<int>(rank) + q * 32;  // this warp's 32 columns
      constexpr int NOUT = MODE == 1 ? 1 : NACC;          // outputs per chunk
      constexpr int NP = (MODE == 1 || NACC == 2) ? 2 : 1;  // accumulators per chunk
      // A K-split part (two per tile): its fp32 sums for this warp's chunks,
      // [chunk / 2][acc][token / 4][lane][token % 4], so that a warp moves 512
      // contiguous bytes per float4 access.
      const size_t wslot = static_cast<size_t>((static_cast<int>(rank) * 8 + (warp - 2)) * 4 * 2 * 1024);
      // the tile inside the output and, for a K-split part, inside the split areas
      bool emit = MOE_DCHECK(ti.row0 >= 0 && ti.row0 + ti.rows <= args.R_max && ti.col0 < args.N &&
                                 (ti.unit < 0 || (ti.unit < args.split_units &&
                                                  ti.stile < args.split_tiles)),
                             args.status);
      if (ti.unit >= 0 && emit) {
        float* mine = args.split_ws + static_cast<size_t>(ti.unit) * kSplitUnitFloats + wslot;
#pragma unroll 1
        for (int c = half; c < nch; c += 2) {
#pragma unroll
          for (int j = 0; j < NP; ++j) {
            float v[32];
            tmem_ld32(t_lane + j * 256 + c * 32, v);
            tmem_ld_wait();
            reg_fence32(v);
            float4* dst = reinterpret_cast<float4*>(mine + ((c >> 1) * 2 + j) * 1024) + lane;
#pragma unroll
            for (int i = 0; i < 8; ++i)
              __stcg(dst + i * 32, make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]));
          }
        }
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0)
          last = atomicAdd(&args.split_tickets[ti.stile * kSplitTileTickets +
                                               static_cast<int>(rank) * 8 + (warp - 2)],
                           1) == 1;
        emit = __shfl_sync(0xffffffffu, last, 0) != 0;
        if (emit) __threadfence();  // the other part's sums are visible past the ticket
      }
      if (ti.unit >= 0 && emit) {
        // The second part folds the first one's sums into its accumulators
        // (own + other: fp32 addition of two terms is commutative, so the
        // result does not depend on which part finished first).
        const float* other = args.split_ws + static_cast<size_t>(ti.unit ^ 1) * kSplitUnitFloats + wslot;
        const int nu = ((nch - half + 1) >> 1) * NP;  // this warp's (chunk, accumulator) pairs
        auto load_other = [&](float4 (&o)[8], int k) {
          const int c = half + 2 * (k / NP);
          const float4* src =
              reinterpret_cast<const float4*>(other + ((c >> 1) * 2 + k % NP) * 1024) + lane;
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] = __ldcg(src + i * 32);
        };
#pragma unroll 1
        for (int k = 0; k < nu; ++k) {
          float4 cur[8];
          load_other(cur, k);
          const int c = half + 2 * (k / NP);
          const uint32_t ta = t_lane + (k % NP) * 256 + c * 32;
          float v[32];
          tmem_ld32(ta, v);
          tmem_ld_wait();
          reg_fence32(v);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            v[4 * i] += cur[i].x;
            v[4 * i + 1] += cur[i].y;
            v[4 * i + 2] += cur[i].z;
            v[4 * i + 3] += cur[i].w;
          }
          tmem_st32(ta, v);
        }
        tmem_st_wait();
      }
      if constexpr (STASH) {
        // Both accumulators of every chunk of this warp drained, activated and
        // packed into registers; TMEM goes back to the MMA for the next tile
        // before the stores, which then overlap that tile's main loop.
        uint32_t st[4][16];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int c = half + 2 * m;
          if (emit && c < nch) {
            float v[32], u[32];
            tmem_ld32(t_lane + c * 32, v);
            tmem_ld32(t_lane + 256 + c * 32, u);
            tmem_ld_wait();
            reg_fence32(v);
            reg_fence32(u);
            tok_activate<MODE>(v, u);
            tok_pack(v, lane, st[m]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&tempty_bar[acc]), 0));
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int c = half + 2 * m;
          if (emit && c < nch) {
            const int vt = min(32, ti.rows - c * 32);
            if (vt == 32 && lane == 0) bulk_wait_read0();
            __syncwarp();
            tok_store_packed(st[m], &tmO, stg, lane, vt, ti.row0 + c * 32, colw, args.N, out);
          }
        }
      } else {
#pragma unroll 1
        for (int c = half; emit && c < nch; c += 2) {
          const int vt = min(32, ti.rows - c * 32);  // tokens of this chunk inside the group
#pragma unroll
          for (int j = 0; j < NOUT; ++j) {
            float v[32], u[32];
            tmem_ld32(t_lane + j * 256 + c * 32, v);
            if (MODE == 1) tmem_ld32(t_lane + 256 + c * 32, u);
            tmem_ld_wait();
            reg_fence32(v);
            if (MODE == 1) reg_fence32(u);
            tok_activate<MODE>(v, u);
            if (vt == 32 && lane == 0) bulk_wait_read0();
            __syncwarp();
            tok_store_chunk(v, &tmO, stg, lane, vt, ti.row0 + c * 32, colw + j * 256, args.N,
                            out);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&tempty_bar[acc]), 0));
      }
      if (NACC == 1) {
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      } else {
        acc_phase ^= 1u;
      }
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

template <int MODE, int NACC, int BK, bool STASH = false>
static cudaError_t launch_tokn_t(const CUtensorMap* x, const CUtensorMap& w1,
                                 const CUtensorMap& w3, const CUtensorMap& o, const GemmArgs& g,
                                 int num_sms, cudaStream_t s) {
  using C = TokCfg<MODE, NACC, BK, STASH>;
  auto kern = k_gemm_tokn<MODE, NACC, BK, STASH>;
  if (log_enabled())
    log_line("token-as-N GEMM: %d accumulator(s) per tile, K %d per stage, %d stages of %d KB, "
             "%d producer warps, K-split tail %s", NACC, BK, C::STAGES, C::STAGE_BYTES / 1024,
             C::PROD, g.split_max > 1 && g.split_ws != nullptr ? "allowed" : "off");
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (err != cudaSuccess) return err;
  return launch_kernel(kern, dim3((num_sms / 2) * 2), dim3(C::THREADS), C::SMEM, s, 2, x[0], x[1],
                       x[2], w1, w3, o, g);
}

template <int MODE, int NACC, bool STASH = false>
static cudaError_t launch_tokn_bk(int bk, const CUtensorMap* x, const CUtensorMap& w1,
                                  const CUtensorMap& w3, const CUtensorMap& o, const GemmArgs& g,
                                  int num_sms, cudaStream_t s) {
  return bk == 128 ? launch_tokn_t<MODE, NACC, 128, STASH>(x, w1, w3, o, g, num_sms, s)
                   : launch_tokn_t<MODE, NACC, 64, STASH>(x, w1, w3, o, g, num_sms, s);
}

cudaError_t launch_gemm_tokn(int mode, const void* a_src, int a_rows, const void* b1,
                             const void* b3, const GemmArgs& g_in, int num_sms, cudaStream_t s) {
  if (g_in.sched == nullptr) return cudaErrorInvalidValue;
  GemmArgs g = g_in;
  // Tile shape per GEMM (measured on the Mixtral-shaped and page-1 layers):
  // SwiGLU keeps two accumulators (W1, W3) and 4 stages of K = 64; GELU one
  // double-buffered accumulator and 3 stages of K = 128; the down-projection
  // likewise, unless its token rows (R_max x K) outgrow half of L2, where two
  // accumulators per token tile halve their re-reads (4 stages of K = 64).
  bool two = mode == 1;
  if (mode == 2)
    two = static_cast<double>(g.R_max) * g.K * 2.0 > 64.0 * 1024 * 1024;
  if (mode != 1 && tuning().tokn_nacc != 0) two = tuning().tokn_nacc == 2;
  int bk = two ? 64 : 128;
  if (tuning().tokn_bk != 0) bk = tuning().tokn_bk == 64 ? 64 : 128;
  // K-split tail: measured on the Mixtral-shaped, 128-expert and 32-expert
  // layers, the SwiGLU GEMM-1 (W1 and W3 accumulators fill TMEM, epilogue not
  // overlapped) gains 1-2.5%; the down-projection loses up to 1% (two
  // accumulators: page-1 and 32-expert layers) or gains nothing, and the
  // double-buffered GELU GEMM-1 gains nothing, so they keep whole tiles.
  g.split_max = (mode == 1 && gemm_variant() != 4) ? tuning().tokn_split : 1;
  CUtensorMap mx[3], mw1, mw3, mo;
  const uint32_t box_rows[3] = {32, 64, 128};
  for (int i = 0; i < 3; ++i)
    if (!make_map_2d(&mx[i], a_src, static_cast<uint64_t>(a_rows), static_cast<uint64_t>(g.K),
                     box_rows[i]))
      return cudaErrorInvalidValue;
  if (!make_map_w(&mw1, b1, g.E, g.K, g.N, static_cast<uint32_t>(bk))) return cudaErrorInvalidValue;
  if (mode == 1) {
    if (!make_map_w(&mw3, b3, g.E, g.K, g.N, static_cast<uint32_t>(bk)))
      return cudaErrorInvalidValue;
  } else {
    mw3 = mw1;
  }
  if (!make_map_out(&mo, g.out, static_cast<uint64_t>(g.R_max), static_cast<uint64_t>(g.N)))
    return cudaErrorInvalidValue;
  switch (mode) {
    case 0: return two ? launch_tokn_bk<0, 2>(bk, mx, mw1, mw3, mo, g, num_sms, s)
                       : launch_tokn_bk<0, 1>(bk, mx, mw1, mw3, mo, g, num_sms, s);
    case 1: return tuning().tokn_stash
                       ? launch_tokn_bk<1, 2, true>(bk, mx, mw1, mw3, mo, g, num_sms, s)
                       : launch_tokn_bk<1, 2, false>(bk, mx, mw1, mw3, mo, g, num_sms, s);
    case 2: return two ? launch_tokn_bk<2, 2>(bk, mx, mw1, mw3, mo, g, num_sms, s)
                       : launch_tokn_bk<2, 1>(bk, mx, mw1, mw3, mo, g, num_sms, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
