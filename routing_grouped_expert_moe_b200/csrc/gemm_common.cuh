// Pieces shared by the grouped expert GEMM kernels (one CTA per tile, and CTA
// pairs): tile geometry, the device-side tile decode, the activation epilogue
// and the host-side TMA tensor-map encoders.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int G_BM = 128;
constexpr int G_BK = 64;
constexpr int G_STAGES = 4;
constexpr int G_ACC_N = 256;
constexpr int G_A_BYTES = G_BM * G_BK * 2;       // 16 KB
constexpr int G_BCHUNK = 64 * G_BK * 2;          // one 64-column box: 8 KB
constexpr int G_B_BYTES = G_ACC_N * G_BK * 2;    // 32 KB
constexpr int G_STAGE_BYTES = G_A_BYTES + G_B_BYTES;
constexpr int G_THREADS = 320;  // producer, MMA, 8 epilogue warps (2 per TMEM lane quarter)
constexpr int G_EPI_WARPS = 8;
constexpr int G_STG_BYTES = 32 * 32 * 2;  // one epilogue warp's staging box: 32 rows x 32 bf16
constexpr int G_SMEM = G_STAGES * G_STAGE_BYTES + G_EPI_WARPS * G_STG_BYTES + 1024;
constexpr uint32_t G_TMEM_COLS = 512;
// Default L2 prefetch distance of the GEMM producers, in k-blocks (0: off).
constexpr int kGemmPrefetchDist = 0;

template <int MODE>
struct ModeCfg {
  static constexpr int BN_OUT = MODE == 1 ? 128 : 256;
};

struct TileInfo {
  int e, m0, rows, n0;
};

__device__ __forceinline__ TileInfo decode_tile(int tau, const int* prefix, const int* seg_start,
                                                const int* seg_rows, const int* mtiles, int E,
                                                int bn_out) {
  int lo = 0, hi = E;  // largest e with prefix[e] <= tau (empty experts are skipped)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= tau) lo = mid; else hi = mid;
  }
  TileInfo t;
  t.e = lo;
  const int local = tau - prefix[lo];
  const int mt = mtiles[lo];
  const int n_tile = local / mt;
  const int m_tile = local - n_tile * mt;
  t.m0 = seg_start[lo] + m_tile * G_BM;
  t.rows = min(G_BM, seg_rows[lo] - m_tile * G_BM);
  t.n0 = n_tile * bn_out;
  return t;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Activation of one thread's 32 accumulator columns, packed to bf16 pairs.
template <int MODE>
__device__ __forceinline__ void epilogue_pack(const float (&v)[32], const float (&u)[32],
                                              uint32_t (&p)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float a0 = v[2 * i], a1 = v[2 * i + 1];
    if (MODE == 0) { a0 = gelu_f(a0); a1 = gelu_f(a1); }
    if (MODE == 1) { a0 = silu_f(a0) * u[2 * i]; a1 = silu_f(a1) * u[2 * i + 1]; }
    p[i] = pack_bf16x2(a0, a1);
  }
}

// Writes one warp's 32 rows x 32 columns of output.  When all 32 rows belong
// to the tile's expert, the rows go through the warp's 2 KB staging box in
// shared memory and one TMA bulk store (columns past N are clipped by the
// tensor map); otherwise (the ragged end of an expert, whose following rows
// belong to the next expert) each thread stores its own row, masked.
template <int MODE>
__device__ __forceinline__ void epilogue_chunk(const float (&v)[32], const float (&u)[32],
                                               const CUtensorMap* tmO, uint8_t* stg, int lane,
                                               bool box_full, int out_row0, int col0, int N,
                                               __nv_bfloat16* orow, bool row_ok) {
  uint32_t p[16];
  epilogue_pack<MODE>(v, u, p);
  const int cols_left = N - col0;
  if (cols_left <= 0) return;
  if (box_full) {
    if (lane == 0) bulk_wait_read0();  // the previous store has read the box
    __syncwarp();
    // row `lane` = 64 bytes; 16-byte pieces in rotated order spread the banks
    const uint4 q0 = make_uint4(p[0], p[1], p[2], p[3]);
    const uint4 q1 = make_uint4(p[4], p[5], p[6], p[7]);
    const uint4 q2 = make_uint4(p[8], p[9], p[10], p[11]);
    const uint4 q3 = make_uint4(p[12], p[13], p[14], p[15]);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = (j + lane) & 3;
      const uint4 w = c == 0 ? q0 : (c == 1 ? q1 : (c == 2 ? q2 : q3));
      *reinterpret_cast<uint4*>(stg + lane * 64 + c * 16) = w;
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tmO, stg, col0, out_row0);
      bulk_commit();
    }
  } else if (row_ok) {
    uint4* d = reinterpret_cast<uint4*>(orow);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (8 * j < cols_left) d[j] = make_uint4(p[4 * j], p[4 * j + 1], p[4 * j + 2], p[4 * j + 3]);
  }
}

// ----------------------------------------------------------------------------
// Host: TMA tensor maps
// ----------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 map over [rows, cols] (cols contiguous) with box {64, box_rows}, 128-byte swizzle.
inline bool make_map_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                        uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 map over W[E, K, N] (N contiguous), box {64 N, 64 K, 1}, 128-byte swizzle.
inline bool make_map_w(CUtensorMap* m, const void* base, uint64_t E, uint64_t K, uint64_t N) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {N, K, E};
  cuuint64_t strides[2] = {N * 2, K * N * 2};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output [rows, cols] bf16 (cols contiguous), 32 x 32 boxes, no swizzle: the
// epilogue's TMA bulk stores.
inline bool make_map_out(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace moe
