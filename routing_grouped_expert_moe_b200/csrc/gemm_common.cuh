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
constexpr int G_SMEM = G_STAGES * G_STAGE_BYTES + 1024;
constexpr uint32_t G_TMEM_COLS = 512;

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

template <int MODE>
__device__ __forceinline__ void epilogue_store(const float (&v)[32], const float (&u)[32],
                                               __nv_bfloat16* dst, int cols_left) {
  uint32_t p[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float a0 = v[2 * i], a1 = v[2 * i + 1];
    if (MODE == 0) { a0 = gelu_f(a0); a1 = gelu_f(a1); }
    if (MODE == 1) { a0 = silu_f(a0) * u[2 * i]; a1 = silu_f(a1) * u[2 * i + 1]; }
    p[i] = pack_bf16x2(a0, a1);
  }
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int j = 0; j < 4; ++j)
    if (8 * j < cols_left) d[j] = make_uint4(p[4 * j], p[4 * j + 1], p[4 * j + 2], p[4 * j + 3]);
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

}  // namespace moe
