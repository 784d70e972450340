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
__device__ __forceinline__ void bulk_wait_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Registers written by an asynchronous tcgen05.ld are valid only after
// tcgen05.wait::ld; this empty asm makes every later use depend on a point
// after the wait, so the compiler cannot move a use above it.
__device__ __forceinline__ void reg_fence32(float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) asm volatile("" : "+f"(v[i]));
}

// Activations of the bf16 tensor-core epilogue, whose results are rounded to
// bf16 (relative spacing 2^-8), so a few fp32 ulps of error are invisible.
//
// GELU(z) = z Phi(z), Phi(z) = erfc(-z / sqrt 2) / 2.  erfc(x) for x >= 0 by the
// Chebyshev fit of Press, Teukolsky, Vetterling & Flannery, Numerical Recipes
// (2nd ed., section 6.2), fractional error below 1.2e-7 everywhere:
//   erfc(x) = t exp(-x^2 + P(t)),  t = 1 / (1 + x/2),  P a degree-9 polynomial.
// Then Phi(z) = 1 - erfc(|x|)/2 for z >= 0 and erfc(|x|)/2 for z < 0, so the
// negative tail keeps its relative accuracy (1 + erf(x) would cancel).
// SiLU(z) = z / (1 + e^-z).  Both use the special-function unit's exp and
// reciprocal and evaluate two columns per instruction.

// Reciprocal by the special-function unit (about 1 ulp; denominators here are
// at least 1, or infinite, giving 0).
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Packed fp32 arithmetic (two values per instruction, sm_100): the epilogue
// evaluates its activations on pairs of columns, halving the FMA-pipe
// instructions that compete with the producer and MMA warps for issue slots.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float2 splat2(float v) { return make_float2(v, v); }

// 2^x by the special-function unit.
__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// GELU of two values (see above): x = |z| / sqrt 2, t = 1 / (1 + x/2),
// erfc(x) = t 2^(log2(e) (P(t) - z^2/2)), Phi = 1 - erfc/2 (z >= 0) or erfc/2.
__device__ __forceinline__ float2 gelu_epi2(float2 z) {
  constexpr float kLog2e = 1.4426950408889634f;
  const float2 az = make_float2(fabsf(z.x), fabsf(z.y));
  const float2 den = ffma2(az, splat2(0.35355339059327376f), splat2(1.0f));  // 1 + |z|/(2 sqrt 2)
  const float2 t = make_float2(rcp_approx(den.x), rcp_approx(den.y));
  float2 p = splat2(0.17087277f);
  p = ffma2(p, t, splat2(-0.82215223f));
  p = ffma2(p, t, splat2(1.48851587f));
  p = ffma2(p, t, splat2(-1.13520398f));
  p = ffma2(p, t, splat2(0.27886807f));
  p = ffma2(p, t, splat2(-0.18628806f));
  p = ffma2(p, t, splat2(0.09678418f));
  p = ffma2(p, t, splat2(0.37409196f));
  p = ffma2(p, t, splat2(1.00002368f));
  p = ffma2(p, t, splat2(-1.26551223f));
  const float2 arg = ffma2(fmul2(z, z), splat2(-0.5f), p);  // P(t) - z^2/2
  const float2 a2 = fmul2(arg, splat2(kLog2e));
  const float2 e = fmul2(t, make_float2(ex2_approx(a2.x), ex2_approx(a2.y)));  // erfc(|z|/sqrt 2)
  const float2 h = fmul2(e, splat2(0.5f));
  const float2 phi = make_float2(z.x >= 0.f ? 1.0f - h.x : h.x, z.y >= 0.f ? 1.0f - h.y : h.y);
  return fmul2(z, phi);
}

// SiLU of two values: z / (1 + 2^(-z log2 e)).
__device__ __forceinline__ float2 silu_epi2(float2 z) {
  const float2 a = fmul2(z, splat2(-1.4426950408889634f));
  const float2 d = make_float2(1.0f + ex2_approx(a.x), 1.0f + ex2_approx(a.y));
  return fmul2(z, make_float2(rcp_approx(d.x), rcp_approx(d.y)));
}

// Activation of one thread's 32 accumulator columns, packed to bf16 pairs.
template <int MODE>
__device__ __forceinline__ void epilogue_pack(const float (&v)[32], const float (&u)[32],
                                              uint32_t (&p)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float2 a = make_float2(v[2 * i], v[2 * i + 1]);
    if (MODE == 0) a = gelu_epi2(a);
    if (MODE == 1) a = fmul2(silu_epi2(a), make_float2(u[2 * i], u[2 * i + 1]));
    p[i] = pack_bf16x2(a.x, a.y);
  }
}

// Writes one warp's 32 rows x 32 columns of output.  When all 32 rows belong
// to the tile's expert, the rows go through one of the warp's staging boxes in
// shared memory and one TMA bulk store (columns past N are clipped by the
// tensor map); otherwise (the ragged end of an expert, whose following rows
// belong to the next expert) each thread stores its own row, masked.  With
// two boxes used in turn, a box is rewritten only after the store issued from
// it two chunks earlier has read it (wait_group.read 1), unless the last
// committed store came from the same box (then wait for all).
template <int MODE>
__device__ __forceinline__ void epilogue_chunk(const float (&v)[32], const float (&u)[32],
                                               const CUtensorMap* tmO, uint8_t* stg_base, int box,
                                               int& last_box, int lane, bool box_full,
                                               int out_row0, int col0, int N,
                                               __nv_bfloat16* orow, bool row_ok) {
  uint32_t p[16];
  epilogue_pack<MODE>(v, u, p);
  const int cols_left = N - col0;
  if (cols_left <= 0) return;
  if (box_full) {
    uint8_t* stg = stg_base + box * G_STG_BYTES;
    if (lane == 0) {
      if (box == last_box) bulk_wait_read0();
      else bulk_wait_read1();
    }
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
    last_box = box;
  } else if (row_ok) {
    uint4* d = reinterpret_cast<uint4*>(orow);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (8 * j < cols_left) d[j] = make_uint4(p[4 * j], p[4 * j + 1], p[4 * j + 2], p[4 * j + 3]);
  }
}

// One epilogue warp's share of a finished accumulator tile (its 32 TMEM lanes,
// one half of the columns): TMEM -> registers -> activation -> bf16 -> global.
// Modes 0 and 2 (four 32-column chunks) load the next chunk from TMEM before
// working on the current one, so the load latency hides behind the
// activation; mode 1 reads the W1 and W3 halves of two chunks.  NBOX staging
// boxes (1 or 2) are used in turn.
template <int MODE, int NBOX>
__device__ __forceinline__ void epilogue_tile(uint32_t t_row, int half, const CUtensorMap* tmO,
                                              uint8_t* stg, int& last_box, int lane,
                                              bool box_full, bool row_ok, int out_row0, int n0,
                                              int N, __nv_bfloat16* orow) {
  constexpr int B1 = NBOX > 1 ? 1 : 0;
  if (MODE == 1) {
#pragma unroll 1
    for (int c = 2 * half; c < 2 * half + 2; ++c) {
      float g[32], u[32];
      tmem_ld32(t_row + c * 32, g);
      tmem_ld32(t_row + 128 + c * 32, u);
      tmem_ld_wait();
      reg_fence32(g);
      reg_fence32(u);
      epilogue_chunk<1>(g, u, tmO, stg, (c & 1) ? B1 : 0, last_box, lane, box_full, out_row0,
                        n0 + c * 32, N, row_ok ? orow + c * 32 : nullptr, row_ok);
    }
  } else {
    const int c0 = 4 * half;
    float va[32], vb[32];
    tmem_ld32(t_row + c0 * 32, va);
    tmem_ld_wait();
    reg_fence32(va);
#pragma unroll 1
    for (int i = 0; i < 4; i += 2) {
      const int c = c0 + i;
      tmem_ld32(t_row + (c + 1) * 32, vb);
      epilogue_chunk<MODE>(va, va, tmO, stg, 0, last_box, lane, box_full, out_row0, n0 + c * 32,
                           N, row_ok ? orow + c * 32 : nullptr, row_ok);
      tmem_ld_wait();
      reg_fence32(vb);
      if (i + 2 < 4) tmem_ld32(t_row + (c + 2) * 32, va);
      epilogue_chunk<MODE>(vb, vb, tmO, stg, B1, last_box, lane, box_full, out_row0,
                           n0 + (c + 1) * 32, N, row_ok ? orow + (c + 1) * 32 : nullptr, row_ok);
      if (i + 2 < 4) {
        tmem_ld_wait();
        reg_fence32(va);
      }
    }
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

// 3-D bf16 map over W[E, K, N] (N contiguous), box {64 N, box_k K, 1}, 128-byte swizzle.
inline bool make_map_w(CUtensorMap* m, const void* base, uint64_t E, uint64_t K, uint64_t N,
                       uint32_t box_k = 64) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {N, K, E};
  cuuint64_t strides[2] = {N * 2, K * N * 2};
  cuuint32_t box[3] = {64, box_k, 1};
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
