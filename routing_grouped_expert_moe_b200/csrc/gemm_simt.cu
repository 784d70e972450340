// fp32 grouped expert GEMM on CUDA cores, and the identity-expert row copy.
//
// Same contract as the tensor-core path (lshu.cn torch_npu fused-operator
// article §3: x[tokens, hidden] x expert_weight[num_experts, hidden,
// intermediate], activation, down-projection) for fp32 storage, where TF32
// tensor-core inputs would lose precision.  A persistent CTA walks the same
// (expert, n-tile, m-tile) list built from expert_offsets; each CTA computes a
// 64 x 64 output tile with 256 threads (4 x 4 outputs per thread), staging
// 16-wide K slices of A (optionally gathered through row_token) and W in
// shared memory.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int S_BM = 64, S_BN = 64, S_BK = 16, S_THREADS = 256;

template <int MODE, bool GATHER>
__global__ void __launch_bounds__(S_THREADS)
    k_gemm_simt(const float* __restrict__ A, const float* __restrict__ B1,
                const float* __restrict__ B3, const GemmArgs args) {
  __shared__ float As[S_BK][S_BM + 4];
  __shared__ float Bs[S_BK][S_BN];
  __shared__ float B3s[MODE == 1 ? S_BK : 1][MODE == 1 ? S_BN : 1];
  __shared__ int s_prefix[kMaxE + 1], s_start[kMaxE], s_rows[kMaxE], s_mt[kMaxE];
  pdl_wait_and_trigger();
  __shared__ int s_arow[S_BM];
  const int E = args.E, N = args.N, K = args.K;
  const int ntn = (N + S_BN - 1) / S_BN;
  if (threadIdx.x == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
      int s0 = args.offsets[e], rows = args.offsets[e + 1] - s0;
      if (rows < 0 || s0 < 0 || s0 + rows > args.R_max) {
        record_status(args.status, 1);
        rows = 0;
      }
      s_start[e] = s0;
      s_rows[e] = rows;
      s_mt[e] = (rows + S_BM - 1) / S_BM;
      s_prefix[e] = run;
      run += s_mt[e] * ntn;
    }
    s_prefix[E] = run;
  }
  __syncthreads();
  const int total = s_prefix[E];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float* out = static_cast<float*>(args.out);
  for (int tau = blockIdx.x; tau < total; tau += gridDim.x) {
    int e = 0;
    while (e + 1 < E && s_prefix[e + 1] <= tau) ++e;
    const int local = tau - s_prefix[e];
    const int nt = local / s_mt[e], mtile = local % s_mt[e];
    const int m0 = s_start[e] + mtile * S_BM;
    const int rows = min(S_BM, s_rows[e] - mtile * S_BM);
    const int n0 = nt * S_BN;
    const int tid = static_cast<int>(threadIdx.x);
    if (tid < S_BM) {
      const int r = tid < rows ? m0 + tid : -1;
      s_arow[tid] = r < 0 ? -1 : (GATHER ? args.row_token[r] : r);
    }
    float acc[4][4], acc3[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = acc3[i][j] = 0.f;
    const float* W1 = B1 + static_cast<size_t>(e) * K * N;
    const float* W3 = MODE == 1 ? B3 + static_cast<size_t>(e) * K * N : nullptr;
    for (int k0 = 0; k0 < K; k0 += S_BK) {
      __syncthreads();
      for (int i = threadIdx.x; i < S_BK * S_BM; i += S_THREADS) {
        const int m = i / S_BK, kk = i % S_BK;
        const int ar = s_arow[m];
        As[kk][m] = (ar >= 0 && k0 + kk < K) ? A[static_cast<size_t>(ar) * K + k0 + kk] : 0.f;
      }
      for (int i = threadIdx.x; i < S_BK * S_BN; i += S_THREADS) {
        const int kk = i / S_BN, n = i % S_BN;
        const bool ok = (k0 + kk < K) && (n0 + n < N);
        Bs[kk][n] = ok ? W1[static_cast<size_t>(k0 + kk) * N + n0 + n] : 0.f;
        if (MODE == 1) B3s[kk][n] = ok ? W3[static_cast<size_t>(k0 + kk) * N + n0 + n] : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < S_BK; ++kk) {
        float a[4], b[4], b3[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          b[j] = Bs[kk][tx * 4 + j];
          if (MODE == 1) b3[j] = B3s[kk][tx * 4 + j];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
            if (MODE == 1) acc3[i][j] = fmaf(a[i], b3[j], acc3[i][j]);
          }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty * 4 + i;
      if (r >= rows) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = n0 + tx * 4 + j;
        if (c >= N) continue;
        float v = acc[i][j];
        if (MODE == 0) v = gelu_f(v);
        if (MODE == 1) v = silu_f(v) * acc3[i][j];
        out[static_cast<size_t>(m0 + r) * N + c] = v;
      }
    }
  }
}

cudaError_t launch_gemm_simt(int mode, const void* a_src, const void* b1, const void* b3,
                             const GemmArgs& g, int num_sms, cudaStream_t s) {
  const float* A = static_cast<const float*>(a_src);
  const float* W1 = static_cast<const float*>(b1);
  const float* W3 = static_cast<const float*>(b3);
  const bool gather = g.row_token != nullptr;
  const int grid = num_sms * 2;
  const dim3 gd(grid), bd(S_THREADS);
  switch (mode * 2 + (gather ? 1 : 0)) {
    case 0: return launch_kernel(k_gemm_simt<0, false>, gd, bd, 0, s, 1, A, W1, W3, g);
    case 1: return launch_kernel(k_gemm_simt<0, true>, gd, bd, 0, s, 1, A, W1, W3, g);
    case 2: return launch_kernel(k_gemm_simt<1, false>, gd, bd, 0, s, 1, A, W1, W3, g);
    case 3: return launch_kernel(k_gemm_simt<1, true>, gd, bd, 0, s, 1, A, W1, W3, g);
    case 4: return launch_kernel(k_gemm_simt<2, false>, gd, bd, 0, s, 1, A, W1, W3, g);
    case 5: return launch_kernel(k_gemm_simt<2, true>, gd, bd, 0, s, 1, A, W1, W3, g);
    default: return cudaErrorInvalidValue;
  }
}

// Rows of the expert segments: out[r] = A[row_token[r]] (gather) or A[r], for
// offsets[0] <= r < offsets[E] (identity experts, and the gather ahead of the
// dense GEMM).  A gathered row outside [0, T) is reported (invalid argument)
// and skipped.
__global__ void k_copy_rows(const uint8_t* __restrict__ A, const GemmArgs g, int row_bytes) {
  pdl_wait_and_trigger();
  const int R = min(g.offsets[g.E], g.R_max);
  const int r0 = max(0, g.offsets[0]);
  const int vecs = row_bytes / 16;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int r = r0 + warp; r < R; r += nwarps) {
    const int src_row = g.row_token ? g.row_token[r] : r;
    if (g.row_token && (src_row < 0 || src_row >= g.T)) {
      if (lane == 0) record_status(g.status, 1);
      continue;
    }
    const int4* src = reinterpret_cast<const int4*>(A + static_cast<size_t>(src_row) * row_bytes);
    int4* dst = reinterpret_cast<int4*>(static_cast<uint8_t*>(g.out) +
                                        static_cast<size_t>(r) * row_bytes);
    for (int v = lane; v < vecs; v += 32) dst[v] = __ldg(src + v);
  }
}

cudaError_t launch_copy_rows(const void* a_src, const GemmArgs& g, int elem_bytes, cudaStream_t s) {
  return launch_kernel(k_copy_rows, dim3(1184), dim3(256), 0, s, 1,
                       static_cast<const uint8_t*>(a_src), g, g.N * elem_bytes);
}

}  // namespace moe
