// CPU oracle for the forward pass of one Mixture-of-Experts layer, in plain C++.
//
// TEST INFRASTRUCTURE.  A plain, slow, obviously-correct restatement of what the
// layer computes, used only to check the CUDA path (and timed as its CPU
// baseline).  Only the test suite, the smoke entry point and the bench's CPU leg
// load it; the product path never does.  It shares no code, header, table or
// helper with the CUDA library and includes nothing from it.
//
// It restates the same passages as the numpy oracle beside it (moe_oracle.py),
// in plain loops: no BLAS, float64 sums, OpenMP over independent rows.
//   "MoE模型高效推理：CANN算子库优化实践" §2.1 (gates = softmax(x @ W_gate), top-2,
//     sum of gate-weighted expert outputs) and §3.2.1 (renormalise kept gates);
//   "ops-transformer 仓库 - MoE 算子优化实战", 核心代码解析 (per expert: mask,
//     SparseGather, expert forward, SparseScatterAdd);
//   lshu.cn torch_npu fused-operator article §3 (x[tokens, hidden],
//     expert_weight[num_experts, hidden, intermediate], int32 token_expert_idx),
//     §5.2 (ids outside [0, num_experts) are errors), §5.3 (fixed per-expert
//     buffer that skewed routing overflows);
//   hnwysp.cn ops-transformer MoE article §3.2 (capacity_factor = 1.2 as an
//     over-allocation coefficient);
//   "ops-transformer 算子精讲" ch.8 (moe_router ..., normalize_scores=True).
// Readings where the pages are silent: C = ceil(cf*T*k/E) with cf the float32
// received and the ceiling exact; overflow dropped first-come in token order,
// then slot order; no second renormalisation after a drop; selection on fp32
// logits, ties to the lower expert id, NaN below -inf; slot 0 = largest logit;
// exact erf GELU; SwiGLU = silu(x W1) * (x W3); h, y and out rounded to the
// storage dtype (bf16: round to nearest, ties to even) where the layer stores them.
//
// Inputs (x, router and expert weights, bias) arrive as float32 arrays holding
// the exact stored values (every bf16 and fp32 value is exact in float32); all
// arithmetic is float64.  Status: 0 ok, 1 bad argument, 2 an
// expert id outside [0, E).
//
// Parity status: every function is pinned by tests/test_oracle_pins.py, which
// runs the same pins on this library and on the numpy oracle.
#include <cmath>
#include <cstdint>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

enum { DT_F32 = 0, DT_BF16 = 1 };
enum { ACT_SWIGLU = 0, ACT_GELU = 1, ACT_IDENTITY = 2 };

// Nearest bfloat16 of a float64 (ties to even), in one rounding step.  A normal
// v = m * 2^e (0.5 <= |m| < 1) rounds to a multiple of 2^(e-8); below the
// smallest normal exponent the spacing stays 2^-133.
double round_bf16(double a) {
  if (!std::isfinite(a) || a == 0.0) return a;
  int e = 0;
  std::frexp(a, &e);
  if (e < -125) e = -125;
  const double q = std::nearbyint(std::ldexp(a, 8 - e));  // default mode: ties to even
  const double r = std::ldexp(q, e - 8);
  if (std::fabs(r) >= std::ldexp(1.0, 128)) return std::copysign(INFINITY, a);
  return r;
}

double round_f32(double a) { return static_cast<double>(static_cast<float>(a)); }

double round_to(int dtype, double a) { return dtype == DT_BF16 ? round_bf16(a) : round_f32(a); }

// a ranks before b: larger logit first, NaN after everything, equal logits to
// the lower expert id.
bool ranks_before(float va, int ea, float vb, int eb) {
  const bool na = std::isnan(va), nb = std::isnan(vb);
  if (na != nb) return nb;
  if (!na && va != vb) return va > vb;
  return ea < eb;
}

// GELU(z) = z Phi(z) = 0.5 z (1 + erf(z / sqrt 2)), evaluated as 0.5 z erfc(-z / sqrt 2):
// the same function without the cancellation of 1 + erf for z below about -5.
double gelu(double z) { return 0.5 * z * std::erfc(-z / std::sqrt(2.0)); }
double silu(double z) { return z / (1.0 + std::exp(-z)); }

}  // namespace

extern "C" {

int oracle_round_bf16(const double* a, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = round_bf16(a[i]);
  return 0;
}

// logits[t][e] = fp32( sum_h x[t][h] * Wg[h][e] + b[e] ), the sum in float64 in h order.
int oracle_router_logits(const float* x, const float* wg, const float* bias, int T, int H, int E,
                         float* logits) {
  if (T < 0 || H < 0 || E < 1) return 1;
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) {
      double s = 0.0;
      for (int h = 0; h < H; ++h)
        s += static_cast<double>(x[static_cast<int64_t>(t) * H + h]) *
             static_cast<double>(wg[static_cast<int64_t>(h) * E + e]);
      if (bias) s += static_cast<double>(bias[e]);
      logits[static_cast<int64_t>(t) * E + e] = static_cast<float>(s);
    }
  }
  return 0;
}

// Top-k ids per token (slot 0 = largest logit) by insertion into a sorted list.
int oracle_topk_select(const float* logits, int T, int E, int k, int32_t* idx) {
  if (k < 1 || k > E) return 1;
  for (int t = 0; t < T; ++t) {
    const float* l = logits + static_cast<int64_t>(t) * E;
    std::vector<int> order;
    for (int e = 0; e < E; ++e) {
      size_t pos = order.size();
      while (pos > 0 && ranks_before(l[e], e, l[order[pos - 1]], order[pos - 1])) --pos;
      order.insert(order.begin() + pos, e);
    }
    for (int s = 0; s < k; ++s) idx[static_cast<int64_t>(t) * k + s] = order[s];
  }
  return 0;
}

// g[t][s] = exp(l_s - l_0) / sum_j exp(l_j - l_0) over the k selected, float64, stored fp32.
int oracle_topk_gates(const float* logits, const int32_t* idx, int T, int E, int k, float* gates) {
  for (int t = 0; t < T; ++t) {
    const float* l = logits + static_cast<int64_t>(t) * E;
    const int32_t* id = idx + static_cast<int64_t>(t) * k;
    if (k > 64) return 1;
    const double l0 = l[id[0]];
    double z[64], sum = 0.0;
    for (int s = 0; s < k; ++s) {
      z[s] = std::exp(static_cast<double>(l[id[s]]) - l0);
      sum += z[s];
    }
    for (int s = 0; s < k; ++s) gates[static_cast<int64_t>(t) * k + s] = static_cast<float>(z[s] / sum);
  }
  return 0;
}

// The literal form: p = softmax over all E, then p_s / sum of the kept p (float64).
int oracle_topk_gates_literal(const float* logits, const int32_t* idx, int T, int E, int k,
                              double* gates) {
  for (int t = 0; t < T; ++t) {
    const float* l = logits + static_cast<int64_t>(t) * E;
    double mx = -INFINITY;
    for (int e = 0; e < E; ++e) mx = std::fmax(mx, static_cast<double>(l[e]));
    double den = 0.0;
    for (int e = 0; e < E; ++e) den += std::exp(l[e] - mx);
    double kept = 0.0;
    for (int s = 0; s < k; ++s) kept += std::exp(l[idx[static_cast<int64_t>(t) * k + s]] - mx) / den;
    for (int s = 0; s < k; ++s)
      gates[static_cast<int64_t>(t) * k + s] =
          std::exp(l[idx[static_cast<int64_t>(t) * k + s]] - mx) / den / kept;
  }
  return 0;
}

// Threshold gating: p = softmax over all E (float64, NaN logits carry no mass);
// keep the experts with p > delta, largest first (ties to the lower id), at most
// k_max, the largest always; g_s = exp(l_s - l_0) / sum_kept exp(l_j - l_0).
// delta <= 0: 1/E (as float32).  idx/gate padded with -1 / 0.
int oracle_threshold_select(const float* logits, int T, int E, int k_max, float delta,
                            int32_t* idx, float* gate, int32_t* n_sel) {
  if (k_max < 1 || k_max > E || k_max > 64) return 1;
  const double d = delta > 0.0f ? static_cast<double>(delta)
                                : static_cast<double>(1.0f / static_cast<float>(E));
  for (int t = 0; t < T; ++t) {
    const float* l = logits + static_cast<int64_t>(t) * E;
    std::vector<int> order;  // insertion into descending order, as oracle_topk_select
    for (int e = 0; e < E; ++e) {
      size_t pos = order.size();
      while (pos > 0 && ranks_before(l[e], e, l[order[pos - 1]], order[pos - 1])) --pos;
      order.insert(order.begin() + pos, e);
    }
    double mx = -INFINITY;
    for (int e = 0; e < E; ++e)
      if (!std::isnan(l[e])) mx = std::fmax(mx, static_cast<double>(l[e]));
    double den = 0.0;
    for (int e = 0; e < E; ++e)
      if (!std::isnan(l[e])) den += std::exp(static_cast<double>(l[e]) - mx);
    int n = 1;
    while (n < k_max && std::exp(static_cast<double>(l[order[n]]) - mx) / den > d) ++n;
    double z[64], zs = 0.0;
    for (int s = 0; s < n; ++s) {
      z[s] = std::exp(static_cast<double>(l[order[s]]) - static_cast<double>(l[order[0]]));
      zs += z[s];
    }
    for (int s = 0; s < k_max; ++s) {
      idx[static_cast<int64_t>(t) * k_max + s] = s < n ? order[s] : -1;
      gate[static_cast<int64_t>(t) * k_max + s] = s < n ? static_cast<float>(z[s] / zs) : 0.0f;
    }
    n_sel[t] = n;
  }
  return 0;
}

// C = ceil(cf * T * k / E), exact for the float32 cf (cf = m * 2^x with integer m);
// *cap = -1 when cf <= 0 (no limit).
int oracle_capacity(float cf, int T, int k, int E, int64_t* cap) {
  if (E < 1 || T < 0 || k < 1) return 1;
  if (!(cf > 0.0f)) {
    *cap = -1;
    return 0;
  }
  int x = 0;
  const double m = std::frexp(static_cast<double>(cf), &x);  // cf = m * 2^x, 0.5 <= m < 1
  const int64_t mi = static_cast<int64_t>(std::ldexp(m, 24));  // exact: fp32 has 24 bits
  x -= 24;                                                     // cf = mi * 2^x
  const __int128 num0 = static_cast<__int128>(mi) * T * k;
  if (num0 == 0) {
    *cap = 0;
    return 0;
  }
  if (x >= 0) {
    if (x > 60) { *cap = INT64_MAX; return 0; }
    const __int128 num = num0 << x;
    *cap = static_cast<int64_t>((num + E - 1) / E);
    return 0;
  }
  if (-x > 120) {  // cf*T*k/E < 1: the ceiling is 1
    *cap = 1;
    return 0;
  }
  const __int128 den = static_cast<__int128>(E) << (-x);
  *cap = static_cast<int64_t>((num0 + den - 1) / den);
  return 0;
}

// Stable, capacity-limited permutation of (token, slot) pairs into expert-major
// rows, first come first kept (t ascending, then s).  cap < 0: no limit.
// empty_slots: id -1 marks an unused slot (threshold gating), skipped silently.
int oracle_permute(const int32_t* idx, int T, int k, int E, int64_t cap, int empty_slots,
                   int64_t* counts, int64_t* kept, int64_t* offsets, int64_t* row_token,
                   int64_t* row_slot, int64_t* row_map, int64_t* R_out) {
  const int64_t n = static_cast<int64_t>(T) * k;
  for (int64_t i = 0; i < n; ++i)
    if ((idx[i] < 0 || idx[i] >= E) && !(empty_slots && idx[i] == -1)) return 2;
  const int64_t limit = cap < 0 ? n : cap;
  std::vector<int64_t> arrival(n, -1);
  for (int e = 0; e < E; ++e) { counts[e] = 0; kept[e] = 0; }
  for (int64_t i = 0; i < n; ++i) {
    const int e = idx[i];
    if (e == -1) continue;
    counts[e] += 1;
    if (kept[e] < limit) arrival[i] = kept[e]++;
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + kept[e];
  const int64_t R = offsets[E];
  for (int64_t r = 0; r < R; ++r) { row_token[r] = -1; row_slot[r] = -1; }
  for (int64_t i = 0; i < n; ++i) {
    row_map[i] = -1;
    if (arrival[i] >= 0) {
      const int64_t r = offsets[idx[i]] + arrival[i];
      row_token[r] = i / k;
      row_slot[r] = i % k;
      row_map[i] = r;
    }
  }
  *R_out = R;
  return 0;
}

// y[r] = expert(e of r) applied to x[row_token[r]] for every kept row r:
// h = gelu(x W1) or silu(x W1) * (x W3) (rounded to dtype), y = h W2 (rounded);
// identity experts: y = x.  W1, W3 are [E][H][F]; W2 is [E][F][H].  Every sum
// runs over the reduction index in ascending order (the loops visit the weight
// rows in memory order and accumulate each output in its own float64 slot).
int oracle_grouped_ffn(const float* x, int T, int H, int F, int E, const int64_t* offsets,
                       const int64_t* row_token, const float* w1, const float* w3, const float* w2,
                       int act, int dtype, double* y) {
  if (act != ACT_SWIGLU && act != ACT_GELU && act != ACT_IDENTITY) return 1;
  for (int e = 0; e < E; ++e) {
    const int64_t r0 = offsets[e], r1 = offsets[e + 1];
    const float* W1 = w1 ? w1 + static_cast<int64_t>(e) * H * F : nullptr;
    const float* W3 = w3 ? w3 + static_cast<int64_t>(e) * H * F : nullptr;
    const float* W2 = w2 ? w2 + static_cast<int64_t>(e) * F * H : nullptr;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = r0; r < r1; ++r) {
      const int64_t t = row_token[r];
      double* yr = y + r * H;
      if (t < 0 || t >= T) continue;
      const float* xr = x + t * H;
      if (act == ACT_IDENTITY) {
        for (int j = 0; j < H; ++j) yr[j] = xr[j];
        continue;
      }
      std::vector<double> z1(F, 0.0), z3(act == ACT_SWIGLU ? F : 0, 0.0), h(F);
      for (int j = 0; j < H; ++j) {  // z1[f] = sum_j x[j] W1[j][f]
        const double xj = xr[j];
        const float* w1j = W1 + static_cast<int64_t>(j) * F;
        for (int f = 0; f < F; ++f) z1[f] += xj * static_cast<double>(w1j[f]);
        if (act == ACT_SWIGLU) {
          const float* w3j = W3 + static_cast<int64_t>(j) * F;
          for (int f = 0; f < F; ++f) z3[f] += xj * static_cast<double>(w3j[f]);
        }
      }
      for (int f = 0; f < F; ++f)
        h[f] = round_to(dtype, act == ACT_GELU ? gelu(z1[f]) : silu(z1[f]) * z3[f]);
      for (int j = 0; j < H; ++j) yr[j] = 0.0;
      for (int f = 0; f < F; ++f) {  // y[j] = sum_f h[f] W2[f][j]
        const double hf = h[f];
        const float* w2f = W2 + static_cast<int64_t>(f) * H;
        for (int j = 0; j < H; ++j) yr[j] += hf * static_cast<double>(w2f[j]);
      }
      for (int j = 0; j < H; ++j) yr[j] = round_to(dtype, yr[j]);
    }
  }
  return 0;
}

// out[t] = sum over s = 0..k-1 (in order) of g[t][s] * y[row_map[t][s]], float64,
// rounded once to dtype; dropped slots (-1) contribute nothing.
int oracle_combine(const double* y, int H, const float* gates, const int64_t* row_map, int T,
                   int k, int dtype, double* out) {
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t) {
    for (int j = 0; j < H; ++j) {
      double s = 0.0;
      for (int q = 0; q < k; ++q) {
        const int64_t r = row_map[static_cast<int64_t>(t) * k + q];
        if (r >= 0) s += static_cast<double>(gates[static_cast<int64_t>(t) * k + q]) * y[r * H + j];
      }
      out[static_cast<int64_t>(t) * H + j] = round_to(dtype, s);
    }
  }
  return 0;
}

// prob_mean[e] = (1/T) sum_t softmax(logits[t])[e], the softmax over all E, float64.
int oracle_router_prob_mean(const float* logits, int T, int E, double* prob_mean) {
  if (T < 0 || E < 1) return 1;
  for (int e = 0; e < E; ++e) prob_mean[e] = 0.0;
  std::vector<double> z(E);
  for (int t = 0; t < T; ++t) {
    const float* l = logits + static_cast<int64_t>(t) * E;
    double mx = -INFINITY;
    for (int e = 0; e < E; ++e) mx = std::fmax(mx, static_cast<double>(l[e]));
    double den = 0.0;
    for (int e = 0; e < E; ++e) { z[e] = std::exp(static_cast<double>(l[e]) - mx); den += z[e]; }
    for (int e = 0; e < E; ++e) prob_mean[e] += z[e] / den;
  }
  if (T > 0)
    for (int e = 0; e < E; ++e) prob_mean[e] /= T;
  return 0;
}

// out[t][i] = sum_j x[t][j] * W[idx[t]][j][i] (float64, j ascending), rounded to dtype.
// W is [E][H][I]; an id outside [0, E) is an error (status 2).
int oracle_expert_matmul(const float* x, const float* w, const int32_t* idx, int T, int H, int I,
                         int E, int dtype, double* out) {
  for (int t = 0; t < T; ++t)
    if (idx[t] < 0 || idx[t] >= E) return 2;
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < T; ++t) {
    const float* W = w + static_cast<int64_t>(idx[t]) * H * I;
    double* o = out + static_cast<int64_t>(t) * I;
    for (int i = 0; i < I; ++i) o[i] = 0.0;
    for (int j = 0; j < H; ++j) {
      const double xj = x[static_cast<int64_t>(t) * H + j];
      const float* wj = W + static_cast<int64_t>(j) * I;
      for (int i = 0; i < I; ++i) o[i] += xj * static_cast<double>(wj[i]);
    }
    for (int i = 0; i < I; ++i) o[i] = round_to(dtype, o[i]);
  }
  return 0;
}

// Elementwise activation (0: SiLU z / (1 + exp(-z)), 1: exact GELU), float64.
int oracle_activation(const double* z, int64_t n, int which, double* out) {
  if (which != 0 && which != 1) return 1;
  for (int64_t i = 0; i < n; ++i) out[i] = which == 1 ? gelu(z[i]) : silu(z[i]);
  return 0;
}

int oracle_num_threads(void) {
  int n = 1;
#pragma omp parallel
  {
#pragma omp single
    {
#ifdef _OPENMP
      n = omp_get_num_threads();
#endif
    }
  }
  return n;
}

}  // extern "C"
