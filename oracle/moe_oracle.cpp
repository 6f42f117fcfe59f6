// Plain CPU oracle of the GPT-OSS-style MoE feed-forward layer.
//
// TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
// benchmark's CPU-baseline leg may load this library. The CUDA path shares no
// code with it, and it includes nothing from the CUDA path.
//
// What it computes, per token t (every step cites where the layer is stated):
//   1. router linear with bias: l[e] = sum_d x[t,d] * Wr[e,d] + br[e]
//      (torchtitan GPT-OSS guide, "HuggingFace weight adapter": the router is
//      moe.router.gate.weight/bias, a linear layer with bias; from-scratch
//      GPT-OSS write-up, "model flow" diagram, "expert routing (top-4)").
//      Accumulated in double, then rounded once to float.
//   2. top-k: the k largest logits, ordered by (logit descending, expert index
//      ascending), so ties go to the lower expert index.
//   3. gate weights: softmax over the k chosen logits only,
//      w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0); computed in double, stored
//      as float.
//   4. expert FFN for each chosen expert e (torchtitan GPT-OSS guide,
//      "grouped matrix multiplication": weights stored (num_experts, out_dim,
//      in_dim), mlp1 then SwiGLU then mlp2, each with a bias):
//        u[n] = sum_d x[t,d] * W1[e,n,d] + b1[e,n],   n < 2I
//        h[i] = bf16( act(u[i], u[I+i]) ),            i < I
//      act = plain SwiGLU silu(g) * u with silu(g) = g/(1+e^-g) (act 0), or
//      the GPT-OSS variant (act 1; torchtitan GPT-OSS guide, paragraph on
//      GptOssGroupedExperts' SwiGLU variant): the gate branch is clamped from
//      above at `limit` and multiplied by sigmoid(alpha * gate), the linear
//      branch is clipped to [-limit, limit] and offset by 1:
//        gc = min(g, limit), uc = min(max(u, -limit), limit),
//        act = gc * sigmoid(alpha * gc) * (uc + 1);
//      alpha and limit are the caller's (the pages do not give them).
//        o[c] = sum_i h[i] * W2[e,c,i] + b2[e,c],     c < D
//      rows [0,I) of W1[e] are the gate half, rows [I,2I) the up half.
//   5. weighted combine (from-scratch GPT-OSS write-up, "model flow" diagram,
//      "weighted combination"): y[t,c] = bf16( sum_j w_j * o_j[c] ), j in
//      order; the gate weight scales the whole expert output, bias included.
//   Permutation (torchtitan GPT-OSS guide, "grouped matrix multiplication":
//   num_tokens_per_expert and offsets = cumsum of it): assignments a = t*k+j
//   sorted stably by expert, counts[e], exclusive offsets[0..E],
//   perm[row] = a and inv[a] = row.
//   MXFP4 expert weights (GPT-OSS in Transformers blog, MXFP4 paragraph: 4-bit
//   floats laid out E2M1 -- 1 sign, 2 exponent, 1 mantissa bit -- with one
//   scale per 32-element block): value = e2m1(code) * 2^(scale - 127), codes
//   two per byte along the reduction dim with the even element in the low
//   nibble, scales one E8M0 byte per 32 consecutive reduction elements.
//
// All accumulations are in double; rounding points are only those listed
// above (logits and gate weights to float, h and y to bf16).
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <algorithm>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

double bf16_to_double(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return static_cast<double>(f);
}

// Round a double to the nearest bf16 (8 significant bits, float's exponent
// range), ties to even, in one rounding step.
uint16_t double_to_bf16(double v) {
  if (std::isnan(v)) return 0x7fc0;
  if (std::isinf(v)) return v > 0 ? 0x7f80 : 0xff80;
  double a = std::fabs(v);
  double r;
  const double min_normal = std::ldexp(1.0, -126);
  if (a < min_normal) {
    // subnormal bf16 spacing is 2^-133
    r = std::nearbyint(std::ldexp(a, 133));
    r = std::ldexp(r, -133);
  } else {
    int ex;
    double m = std::frexp(a, &ex);  // a = m * 2^ex, m in [0.5, 1)
    r = std::nearbyint(std::ldexp(m, 8));  // 8 significant bits
    r = std::ldexp(r, ex - 8);
  }
  float f = static_cast<float>(std::copysign(r, v));  // exact (or inf on overflow)
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return static_cast<uint16_t>(u >> 16);
}

// E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa; exponent 0
// is subnormal (0.m * 2^0).
double e2m1_value(unsigned code) {
  unsigned s = (code >> 3) & 1u, ex = (code >> 1) & 3u, m = code & 1u;
  double mag = ex == 0 ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, static_cast<int>(ex) - 1);
  return s ? -mag : mag;
}

double e8m0_value(uint8_t s) {
  if (s == 0xff) return std::nan("");
  return std::ldexp(1.0, static_cast<int>(s) - 127);
}

// Expert weight element W[e][n][kk] of an (E, N, K) tensor.
struct Weights {
  int fmt;  // 0 bf16, 1 mxfp4
  const uint16_t* bf16;
  const uint8_t* codes;
  const uint8_t* scales;
  int64_t N, K;
  double at(int64_t e, int64_t n, int64_t kk) const {
    if (fmt == 0) return bf16_to_double(bf16[(e * N + n) * K + kk]);
    uint8_t byte = codes[(e * N + n) * (K / 2) + kk / 2];
    unsigned code = (kk & 1) ? (byte >> 4) : (byte & 0xf);
    return e2m1_value(code) * e8m0_value(scales[(e * N + n) * (K / 32) + kk / 32]);
  }
};

double silu(double g) { return g / (1.0 + std::exp(-g)); }

struct Act {
  int kind;  // 0 plain SwiGLU, 1 GPT-OSS variant
  double alpha, limit;
  double operator()(double g, double u) const {
    if (kind == 0) return silu(g) * u;
    const double gc = std::min(g, limit);
    const double uc = std::min(std::max(u, -limit), limit);
    return gc / (1.0 + std::exp(-alpha * gc)) * (uc + 1.0);
  }
};

void route_token(int64_t t, int D, int E, int k, const uint16_t* x, const uint16_t* Wr,
                 const uint16_t* br, float* logits_row, int32_t* idx_row, float* w_row) {
  std::vector<float> l(E);
  for (int e = 0; e < E; ++e) {
    double acc = 0.0;
    for (int d = 0; d < D; ++d)
      acc += bf16_to_double(x[t * D + d]) * bf16_to_double(Wr[static_cast<int64_t>(e) * D + d]);
    acc += bf16_to_double(br[e]);
    l[e] = static_cast<float>(acc);
    if (logits_row) logits_row[e] = l[e];
  }
  std::vector<int> order(E);
  for (int e = 0; e < E; ++e) order[e] = e;
  std::sort(order.begin(), order.end(), [&](int a, int b) {
    if (l[a] != l[b]) return l[a] > l[b];
    return a < b;
  });
  double lmax = l[order[0]];
  double denom = 0.0;
  for (int j = 0; j < k; ++j) denom += std::exp(static_cast<double>(l[order[j]]) - lmax);
  for (int j = 0; j < k; ++j) {
    idx_row[j] = order[j];
    w_row[j] = static_cast<float>(std::exp(static_cast<double>(l[order[j]]) - lmax) / denom);
  }
}

// Expert FFN output o (length D, double) of token row x_row for expert e.
void expert_ffn(const uint16_t* x_row, int D, int I, int64_t e, const Weights& W1, const uint16_t* b1,
                const Weights& W2, const uint16_t* b2, const Act& act, std::vector<double>& u, std::vector<double>& h,
                std::vector<double>& o) {
  const int64_t twoI = 2 * static_cast<int64_t>(I);
  for (int64_t n = 0; n < twoI; ++n) {
    double acc = 0.0;
    for (int d = 0; d < D; ++d) acc += bf16_to_double(x_row[d]) * W1.at(e, n, d);
    u[n] = acc + bf16_to_double(b1[e * twoI + n]);
  }
  for (int i = 0; i < I; ++i) h[i] = bf16_to_double(double_to_bf16(act(u[i], u[I + i])));
  for (int c = 0; c < D; ++c) {
    double acc = 0.0;
    for (int i = 0; i < I; ++i) acc += h[i] * W2.at(e, c, i);
    o[c] = acc + bf16_to_double(b2[e * D + c]);
  }
}

bool dims_ok(int64_t T, int D, int E, int k, int I) {
  return T >= 0 && D > 0 && E > 0 && k > 0 && k <= E && I > 0;
}

}  // namespace

extern "C" {

// Number of OpenMP threads the oracle uses.
int oracle_num_threads() {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

// Round n doubles to bf16 bit patterns (round to nearest, ties to even).
void oracle_round_bf16(const double* in, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = double_to_bf16(in[i]);
}

// Dequantize an MXFP4 (N, K) matrix to doubles.
int oracle_dequant_mxfp4(const uint8_t* codes, const uint8_t* scales, int64_t N, int64_t K, double* out) {
  if (K % 32) return 1;
  Weights w{1, nullptr, codes, scales, N, K};
  for (int64_t n = 0; n < N; ++n)
    for (int64_t kk = 0; kk < K; ++kk) out[n * K + kk] = w.at(0, n, kk);
  return 0;
}

// Router + top-k + softmax for all T tokens. logits (T x E) may be null.
int oracle_route(int64_t T, int D, int E, int k, const uint16_t* x, const uint16_t* Wr, const uint16_t* br,
                 float* logits, int32_t* topk_idx, float* topk_w) {
  if (!dims_ok(T, D, E, k, 1)) return 1;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t)
    route_token(t, D, E, k, x, Wr, br, logits ? logits + t * E : nullptr, topk_idx + t * k, topk_w + t * k);
  return 0;
}

// Stable counting sort of the T*k assignments by expert.
int oracle_permute(int64_t T, int E, int k, const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                   int32_t* perm, int32_t* inv) {
  const int64_t R = T * k;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t a = 0; a < R; ++a) {
    if (topk_idx[a] < 0 || topk_idx[a] >= E) return 2;
    counts[topk_idx[a]]++;
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  std::vector<int64_t> next(offsets, offsets + E);
  for (int64_t a = 0; a < R; ++a) {
    int64_t row = next[topk_idx[a]]++;
    perm[row] = static_cast<int32_t>(a);
    inv[a] = static_cast<int32_t>(row);
  }
  return 0;
}

// Expert FFN + weighted combine for the listed tokens, given the routing.
// wfmt 0: W1 (E,2I,D) and W2 (E,D,I) are bf16. wfmt 1: they are MXFP4 codes
// (E,2I,D/2), (E,D,I/2) with scales (E,2I,D/32), (E,D,I/32).
// y_out: ntok x D bf16. o_out (nullable): ntok x k x D doubles, the unweighted
// expert outputs o_j. y_exact (nullable): ntok x D doubles, the weighted sum
// before its final bf16 rounding.
int oracle_ffn_tokens(int64_t T, int D, int E, int k, int I, int wfmt, int act_kind, double act_alpha,
                      double act_limit, const uint16_t* x, const int32_t* topk_idx, const float* topk_w,
                      const void* W1, const uint8_t* W1_scales, const uint16_t* b1, const void* W2,
                      const uint8_t* W2_scales, const uint16_t* b2, const int64_t* tokens, int64_t ntok,
                      uint16_t* y_out, double* o_out, double* y_exact) {
  if (!dims_ok(T, D, E, k, I)) return 1;
  if (act_kind != 0 && act_kind != 1) return 1;
  const Act act{act_kind, act_alpha, act_limit};
  if (wfmt != 0 && wfmt != 1) return 1;
  if (wfmt == 1 && (D % 32 || I % 32)) return 1;
  Weights w1{wfmt, static_cast<const uint16_t*>(W1), static_cast<const uint8_t*>(W1), W1_scales, 2 * static_cast<int64_t>(I), D};
  Weights w2{wfmt, static_cast<const uint16_t*>(W2), static_cast<const uint8_t*>(W2), W2_scales, D, I};
  int err = 0;
#pragma omp parallel
  {
    std::vector<double> u(2 * static_cast<size_t>(I)), h(I), o(D), y(D);
#pragma omp for schedule(dynamic, 1)
    for (int64_t s = 0; s < ntok; ++s) {
      int64_t t = tokens[s];
      if (t < 0 || t >= T) {
#pragma omp atomic write
        err = 2;
        continue;
      }
      std::fill(y.begin(), y.end(), 0.0);
      for (int j = 0; j < k; ++j) {
        int e = topk_idx[t * k + j];
        if (e < 0 || e >= E) {
#pragma omp atomic write
          err = 2;
          break;
        }
        expert_ffn(x + t * D, D, I, e, w1, b1, w2, b2, act, u, h, o);
        double wj = static_cast<double>(topk_w[t * k + j]);
        for (int c = 0; c < D; ++c) y[c] += wj * o[c];
        if (o_out)
          for (int c = 0; c < D; ++c) o_out[(s * k + j) * D + c] = o[c];
      }
      for (int c = 0; c < D; ++c) y_out[s * D + c] = double_to_bf16(y[c]);
      if (y_exact)
        for (int c = 0; c < D; ++c) y_exact[s * D + c] = y[c];
    }
  }
  return err;
}

// The whole layer for all tokens: route, then FFN + combine.
int oracle_forward(int64_t T, int D, int E, int k, int I, int wfmt, int act_kind, double act_alpha,
                   double act_limit, const uint16_t* x, const uint16_t* Wr, const uint16_t* br, const void* W1,
                   const uint8_t* W1_scales, const uint16_t* b1, const void* W2, const uint8_t* W2_scales,
                   const uint16_t* b2, uint16_t* y, int32_t* topk_idx, float* topk_w) {
  int rc = oracle_route(T, D, E, k, x, Wr, br, nullptr, topk_idx, topk_w);
  if (rc) return rc;
  std::vector<int64_t> tokens(T);
  for (int64_t t = 0; t < T; ++t) tokens[t] = t;
  return oracle_ffn_tokens(T, D, E, k, I, wfmt, act_kind, act_alpha, act_limit, x, topk_idx, topk_w, W1, W1_scales,
                           b1, W2, W2_scales, b2, tokens.data(), T, y, nullptr, nullptr);
}

}  // extern "C"
