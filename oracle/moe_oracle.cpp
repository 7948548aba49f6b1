// Oracle for the DeepSeekMoE layer forward — TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, obviously correct CPU restatement of what one DeepSeekMoE
// layer computes, used to check the CUDA path. Only tests/, the package's
// smoke() entry and bench.py's CPU-baseline leg may load it. It shares no code,
// header, table or helper with the CUDA library and includes no CUDA header.
//
// Sources (the pages this follows):
//  [V3-notes]  DeepSeek-V3 model.py notes (73biji.xyz/llm_pp_dsv3):
//              - "DeepSeekMoE 三改进" passage and its total-output equation
//                h'_t = u_t + FFN_share(u_t) + sum_r g_{i,t} FFN_r(u_t);
//              - "V3 改进①：无辅助损失负载均衡" (s_{i,t} + b_i enters top-k only);
//              - "Gate 选专家流程（model.py，五步）" (the five gate steps);
//              - "MoE 前向四步" (gate -> y[idx] += expert(x[idx]) * w -> + z).
//  [V2-card]   DeepSeek-V2 model card (aigallery), "架构简图" (160 routed, top-6,
//              2 shared).
// The expert body is SwiGLU, W2 (silu(W1 v) * W3 v), with silu(g) = g*sigmoid(g)
// (the pages only say "FFN"; SwiGLU is the stated reading).
//
// Precision: dot products and the FFN are accumulated in double; logits and
// scores are rounded to fp32; the selection arithmetic of gate steps 2-5
// (s + b, group score, renormalisation, route_scale) runs in fp32, in the order
// written below, so that a GPU gate fed the same fp32 scores can be compared
// index for index.
//
// Readings where the pages are silent:
//  - ties in both top-k's go to the lower index (groups and experts);
//  - idx is returned in descending key order;
//  - renormalisation is a config switch (on for sigmoid, off for softmax);
//  - the group score is the max of the group's keys (AMAX) or the fp32 sum of
//    its two largest keys (TOP2SUM);
//  - the bias enters only the selection; the weights gather raw scores.
//
// Parity pins for every function here are in tests/test_oracle_pins.py.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {

// Mirrors the fields a caller fixes for one layer. All "auto" choices are
// resolved by the Python wrapper before the call.
typedef struct {
  int32_t n_experts;    // E, routed experts
  int32_t n_groups;     // G
  int32_t topk_groups;  // TG
  int32_t topk;         // k
  float route_scale;
  int32_t score_func;   // 0 sigmoid, 1 softmax
  int32_t dim;          // d
  int32_t inter;        // I, per-expert SwiGLU hidden size
  int32_t n_shared;     // S
  int32_t norm_topk;    // 0/1: divide gathered scores by their sum
  int32_t group_score;  // 1 AMAX, 2 TOP2SUM (ignored when n_groups == 1)
  int32_t add_residual; // 0/1: add u_t to the output
} oracle_cfg;

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"

namespace {

// bf16 -> fp32 is exact: the 16 stored bits are the top half of an fp32.
inline double load_elem(const void* base, int dtype, int64_t i) {
  if (dtype == 0) return (double)((const float*)base)[i];
  uint32_t bits = (uint32_t)((const uint16_t*)base)[i] << 16;
  float f;
  std::memcpy(&f, &bits, sizeof f);
  return (double)f;
}

const float kNegInf = -std::numeric_limits<float>::infinity();

// Order used by both top-k's: larger key first, lower index on equal keys.
struct KeyIdx {
  float key;
  int idx;
};
inline bool before(const KeyIdx& a, const KeyIdx& b) {
  if (a.key != b.key) return a.key > b.key;
  return a.idx < b.idx;
}

// Gate steps 2-5 for one token, from its fp32 scores s[E] (post score function).
// Outputs: key[E] (s + b, -inf outside the kept groups), gsc[G], idx[k], w[k],
// and the two selection margins.
void select_one(const oracle_cfg& c, const float* s, const float* bias, float* key,
                float* gsc, int32_t* idx, float* w, float* kth_margin,
                float* grp_margin) {
  const int E = c.n_experts, G = c.n_groups, TG = c.topk_groups, k = c.topk;
  const int gs = E / G;

  // s_{i,t} + b_i takes part in the selection only ("V3 改进①").
  for (int e = 0; e < E; ++e) key[e] = bias ? (float)(s[e] + bias[e]) : s[e];

  // Group-limited routing ("Gate 选专家流程", steps 2-3).
  *grp_margin = std::numeric_limits<float>::infinity();
  if (G > 1) {
    std::vector<float> grp(gs);
    for (int g = 0; g < G; ++g) {
      for (int i = 0; i < gs; ++i) grp[i] = key[g * gs + i];
      std::sort(grp.begin(), grp.end(), [](float a, float b) { return a > b; });
      gsc[g] = (c.group_score == 2) ? (float)(grp[0] + grp[1]) : grp[0];
    }
    std::vector<KeyIdx> order(G);
    for (int g = 0; g < G; ++g) order[g] = {gsc[g], g};
    std::sort(order.begin(), order.end(), before);
    std::vector<char> keep(G, 0);
    for (int r = 0; r < TG; ++r) keep[order[r].idx] = 1;
    if (TG < G) *grp_margin = order[TG - 1].key - order[TG].key;
    for (int e = 0; e < E; ++e)
      if (!keep[e / gs]) key[e] = kNegInf;
  } else if (gsc) {
    gsc[0] = 0.f;
  }

  // Global top-k over the masked keys (step 4).
  std::vector<KeyIdx> order(E);
  for (int e = 0; e < E; ++e) order[e] = {key[e], e};
  std::sort(order.begin(), order.end(), before);
  for (int j = 0; j < k; ++j) idx[j] = order[j].idx;
  *kth_margin = std::numeric_limits<float>::infinity();
  if (k < E && order[k].key != kNegInf) *kth_margin = order[k - 1].key - order[k].key;

  // Gather the raw scores, renormalise, times route_scale (step 5).
  float sum = 0.f;
  for (int j = 0; j < k; ++j) sum = sum + s[idx[j]];
  for (int j = 0; j < k; ++j) {
    float v = s[idx[j]];
    if (c.norm_topk) v = v / sum;
    w[j] = v * c.route_scale;
  }
}

// One SwiGLU expert on one token, accumulating weight * FFN(u) into acc[d].
void expert_ffn_acc(const oracle_cfg& c, int dtype, const double* u, const void* w1,
                    const void* w3, const void* w2, double weight, double* acc) {
  const int d = c.dim, I = c.inter;
  std::vector<double> h(I);
  for (int f = 0; f < I; ++f) {
    double g = 0.0, v = 0.0;
    for (int i = 0; i < d; ++i) {
      g += load_elem(w1, dtype, (int64_t)f * d + i) * u[i];
      v += load_elem(w3, dtype, (int64_t)f * d + i) * u[i];
    }
    double silu = g / (1.0 + std::exp(-g));
    h[f] = silu * v;
  }
  for (int o = 0; o < d; ++o) {
    double y = 0.0;
    for (int f = 0; f < I; ++f) y += load_elem(w2, dtype, (int64_t)o * I + f) * h[f];
    acc[o] += weight * y;
  }
}

}  // namespace

extern "C" {

// Gate logits l = u W_g^T ("DeepSeekMoE 三改进": W_g u_t), double accumulate,
// rounded to fp32. x [T, d], w_gate [E, d], both row-major in `dtype`.
int oracle_gate_logits(const oracle_cfg* c, int64_t T, int dtype, const void* x,
                       const void* w_gate, float* logits) {
  const int E = c->n_experts, d = c->dim;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t t = 0; t < T; ++t) {
    std::vector<double> u(d);
    for (int i = 0; i < d; ++i) u[i] = load_elem(x, dtype, t * d + i);
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int i = 0; i < d; ++i) acc += load_elem(w_gate, dtype, (int64_t)e * d + i) * u[i];
      logits[t * E + e] = (float)acc;
    }
  }
  return 0;
}

// Score function ("三改进" item 3 for sigmoid; the traditional-MoE softmax).
// Computed in double from the fp32 logits, rounded to fp32.
int oracle_scores(const oracle_cfg* c, int64_t T, const float* logits, float* scores) {
  const int E = c->n_experts;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    const float* l = logits + t * E;
    float* s = scores + t * E;
    if (c->score_func == 0) {
      for (int e = 0; e < E; ++e) s[e] = (float)(1.0 / (1.0 + std::exp(-(double)l[e])));
    } else {
      double m = -std::numeric_limits<double>::infinity();
      for (int e = 0; e < E; ++e) m = std::max(m, (double)l[e]);
      double z = 0.0;
      for (int e = 0; e < E; ++e) z += std::exp((double)l[e] - m);
      for (int e = 0; e < E; ++e) s[e] = (float)(std::exp((double)l[e] - m) / z);
    }
  }
  return 0;
}

// Gate steps 2-5 for T tokens from fp32 scores [T, E]. Any output pointer
// except idx/w may be NULL. gsc is [T, G]; margins are [T].
int oracle_select(const oracle_cfg* c, int64_t T, const float* scores, const float* bias,
                  float* keys, float* gsc, int32_t* idx, float* w, float* kth_margin,
                  float* grp_margin) {
  const int E = c->n_experts, G = c->n_groups, k = c->topk;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    std::vector<float> key(E), g(G);
    float km, gm;
    select_one(*c, scores + t * E, bias, key.data(), g.data(), idx + t * k, w + t * k, &km, &gm);
    if (keys) std::copy(key.begin(), key.end(), keys + t * E);
    if (gsc) std::copy(g.begin(), g.end(), gsc + t * G);
    if (kth_margin) kth_margin[t] = km;
    if (grp_margin) grp_margin[t] = gm;
  }
  return 0;
}

// The literal MoE forward ("MoE 前向四步", single card) for n_tok selected
// tokens: y = sum_shared FFN_s(u) + sum_j w_j FFN_{idx_j}(u) [+ u].
// w1/w3/w2 are arrays of E+S per-expert pointers (routed 0..E-1, shared
// E..E+S-1); W1/W3 are [I, d], W2 is [d, I]. An expert a token needs must not
// be NULL (returns -1 otherwise). idx/w are the gate's [T, k] outputs. y is
// [n_tok, d] double.
int oracle_forward(const oracle_cfg* c, int64_t T, int dtype, const void* x,
                   const int32_t* idx, const float* w, const void* const* w1,
                   const void* const* w3, const void* const* w2, int64_t n_tok,
                   const int64_t* tok_ids, double* y) {
  const int d = c->dim, k = c->topk, E = c->n_experts, S = c->n_shared;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t n = 0; n < n_tok; ++n) {
    const int64_t t = tok_ids[n];
    if (t < 0 || t >= T) { bad |= 1; continue; }
    std::vector<double> u(d), acc(d, 0.0);
    for (int i = 0; i < d; ++i) u[i] = load_elem(x, dtype, t * d + i);
    for (int s = 0; s < S; ++s) {
      const int e = E + s;
      if (!w1[e] || !w3[e] || !w2[e]) { bad |= 1; continue; }
      expert_ffn_acc(*c, dtype, u.data(), w1[e], w3[e], w2[e], 1.0, acc.data());
    }
    for (int j = 0; j < k; ++j) {
      const int e = idx[t * k + j];
      if (e < 0 || e >= E || !w1[e] || !w3[e] || !w2[e]) { bad |= 1; continue; }
      expert_ffn_acc(*c, dtype, u.data(), w1[e], w3[e], w2[e], (double)w[t * k + j], acc.data());
    }
    if (c->add_residual)
      for (int i = 0; i < d; ++i) acc[i] += u[i];
    std::copy(acc.begin(), acc.end(), y + n * d);
  }
  return bad ? -1 : 0;
}

// Expert load: how many (token, slot) picks each routed expert received, i.e.
// the histogram of idx [T, k]. counts is [E]. Returns -1 if an index is out of
// range (and counts only the valid ones).
int oracle_expert_load(const oracle_cfg* c, int64_t T, const int32_t* idx, int64_t* counts) {
  const int E = c->n_experts, k = c->topk;
  int bad = 0;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t i = 0; i < T * k; ++i) {
    if (idx[i] < 0 || idx[i] >= E) {
      bad = 1;
      continue;
    }
    ++counts[idx[i]];
  }
  return bad ? -1 : 0;
}

// Aux-loss-free bias update ("V3 改进①：无辅助损失负载均衡": the bias follows the
// expert's load, at a speed set by gamma). Reading of the rule: the mean load is
// T*k/E picks per expert; an expert above it is overloaded and its bias drops
// by gamma, one below it is underloaded and its bias rises by gamma, one exactly
// at it keeps its bias. The comparison load_i > T*k/E is done in integers
// (load_i * E > T * k); the update is one fp32 addition. bias [E] is in-out.
int oracle_bias_update(const oracle_cfg* c, int64_t T, const int32_t* idx, float gamma,
                       float* bias) {
  const int E = c->n_experts, k = c->topk;
  std::vector<int64_t> load(E);
  const int rc = oracle_expert_load(c, T, idx, load.data());
  const int64_t total = T * (int64_t)k;
  for (int e = 0; e < E; ++e) {
    const int64_t scaled = load[e] * (int64_t)E;
    if (scaled > total)
      bias[e] = bias[e] - gamma;
    else if (scaled < total)
      bias[e] = bias[e] + gamma;
  }
  return rc;
}

// Sequence-wise balance statistics ("V3 改进②：序列级平衡损失",
// L_Bal = alpha * sum_i f_i * P_i) over the T tokens given:
//   f_i = (1/T) * #{t : i is among idx_t}      (top-k activation frequency),
//   P_i = (1/T) * sum_t s_{i,t} / sum_j s_{j,t} (time mean of the normalised
//                                                affinity s'),
// with s the fp32 scores [T, E] (after the score function, before any bias).
// Everything in double; f, P are [E], loss is one value.
int oracle_balance_stats(const oracle_cfg* c, int64_t T, const float* scores,
                         const int32_t* idx, double alpha, double* f, double* P,
                         double* loss) {
  const int E = c->n_experts;
  std::vector<int64_t> load(E);
  const int rc = oracle_expert_load(c, T, idx, load.data());
  for (int e = 0; e < E; ++e) P[e] = 0.0;
  for (int64_t t = 0; t < T; ++t) {
    double z = 0.0;
    for (int e = 0; e < E; ++e) z += (double)scores[t * E + e];
    for (int e = 0; e < E; ++e) P[e] += (double)scores[t * E + e] / z;
  }
  double l = 0.0;
  for (int e = 0; e < E; ++e) {
    f[e] = (double)load[e] / (double)T;
    P[e] = P[e] / (double)T;
    l += f[e] * P[e];
  }
  *loss = alpha * l;
  return rc;
}

// One rank's part of the expert-parallel forward ("MoE 前向四步": each rank
// loops over its own experts [expert_begin, expert_end), y is all-reduced over
// the ranks, and the shared experts' z is added after the reduction):
//   y_routed = sum over slots j with expert_begin <= idx_j < expert_end of
//              w_j FFN_{idx_j}(u)                    (slot order, double);
//   y_shared = sum_s FFN_s(u)                        (if y_shared is not NULL).
// Weights as for oracle_forward (E+S per-expert pointers; unused ones may be
// NULL). Both outputs are [n_tok, d] double.
int oracle_forward_part(const oracle_cfg* c, int64_t T, int dtype, const void* x,
                        const int32_t* idx, const float* w, const void* const* w1,
                        const void* const* w3, const void* const* w2, int expert_begin,
                        int expert_end, int64_t n_tok, const int64_t* tok_ids, double* y_routed,
                        double* y_shared) {
  const int d = c->dim, k = c->topk, E = c->n_experts, S = c->n_shared;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t n = 0; n < n_tok; ++n) {
    const int64_t t = tok_ids[n];
    if (t < 0 || t >= T) {
      bad |= 1;
      continue;
    }
    std::vector<double> u(d), acc(d, 0.0), sh(d, 0.0);
    for (int i = 0; i < d; ++i) u[i] = load_elem(x, dtype, t * d + i);
    for (int j = 0; j < k; ++j) {
      const int e = idx[t * k + j];
      if (e < expert_begin || e >= expert_end) continue;
      if (e < 0 || e >= E || !w1[e] || !w3[e] || !w2[e]) {
        bad |= 1;
        continue;
      }
      expert_ffn_acc(*c, dtype, u.data(), w1[e], w3[e], w2[e], (double)w[t * k + j], acc.data());
    }
    std::copy(acc.begin(), acc.end(), y_routed + n * d);
    if (y_shared) {
      for (int s = 0; s < S; ++s) {
        const int e = E + s;
        if (!w1[e] || !w3[e] || !w2[e]) {
          bad |= 1;
          continue;
        }
        expert_ffn_acc(*c, dtype, u.data(), w1[e], w3[e], w2[e], 1.0, sh.data());
      }
      std::copy(sh.begin(), sh.end(), y_shared + n * d);
    }
  }
  return bad ? -1 : 0;
}

// One expert's SwiGLU hidden vector h = silu(W1 u) * W3 u for n_tok tokens,
// double. h is [n_tok, I]. Used to localise a mismatch to the first GEMM.
int oracle_expert_hidden(const oracle_cfg* c, int64_t T, int dtype, const void* x,
                         const void* w1, const void* w3, int64_t n_tok,
                         const int64_t* tok_ids, double* h) {
  const int d = c->dim, I = c->inter;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t n = 0; n < n_tok; ++n) {
    const int64_t t = tok_ids[n];
    if (t < 0 || t >= T) { bad |= 1; continue; }
    std::vector<double> u(d);
    for (int i = 0; i < d; ++i) u[i] = load_elem(x, dtype, t * d + i);
    for (int f = 0; f < I; ++f) {
      double g = 0.0, v = 0.0;
      for (int i = 0; i < d; ++i) {
        g += load_elem(w1, dtype, (int64_t)f * d + i) * u[i];
        v += load_elem(w3, dtype, (int64_t)f * d + i) * u[i];
      }
      h[n * I + f] = g / (1.0 + std::exp(-g)) * v;
    }
  }
  return bad ? -1 : 0;
}

}  // extern "C"

// ===========================================================================
// MXFP8 expert weights (the FP8 form of the layer).
//
// Format: MX FP8 E4M3. Blocks of 32 consecutive elements along the reduction
// dimension (K) share one power-of-two scale 2^e, stored as an 8-bit biased
// exponent (e + 127); each element is FP8 E4M3 (1 sign bit, 4 exponent bits
// with bias 7, 3 mantissa bits, subnormals, no infinities, largest finite
// value 448 = 1.75 * 2^8, code 0x7F / 0xFF is NaN). The pages name the family
// (the DeepSeek-V3 notes' "FP8 混合精度训练" and the KTransformers page's native
// MXFP4 routed experts) but give no quantisation rule; the rule taken here:
//   scale : e = the smallest integer with amax <= 448 * 2^e, so that no element
//           of the block saturates; for amax = m * 2^E with m in [1, 2) that is
//           e = E - 8 + (m > 1.75); amax = 0 gives e = -127; e is clamped to
//           [-127, 127];
//   element: code = E4M3 round-to-nearest-even of v / 2^e (exact division).
// The FP8 forward quantises each token's u (blocks of 32 along d) and each
// SwiGLU hidden vector (blocks of 32 along I) by the same rule and runs the
// literal loop in double on the dequantised values.
// ===========================================================================
namespace {

uint8_t e4m3_from_double(double v) {
  if (std::isnan(v)) return 0x7F;
  const uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
  const double a = std::fabs(v);
  if (a < std::ldexp(1.0, -6)) {
    // Subnormal range: multiples of 2^-9; 8 * 2^-9 is the smallest normal.
    const double q = std::nearbyint(std::ldexp(a, 9));
    return (uint8_t)(sign | (q >= 8.0 ? 0x08 : (uint8_t)q));
  }
  int E = 0;
  std::frexp(a, &E);            // a = f * 2^E, f in [0.5, 1)
  int ex = E - 1;               // a in [2^ex, 2^(ex+1))
  double q = std::nearbyint(std::ldexp(a, 3 - ex));   // 1.mmm as an integer in [8, 16]
  if (q == 16.0) {
    ex += 1;
    q = 8.0;
  }
  if (ex > 8 || (ex == 8 && q > 14.0)) return (uint8_t)(sign | 0x7E);   // saturate at 448
  return (uint8_t)(sign | ((ex + 7) << 3) | ((int)q - 8));
}

double e4m3_to_double(uint8_t c) {
  const int ex = (c >> 3) & 15, man = c & 7;
  if (ex == 15 && man == 7) return std::numeric_limits<double>::quiet_NaN();
  const double mag = ex == 0 ? std::ldexp((double)man, -9) : std::ldexp((double)(8 + man), ex - 10);
  return (c & 0x80) ? -mag : mag;
}

int mx_exponent(double amax) {
  if (!(amax > 0.0)) return -127;
  int E = 0;
  const double f = std::frexp(amax, &E);   // amax = (2f) * 2^(E-1), 2f in [1, 2)
  int e = (E - 1) - 8 + (2.0 * f > 1.75 ? 1 : 0);
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// One row of K values (K a multiple of 32) to codes and biased scale bytes.
void mx_quantize_row(const double* v, int64_t K, uint8_t* codes, uint8_t* scales) {
  for (int64_t b = 0; b < K / 32; ++b) {
    double amax = 0.0;
    for (int i = 0; i < 32; ++i) amax = std::max(amax, std::fabs(v[b * 32 + i]));
    const int e = mx_exponent(amax);
    scales[b] = (uint8_t)(e + 127);
    for (int i = 0; i < 32; ++i) codes[b * 32 + i] = e4m3_from_double(std::ldexp(v[b * 32 + i], -e));
  }
}

double mx_value(const uint8_t* codes, const uint8_t* scales, int64_t i) {
  return std::ldexp(e4m3_to_double(codes[i]), (int)scales[i / 32] - 127);
}

double load_any(const void* src, int dtype, int64_t i) {
  if (dtype == 2) return ((const double*)src)[i];
  return load_elem(src, dtype, i);
}

}  // namespace

extern "C" {

// E4M3 round-to-nearest-even of n doubles (saturating at +-448) and back.
int oracle_e4m3_encode(int64_t n, const double* v, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_from_double(v[i]);
  return 0;
}
int oracle_e4m3_decode(int64_t n, const uint8_t* c, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_to_double(c[i]);
  return 0;
}

// MX quantisation of a row-major [rows, K] matrix (K a multiple of 32) held as
// fp32 (dtype 0), bf16 (1) or double (2): codes [rows, K], scales [rows, K/32]
// (biased exponents). Returns -1 if K is not a multiple of 32.
int oracle_mx_quantize(int64_t rows, int64_t K, int dtype, const void* src, uint8_t* codes,
                       uint8_t* scales) {
  if (K % 32 != 0) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    std::vector<double> v(K);
    for (int64_t i = 0; i < K; ++i) v[i] = load_any(src, dtype, r * K + i);
    mx_quantize_row(v.data(), K, codes + r * K, scales + r * (K / 32));
  }
  return 0;
}

// codes * 2^(scale - 127), double [rows, K].
int oracle_mx_dequantize(int64_t rows, int64_t K, const uint8_t* codes, const uint8_t* scales,
                         double* out) {
  if (K % 32 != 0) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t i = 0; i < K; ++i) out[r * K + i] = mx_value(codes + r * K, scales + r * (K / 32), i);
  return 0;
}

// The literal forward ("MoE 前向四步") with MXFP8 expert weights, in the page's
// loop order: expert by expert (routed experts 0..E-1, then the shared ones),
// each over the tokens that use it, y[token] += weight * expert(u). Per token, u
// is quantised (blocks of 32 along d); an expert's weights are decoded once to
// double, and each of its tokens computes h = silu(W1 u) * W3 u in double on the
// dequantised values, quantises h (blocks of 32 along I; skipped if
// quantize_hidden == 0) and adds weight * W2 h. x is bf16 [T, d]. w1q/w3q are
// per-expert code arrays [I, d] with scales [I, d/32]; w2q codes [d, I] with
// scales [d, I/32]; E+S entries each (NULL where unused). y [n_tok, d].
int oracle_forward_mxfp8(const oracle_cfg* c, int64_t T, const void* x, const int32_t* idx,
                         const float* w, const uint8_t* const* w1q, const uint8_t* const* w1s,
                         const uint8_t* const* w3q, const uint8_t* const* w3s,
                         const uint8_t* const* w2q, const uint8_t* const* w2s,
                         int quantize_hidden, int64_t n_tok, const int64_t* tok_ids, double* y) {
  const int d = c->dim, I = c->inter, k = c->topk, E = c->n_experts, S = c->n_shared;
  if (d % 32 != 0 || I % 32 != 0) return -1;
  // The users of each expert: (position in tok_ids, routing weight); the shared
  // experts take every token with weight 1.
  std::vector<std::vector<std::pair<int64_t, double>>> users(E + S);
  for (int64_t n = 0; n < n_tok; ++n) {
    const int64_t t = tok_ids[n];
    if (t < 0 || t >= T) return -1;
    for (int j = 0; j < k; ++j) {
      const int e = idx[t * k + j];
      if (e < 0 || e >= E) return -1;
      // (an expert named twice by one token contributes with both weights)
      if (!users[e].empty() && users[e].back().first == n)
        users[e].back().second += (double)w[t * k + j];
      else
        users[e].push_back({n, (double)w[t * k + j]});
    }
    for (int s = 0; s < S; ++s) users[E + s].push_back({n, 1.0});
  }
  // Quantised tokens.
  std::vector<double> u((size_t)n_tok * d), uq((size_t)n_tok * d);
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < n_tok; ++n) {
    std::vector<uint8_t> cu(d), su(d / 32);
    for (int i = 0; i < d; ++i) u[n * d + i] = load_elem(x, 1, tok_ids[n] * d + i);
    mx_quantize_row(&u[n * d], d, cu.data(), su.data());
    for (int i = 0; i < d; ++i) uq[n * d + i] = mx_value(cu.data(), su.data(), i);
  }
  std::vector<double> acc((size_t)n_tok * d, 0.0);
  std::vector<double> w1d((size_t)I * d), w3d((size_t)I * d), w2d((size_t)d * I);
  for (int e = 0; e < E + S; ++e) {
    if (users[e].empty()) continue;
    if (!w1q[e] || !w1s[e] || !w3q[e] || !w3s[e] || !w2q[e] || !w2s[e]) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < (int64_t)I * d; ++j) {
      w1d[j] = mx_value(w1q[e], w1s[e], j);
      w3d[j] = mx_value(w3q[e], w3s[e], j);
      w2d[j] = mx_value(w2q[e], w2s[e], j);
    }
    const auto& us = users[e];
#pragma omp parallel for schedule(dynamic, 1)
    for (size_t q = 0; q < us.size(); ++q) {
      const int64_t n = us[q].first;
      const double* un = &uq[n * d];
      std::vector<double> h(I), hq(I);
      std::vector<uint8_t> ch(I), sh(I / 32);
      for (int f = 0; f < I; ++f) {
        double g = 0.0, v = 0.0;
        for (int i = 0; i < d; ++i) {
          g += w1d[(int64_t)f * d + i] * un[i];
          v += w3d[(int64_t)f * d + i] * un[i];
        }
        h[f] = g / (1.0 + std::exp(-g)) * v;
      }
      if (quantize_hidden) {
        mx_quantize_row(h.data(), I, ch.data(), sh.data());
        for (int f = 0; f < I; ++f) hq[f] = mx_value(ch.data(), sh.data(), f);
      } else {
        hq = h;
      }
      double* an = &acc[n * d];
      for (int o = 0; o < d; ++o) {
        double sum = 0.0;
        for (int f = 0; f < I; ++f) sum += w2d[(int64_t)o * I + f] * hq[f];
        an[o] += us[q].second * sum;
      }
    }
  }
  for (int64_t n = 0; n < n_tok; ++n) {
    if (c->add_residual)
      for (int i = 0; i < d; ++i) acc[n * d + i] += u[n * d + i];
    std::copy(acc.begin() + n * d, acc.begin() + (n + 1) * d, y + n * d);
  }
  return 0;
}

}  // extern "C"

// ===========================================================================
// MXFP4 expert weights (the 4-bit form of the layer).
//
// Format: MX FP4 E2M1. Blocks of 32 consecutive elements along K share one
// power-of-two scale 2^e (8-bit biased exponent e + 127, as for MXFP8); each
// element is FP4 E2M1: 1 sign bit, 2 exponent bits with bias 1, 1 mantissa
// bit, a subnormal at exponent 0, no infinities or NaN. Its magnitudes are
// 0, 0.5, 1, 1.5, 2, 3, 4 and 6. The KTransformers DeepSeek page ("DeepSeek
// V4-Flash", its training notes) runs routed experts held natively in MXFP4;
// the pages give no quantisation rule, and the one taken mirrors the MXFP8
// rule above:
//   scale  : e = the smallest integer with amax <= 6 * 2^e (no element
//            saturates); for amax = m * 2^E with m in [1, 2) that is
//            e = E - 2 + (m > 1.5); amax = 0 gives e = -127; clamped to
//            [-127, 127];
//   element: code = E2M1 round-to-nearest-even of v / 2^e (ties go to the
//            code whose mantissa bit is 0).
// Codes here are one per byte (0..15, sign in bit 3); the library packs two
// per byte. Tokens and SwiGLU hidden vectors stay MXFP8 (E4M3), so the 4-bit
// forward is the FP8 forward on weights whose every element is an E2M1 value
// times its block scale (each of those is exactly an E4M3 value times the same
// scale, which is how oracle.py evaluates it).
// ===========================================================================
namespace {

double e2m1_to_double(uint8_t c) {
  const int ex = (c >> 1) & 3, man = c & 1;
  const double mag = ex == 0 ? 0.5 * man : std::ldexp(1.0 + 0.5 * man, ex - 1);
  return (c & 8) ? -mag : mag;
}

uint8_t e2m1_from_double(double v) {
  const uint8_t sign = std::signbit(v) ? 8 : 0;
  const double a = std::fabs(v);
  // Above the largest magnitude the code saturates at 6 (decided before the
  // distance search, whose differences lose 6 - 4 for huge values).
  if (a >= 6.0) return (uint8_t)(sign | 7);
  // The nearest of the eight magnitudes; on a tie the even code (mantissa 0).
  uint8_t best = 0;
  double best_err = a;
  for (uint8_t c = 1; c < 8; ++c) {
    const double err = std::fabs(a - e2m1_to_double(c));
    if (err < best_err || (err == best_err && (c & 1) == 0)) {
      best = c;
      best_err = err;
    }
  }
  return (uint8_t)(sign | best);
}

int mx4_exponent(double amax) {
  if (!(amax > 0.0)) return -127;
  int E = 0;
  const double f = std::frexp(amax, &E);   // amax = (2f) * 2^(E-1), 2f in [1, 2)
  int e = (E - 1) - 2 + (2.0 * f > 1.5 ? 1 : 0);
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

}  // namespace

extern "C" {

// E2M1 round-to-nearest-even of n doubles (saturating at +-6) and back.
int oracle_e2m1_encode(int64_t n, const double* v, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e2m1_from_double(v[i]);
  return 0;
}
int oracle_e2m1_decode(int64_t n, const uint8_t* c, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e2m1_to_double(c[i]);
  return 0;
}

// MXFP4 quantisation of a row-major [rows, K] matrix (K a multiple of 32) held
// as fp32 (dtype 0), bf16 (1) or double (2): codes [rows, K] (one per byte),
// scales [rows, K/32] (biased exponents). Returns -1 if K % 32 != 0.
int oracle_mx4_quantize(int64_t rows, int64_t K, int dtype, const void* src, uint8_t* codes,
                        uint8_t* scales) {
  if (K % 32 != 0) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < K / 32; ++b) {
      double v[32], amax = 0.0;
      for (int i = 0; i < 32; ++i) {
        v[i] = load_any(src, dtype, r * K + b * 32 + i);
        amax = std::max(amax, std::fabs(v[i]));
      }
      const int e = mx4_exponent(amax);
      scales[r * (K / 32) + b] = (uint8_t)(e + 127);
      for (int i = 0; i < 32; ++i) codes[r * K + b * 32 + i] = e2m1_from_double(std::ldexp(v[i], -e));
    }
  }
  return 0;
}

// codes * 2^(scale - 127), double [rows, K].
int oracle_mx4_dequantize(int64_t rows, int64_t K, const uint8_t* codes, const uint8_t* scales,
                          double* out) {
  if (K % 32 != 0) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t i = 0; i < K; ++i)
      out[r * K + i] = std::ldexp(e2m1_to_double(codes[r * K + i]),
                                  (int)scales[r * (K / 32) + i / 32] - 127);
  return 0;
}

}  // extern "C"
