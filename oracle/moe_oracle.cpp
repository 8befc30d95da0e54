// moe_oracle.cpp -- plain, slow, fp64 CPU definition of the stacked MoE FFN
// forward pass.  TEST INFRASTRUCTURE ONLY: nothing in the product library
// links, loads or calls this file.  Only the tests, the smoke check and the
// CPU-baseline leg of the benchmark use it.  It shares no code, header,
// table or helper with the CUDA path.
//
// What it follows (all citations are to the documentation pages that define
// the method):
//   * max.nn.moe.StackedMoE page, "Weight tensor shapes": gate_up_proj is
//     [num_experts, hidden_dim, 2*moe_dim], down_proj is
//     [num_experts, moe_dim, hidden_dim]; gate/up formats concatenated or
//     interleaved; optional projection bias; router weights applied after the
//     experts (apply_router_weight_first=False).
//   * max.nn.moe.GatedActivation page, the fused_activation list: "silu",
//     "swigluoai", "gelu_tanh" and the alpha / limit rules.
//   * Mojo sink_gate_router_kernel page, description and Args: sigmoid(logit)
//     + bias for selection only, top-k, softmax over the log-sigmoid of the
//     selected raw logits concatenated with the always-on sink logits, scaled
//     by route_scale * global_scale.
//   * NeMo AutoModel components/moe/experts page: GroupedExperts._forward_loop
//     (per-expert gather -> FFN -> scatter), _permute_tokens_for_grouped_mm
//     (tokens sorted by expert, tokens_per_expert, cumulative offsets),
//     _apply_bias (down bias weighted by the routing probabilities),
//     swiglu_clamped_deepep / swiglu_oai_deepep (concatenated [gate | up]),
//     quick_geglu_deepep (interleaved gate = x[..., ::2], up = x[..., 1::2]).
//
// Readings where the pages are silent (each is listed with its reason in the
// design notes of this repository):
//   R1  Softmax top-k router: the k largest logits (ties -> lowest expert
//       index), ordered by descending logit; weights are the softmax over the
//       k selected logits.
//   R2  Sink router selection score: the single-precision value
//       fl32(fl32(sigmoid(z)) + b), where fl32(sigmoid(z)) is the float
//       nearest the exact sigmoid.  The page gives the scores in the logits'
//       dtype (float32), and an argmax must be decided in one precision on
//       both sides.  Weights are computed in fp64 from the raw logits.
//   R3  limit <= 0 means "no clamp" for silu and swigluoai.
//   R4  The gate_up bias is added before the clamps and the activation; the
//       down bias is added inside the expert, so it is weighted by the
//       routing weight.
//   R5  The CSR permutation lists flat slots t*k+j sorted by expert, stable
//       (ascending slot inside one expert).
//   R6  apply_router_weight_first (StackedMoE page): the weight scales the
//       expert input, so the down bias is not weighted.  token_mask (NeMo
//       GroupedExperts.forward): a masked token uses no expert and outputs a
//       zero row.  Shared experts (StackedMoE has_shared_experts; the sink
//       router page's "sink lanes are gated shared experts") are evaluated by
//       the caller as this same FFN with every token routed to all of them.
//
// Inputs arrive as their stored bit patterns (bf16 as uint16, fp32 as float)
// and are converted exactly to double; every operation after that is fp64.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

double bf16_bits_to_double(uint16_t bits) {
  uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

// Round a double to the nearest bf16 value (8 significant bits, ties to
// even).  Used only by the diagnostic option that rounds h like a bf16
// intermediate would be rounded.
double round_to_bf16(double v) {
  if (v == 0.0 || !std::isfinite(v)) return v;
  int ex;
  double m = std::frexp(v, &ex);          // v = m * 2^ex, 0.5 <= |m| < 1
  double scaled = std::ldexp(m, 8);       // 8 significant bits before the point
  double r = std::nearbyint(scaled);      // default rounding mode: ties to even
  return std::ldexp(r, ex - 8);
}

double logit_at(const void* logits, int is_bf16, int64_t row, int64_t stride, int64_t col) {
  if (is_bf16) return bf16_bits_to_double(static_cast<const uint16_t*>(logits)[row * stride + col]);
  return static_cast<double>(static_cast<const float*>(logits)[row * stride + col]);
}

// Indices of the k best keys: descending key, ties broken by the lower index.
// A stable sort on the descending comparator keeps ascending index order
// among equal keys.
template <typename Key>
void top_k_desc(const std::vector<Key>& key, int k, int32_t* out) {
  std::vector<int32_t> order(key.size());
  for (size_t i = 0; i < order.size(); ++i) order[i] = static_cast<int32_t>(i);
  std::stable_sort(order.begin(), order.end(),
                   [&](int32_t a, int32_t b) { return key[a] > key[b]; });
  for (int j = 0; j < k; ++j) out[j] = order[j];
}

// log(sigmoid(z)) written so that it stays finite for any finite z.
double log_sigmoid(double z) { return std::min(z, 0.0) - std::log1p(std::exp(-std::fabs(z))); }

}  // namespace

extern "C" {

// The fused gated activation, GatedActivation page ("silu", "swigluoai",
// "gelu_tanh"); activation codes 0, 1, 2 respectively.  The clamp forms
// follow the same page and the NeMo swiglu_clamped_deepep / swiglu_oai_deepep
// descriptions (clamp only when limit > 0, reading R3).
double oracle_activation(int activation, double g, double u, double alpha, double limit) {
  switch (activation) {
    case 0:  // silu(gate) * up, optional clamps
      if (limit > 0.0) {
        g = std::min(g, limit);
        u = std::min(std::max(u, -limit), limit);
      }
      return g / (1.0 + std::exp(-g)) * u;
    case 1:  // g * sigmoid(alpha * g) * (u + 1)
      if (limit > 0.0) {
        g = std::min(g, limit);
        u = std::min(std::max(u, -limit), limit);
      }
      return g * (1.0 / (1.0 + std::exp(-alpha * g))) * (u + 1.0);
    case 2: {  // gelu(gate) * up, tanh form with the page's constants
      double inner = 0.7978845608028654 * (g + 0.044715 * g * g * g);
      return 0.5 * g * (1.0 + std::tanh(inner)) * u;
    }
    default:
      return std::nan("");
  }
}

// Softmax top-k router (reading R1).  logits: [T, stride], first E columns
// used.  Writes idx [T, k] (int32) and w [T, k] (fp64).  Returns 0, or -1 on
// bad arguments.
int oracle_route_softmax_topk(int64_t T, int E, int k, const void* logits, int logits_is_bf16,
                              int64_t stride, int32_t* idx, double* w) {
  if (T < 0 || E < 1 || k < 1 || k > E || stride < E) return -1;
  for (int64_t t = 0; t < T; ++t) {
    std::vector<double> z(E);
    for (int e = 0; e < E; ++e) z[e] = logit_at(logits, logits_is_bf16, t, stride, e);
    top_k_desc(z, k, idx + t * k);
    double m = z[idx[t * k]];
    double sum = 0.0;
    for (int j = 0; j < k; ++j) sum += std::exp(z[idx[t * k + j]] - m);
    for (int j = 0; j < k; ++j) w[t * k + j] = std::exp(z[idx[t * k + j]] - m) / sum;
  }
  return 0;
}

// Sigmoid-gate router with sink lanes, sink_gate_router_kernel page:
// selection on sigmoid(z) + bias (bias for selection only, reading R2);
// weights = softmax over [log sigmoid(z_selected) ..., log sigmoid(z_sink) ...]
// times route_scale * global_scale.  logits: [T, stride], routed columns
// 0..E-1 then sink columns E..E+S-1; a wider tail is not read.  bias may be
// NULL (all zero).  Writes idx [T,k], w [T,k], sink_w [T,S] (may be NULL when
// S == 0).
int oracle_route_sigmoid_sink(int64_t T, int E, int S, int k, const void* logits, int logits_is_bf16,
                              int64_t stride, const float* bias, double route_scale,
                              double global_scale, int32_t* idx, double* w, double* sink_w) {
  if (T < 0 || E < 1 || S < 0 || k < 1 || k > E || stride < E + S) return -1;
  if (S > 0 && sink_w == nullptr) return -1;
  for (int64_t t = 0; t < T; ++t) {
    std::vector<float> score(E);
    for (int e = 0; e < E; ++e) {
      double z = logit_at(logits, logits_is_bf16, t, stride, e);
      float sig = static_cast<float>(1.0 / (1.0 + std::exp(-z)));   // nearest float to sigmoid(z)
      float b = bias ? bias[e] : 0.0f;
      score[e] = sig + b;                                            // one float add
    }
    top_k_desc(score, k, idx + t * k);
    std::vector<double> v(k + S);
    for (int j = 0; j < k; ++j) v[j] = log_sigmoid(logit_at(logits, logits_is_bf16, t, stride, idx[t * k + j]));
    for (int i = 0; i < S; ++i) v[k + i] = log_sigmoid(logit_at(logits, logits_is_bf16, t, stride, E + i));
    double m = *std::max_element(v.begin(), v.end());
    double sum = 0.0;
    for (double vi : v) sum += std::exp(vi - m);
    double scale = route_scale * global_scale;
    for (int j = 0; j < k; ++j) w[t * k + j] = std::exp(v[j] - m) / sum * scale;
    for (int i = 0; i < S; ++i) sink_w[t * S + i] = std::exp(v[k + i] - m) / sum * scale;
  }
  return 0;
}

// moe_create_indices (sink_gate_router_kernel page, bucketing note; NeMo
// _permute_tokens_for_grouped_mm): counting sort of the R = T*k flat slots by
// expert, stable (reading R5).  counts [E], offsets [E+1] (exclusive prefix
// of counts), perm [R] (slot ids sorted by expert), inv [R] (position of each
// slot in perm; may be NULL).  Returns -1 if an index is out of [0, E).
int oracle_create_indices(int64_t R, int E, const int32_t* idx, int32_t* counts, int32_t* offsets,
                          int32_t* perm, int32_t* inv) {
  if (R < 0 || E < 1) return -1;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t s = 0; s < R; ++s) {
    if (idx[s] < 0 || idx[s] >= E) return -1;
    counts[idx[s]] += 1;
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  std::vector<int32_t> fill(offsets, offsets + E);
  for (int64_t s = 0; s < R; ++s) {
    int32_t pos = fill[idx[s]]++;
    perm[pos] = static_cast<int32_t>(s);
    if (inv) inv[s] = pos;
  }
  return 0;
}

// Grouped expert FFN, following the per-expert loop of NeMo
// GroupedExperts._forward_loop:  for every expert e, every slot (t, j) routed
// to e computes
//     a = x[t] . W_gu[e] + b_gu[e]                      (2*D columns)
//     (g, u) = split(a)  concatenated: (a[0:D], a[D:2D]);
//                        interleaved:  (a[0::2], a[1::2])
//     h = act(g, u)                                     (GatedActivation)
//     y_slot = h . W_d[e] + b_d[e]
// and the output is out[t] = sum_j w[t, j] * y_slot(t, j), j ascending
// (router weight after the experts; down bias weighted, NeMo _apply_bias).
//
// Inputs: x [T, H] bf16 bits; idx [T, k]; w [T, k] fp64; W_gu [E, H, 2D],
// b_gu [E, 2D] (NULL = none), W_d [E, D, H], b_d [E, H] (NULL = none), all
// bf16 bits.  gate_up_format 0 = concatenated, 1 = interleaved.
// tokens_sel: NULL for every token (out is [T, H]) or n_sel token ids (out is
// [n_sel, H] in that order).  round_h_bf16 != 0 rounds h to bf16 first (a
// diagnostic, off for parity).  Returns 0, or -1 on bad arguments.
int oracle_expert_ffn_ex(int64_t T, int H, int E, int k, int D, const uint16_t* x, const int32_t* idx,
                         const double* w, const uint16_t* W_gu, const uint16_t* b_gu, const uint16_t* W_d,
                         const uint16_t* b_d, int gate_up_format, int activation, double alpha, double limit,
                         int64_t n_sel, const int64_t* tokens_sel, int round_h_bf16, int weight_first,
                         const uint8_t* token_mask, double* out);

int oracle_expert_ffn(int64_t T, int H, int E, int k, int D, const uint16_t* x, const int32_t* idx,
                      const double* w, const uint16_t* W_gu, const uint16_t* b_gu, const uint16_t* W_d,
                      const uint16_t* b_d, int gate_up_format, int activation, double alpha, double limit,
                      int64_t n_sel, const int64_t* tokens_sel, int round_h_bf16, double* out) {
  return oracle_expert_ffn_ex(T, H, E, k, D, x, idx, w, W_gu, b_gu, W_d, b_d, gate_up_format, activation, alpha,
                              limit, n_sel, tokens_sel, round_h_bf16, 0, nullptr, out);
}

// The same expert FFN with the two options of the layer pages:
//   weight_first != 0 (StackedMoE apply_router_weight_first): the routing
//     weight scales the expert's INPUT, out[t] = sum_j FFN_e(w[t,j] * x[t]),
//     so the down bias is not weighted;
//   token_mask (NeMo GroupedExperts.forward token_mask, NULL = all valid):
//     a token whose mask byte is 0 goes through no expert and its output row
//     is zero.
int oracle_expert_ffn_ex(int64_t T, int H, int E, int k, int D, const uint16_t* x, const int32_t* idx,
                         const double* w, const uint16_t* W_gu, const uint16_t* b_gu, const uint16_t* W_d,
                         const uint16_t* b_d, int gate_up_format, int activation, double alpha, double limit,
                         int64_t n_sel, const int64_t* tokens_sel, int round_h_bf16, int weight_first,
                         const uint8_t* token_mask, double* out) {
  if (T < 0 || H < 1 || E < 1 || k < 1 || D < 1) return -1;
  const int64_t n_tok = tokens_sel ? n_sel : T;
  for (int64_t i = 0; i < n_tok; ++i) {
    int64_t t = tokens_sel ? tokens_sel[i] : i;
    if (t < 0 || t >= T) return -1;
    for (int j = 0; j < k; ++j)
      if (idx[t * k + j] < 0 || idx[t * k + j] >= E) return -1;
  }
  const int64_t n_slots = n_tok * k;
  std::vector<double> y(static_cast<size_t>(n_slots) * H, 0.0);
  const int64_t N1 = 2 * static_cast<int64_t>(D);

  for (int e = 0; e < E; ++e) {
    std::vector<int64_t> slots;  // local slot s = i*k + j, ascending; masked tokens take none
    for (int64_t s = 0; s < n_slots; ++s) {
      int64_t t = tokens_sel ? tokens_sel[s / k] : s / k;
      if (token_mask && token_mask[t] == 0) continue;
      if (idx[t * k + s % k] == e) slots.push_back(s);
    }
    if (slots.empty()) continue;  // an expert with no tokens contributes nothing
    const uint16_t* Wg = W_gu + static_cast<int64_t>(e) * H * N1;
    const uint16_t* Wd = W_d + static_cast<int64_t>(e) * D * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t q = 0; q < static_cast<int64_t>(slots.size()); ++q) {
      const int64_t s = slots[q];
      const int64_t t = tokens_sel ? tokens_sel[s / k] : s / k;
      std::vector<double> a(N1, 0.0), h(D);
      for (int64_t n = 0; n < N1; ++n) a[n] = b_gu ? bf16_bits_to_double(b_gu[e * N1 + n]) : 0.0;
      // the routing weight scales the input instead of the output
      const double in_scale = weight_first ? w[t * k + s % k] : 1.0;
      for (int64_t c = 0; c < H; ++c) {
        const double xc = in_scale * bf16_bits_to_double(x[t * H + c]);
        const uint16_t* row = Wg + c * N1;
        for (int64_t n = 0; n < N1; ++n) a[n] += xc * bf16_bits_to_double(row[n]);
      }
      for (int64_t i = 0; i < D; ++i) {
        double g = gate_up_format == 0 ? a[i] : a[2 * i];
        double u = gate_up_format == 0 ? a[D + i] : a[2 * i + 1];
        h[i] = oracle_activation(activation, g, u, alpha, limit);
        if (round_h_bf16) h[i] = round_to_bf16(h[i]);
      }
      double* ys = y.data() + s * H;
      for (int64_t c = 0; c < H; ++c) ys[c] = b_d ? bf16_bits_to_double(b_d[static_cast<int64_t>(e) * H + c]) : 0.0;
      for (int64_t i = 0; i < D; ++i) {
        const double hi = h[i];
        const uint16_t* row = Wd + i * H;
        for (int64_t c = 0; c < H; ++c) ys[c] += hi * bf16_bits_to_double(row[c]);
      }
    }
  }
  for (int64_t i = 0; i < n_tok; ++i) {
    const int64_t t = tokens_sel ? tokens_sel[i] : i;
    double* o = out + i * H;
    for (int64_t c = 0; c < H; ++c) o[c] = 0.0;
    for (int j = 0; j < k; ++j) {  // a masked token's slots were never computed: y is zero
      const double wj = weight_first ? 1.0 : w[t * k + j];
      const double* ys = y.data() + (i * k + j) * H;
      for (int64_t c = 0; c < H; ++c) o[c] += wj * ys[c];
    }
  }
  return 0;
}

// Threads the OpenMP runtime would use (reported next to the CPU timing).
int oracle_num_threads(void);

}  // extern "C"

#ifdef _OPENMP
#include <omp.h>
extern "C" int oracle_num_threads(void) { return omp_get_max_threads(); }
#else
extern "C" int oracle_num_threads(void) { return 1; }
#endif
