// CPU oracle for the greedy MoE speculative-verify step of the jina-ocr-v1 decoder.
//
// TEST INFRASTRUCTURE ONLY.  This file is a plain, slow, obviously correct
// statement of what the verify step computes.  Only the test suite, the
// package's smoke check and the benchmark's CPU-baseline leg may call it; the
// product path never links or executes it.  It shares no code, header, helper
// or table with the CUDA library.
//
// What it follows (page, paragraph):
//   * jina-ocr-v1 model card (jina.ai/models/jina-ocr-v1), architecture
//     paragraph: the decoder is a DeepSeek-3B-MoE stack with 12 layers, hidden
//     size 1280, 64 routed experts plus 2 shared under top-6 routing, and a
//     129,280-token vocabulary.
//   * same page, decoding-speed paragraph, and the introduction: drafts are
//     verified greedily, so the emitted text equals plain autoregressive
//     decoding; the verifier commits up to K+1 tokens per pass.
//   * tldrocket write-up ("Jina AI Releases jina-ocr-v1 ..."), speculative
//     paragraph: the decoder keeps only the drafts that match its own choice.
//   * model card, decoding-speed paragraph, and the write-up's speculative
//     paragraph: the drafts come from FastMTP, one dense draft block applied
//     recursively for K steps (not K separate heads).  The pages give the
//     block no shape; the reading taken is in fastmtp_draft_row below.
//   * model card, architecture paragraph: a 32,768-position limit, the only
//     fact the pages give about the decoder's self-attention.  The reading
//     taken is in decode_attention_row below.
// The pages give no formulas; the readings taken where they are silent are:
//   gating = softmax over the E routed logits, keep the top k (selected on the
//   logits, ties to the lower expert id, slots in descending-logit order), then
//   divide by the kept mass; each expert is a SwiGLU FFN; the two shared
//   experts are one SwiGLU of twice the intermediate size added with weight 1;
//   each layer adds its MoE output to the residual stream (no norm); bf16
//   rounding happens at the SwiGLU activation and once per layer on h.
//
// Precision: inputs and weights are bf16 bit patterns.  Every dot product
// accumulates in Acc (float by default, double in the checking mode) in
// ascending index order, with no blocking or reordering.  A bf16 x bf16
// product is exact in float, so only the additions round.
//
// Build: g++ -std=c++17 -O2 -ffp-contract=off -fopenmp -shared -fPIC
// (no -ffast-math: the summation order must stay as written).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <numeric>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

float bf16_to_float(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// Round a float to the nearest bf16, ties to even.
uint16_t float_to_bf16(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return static_cast<uint16_t>((u >> 16) | 0x40u);  // NaN stays NaN
  u += 0x7fffu + ((u >> 16) & 1u);
  return static_cast<uint16_t>(u >> 16);
}

template <class Acc>
Acc dot_bf16(const uint16_t* a, const uint16_t* b, int n) {
  Acc s = 0;
  for (int i = 0; i < n; ++i)
    s += static_cast<Acc>(bf16_to_float(a[i])) * static_cast<Acc>(bf16_to_float(b[i]));
  return s;
}

template <class Acc>
Acc silu(Acc g) {
  return g / (static_cast<Acc>(1) + std::exp(-g));
}

// ---------------------------------------------------------------------------
// Router: logits, top-k selection, renormalised softmax weights.
// weight_form 0: softmax over all E, keep the selected, divide by their sum.
// weight_form 1: exp(l_j - l_max_sel) / sum over the selected (same value).
// ---------------------------------------------------------------------------
template <class Acc>
void router_row(const uint16_t* x, int H, int E, int k, const uint16_t* w_router,
                const float* bias, int32_t* idx, float* w, float* logits_out,
                float* gap_out, int weight_form) {
  std::vector<Acc> l(E);
  for (int e = 0; e < E; ++e) {
    Acc v = dot_bf16<Acc>(x, w_router + static_cast<size_t>(e) * H, H);
    if (bias) v += static_cast<Acc>(bias[e]);
    l[e] = v;
  }
  // Order experts by logit, largest first; equal logits keep the lower id
  // first (stable sort).  A NaN logit comes after every number, so a row with
  // fewer than k numbers still selects k distinct experts: the -inf ones next
  // by id, then the NaN ones by id.
  std::vector<int> order(E);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
    const bool na = std::isnan(l[a]), nb = std::isnan(l[b]);
    if (na || nb) return !na && nb;
    return l[a] > l[b];
  });
  for (int j = 0; j < k; ++j) idx[j] = order[j];

  if (gap_out)
    gap_out[0] = (k < E) ? static_cast<float>(l[order[k - 1]] - l[order[k]])
                         : std::numeric_limits<float>::infinity();
  if (logits_out)
    for (int e = 0; e < E; ++e) logits_out[e] = static_cast<float>(l[e]);

  if (weight_form == 0) {
    Acc mx = l[order[0]];
    std::vector<Acc> p(E);
    Acc z = 0;
    for (int e = 0; e < E; ++e) {
      p[e] = std::exp(l[e] - mx);
      z += p[e];
    }
    for (int e = 0; e < E; ++e) p[e] = p[e] / z;
    Acc kept = 0;
    for (int j = 0; j < k; ++j) kept += p[idx[j]];
    for (int j = 0; j < k; ++j) w[j] = static_cast<float>(p[idx[j]] / kept);
  } else {
    Acc mx = l[idx[0]];
    Acc s = 0;
    std::vector<Acc> q(k);
    for (int j = 0; j < k; ++j) {
      q[j] = std::exp(l[idx[j]] - mx);
      s += q[j];
    }
    for (int j = 0; j < k; ++j) w[j] = static_cast<float>(q[j] / s);
  }
}

// One SwiGLU expert on one row: a = bf16(silu(x Wg^T) * (x Wu^T)), y = a Wd^T.
template <class Acc>
void swiglu_row(const uint16_t* x, int H, int I, const uint16_t* wg, const uint16_t* wu,
                const uint16_t* wd, uint16_t* a, Acc* y) {
  for (int i = 0; i < I; ++i) {
    Acc g = dot_bf16<Acc>(x, wg + static_cast<size_t>(i) * H, H);
    Acc u = dot_bf16<Acc>(x, wu + static_cast<size_t>(i) * H, H);
    a[i] = float_to_bf16(static_cast<float>(silu<Acc>(g) * u));
  }
  for (int h = 0; h < H; ++h) y[h] = dot_bf16<Acc>(a, wd + static_cast<size_t>(h) * I, I);
}

// One MoE layer on one row: m = sum_j w_j * y_{e_j} + y_shared  (slot order,
// shared added last); out = bf16(residual + m), or bf16(m) without residual.
template <class Acc>
void moe_row(const uint16_t* x, int H, int I, int Ish, int k, const uint16_t* w_gate,
             const uint16_t* w_up, const uint16_t* w_down, const uint16_t* ws_gate,
             const uint16_t* ws_up, const uint16_t* ws_down, const int32_t* idx,
             const float* w, const uint16_t* residual, float* m_out, uint16_t* out) {
  std::vector<Acc> m(H, static_cast<Acc>(0)), y(H);
  std::vector<uint16_t> a(std::max(I, Ish));
  const size_t expert_stride = static_cast<size_t>(I) * H;
  for (int j = 0; j < k; ++j) {
    const int e = idx[j];
    swiglu_row<Acc>(x, H, I, w_gate + e * expert_stride, w_up + e * expert_stride,
                    w_down + e * expert_stride, a.data(), y.data());
    const Acc wj = static_cast<Acc>(w[j]);
    for (int h = 0; h < H; ++h) m[h] += wj * y[h];
  }
  if (Ish > 0) {
    swiglu_row<Acc>(x, H, Ish, ws_gate, ws_up, ws_down, a.data(), y.data());
    for (int h = 0; h < H; ++h) m[h] += y[h];
  }
  for (int h = 0; h < H; ++h) {
    if (m_out) m_out[h] = static_cast<float>(m[h]);
    Acc v = m[h];
    if (residual) v = static_cast<Acc>(bf16_to_float(residual[h])) + m[h];
    out[h] = float_to_bf16(static_cast<float>(v));
  }
}

// LM head + greedy choice on one row: argmax over v of h . W_lm[v] (first
// index wins on equality; -0 and +0 compare equal), plus the top-2 gap.
template <class Acc>
void lm_row(const uint16_t* h, int H, const uint16_t* w_lm, int V, int32_t* am, float* zmax,
            float* gap) {
  int best = 0;
  Acc bz = dot_bf16<Acc>(h, w_lm, H);
  Acc second = -std::numeric_limits<Acc>::infinity();
  for (int v = 1; v < V; ++v) {
    Acc z = dot_bf16<Acc>(h, w_lm + static_cast<size_t>(v) * H, H);
    if (z > bz) {
      second = bz;
      bz = z;
      best = v;
    } else if (z > second) {
      second = z;
    }
  }
  am[0] = best;
  if (zmax) zmax[0] = static_cast<float>(bz);
  if (gap) gap[0] = (V > 1) ? static_cast<float>(bz - second) : std::numeric_limits<float>::infinity();
}

// RMSNorm of one row: out_i = bf16((x_i * r) * gain_i) with
// r = 1 / sqrt(sum_i x_i^2 / n + eps), the sum in Acc in ascending order.
template <class Acc>
void rmsnorm_row(const uint16_t* x, int n, const uint16_t* gain, float eps, uint16_t* out) {
  Acc ss = 0;
  for (int i = 0; i < n; ++i) {
    const Acc v = static_cast<Acc>(bf16_to_float(x[i]));
    ss += v * v;
  }
  const Acc r = static_cast<Acc>(1) / std::sqrt(ss / static_cast<Acc>(n) + static_cast<Acc>(eps));
  for (int i = 0; i < n; ++i)
    out[i] = float_to_bf16(static_cast<float>((static_cast<Acc>(bf16_to_float(x[i])) * r) *
                                              static_cast<Acc>(bf16_to_float(gain[i]))));
}

// One step of the FastMTP draft block on one row (the reading of "a single
// dense draft block applied recursively"): the block takes the previous
// hidden state h (the verifier's last hidden state at the first step, the
// block's own output after that) and the token t drafted last (the verifier's
// next token at the first step), and returns the next hidden state:
//   u  = [ RMSNorm(h) * g_h ; RMSNorm(E[t]) * g_e ]      (2H, bf16)
//   z  = bf16(u . W_proj^T)                              (W_proj [H][2H])
//   h' = bf16(z + SwiGLU(z))                             (dense, intermediate I_d)
// and the draft is the shared LM head's greedy choice on h'.
template <class Acc>
void draft_step_row(const uint16_t* h, int32_t t, int H, int Id, const uint16_t* w_emb,
                    const uint16_t* g_h, const uint16_t* g_e, const uint16_t* w_proj,
                    const uint16_t* wg, const uint16_t* wu, const uint16_t* wd, float eps,
                    uint16_t* h_out) {
  std::vector<uint16_t> u(2 * static_cast<size_t>(H)), z(H), a(Id);
  rmsnorm_row<Acc>(h, H, g_h, eps, u.data());
  rmsnorm_row<Acc>(w_emb + static_cast<size_t>(t) * H, H, g_e, eps, u.data() + H);
  for (int i = 0; i < H; ++i)
    z[i] = float_to_bf16(static_cast<float>(dot_bf16<Acc>(u.data(), w_proj + static_cast<size_t>(i) * 2 * H, 2 * H)));
  std::vector<Acc> y(H);
  swiglu_row<Acc>(z.data(), H, Id, wg, wu, wd, a.data(), y.data());
  for (int i = 0; i < H; ++i)
    h_out[i] = float_to_bf16(static_cast<float>(static_cast<Acc>(bf16_to_float(z[i])) + y[i]));
}

// Rotary position embedding of one head vector x[d] at position pos (the
// reading of the decoder's positions): pairs (i, i + d/2) for i < d/2 turn by
// the angle pos * theta^(-2i/d):
//   y_i       = x_i cos(a) - x_{i+d/2} sin(a)
//   y_{i+d/2} = x_{i+d/2} cos(a) + x_i sin(a)
// computed in double and rounded to bf16 once.
void rope_head(const uint16_t* x, int d, int32_t pos, double theta, uint16_t* y) {
  const int half = d / 2;
  for (int i = 0; i < half; ++i) {
    const double a = static_cast<double>(pos) * std::pow(theta, -2.0 * i / d);
    const double c = std::cos(a), s = std::sin(a);
    const double x0 = bf16_to_float(x[i]), x1 = bf16_to_float(x[i + half]);
    y[i] = float_to_bf16(static_cast<float>(x0 * c - x1 * s));
    y[i + half] = float_to_bf16(static_cast<float>(x1 * c + x0 * s));
  }
}

// Causal self-attention of one query row of one head over a sequence's key /
// value cache (the reading of the decoder's attention on the verify rows):
// the query at position p sees the cached positions 0..p, scores
// s_j = (q . k_j) / sqrt(d), weights softmax(s) over those positions, output
// o = sum_j softmax_j * v_j.  Everything in double, in ascending position and
// index order; k_j, v_j are rows of the cache (stride d between positions).
void decode_attention_row(const uint16_t* q, const uint16_t* k, const uint16_t* v, int d, int p, double* o) {
  const double scale = 1.0 / std::sqrt(static_cast<double>(d));
  std::vector<double> s(static_cast<size_t>(p) + 1);
  double mx = -std::numeric_limits<double>::infinity();
  for (int j = 0; j <= p; ++j) {
    double acc = 0.0;
    for (int i = 0; i < d; ++i)
      acc += static_cast<double>(bf16_to_float(q[i])) * bf16_to_float(k[static_cast<size_t>(j) * d + i]);
    s[j] = acc * scale;
    mx = std::max(mx, s[j]);
  }
  double z = 0.0;
  for (int j = 0; j <= p; ++j) {
    s[j] = std::exp(s[j] - mx);
    z += s[j];
  }
  for (int i = 0; i < d; ++i) o[i] = 0.0;
  for (int j = 0; j <= p; ++j) {
    const double w = s[j] / z;
    for (int i = 0; i < d; ++i) o[i] += w * bf16_to_float(v[static_cast<size_t>(j) * d + i]);
  }
}

void set_threads(int n_threads) {
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#else
  (void)n_threads;
#endif
}

}  // namespace

extern "C" {

// Returns 0 on success, 1 on invalid arguments.
int oracle_router(const uint16_t* x, int T, int H, int E, int k, const uint16_t* w_router,
                  const float* bias, int32_t* topk_idx, float* topk_w, float* logits,
                  float* gap, int weight_form, int acc_double, int n_threads) {
  if (!x || !w_router || !topk_idx || !topk_w || T < 0 || H <= 0 || E <= 0 || k <= 0 || k > E)
    return 1;
  set_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < T; ++r) {
    const uint16_t* xr = x + static_cast<size_t>(r) * H;
    float* lo = logits ? logits + static_cast<size_t>(r) * E : nullptr;
    float* go = gap ? gap + r : nullptr;
    if (acc_double)
      router_row<double>(xr, H, E, k, w_router, bias, topk_idx + r * k, topk_w + r * k, lo, go,
                         weight_form);
    else
      router_row<float>(xr, H, E, k, w_router, bias, topk_idx + r * k, topk_w + r * k, lo, go,
                        weight_form);
  }
  return 0;
}

int oracle_moe_ffn(const uint16_t* x, int T, int H, int E, int I, int Ish, int k,
                   const uint16_t* w_gate, const uint16_t* w_up, const uint16_t* w_down,
                   const uint16_t* ws_gate, const uint16_t* ws_up, const uint16_t* ws_down,
                   const int32_t* topk_idx, const float* topk_w, const uint16_t* residual,
                   float* m_out, uint16_t* out, int acc_double, int n_threads) {
  if (!x || !w_gate || !w_up || !w_down || !topk_idx || !topk_w || !out || T < 0 || H <= 0 ||
      E <= 0 || I <= 0 || k <= 0 || k > E || Ish < 0)
    return 1;
  if (Ish > 0 && (!ws_gate || !ws_up || !ws_down)) return 1;
  for (int r = 0; r < T * k; ++r)
    if (topk_idx[r] < 0 || topk_idx[r] >= E) return 1;
  set_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < T; ++r) {
    const size_t o = static_cast<size_t>(r) * H;
    const uint16_t* res = residual ? residual + o : nullptr;
    float* mo = m_out ? m_out + o : nullptr;
    if (acc_double)
      moe_row<double>(x + o, H, I, Ish, k, w_gate, w_up, w_down, ws_gate, ws_up, ws_down,
                      topk_idx + r * k, topk_w + r * k, res, mo, out + o);
    else
      moe_row<float>(x + o, H, I, Ish, k, w_gate, w_up, w_down, ws_gate, ws_up, ws_down,
                     topk_idx + r * k, topk_w + r * k, res, mo, out + o);
  }
  return 0;
}

// A single expert on a single row, exposing the bf16 activation a[I] and y[H].
int oracle_swiglu(const uint16_t* x, int H, int I, const uint16_t* wg, const uint16_t* wu,
                  const uint16_t* wd, uint16_t* a_out, float* y_out, int acc_double) {
  if (!x || !wg || !wu || !wd || !a_out || !y_out || H <= 0 || I <= 0) return 1;
  if (acc_double) {
    std::vector<double> y(H);
    swiglu_row<double>(x, H, I, wg, wu, wd, a_out, y.data());
    for (int h = 0; h < H; ++h) y_out[h] = static_cast<float>(y[h]);
  } else {
    std::vector<float> y(H);
    swiglu_row<float>(x, H, I, wg, wu, wd, a_out, y.data());
    for (int h = 0; h < H; ++h) y_out[h] = y[h];
  }
  return 0;
}

int oracle_lm_head_argmax(const uint16_t* h, int T, int H, const uint16_t* w_lm, int V,
                          int32_t* argmax, float* zmax, float* gap, int acc_double,
                          int n_threads) {
  if (!h || !w_lm || !argmax || T < 0 || H <= 0 || V <= 0) return 1;
  set_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < T; ++r) {
    const uint16_t* hr = h + static_cast<size_t>(r) * H;
    float* zo = zmax ? zmax + r : nullptr;
    float* go = gap ? gap + r : nullptr;
    if (acc_double)
      lm_row<double>(hr, H, w_lm, V, argmax + r, zo, go);
    else
      lm_row<float>(hr, H, w_lm, V, argmax + r, zo, go);
  }
  return 0;
}

// Greedy acceptance.  Row b*(K+1)+j holds the verifier's choice after the
// j-th token of sequence b (j = 0: the current token, j >= 1: draft j).  Draft
// i+1 (drafts[b][i]) is kept while it equals the verifier's choice at row i.
// accepted[b] = number of drafts kept (0..K); next_token[b] = the verifier's
// choice after the last kept token; emitted[b][0..accepted] = the committed
// tokens (accepted + 1 of them), the rest of the row is -1.
int oracle_greedy_accept(const int32_t* argmax, const int32_t* drafts, int B, int K,
                         int32_t* accepted, int32_t* next_token, int32_t* emitted) {
  if (!argmax || !accepted || !next_token || B < 0 || K < 0 || (K > 0 && !drafts)) return 1;
  for (int b = 0; b < B; ++b) {
    const int32_t* g = argmax + static_cast<size_t>(b) * (K + 1);
    const int32_t* d = drafts ? drafts + static_cast<size_t>(b) * K : nullptr;
    int a = 0;
    while (a < K && d[a] == g[a]) ++a;
    accepted[b] = a;
    next_token[b] = g[a];
    if (emitted) {
      for (int j = 0; j <= K; ++j) emitted[static_cast<size_t>(b) * (K + 1) + j] = (j <= a) ? g[j] : -1;
    }
  }
  return 0;
}

// RMSNorm of T rows of n values (see rmsnorm_row).
int oracle_rmsnorm(const uint16_t* x, int T, int n, const uint16_t* gain, float eps, uint16_t* out,
                   int acc_double) {
  if (!x || !gain || !out || T < 0 || n <= 0 || !(eps >= 0.f)) return 1;
  for (int r = 0; r < T; ++r) {
    const size_t o = static_cast<size_t>(r) * n;
    if (acc_double)
      rmsnorm_row<double>(x + o, n, gain, eps, out + o);
    else
      rmsnorm_row<float>(x + o, n, gain, eps, out + o);
  }
  return 0;
}

// FastMTP drafting: K recursive steps of the draft block (draft_step_row) per
// sequence, starting from h0[b] and t0[b]; drafts[b][j] = the LM head's greedy
// choice on the j-th step's output.  h_steps[j][b][H] (nullable) receives the
// step outputs, gaps[j][b] (nullable) the LM top-2 gap of each step.
int oracle_fastmtp_draft(const uint16_t* h0, const int32_t* t0, int B, int K, int H, int Id, int V,
                         const uint16_t* w_emb, const uint16_t* g_h, const uint16_t* g_e,
                         const uint16_t* w_proj, const uint16_t* wg, const uint16_t* wu,
                         const uint16_t* wd, const uint16_t* w_lm, float eps, int32_t* drafts,
                         uint16_t* h_steps, float* gaps, int acc_double, int n_threads) {
  if (!h0 || !t0 || !w_emb || !g_h || !g_e || !w_proj || !wg || !wu || !wd || !w_lm || B < 0 ||
      K < 0 || H <= 0 || Id <= 0 || V <= 0 || !(eps >= 0.f) || (K > 0 && B > 0 && !drafts))
    return 1;
  for (int b = 0; b < B; ++b)
    if (t0[b] < 0 || t0[b] >= V) return 1;
  set_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
  for (int b = 0; b < B; ++b) {
    std::vector<uint16_t> h(h0 + static_cast<size_t>(b) * H, h0 + static_cast<size_t>(b + 1) * H), hn(H);
    int32_t t = t0[b];
    for (int j = 0; j < K; ++j) {
      int32_t d = 0;
      float gp = 0.f;
      if (acc_double) {
        draft_step_row<double>(h.data(), t, H, Id, w_emb, g_h, g_e, w_proj, wg, wu, wd, eps, hn.data());
        lm_row<double>(hn.data(), H, w_lm, V, &d, nullptr, &gp);
      } else {
        draft_step_row<float>(h.data(), t, H, Id, w_emb, g_h, g_e, w_proj, wg, wu, wd, eps, hn.data());
        lm_row<float>(hn.data(), H, w_lm, V, &d, nullptr, &gp);
      }
      drafts[static_cast<size_t>(b) * K + j] = d;
      if (h_steps) std::copy(hn.begin(), hn.end(), h_steps + (static_cast<size_t>(j) * B + b) * H);
      if (gaps) gaps[static_cast<size_t>(j) * B + b] = gp;
      h.swap(hn);
      t = d;
    }
  }
  return 0;
}

// RoPE of T rows of nh heads of d values (row r at position pos[r]); x and y
// are [T][nh*d] bf16.  d must be even.
int oracle_rope(const uint16_t* x, int T, int nh, int d, const int32_t* pos, double theta, uint16_t* y) {
  if (!x || !pos || !y || T < 0 || nh <= 0 || d <= 0 || (d & 1) || !(theta > 0.0)) return 1;
  for (int r = 0; r < T; ++r)
    for (int h = 0; h < nh; ++h) {
      const size_t o = (static_cast<size_t>(r) * nh + h) * d;
      rope_head(x + o, d, pos[r], theta, y + o);
    }
  return 0;
}

// Self-attention of the verify rows over the key/value cache.  B sequences of
// K+1 query rows each (row r = b*(K+1) + j); sequence b holds ctx_len[b]
// earlier positions and this step's K+1 rows at positions ctx_len[b] + j, so
// query row j sees positions 0..ctx_len[b]+j.  q [B*(K+1)][nh][d] bf16;
// k_cache, v_cache [B][nh][L_max][d] bf16; out [B*(K+1)][nh][d] double.
int oracle_decode_attention(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                            const int32_t* ctx_len, int B, int K, int nh, int d, int L_max, double* out,
                            int n_threads) {
  if (!q || !k_cache || !v_cache || !ctx_len || !out || B < 0 || K < 0 || nh <= 0 || d <= 0 || L_max <= 0)
    return 1;
  for (int b = 0; b < B; ++b)
    if (ctx_len[b] < 0 || ctx_len[b] + K + 1 > L_max) return 1;
  set_threads(n_threads);
  const int T = B * (K + 1);
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int r = 0; r < T; ++r)
    for (int h = 0; h < nh; ++h) {
      const int b = r / (K + 1), j = r % (K + 1);
      const size_t head = (static_cast<size_t>(b) * nh + h) * static_cast<size_t>(L_max) * d;
      decode_attention_row(q + (static_cast<size_t>(r) * nh + h) * d, k_cache + head, v_cache + head, d,
                           ctx_len[b] + j, out + (static_cast<size_t>(r) * nh + h) * d);
    }
  return 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
