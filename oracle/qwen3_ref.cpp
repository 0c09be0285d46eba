// fp64 C++ CPU oracle of the Qwen3 decoder block -- TEST INFRASTRUCTURE ONLY.
//
// A second, independent statement of the same definitions as oracle/qwen3_ref.py, in
// plain loops over double (OpenMP over independent rows and heads only). Only the
// tests and the benchmark's CPU-baseline leg may load it (through oracle/cpp_ref.py);
// the CUDA library never does, and nothing here is shared with it. Every sum runs in
// index order; there is no blocking, fusion or reordering beyond what each
// definition states.
//
// Pages cited (title, site):
//   [P-Mini] "从零实现 Qwen3：拆解 mini-qwen3 的 0.6B Dense 架构" (quarkcode.cn)
//   [P-MoE]  "从零构建 Qwen-3 MoE" (adg.csdn.net)
//   [P-SGL]  "从0实现SGLang 3: Qwen3-0.6B" (wmrh.cn)
//
// Layouts: row-major; a linear weight is [out_features][in_features] and is applied as
// x W^T; q/k/v are [tokens][heads][head_dim]. Pinned by the same pins as the numpy
// oracle (tests/test_oracle_cpp.py), and checked against it.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <numeric>
#include <vector>

namespace {

using i64 = int64_t;

// out[m][n] = sum_k a[m][k] * w[n][k]   (x W^T, the pages' nn.Linear without bias)
void linear(const double* a, const double* w, i64 M, i64 N, i64 K, double* out) {
#pragma omp parallel for schedule(static) if (M * N * K > (1 << 16))
  for (i64 m = 0; m < M; ++m)
    for (i64 n = 0; n < N; ++n) {
      double s = 0.0;
      const double* ar = a + m * K;
      const double* wr = w + n * K;
      for (i64 k = 0; k < K; ++k) s += ar[k] * wr[k];
      out[m * N + n] = s;
    }
}

// [P-Mini] section RMSNorm: x / sqrt(mean(x^2) + eps) * w, per row of n values
void rms_rows(const double* x, const double* w, i64 rows, i64 n, double eps, double* out) {
  for (i64 r = 0; r < rows; ++r) {
    double ss = 0.0;
    for (i64 j = 0; j < n; ++j) ss += x[r * n + j] * x[r * n + j];
    const double inv = 1.0 / std::sqrt(ss / (double)n + eps);
    for (i64 j = 0; j < n; ++j) out[r * n + j] = x[r * n + j] * inv * w[j];
  }
}

double silu1(double z) { return z / (1.0 + std::exp(-z)); }

}  // namespace

extern "C" {

struct Q3RefConfig {
  i64 hidden, n_q_heads, n_kv_heads, head_dim, intermediate, vocab, n_layers, max_pos;
  i64 n_experts, top_k, moe_intermediate, norm_topk_prob;
  double rope_theta, rms_eps;
};

struct Q3RefLayer {
  const double *in_norm, *wq, *wk, *wv, *q_norm, *k_norm, *wo, *post_norm;
  const double *w_gate, *w_up, *w_down;     // dense FFN
  const double *router, *gate_up, *down;    // MoE: [E][H], [E][2Im][H] (gate rows first), [E][H][Im]
};

void q3ref_rms_norm(const double* x, const double* w, i64 rows, i64 n, double eps, double* out) {
  rms_rows(x, w, rows, n, eps, out);
}

// [P-Mini] section RoPE: theta_i = base^(-2i/d), i < d/2
void q3ref_rope_frequencies(i64 d, double theta, double* out) {
  for (i64 i = 0; i < d / 2; ++i) out[i] = std::pow(theta, -2.0 * (double)i / (double)d);
}

// Rotate-half pairing (dimension i with i + d/2) at absolute position m:
// (a, b) -> (a cos(m theta_i) - b sin(m theta_i), a sin(m theta_i) + b cos(m theta_i)).
void q3ref_rope_rotate_half(const double* u, const double* pos, i64 T, i64 nh, i64 d, double theta, double* out) {
  const i64 half = d / 2;
  std::vector<double> f(half);
  q3ref_rope_frequencies(d, theta, f.data());
  for (i64 t = 0; t < T; ++t)
    for (i64 h = 0; h < nh; ++h)
      for (i64 i = 0; i < half; ++i) {
        const double ang = pos[t] * f[i];
        const double c = std::cos(ang), s = std::sin(ang);
        const double a = u[(t * nh + h) * d + i], b = u[(t * nh + h) * d + half + i];
        out[(t * nh + h) * d + i] = a * c - b * s;
        out[(t * nh + h) * d + half + i] = a * s + b * c;
      }
}

// Key j is visible to query i when its position is not after the query's ([P-Mini]
// section GQA, the causal mask).
void q3ref_causal_allowed(const double* qpos, const double* kpos, i64 Tq, i64 Tk, uint8_t* out) {
  for (i64 i = 0; i < Tq; ++i)
    for (i64 j = 0; j < Tk; ++j) out[i * Tk + j] = kpos[j] <= qpos[i] ? 1 : 0;
}

// softmax(q k^T / sqrt(d) + M) v per query head h, with the KV group h / (Hq / Hkv)
// ([P-Mini] section GQA; [P-MoE] section 12).
void q3ref_causal_gqa_attention(const double* q, const double* k, const double* v, const double* qpos,
                                const double* kpos, i64 Tq, i64 Tk, i64 Hq, i64 Hkv, i64 d, double* out) {
  const i64 group = Hq / Hkv;
  const double scale = 1.0 / std::sqrt((double)d);
#pragma omp parallel for collapse(2) schedule(static)
  for (i64 i = 0; i < Tq; ++i)
    for (i64 h = 0; h < Hq; ++h) {
      const i64 g = h / group;
      std::vector<double> s(Tk);
      double mx = -std::numeric_limits<double>::infinity();
      for (i64 j = 0; j < Tk; ++j) {
        if (kpos[j] > qpos[i]) { s[j] = -std::numeric_limits<double>::infinity(); continue; }
        double dot = 0.0;
        for (i64 e = 0; e < d; ++e) dot += q[(i * Hq + h) * d + e] * k[(j * Hkv + g) * d + e];
        s[j] = dot * scale;
        mx = std::max(mx, s[j]);
      }
      double den = 0.0;
      for (i64 j = 0; j < Tk; ++j) {
        s[j] = std::exp(s[j] - mx);
        den += s[j];
      }
      for (i64 e = 0; e < d; ++e) {
        double acc = 0.0;
        for (i64 j = 0; j < Tk; ++j) acc += s[j] * v[(j * Hkv + g) * d + e];
        out[(i * Hq + h) * d + e] = acc / den;
      }
    }
}

// silu(z) = z sigmoid(z) ([P-MoE] section 1.2: Swish with beta = 1)
void q3ref_silu(const double* z, i64 n, double* out) {
  for (i64 i = 0; i < n; ++i) out[i] = silu1(z[i]);
}

// [P-Mini] section SwiGLU FFN: down(silu(gate(h)) * up(h))
void q3ref_swiglu_ffn(const double* h, const double* wg, const double* wu, const double* wd, i64 T, i64 H, i64 I,
                      double* out) {
  std::vector<double> g(T * I), u(T * I);
  linear(h, wg, T, I, H, g.data());
  linear(h, wu, T, I, H, u.data());
  for (i64 i = 0; i < T * I; ++i) g[i] = silu1(g[i]) * u[i];
  linear(g.data(), wd, T, H, I, out);
}

// First half of the block for one sequence ([P-Mini] sections TransformerBlock and GQA):
// h = norm1(x); q, k, v projections; per-head QK RMSNorm, then RoPE at the absolute
// positions; keys and values appended after the S cached ones; causal GQA over all of
// them for the selected rows; x1 = x + o W_o^T. k_new / v_new receive the T new keys
// (post norm and RoPE) and values, [T][Hkv][d].
void q3ref_attention_half(const Q3RefConfig* c, const Q3RefLayer* L, const double* x, i64 T, const double* pos,
                          const double* ck, const double* cv, const double* cpos, i64 S, const i64* rows,
                          i64 n_rows, double* x1, double* k_new, double* v_new) {
  const i64 H = c->hidden, d = c->head_dim, hq = c->n_q_heads, hkv = c->n_kv_heads;
  std::vector<double> h(T * H), q(T * hq * d), k(T * hkv * d), v(T * hkv * d);
  rms_rows(x, L->in_norm, T, H, c->rms_eps, h.data());
  linear(h.data(), L->wq, T, hq * d, H, q.data());
  linear(h.data(), L->wk, T, hkv * d, H, k.data());
  linear(h.data(), L->wv, T, hkv * d, H, v.data());
  std::vector<double> qn(q.size()), kn(k.size());
  rms_rows(q.data(), L->q_norm, T * hq, d, c->rms_eps, qn.data());
  rms_rows(k.data(), L->k_norm, T * hkv, d, c->rms_eps, kn.data());
  q3ref_rope_rotate_half(qn.data(), pos, T, hq, d, c->rope_theta, q.data());
  q3ref_rope_rotate_half(kn.data(), pos, T, hkv, d, c->rope_theta, k.data());
  std::memcpy(k_new, k.data(), sizeof(double) * k.size());
  std::memcpy(v_new, v.data(), sizeof(double) * v.size());
  const i64 Tk = S + T;
  std::vector<double> keys(Tk * hkv * d), vals(Tk * hkv * d), kpos(Tk);
  if (S > 0) {
    std::memcpy(keys.data(), ck, sizeof(double) * S * hkv * d);
    std::memcpy(vals.data(), cv, sizeof(double) * S * hkv * d);
    std::memcpy(kpos.data(), cpos, sizeof(double) * S);
  }
  std::memcpy(keys.data() + S * hkv * d, k.data(), sizeof(double) * k.size());
  std::memcpy(vals.data() + S * hkv * d, v.data(), sizeof(double) * v.size());
  std::memcpy(kpos.data() + S, pos, sizeof(double) * T);
  std::vector<double> qs(n_rows * hq * d), qp(n_rows), o(n_rows * hq * d);
  for (i64 r = 0; r < n_rows; ++r) {
    const i64 t = rows ? rows[r] : r;
    std::memcpy(qs.data() + r * hq * d, q.data() + t * hq * d, sizeof(double) * hq * d);
    qp[r] = pos[t];
  }
  q3ref_causal_gqa_attention(qs.data(), keys.data(), vals.data(), qp.data(), kpos.data(), n_rows, Tk, hq, hkv, d,
                             o.data());
  linear(o.data(), L->wo, n_rows, H, hq * d, x1);
  for (i64 r = 0; r < n_rows; ++r) {
    const i64 t = rows ? rows[r] : r;
    for (i64 j = 0; j < H; ++j) x1[r * H + j] += x[t * H + j];
  }
}

// [P-Mini] section TransformerBlock, second half: x1 + FFN(norm2(x1))
void q3ref_dense_ffn_half(const Q3RefConfig* c, const Q3RefLayer* L, const double* x1, i64 T, double* out) {
  const i64 H = c->hidden;
  std::vector<double> h2(T * H);
  rms_rows(x1, L->post_norm, T, H, c->rms_eps, h2.data());
  q3ref_swiglu_ffn(h2.data(), L->w_gate, L->w_up, L->w_down, T, H, c->intermediate, out);
  for (i64 i = 0; i < T * H; ++i) out[i] += x1[i];
}

void q3ref_block_forward(const Q3RefConfig* c, const Q3RefLayer* L, const double* x, i64 T, const double* pos,
                         const double* ck, const double* cv, const double* cpos, i64 S, const i64* rows, i64 n_rows,
                         double* out, double* k_new, double* v_new) {
  std::vector<double> x1(n_rows * c->hidden);
  q3ref_attention_half(c, L, x, T, pos, ck, cv, cpos, S, rows, n_rows, x1.data(), k_new, v_new);
  q3ref_dense_ffn_half(c, L, x1.data(), n_rows, out);
}

// [P-Mini] section MoE: probabilities = softmax of the router logits; the top k by
// descending probability (equal probabilities: lower expert index first); weights
// renormalised to sum 1 when norm; margin = k-th minus (k+1)-th probability.
void q3ref_moe_route(const double* h2, const double* router, i64 T, i64 E, i64 H, i64 k, int norm, int32_t* idx,
                     double* w, double* probs, double* margin) {
  std::vector<double> logits(T * E);
  linear(h2, router, T, E, H, logits.data());
  for (i64 t = 0; t < T; ++t) {
    double mx = -std::numeric_limits<double>::infinity();
    for (i64 e = 0; e < E; ++e) mx = std::max(mx, logits[t * E + e]);
    double den = 0.0;
    for (i64 e = 0; e < E; ++e) den += std::exp(logits[t * E + e] - mx);
    for (i64 e = 0; e < E; ++e) probs[t * E + e] = std::exp(logits[t * E + e] - mx) / den;
    std::vector<i64> order(E);
    std::iota(order.begin(), order.end(), 0);
    const double* p = probs + t * E;
    std::stable_sort(order.begin(), order.end(), [p](i64 a, i64 b) { return p[a] > p[b]; });
    double tot = 0.0;
    for (i64 j = 0; j < k; ++j) tot += p[order[j]];
    for (i64 j = 0; j < k; ++j) {
      idx[t * k + j] = (int32_t)order[j];
      w[t * k + j] = norm ? p[order[j]] / tot : p[order[j]];
    }
    margin[t] = k < E ? p[order[k - 1]] - p[order[k]] : std::numeric_limits<double>::infinity();
  }
}

// (token, slot) pairs grouped by expert: expert ascending, then token ascending.
void q3ref_moe_permutation(const int32_t* idx, i64 T, i64 k, i64 E, i64* offsets, i64* perm_token, i64* perm_slot) {
  std::vector<i64> count(E, 0);
  for (i64 i = 0; i < T * k; ++i) ++count[idx[i]];
  offsets[0] = 0;
  for (i64 e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + count[e];
  std::vector<i64> fill(offsets, offsets + E);
  for (i64 t = 0; t < T; ++t)  // tokens in ascending order fill each expert's range
    for (i64 j = 0; j < k; ++j) {
      const i64 e = idx[t * k + j];
      perm_token[fill[e]] = t;
      perm_slot[fill[e]] = j;
      ++fill[e];
    }
}

// sum over slots j = 0..k-1 of w[t][j] * Expert_{idx[t][j]}(h2[t]); an expert is the
// SwiGLU FFN with gate rows [0, Im) and up rows [Im, 2Im) of gate_up[e] ([P-Mini] MoE,
// chunk(2)), then down[e].
void q3ref_moe_ffn(const double* h2, const int32_t* idx, const double* w, const double* gate_up, const double* down,
                   i64 T, i64 k, i64 H, i64 Im, double* out) {
#pragma omp parallel for schedule(static)
  for (i64 t = 0; t < T; ++t) {
    std::vector<double> gu(2 * Im), a(Im), y(H);
    for (i64 j = 0; j < H; ++j) out[t * H + j] = 0.0;
    for (i64 s = 0; s < k; ++s) {
      const i64 e = idx[t * k + s];
      linear(h2 + t * H, gate_up + e * 2 * Im * H, 1, 2 * Im, H, gu.data());
      for (i64 i = 0; i < Im; ++i) a[i] = silu1(gu[i]) * gu[Im + i];
      linear(a.data(), down + e * H * Im, 1, H, Im, y.data());
      for (i64 j = 0; j < H; ++j) out[t * H + j] += w[t * k + s] * y[j];
    }
  }
}

// x1 + MoE(norm2(x1)) ([P-Mini] sections TransformerBlock and MoE); the router's own
// routing unless idx_in / w_in are given. Routing outputs (idx, w, probs, margin) are
// written when their pointers are set.
void q3ref_moe_ffn_half(const Q3RefConfig* c, const Q3RefLayer* L, const double* x1, i64 T, const int32_t* idx_in,
                        const double* w_in, double* out, int32_t* idx, double* w, double* probs, double* margin) {
  const i64 H = c->hidden, E = c->n_experts, k = c->top_k;
  std::vector<double> h2(T * H);
  rms_rows(x1, L->post_norm, T, H, c->rms_eps, h2.data());
  std::vector<int32_t> ri(T * k);
  std::vector<double> rw(T * k), rp(T * E), rm(T);
  if (!idx_in) {
    q3ref_moe_route(h2.data(), L->router, T, E, H, k, (int)c->norm_topk_prob, ri.data(), rw.data(), rp.data(),
                    rm.data());
    idx_in = ri.data();
    w_in = rw.data();
    if (probs) std::memcpy(probs, rp.data(), sizeof(double) * rp.size());
    if (margin) std::memcpy(margin, rm.data(), sizeof(double) * rm.size());
  }
  if (idx) std::memcpy(idx, idx_in, sizeof(int32_t) * T * k);
  if (w) std::memcpy(w, w_in, sizeof(double) * T * k);
  q3ref_moe_ffn(h2.data(), idx_in, w_in, L->gate_up, L->down, T, k, H, c->moe_intermediate, out);
  for (i64 i = 0; i < T * H; ++i) out[i] += x1[i];
}

// One sequence through the stack ([P-Mini] section 骨架: embedding, the layers in order,
// final RMSNorm, LM head = the embedding matrix ([P-SGL] section 一, tied)).
// Layer l's cache: cache_len[l] rows of ck[l] / cv[l] at positions cpos[l] (S = 0: none).
// logits [n_rows][vocab] for the selected token rows; k_new[l] / v_new[l]: [T][Hkv][d].
void q3ref_stack_forward(const Q3RefConfig* c, const i64* ids, i64 T, const double* embed, const Q3RefLayer* layers,
                         const double* final_norm, const double* pos, const double* const* ck,
                         const double* const* cv, const double* const* cpos, const i64* cache_len,
                         const i64* logit_rows, i64 n_rows, double* logits, double* const* k_new,
                         double* const* v_new) {
  const i64 H = c->hidden;
  std::vector<double> x(T * H), y(T * H);
  for (i64 t = 0; t < T; ++t) std::memcpy(x.data() + t * H, embed + ids[t] * H, sizeof(double) * H);
  for (i64 l = 0; l < c->n_layers; ++l) {
    const i64 S = cache_len ? cache_len[l] : 0;
    q3ref_block_forward(c, &layers[l], x.data(), T, pos, S ? ck[l] : nullptr, S ? cv[l] : nullptr,
                        S ? cpos[l] : nullptr, S, nullptr, T, y.data(), k_new[l], v_new[l]);
    std::swap(x, y);
  }
  std::vector<double> xs(n_rows * H), xf(n_rows * H);
  for (i64 r = 0; r < n_rows; ++r) std::memcpy(xs.data() + r * H, x.data() + logit_rows[r] * H, sizeof(double) * H);
  rms_rows(xs.data(), final_norm, n_rows, H, c->rms_eps, xf.data());
  linear(xf.data(), embed, n_rows, c->vocab, H, logits);
}

// [P-Mini] section 测试与实测数字: parameters per layer (attention with q/k norms, SwiGLU FFN,
// two RMSNorms), the embedding (and an untied LM head), the final norm.
i64 q3ref_param_count(const Q3RefConfig* c, int tied) {
  const i64 H = c->hidden, d = c->head_dim, hq = c->n_q_heads, hkv = c->n_kv_heads;
  const i64 attn = H * hq * d + H * hkv * d + H * hkv * d + hq * d * H + 2 * d;
  const i64 ffn = 3 * H * c->intermediate;
  const i64 per_layer = attn + ffn + 2 * H;
  const i64 emb = c->vocab * H;
  return c->n_layers * per_layer + emb * (tied ? 1 : 2) + H;
}

// [P-Mini] section GQA: K and V, n_kv_heads x head_dim each, per token and layer
i64 q3ref_kv_bytes_per_token_layer(const Q3RefConfig* c, int bytes_per_elem) {
  return 2 * c->n_kv_heads * c->head_dim * bytes_per_elem;
}

}  // extern "C"
