"""fp64 CPU oracle of the Qwen3 decoder block -- TEST INFRASTRUCTURE ONLY.

Only tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this module. The CUDA library never calls it, and it shares no code with
the CUDA library: it is written directly from the definitions on the pages, in
float64, with numpy's matrix product as the only library primitive. There is no
blocking, fusion or reordering beyond what each definition states.

Pages cited (title, site):
  [P-MoE]   "从零构建 Qwen-3 MoE" (adg.csdn.net), op-by-op notebook, sections 1-13
  [P-Hand]  "手搓一个Qwen3" (news.43b.com.cn), module listing, sections 2-6
  [P-Mini]  "从零实现 Qwen3：拆解 mini-qwen3 的 0.6B Dense 架构" (quarkcode.cn)
  [P-SGL]   "从0实现SGLang 3: Qwen3-0.6B" (wmrh.cn), sections 一-七 and 3.1-3.8

Inputs are bf16 tensors given as their uint16 bit patterns; they are widened to
float64 exactly and nothing is rounded afterwards.

Pins (what ties each function to something other than itself; the tests live in
tests/test_oracle_pins.py):
  rms_norm                 constant-vector closed form, scale invariance, unit RMS
  rope_rotate_half         norm preservation, relative-position property, m=0 identity,
                           half-split pairing of the 8-dim example, explicit angle values
  causal_gqa_attention     single key -> v, zero query -> prefix mean of v, GQA == MHA on
                           repeated K/V (independent path), brute force on tiny shapes with an
                           explicit mask matrix, the printed 17x17 mask, causality
  swiglu_ffn / silu        silu(0)=0, silu(z)->z, silu(-z)->0, one-hot weights closed form
  block_forward            decode-with-cache == row of a longer prefill; causality; identity
                           block when o_proj and down weights are zero
  moe_route / moe_ffn      the 0.7*E2 + 0.3*E4 worked example, k = E dense weighted sum,
                           sparse == token-wise dense reference, permutation order
  moe_ffn_half /           the block-level 0.7*E2 + 0.3*E4 example and k = E dense sum on
  moe_block_forward        norm_2(x1); a per-token loop over an independently restated
                           post-attention norm, router, top-k and experts; given routing
  stack_forward            zero-residual stack closed form (argmax logit = own token),
                           last-only == last row, causality across 2 layers
  param_count              0.752B untied parameter count and 3.01 GB fp32 of [P-Mini]
  kv_bytes_per_token       4 KB / token / layer of [P-Mini] section GQA
There is no function whose parity is unpinned.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np


# ---------------------------------------------------------------------------
# Configuration ([P-Mini] section 配置文件, table; [P-SGL] section 一)
# ---------------------------------------------------------------------------
@dataclass
class Config:
    hidden: int = 1024
    n_q_heads: int = 16
    n_kv_heads: int = 8
    head_dim: int = 128
    intermediate: int = 3072
    vocab: int = 151936
    n_layers: int = 28
    max_pos: int = 40960
    rope_theta: float = 1.0e6
    rms_eps: float = 1.0e-6
    n_experts: int = 0
    top_k: int = 0
    moe_intermediate: int = 0
    norm_topk_prob: bool = True


QWEN3_0_6B = Config()


def bf16_to_f64(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# RMSNorm ([P-Mini] section RMSNorm, the x-hat formula; [P-MoE] section 6)
#   x_hat_i = x_i / sqrt(mean_j x_j^2 + eps) * w_i
# ---------------------------------------------------------------------------
def rms_norm(x: np.ndarray, w: np.ndarray, eps: float) -> np.ndarray:
    mean_sq = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(mean_sq + eps) * w


# ---------------------------------------------------------------------------
# RoPE ([P-Mini] section RoPE: theta_i = base^(-2i/d); dimension i pairs with
# i + d/2 ("rotate half"); (a, b) -> (a cos(m theta_i) - b sin(m theta_i),
# a sin(m theta_i) + b cos(m theta_i)); the table row is the absolute position m)
# ---------------------------------------------------------------------------
def rope_frequencies(head_dim: int, theta: float) -> np.ndarray:
    i = np.arange(head_dim // 2, dtype=np.float64)
    return theta ** (-2.0 * i / head_dim)


def rope_rotate_half(u: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """u: [T, n_heads, d]; positions: [T] absolute positions."""
    d = u.shape[-1]
    half = d // 2
    angle = np.asarray(positions, dtype=np.float64)[:, None] * rope_frequencies(d, theta)[None, :]
    c = np.cos(angle)[:, None, :]
    s = np.sin(angle)[:, None, :]
    a = u[..., :half]
    b = u[..., half:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


# ---------------------------------------------------------------------------
# Causal grouped-query attention ([P-Mini] section GQA: softmax(QK^T/sqrt(d_head) + M) V
# with M_ij = -inf for key position after query position; query head h uses KV
# group h // (Hq / Hkv) ([P-MoE] section 12, head // (n_heads // n_kv_heads)))
# ---------------------------------------------------------------------------
def causal_allowed(q_pos: np.ndarray, k_pos: np.ndarray) -> np.ndarray:
    """Boolean [Tq, Tk]: key j is visible to query i iff its position is not after i's."""
    return np.asarray(k_pos)[None, :] <= np.asarray(q_pos)[:, None]


def softmax_rows(s: np.ndarray) -> np.ndarray:
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def causal_gqa_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                         q_pos: np.ndarray, k_pos: np.ndarray) -> np.ndarray:
    """q: [Tq, Hq, d]; k, v: [Tk, Hkv, d]; returns [Tq, Hq, d]."""
    tq, hq, d = q.shape
    hkv = k.shape[1]
    group = hq // hkv
    allowed = causal_allowed(q_pos, k_pos)
    out = np.empty((tq, hq, d), dtype=np.float64)
    for h in range(hq):
        g = h // group
        s = (q[:, h, :] @ k[:, g, :].T) / np.sqrt(d)
        s = np.where(allowed, s, -np.inf)
        out[:, h, :] = softmax_rows(s) @ v[:, g, :]
    return out


# ---------------------------------------------------------------------------
# SwiGLU FFN ([P-Mini] section SwiGLU FFN: FFN(x) = W_down (SiLU(W_gate x) * W_up x);
# [P-MoE] section 1.2: Swish with beta = 1 is x * sigmoid(x))
# ---------------------------------------------------------------------------
def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def swiglu_ffn(h: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    return (silu(h @ w_gate.T) * (h @ w_up.T)) @ w_down.T


# ---------------------------------------------------------------------------
# Layer weights in the pages' layouts (nn.Linear [out, in]; [P-Mini] section GQA)
# ---------------------------------------------------------------------------
@dataclass
class LayerWeights:
    in_norm: np.ndarray            # [H]
    wq: np.ndarray                 # [Hq*d, H]
    wk: np.ndarray                 # [Hkv*d, H]
    wv: np.ndarray                 # [Hkv*d, H]
    q_norm: np.ndarray             # [d]
    k_norm: np.ndarray             # [d]
    wo: np.ndarray                 # [H, Hq*d]
    post_norm: np.ndarray          # [H]
    w_gate: Optional[np.ndarray] = None    # [I, H]
    w_up: Optional[np.ndarray] = None      # [I, H]
    w_down: Optional[np.ndarray] = None    # [H, I]
    router: Optional[np.ndarray] = None    # [E, H]
    gate_up: Optional[np.ndarray] = None   # [E, 2*Im, H]: rows [0, Im) gate, [Im, 2Im) up
    down: Optional[np.ndarray] = None      # [E, H, Im]


# ---------------------------------------------------------------------------
# Decoder block, attention half ([P-Mini] sections TransformerBlock and GQA:
# pre-norm, q/k/v projections, per-head QK RMSNorm before RoPE, KV cache
# concatenation along the sequence, causal GQA, o_proj, residual)
# ---------------------------------------------------------------------------
def attention_half(x: np.ndarray, L: LayerWeights, cfg: Config, positions: np.ndarray,
                   cache_k: Optional[np.ndarray] = None, cache_v: Optional[np.ndarray] = None,
                   cache_pos: Optional[np.ndarray] = None, rows: Optional[np.ndarray] = None):
    """x: [T, H] for one sequence at absolute positions `positions` [T].
    cache_k/cache_v: [S, Hkv, d] keys/values already stored (post QK-norm, post RoPE)
    at positions cache_pos [S]. rows: subset of the T query rows to finish (all if None).
    Returns (x1[rows], k_new [T, Hkv, d], v_new [T, Hkv, d])."""
    T = x.shape[0]
    d = cfg.head_dim
    h = rms_norm(x, L.in_norm, cfg.rms_eps)
    q = (h @ L.wq.T).reshape(T, cfg.n_q_heads, d)
    k = (h @ L.wk.T).reshape(T, cfg.n_kv_heads, d)
    v = (h @ L.wv.T).reshape(T, cfg.n_kv_heads, d)
    q = rms_norm(q, L.q_norm, cfg.rms_eps)
    k = rms_norm(k, L.k_norm, cfg.rms_eps)
    q = rope_rotate_half(q, positions, cfg.rope_theta)
    k = rope_rotate_half(k, positions, cfg.rope_theta)
    if cache_k is not None and cache_k.shape[0] > 0:
        keys = np.concatenate([cache_k, k], axis=0)
        values = np.concatenate([cache_v, v], axis=0)
        key_pos = np.concatenate([np.asarray(cache_pos), np.asarray(positions)])
    else:
        keys, values, key_pos = k, v, np.asarray(positions)
    sel = np.arange(T) if rows is None else np.asarray(rows)
    o = causal_gqa_attention(q[sel], keys, values, np.asarray(positions)[sel], key_pos)
    x1 = x[sel] + o.reshape(len(sel), cfg.n_q_heads * d) @ L.wo.T
    return x1, k, v


def dense_ffn_half(x1: np.ndarray, L: LayerWeights, cfg: Config) -> np.ndarray:
    """[P-Mini] section TransformerBlock: x + FFN(norm_2(x))."""
    h2 = rms_norm(x1, L.post_norm, cfg.rms_eps)
    return x1 + swiglu_ffn(h2, L.w_gate, L.w_up, L.w_down)


def block_forward(x, L, cfg, positions, cache_k=None, cache_v=None, cache_pos=None, rows=None):
    """Dense decoder block; returns (out[rows], k_new, v_new)."""
    x1, k, v = attention_half(x, L, cfg, positions, cache_k, cache_v, cache_pos, rows)
    return dense_ffn_half(x1, L, cfg), k, v


# ---------------------------------------------------------------------------
# MoE FFN ([P-Mini] section MoE: router logits = linear(h), probabilities by a
# float softmax, top-k, renormalised within the top-k when norm_topk_prob;
# fused gate_up [E, 2I, H] split by chunk(2) into gate then up; each selected
# expert's SwiGLU output is scaled by its routing weight and accumulated into
# the token's row. [P-MoE] section 1: final output = 0.7 E2(x) + 0.3 E4(x).)
# ---------------------------------------------------------------------------
def moe_route(h2: np.ndarray, router: np.ndarray, top_k: int, norm_topk_prob: bool = True):
    """Returns (idx [T,k] int32, w [T,k], probs [T,E], margin [T]).
    Top-k order: descending probability, ties broken toward the lower expert index.
    margin = p_(k) - p_(k+1) (the k-th largest minus the next), +inf when k == E."""
    logits = h2 @ router.T
    probs = softmax_rows(logits)
    T, E = probs.shape
    order = np.argsort(-probs, axis=1, kind="stable")
    idx = order[:, :top_k]
    sel = np.take_along_axis(probs, idx, axis=1)
    if top_k < E:
        nxt = np.take_along_axis(probs, order[:, top_k:top_k + 1], axis=1)[:, 0]
        margin = sel[:, -1] - nxt
    else:
        margin = np.full(T, np.inf)
    w = sel / np.sum(sel, axis=1, keepdims=True) if norm_topk_prob else sel
    return idx.astype(np.int32), w, probs, margin


def moe_permutation(idx: np.ndarray, n_experts: int):
    """Groups (token, slot) pairs by expert: expert ascending, then token ascending.
    Returns (offsets [E+1], perm_token [T*k], perm_slot [T*k])."""
    T, k = idx.shape
    pairs = [(int(idx[t, j]), t, j) for t in range(T) for j in range(k)]
    pairs.sort(key=lambda p: (p[0], p[1]))
    counts = np.bincount(idx.reshape(-1), minlength=n_experts)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    perm_token = np.array([p[1] for p in pairs], dtype=np.int64)
    perm_slot = np.array([p[2] for p in pairs], dtype=np.int64)
    return offsets, perm_token, perm_slot


def expert_ffn(h: np.ndarray, gate_up_e: np.ndarray, down_e: np.ndarray) -> np.ndarray:
    """One expert: gate, up = chunk(h @ gate_up_e^T, 2); down(silu(gate) * up)."""
    im = gate_up_e.shape[0] // 2
    gu = h @ gate_up_e.T
    return (silu(gu[:, :im]) * gu[:, im:]) @ down_e.T


def moe_ffn(h2: np.ndarray, idx: np.ndarray, w: np.ndarray, gate_up: np.ndarray,
            down: np.ndarray) -> np.ndarray:
    """Sum over slots j = 0..k-1 (in that order) of w[t,j] * Expert_{idx[t,j]}(h2[t])."""
    T, k = idx.shape
    H = down.shape[1]
    y = np.zeros((T, k, H), dtype=np.float64)
    for e in np.unique(idx):
        t_sel, j_sel = np.nonzero(idx == e)
        y[t_sel, j_sel] = expert_ffn(h2[t_sel], gate_up[e], down[e])
    out = np.zeros((T, H), dtype=np.float64)
    for j in range(k):
        out += w[:, j:j + 1] * y[:, j]
    return out


def moe_ffn_half(x1: np.ndarray, L: LayerWeights, cfg: Config, idx: Optional[np.ndarray] = None,
                 w: Optional[np.ndarray] = None):
    """Second half of the MoE block ([P-Mini] sections TransformerBlock and MoE):
    h2 = norm_2(x1) with the post-attention weights, the router reads h2, and the
    selected experts' outputs on h2, weighted, are added to the residual x1.
    With idx and w given, that routing is used instead of the router's (the oracle
    evaluated on another implementation's routing). Returns (out, (idx, w, probs,
    margin)); probs and margin are None when the routing was given."""
    h2 = rms_norm(x1, L.post_norm, cfg.rms_eps)
    probs = margin = None
    if idx is None:
        idx, w, probs, margin = moe_route(h2, L.router, cfg.top_k, cfg.norm_topk_prob)
    return x1 + moe_ffn(h2, idx, w, L.gate_up, L.down), (idx, w, probs, margin)


def moe_block_forward(x, L, cfg, positions, rows=None):
    """Attention half then x1 + MoE(norm_2(x1)). Returns (out, k, v, route) where
    route = (idx, w, probs, margin) for the computed rows."""
    x1, k, v = attention_half(x, L, cfg, positions, rows=rows)
    out, route = moe_ffn_half(x1, L, cfg)
    return out, k, v, route


# ---------------------------------------------------------------------------
# Stack ([P-Mini] section 骨架: embedding lookup, 28 blocks in order, final
# RMSNorm, LM head; [P-SGL] section 一: tie_word_embeddings, so the LM head is
# the embedding matrix; [P-MoE] section 13 computes the last position only)
# ---------------------------------------------------------------------------
def stack_forward(ids: np.ndarray, embed: np.ndarray, layers, final_norm: np.ndarray, cfg: Config,
                  positions: Optional[np.ndarray] = None, caches=None, logit_rows=None):
    """One sequence. ids [T]; caches: list per layer of (k [S,Hkv,d], v, pos [S]) or None.
    Returns (logits [len(logit_rows), V], new_kv list of (k_new, v_new))."""
    T = len(ids)
    if positions is None:
        positions = np.arange(T)
    x = embed[np.asarray(ids)]
    new_kv = []
    for i, L in enumerate(layers):
        ck = cv = cp = None
        if caches is not None and caches[i] is not None:
            ck, cv, cp = caches[i]
        x, k, v = block_forward(x, L, cfg, positions, ck, cv, cp)
        new_kv.append((k, v))
    rows = np.arange(T) if logit_rows is None else np.asarray(logit_rows)
    xf = rms_norm(x[rows], final_norm, cfg.rms_eps)
    return xf @ embed.T, new_kv


# ---------------------------------------------------------------------------
# Sizes ([P-Mini] section 测试与实测数字: 0.752B parameters untied, 3.01 GB fp32;
# section GQA: about 4 KB of KV cache per token per layer in bf16)
# ---------------------------------------------------------------------------
def param_count(cfg: Config, tied: bool) -> int:
    d, H = cfg.head_dim, cfg.hidden
    attn = H * cfg.n_q_heads * d + 2 * H * cfg.n_kv_heads * d + cfg.n_q_heads * d * H + 2 * d
    ffn = 3 * H * cfg.intermediate
    per_layer = attn + ffn + 2 * H
    emb = cfg.vocab * H
    return cfg.n_layers * per_layer + emb * (1 if tied else 2) + H


def kv_bytes_per_token_layer(cfg: Config, bytes_per_elem: int = 2) -> int:
    return 2 * cfg.n_kv_heads * cfg.head_dim * bytes_per_elem
