"""Planted mistakes in the oracle (on the CPU) must each fail at least one pin.

Every mutation below is a plausible slip when writing the block from the pages:
a wrong RoPE pairing or sign, a dropped scale, an off-by-one mask, a swapped
operand. A mutation that no pin catches would mean the pins leave that part of
the oracle unchecked.
"""
import numpy as np
import pytest

import oracle.qwen3_ref as R
from oracle_pins import ALL_PINS


def _rope_adjacent_pairs(u, positions, theta):
    d = u.shape[-1]
    ang = np.asarray(positions, dtype=np.float64)[:, None] * R.rope_frequencies(d, theta)[None, :]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    a, b = u[..., 0::2], u[..., 1::2]
    out = np.empty_like(u)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def _rope_sign_flipped(u, positions, theta):
    d = u.shape[-1]; h = d // 2
    ang = np.asarray(positions, dtype=np.float64)[:, None] * R.rope_frequencies(d, theta)[None, :]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    a, b = u[..., :h], u[..., h:]
    return np.concatenate([a * c + b * s, -a * s + b * c], axis=-1)


def _rope_freq_wrong_exponent(head_dim, theta):
    return theta ** (-np.arange(head_dim // 2, dtype=np.float64) / head_dim)


def _rms_sum_not_mean(x, w, eps):
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps) * w


def _rms_eps_outside(x, w, eps):
    return x / (np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps) * w


def _mask_strict(q_pos, k_pos):
    return np.asarray(k_pos)[None, :] < np.asarray(q_pos)[:, None]


def _attn_gqa_modulo(q, k, v, q_pos, k_pos):
    tq, hq, d = q.shape
    hkv = k.shape[1]
    allowed = R.causal_allowed(q_pos, k_pos)
    out = np.empty((tq, hq, d))
    for h in range(hq):
        g = h % hkv
        s = np.where(allowed, (q[:, h] @ k[:, g].T) / np.sqrt(d), -np.inf)
        out[:, h] = R.softmax_rows(s) @ v[:, g]
    return out


def _silu_is_sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def _swiglu_swapped(h, wg, wu, wd):
    return (R.silu(h @ wu.T) * (h @ wg.T)) @ wd.T


def _route_no_renorm(h2, router, k, norm):
    return _ORIG["moe_route"](h2, router, k, False)


def _route_high_index_first(h2, router, k, norm=True):
    probs = R.softmax_rows(h2 @ router.T)
    E = probs.shape[1]
    order = np.argsort(-probs[:, ::-1], axis=1, kind="stable")
    order = E - 1 - order
    idx = order[:, :k]
    sel = np.take_along_axis(probs, idx, axis=1)
    margin = sel[:, -1] - np.take_along_axis(probs, order[:, k:k + 1], axis=1)[:, 0] if k < E else np.full(len(probs), np.inf)
    w = sel / sel.sum(1, keepdims=True) if norm else sel
    return idx.astype(np.int32), w, probs, margin


def _ffn_on_unnormed(x1, L, cfg):
    return x1 + R.swiglu_ffn(x1, L.w_gate, L.w_up, L.w_down)


def _attn_half_rope_before_norm(x, L, cfg, positions, cache_k=None, cache_v=None, cache_pos=None, rows=None):
    T = x.shape[0]; d = cfg.head_dim
    h = R.rms_norm(x, L.in_norm, cfg.rms_eps)
    q = R.rope_rotate_half((h @ L.wq.T).reshape(T, cfg.n_q_heads, d), positions, cfg.rope_theta)
    k = R.rope_rotate_half((h @ L.wk.T).reshape(T, cfg.n_kv_heads, d), positions, cfg.rope_theta)
    v = (h @ L.wv.T).reshape(T, cfg.n_kv_heads, d)
    q = R.rms_norm(q, L.q_norm, cfg.rms_eps); k = R.rms_norm(k, L.k_norm, cfg.rms_eps)
    if cache_k is not None and cache_k.shape[0] > 0:
        keys = np.concatenate([cache_k, k]); values = np.concatenate([cache_v, v])
        kp = np.concatenate([cache_pos, positions])
    else:
        keys, values, kp = k, v, np.asarray(positions)
    sel = np.arange(T) if rows is None else np.asarray(rows)
    o = R.causal_gqa_attention(q[sel], keys, values, np.asarray(positions)[sel], kp)
    return x[sel] + o.reshape(len(sel), -1) @ L.wo.T, k, v


def _stack_no_final_norm(ids, embed, layers, final_norm, cfg, positions=None, caches=None, logit_rows=None):
    return _ORIG["stack_forward"](ids, embed, layers, np.full_like(final_norm, 1.7), cfg, positions, caches, logit_rows)


def _attn_half_no_residual(x, L, cfg, positions, cache_k=None, cache_v=None, cache_pos=None, rows=None):
    x1, k, v = _ORIG["attention_half"](x, L, cfg, positions, cache_k, cache_v, cache_pos, rows)
    sel = np.arange(x.shape[0]) if rows is None else np.asarray(rows)
    return x1 - x[sel], k, v


def _moe_half_routes_on_x1(x1, L, cfg, idx=None, w=None):
    h2 = R.rms_norm(x1, L.post_norm, cfg.rms_eps)
    probs = margin = None
    if idx is None:
        idx, w, probs, margin = R.moe_route(x1, L.router, cfg.top_k, cfg.norm_topk_prob)
    return x1 + R.moe_ffn(h2, idx, w, L.gate_up, L.down), (idx, w, probs, margin)


def _moe_half_input_norm(x1, L, cfg, idx=None, w=None):
    h2 = R.rms_norm(x1, L.in_norm, cfg.rms_eps)
    probs = margin = None
    if idx is None:
        idx, w, probs, margin = R.moe_route(h2, L.router, cfg.top_k, cfg.norm_topk_prob)
    return x1 + R.moe_ffn(h2, idx, w, L.gate_up, L.down), (idx, w, probs, margin)


def _moe_half_no_residual(x1, L, cfg, idx=None, w=None):
    out, route = _ORIG["moe_ffn_half"](x1, L, cfg, idx, w)
    return out - x1, route


def _moe_half_experts_on_x1(x1, L, cfg, idx=None, w=None):
    h2 = R.rms_norm(x1, L.post_norm, cfg.rms_eps)
    probs = margin = None
    if idx is None:
        idx, w, probs, margin = R.moe_route(h2, L.router, cfg.top_k, cfg.norm_topk_prob)
    return x1 + R.moe_ffn(x1, idx, w, L.gate_up, L.down), (idx, w, probs, margin)


_ORIG = {n: getattr(R, n) for n in ("moe_route", "attention_half", "stack_forward", "causal_gqa_attention",
                                    "moe_ffn_half")}


def _wrap_no_qk(monkeypatch):
    orig_rms = R.rms_norm

    def rms_skip_heads(x, w, eps):
        if x.ndim == 3:      # per-head QK norm is the only 3-D use
            return x
        return orig_rms(x, w, eps)
    monkeypatch.setattr(R, "rms_norm", rms_skip_heads)


MUTATIONS = {
    "rope_adjacent_pairs": ("rope_rotate_half", _rope_adjacent_pairs),
    "rope_sign_flipped": ("rope_rotate_half", _rope_sign_flipped),
    "rope_freq_exponent": ("rope_frequencies", _rope_freq_wrong_exponent),
    "rms_sum_not_mean": ("rms_norm", _rms_sum_not_mean),
    "rms_eps_outside_sqrt": ("rms_norm", _rms_eps_outside),
    "mask_excludes_self": ("causal_allowed", _mask_strict),
    "gqa_modulo_mapping": ("causal_gqa_attention", _attn_gqa_modulo),
    "silu_is_sigmoid": ("silu", _silu_is_sigmoid),
    "swiglu_gate_up_swapped": ("swiglu_ffn", _swiglu_swapped),
    "moe_no_renorm": ("moe_route", _route_no_renorm),
    "moe_tie_high_index": ("moe_route", _route_high_index_first),
    "ffn_reads_unnormed": ("dense_ffn_half", _ffn_on_unnormed),
    "rope_before_qk_norm": ("attention_half", _attn_half_rope_before_norm),
    "final_norm_weights_ignored": ("stack_forward", _stack_no_final_norm),
    "attention_residual_dropped": ("attention_half", _attn_half_no_residual),
    "moe_routes_on_x1": ("moe_ffn_half", _moe_half_routes_on_x1),
    "moe_uses_input_norm": ("moe_ffn_half", _moe_half_input_norm),
    "moe_residual_dropped": ("moe_ffn_half", _moe_half_no_residual),
    "moe_experts_on_x1": ("moe_ffn_half", _moe_half_experts_on_x1),
}


def _failing_pins():
    failed = []
    for name, pin in ALL_PINS.items():
        try:
            with np.errstate(all="ignore"):
                pin(R)
        except Exception:
            failed.append(name)
    return failed


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_mutation_is_caught(mutation, monkeypatch):
    attr, fn = MUTATIONS[mutation]
    monkeypatch.setattr(R, attr, fn)
    assert _failing_pins(), f"no pin catches the planted mistake {mutation}"


def test_missing_qk_norm_is_caught(monkeypatch):
    _wrap_no_qk(monkeypatch)
    assert _failing_pins()


def test_missing_attention_scale_is_caught(monkeypatch):
    orig = _ORIG["causal_gqa_attention"]

    def no_scale(q, k, v, q_pos, k_pos):
        return orig(q * np.sqrt(q.shape[-1]), k, v, q_pos, k_pos)
    monkeypatch.setattr(R, "causal_gqa_attention", no_scale)
    assert _failing_pins()


def test_unmutated_oracle_passes_every_pin():
    assert _failing_pins() == []
