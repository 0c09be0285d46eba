"""Pins of the fp64 oracle: checks against facts the pages and mathematics fix.

Each pin takes the oracle module ``R`` (so that the planted-mistake tests can
hand in a mutated copy) and raises AssertionError when the oracle disagrees.
None of them re-types the function it checks: they use closed forms, invariants,
brute force on tiny shapes, independent code paths and the values the pages
print (tests/golden/).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _cfg(R, **kw):
    base = dict(hidden=64, n_q_heads=4, n_kv_heads=2, head_dim=16, intermediate=96, vocab=50,
                n_layers=2, max_pos=4096, rope_theta=1.0e6, rms_eps=1.0e-6)
    base.update(kw)
    return R.Config(**base)


def _layer(R, cfg, rng, scale=0.2, moe=False):
    H, d, hq, hkv, I = cfg.hidden, cfg.head_dim, cfg.n_q_heads, cfg.n_kv_heads, cfg.intermediate
    kw = dict(in_norm=1 + 0.1 * rng.standard_normal(H), wq=scale * rng.standard_normal((hq * d, H)),
              wk=scale * rng.standard_normal((hkv * d, H)), wv=scale * rng.standard_normal((hkv * d, H)),
              q_norm=1 + 0.1 * rng.standard_normal(d), k_norm=1 + 0.1 * rng.standard_normal(d),
              wo=scale * rng.standard_normal((H, hq * d)), post_norm=1 + 0.1 * rng.standard_normal(H),
              w_gate=scale * rng.standard_normal((I, H)), w_up=scale * rng.standard_normal((I, H)),
              w_down=scale * rng.standard_normal((H, I)))
    if moe:
        E, Im = cfg.n_experts, cfg.moe_intermediate
        kw.update(router=rng.standard_normal((E, H)), gate_up=scale * rng.standard_normal((E, 2 * Im, H)),
                  down=scale * rng.standard_normal((E, H, Im)))
    return R.LayerWeights(**kw)


# ----------------------------------------------------------------------------- RMSNorm
def pin_rmsnorm_constant_vector(R):
    """x = c * 1: mean square is c^2, so out = c / sqrt(c^2 + eps) * w exactly."""
    n, eps = 1024, 1e-2
    w = 1 + 0.1 * _rng(1).standard_normal(n)
    for c in (0.5, -3.0, 7.25):
        out = R.rms_norm(np.full(n, c), w, eps)
        np.testing.assert_allclose(out, c / math.sqrt(c * c + eps) * w, rtol=1e-13, atol=0)


def pin_rmsnorm_scale_invariance_and_unit_rms(R):
    x = _rng(2).standard_normal((5, 300))
    w = np.ones(300)
    a = R.rms_norm(x, w, 0.0)
    np.testing.assert_allclose(R.rms_norm(17.0 * x, w, 0.0), a, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(np.mean(a * a, axis=-1), 1.0, rtol=1e-12)
    # [3, 4]: mean square 12.5
    np.testing.assert_allclose(R.rms_norm(np.array([3.0, 4.0]), np.ones(2), 0.0),
                               [3 / math.sqrt(12.5), 4 / math.sqrt(12.5)], rtol=1e-14)


# ----------------------------------------------------------------------------- RoPE
def pin_rope_identity_at_zero(R):
    u = _rng(3).standard_normal((4, 3, 128))
    np.testing.assert_array_equal(R.rope_rotate_half(u, np.zeros(4), 1e6), u)


def pin_rope_pair_norms(R):
    u = _rng(4).standard_normal((6, 2, 128))
    out = R.rope_rotate_half(u, np.array([1, 5, 77, 1000, 32767, 40959]), 1e6)
    n_in = u[..., :64] ** 2 + u[..., 64:] ** 2
    n_out = out[..., :64] ** 2 + out[..., 64:] ** 2
    np.testing.assert_allclose(n_out, n_in, rtol=1e-12, atol=1e-14)


def pin_rope_relative_position(R):
    rng = _rng(5)
    q = rng.standard_normal((1, 1, 128))
    k = rng.standard_normal((1, 1, 128))
    ref = None
    for shift in (0, 1, 100, 20000):
        m, n = 37 + shift, 5 + shift
        dot = float(np.sum(R.rope_rotate_half(q, np.array([m]), 1e6) * R.rope_rotate_half(k, np.array([n]), 1e6)))
        if ref is None:
            ref = dot
        assert abs(dot - ref) < 1e-10 * max(1.0, abs(ref)), (shift, dot, ref)


def pin_rope_half_split_pairing(R):
    """The 8-dim example: dimension i mixes only with i + 4."""
    g = json.load(open(os.path.join(GOLDEN, "rope_pairing_8dim.json")))
    d = g["head_dim"]
    for a, b in g["pairs"]:
        e = np.zeros((1, 1, d))
        e[0, 0, a] = 1.0
        out = R.rope_rotate_half(e, np.array([3]), 10.0)[0, 0]
        nz = set(np.nonzero(np.abs(out) > 1e-15)[0].tolist())
        assert nz == {a, b}, (a, b, out)


def pin_rope_angle_values(R):
    """theta_i = 1e6^(-2i/128): i=0 gives angle m, i=32 gives m * 1e-3. A unit vector
    on the first half of a pair rotates to (cos phi, sin phi) on (i, i+64)."""
    for i, m, phi in ((0, 1, 1.0), (0, 2, 2.0), (32, 1000, 1.0), (32, 3000, 3.0), (16, 10 ** 3, 10 ** 3 * 10 ** -1.5)):
        e = np.zeros((1, 1, 128))
        e[0, 0, i] = 1.0
        out = R.rope_rotate_half(e, np.array([m]), 1e6)[0, 0]
        np.testing.assert_allclose([out[i], out[i + 64]], [math.cos(phi), math.sin(phi)], rtol=0, atol=1e-12)
        f = np.zeros((1, 1, 128))
        f[0, 0, i + 64] = 1.0
        out = R.rope_rotate_half(f, np.array([m]), 1e6)[0, 0]
        np.testing.assert_allclose([out[i], out[i + 64]], [-math.sin(phi), math.cos(phi)], rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- attention
def pin_attention_single_key(R):
    rng = _rng(6)
    q = rng.standard_normal((1, 4, 16))
    k = rng.standard_normal((1, 2, 16))
    v = rng.standard_normal((1, 2, 16))
    out = R.causal_gqa_attention(q, k, v, np.array([0]), np.array([0]))
    for h in range(4):
        np.testing.assert_allclose(out[0, h], v[0, h // 2], rtol=1e-14)


def pin_attention_zero_query_prefix_mean(R):
    """q = 0 gives equal scores, so row i averages v over keys 0..i (itself included)."""
    rng = _rng(7)
    T = 9
    q = np.zeros((T, 2, 8))
    k = rng.standard_normal((T, 1, 8))
    v = rng.standard_normal((T, 1, 8))
    out = R.causal_gqa_attention(q, k, v, np.arange(T), np.arange(T))
    for i in range(T):
        np.testing.assert_allclose(out[i, 0], v[: i + 1, 0].mean(axis=0), rtol=1e-12, atol=1e-14)


def pin_attention_scale_closed_form(R):
    """Two keys with scores a*b/sqrt(d) and 0, values 1 and 0: output = sigmoid(a*b/sqrt(d))."""
    d = 128
    for a, b in ((1.0, 2.0), (3.0, -4.0), (10.0, 1.5)):
        q = np.zeros((1, 1, d)); q[0, 0, 3] = a
        k = np.zeros((2, 1, d)); k[1, 0, 3] = b
        v = np.zeros((2, 1, d)); v[1, 0, 0] = 1.0
        out = R.causal_gqa_attention(q, k, v, np.array([1]), np.array([0, 1]))
        z = a * b / math.sqrt(d)
        np.testing.assert_allclose(out[0, 0, 0], 1 / (1 + math.exp(-z)), rtol=1e-12)


def pin_attention_gqa_equals_mha_repeated(R):
    """Independent path: K/V repeated per query head (repeat_interleave), an explicit
    additive mask matrix, einsum scores, exp-normalise."""
    rng = _rng(8)
    T, hq, hkv, d = 11, 8, 2, 16
    q = rng.standard_normal((T, hq, d)); k = rng.standard_normal((T, hkv, d)); v = rng.standard_normal((T, hkv, d))
    kr = np.repeat(k, hq // hkv, axis=1); vr = np.repeat(v, hq // hkv, axis=1)
    M = np.triu(np.full((T, T), -np.inf), 1)
    s = np.einsum("ihd,jhd->hij", q, kr) / math.sqrt(d) + M[None]
    p = np.exp(s - s.max(-1, keepdims=True)); p /= p.sum(-1, keepdims=True)
    ref = np.einsum("hij,jhd->ihd", p, vr)
    np.testing.assert_allclose(R.causal_gqa_attention(q, k, v, np.arange(T), np.arange(T)), ref, rtol=1e-11, atol=1e-13)


def pin_attention_brute_force_tiny(R):
    rng = _rng(9)
    for T in (1, 2, 5, 8):
        q = rng.standard_normal((T, 2, 4)); k = rng.standard_normal((T, 1, 4)); v = rng.standard_normal((T, 1, 4))
        out = R.causal_gqa_attention(q, k, v, np.arange(T), np.arange(T))
        for i in range(T):
            for h in range(2):
                w = [math.exp(sum(q[i, h, c] * k[j, 0, c] for c in range(4)) / 2.0) for j in range(i + 1)]
                z = sum(w)
                for c in range(4):
                    ref = sum(w[j] * v[j, 0, c] for j in range(i + 1)) / z
                    assert abs(out[i, h, c] - ref) < 1e-12, (T, i, h, c)


def pin_attention_printed_mask(R):
    lines = [l for l in open(os.path.join(GOLDEN, "causal_mask_17.txt")) if not l.startswith("#")]
    printed = np.array([[0.0 if t == "0" else -np.inf for t in l.split()] for l in lines])
    assert printed.shape == (17, 17)
    allowed = R.causal_allowed(np.arange(17), np.arange(17))
    np.testing.assert_array_equal(allowed, printed == 0.0)


def pin_attention_causality(R):
    rng = _rng(10)
    T = 12
    q = rng.standard_normal((T, 4, 8)); k = rng.standard_normal((T, 2, 8)); v = rng.standard_normal((T, 2, 8))
    a = R.causal_gqa_attention(q, k, v, np.arange(T), np.arange(T))
    k2, v2 = k.copy(), v.copy()
    k2[7:] = rng.standard_normal((T - 7, 2, 8)); v2[7:] = rng.standard_normal((T - 7, 2, 8))
    b = R.causal_gqa_attention(q, k2, v2, np.arange(T), np.arange(T))
    np.testing.assert_array_equal(a[:7], b[:7])
    assert np.abs(a[7:] - b[7:]).max() > 1e-3


# ----------------------------------------------------------------------------- SwiGLU
def pin_silu_values(R):
    assert R.silu(np.array(0.0)) == 0.0
    np.testing.assert_allclose(R.silu(np.array(40.0)), 40.0, rtol=1e-15)
    assert abs(R.silu(np.array(-40.0))) < 1e-15
    # silu(1) = 1 / (1 + e^-1)
    np.testing.assert_allclose(R.silu(np.array(1.0)), 0.7310585786300049, rtol=1e-15)
    np.testing.assert_allclose(R.silu(np.array(-1.0)), -0.2689414213699951, rtol=1e-15)


def pin_swiglu_one_hot(R):
    """gate row selects h_a, up row selects h_b, down column routes to output c:
    out_c = silu(h_a) * h_b, every other output 0."""
    H = 6
    h = np.array([[0.3, -1.2, 2.0, 0.7, -0.4, 1.1]])
    for a, b, c in ((0, 2, 5), (2, 0, 1), (1, 3, 3)):
        wg = np.zeros((1, H)); wg[0, a] = 1.0
        wu = np.zeros((1, H)); wu[0, b] = 1.0
        wd = np.zeros((H, 1)); wd[c, 0] = 1.0
        out = R.swiglu_ffn(h, wg, wu, wd)[0]
        z = h[0, a]
        ref = np.zeros(H); ref[c] = z / (1 + math.exp(-z)) * h[0, b]
        np.testing.assert_allclose(out, ref, rtol=1e-14, atol=1e-16)


# ----------------------------------------------------------------------------- block
def pin_block_decode_equals_prefill_row(R):
    """Prefill T tokens, then decode token T against their cached K/V == row T of a
    prefill over T+1 tokens (the no-cache recompute)."""
    rng = _rng(11)
    cfg = _cfg(R)
    L = _layer(R, cfg, rng)
    T = 10
    x = rng.standard_normal((T + 1, cfg.hidden))
    full, kf, vf = R.block_forward(x, L, cfg, np.arange(T + 1))
    _, k, v = R.block_forward(x[:T], L, cfg, np.arange(T))
    dec, kd, vd = R.block_forward(x[T:], L, cfg, np.array([T]), k, v, np.arange(T))
    np.testing.assert_allclose(dec[0], full[T], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(kd[0], kf[T], rtol=1e-12, atol=1e-13)
    # start offset: a cache that starts at position 40 behaves as the same keys
    _, k2, v2 = R.block_forward(x[:T], L, cfg, 40 + np.arange(T))
    dec2, _, _ = R.block_forward(x[T:], L, cfg, np.array([40 + T]), k2, v2, 40 + np.arange(T))
    full2, _, _ = R.block_forward(x, L, cfg, 40 + np.arange(T + 1))
    np.testing.assert_allclose(dec2[0], full2[T], rtol=1e-11, atol=1e-12)


def pin_block_identity_when_outputs_zero(R):
    rng = _rng(12)
    cfg = _cfg(R)
    L = _layer(R, cfg, rng)
    L.wo = np.zeros_like(L.wo)
    L.w_down = np.zeros_like(L.w_down)
    x = rng.standard_normal((7, cfg.hidden))
    out, _, _ = R.block_forward(x, L, cfg, np.arange(7))
    np.testing.assert_array_equal(out, x)


def pin_block_residual_structure(R):
    """With w_down = 0 the block is x + o_proj(attn); with wo = 0 it is x + FFN(norm2(x)):
    the FFN sees the post-attention norm of x, not x itself."""
    rng = _rng(13)
    cfg = _cfg(R)
    L = _layer(R, cfg, rng)
    x = rng.standard_normal((5, cfg.hidden))
    L.wo = np.zeros_like(L.wo)
    out, _, _ = R.block_forward(x, L, cfg, np.arange(5))
    # independent path: explicit per-row FFN on the normalised row
    for t in range(5):
        r = x[t] / math.sqrt(float(np.mean(x[t] ** 2)) + cfg.rms_eps) * L.post_norm
        g = L.w_gate @ r; u = L.w_up @ r
        ref = x[t] + L.w_down @ (g / (1 + np.exp(-g)) * u)
        np.testing.assert_allclose(out[t], ref, rtol=1e-11, atol=1e-12)


def pin_block_causality(R):
    rng = _rng(14)
    cfg = _cfg(R)
    L = _layer(R, cfg, rng)
    x = rng.standard_normal((9, cfg.hidden))
    a, _, _ = R.block_forward(x, L, cfg, np.arange(9))
    x2 = x.copy(); x2[5:] = rng.standard_normal((4, cfg.hidden))
    b, _, _ = R.block_forward(x2, L, cfg, np.arange(9))
    np.testing.assert_array_equal(a[:5], b[:5])


def pin_block_qk_norm_scale_invariance(R):
    """Per-head QK RMSNorm makes the block invariant to the scale of Wq and Wk
    (eps = 0): without it the scores would scale by c_q * c_k."""
    rng = _rng(22)
    cfg = _cfg(R, rms_eps=0.0)
    L = _layer(R, cfg, rng)
    x = rng.standard_normal((8, cfg.hidden))
    a, _, _ = R.block_forward(x, L, cfg, np.arange(8))
    L.wq = 3.0 * L.wq; L.wk = 0.25 * L.wk
    b, _, _ = R.block_forward(x, L, cfg, np.arange(8))
    np.testing.assert_allclose(b, a, rtol=1e-10, atol=1e-11)


def pin_block_position_shift_invariance(R):
    """QK-norm before RoPE keeps attention a function of position differences only, so
    shifting every position by the same amount leaves the block output unchanged."""
    rng = _rng(23)
    cfg = _cfg(R)
    L = _layer(R, cfg, rng)
    L.q_norm = 1 + 0.5 * rng.standard_normal(cfg.head_dim)
    L.k_norm = 1 + 0.5 * rng.standard_normal(cfg.head_dim)
    x = rng.standard_normal((8, cfg.hidden))
    a, _, _ = R.block_forward(x, L, cfg, np.arange(8))
    b, _, _ = R.block_forward(x, L, cfg, 1234 + np.arange(8))
    np.testing.assert_allclose(b, a, rtol=1e-9, atol=1e-10)


# ----------------------------------------------------------------------------- MoE
def _moe_cfg(R, E=4, k=2, Im=8):
    return _cfg(R, n_experts=E, top_k=k, moe_intermediate=Im)


def pin_moe_worked_example(R):
    """4 experts; router probabilities (0.05, 0.56, 0.15, 0.24) select E2 and E4, which
    renormalise to 0.7 and 0.3; the output is 0.7 E2(x) + 0.3 E4(x)."""
    g = json.load(open(os.path.join(GOLDEN, "moe_worked_example.json")))
    E, k = g["n_experts"], g["top_k"]
    H, Im = 4, 3
    probs = np.array([0.05, 0.56, 0.15, 0.24])
    h2 = np.array([[1.0, 0.0, 0.0, 0.0]])
    router = np.zeros((E, H)); router[:, 0] = np.log(probs)
    idx, w, p, margin = R.moe_route(h2, router, k, True)
    assert [int(i) + 1 for i in idx[0]] == g["selected_experts_1_based"], idx
    np.testing.assert_allclose(w[0], g["weights"], rtol=1e-13)
    np.testing.assert_allclose(margin[0], 0.24 - 0.15, rtol=1e-12)
    # experts with closed-form outputs: expert e maps h to a_e * silu(h0) * h0 on coordinate e
    rng = _rng(15)
    x = np.array([[0.9, -0.3, 0.5, 1.7]])
    gate_up = np.zeros((E, 2 * Im, H)); down = np.zeros((E, H, Im))
    a = 1 + rng.random(E)
    for e in range(E):
        gate_up[e, 0, 0] = 1.0          # gate row 0 reads x0
        gate_up[e, Im, 0] = a[e]        # up row 0 reads a_e x0
        down[e, e, 0] = 1.0             # output coordinate e
    out = R.moe_ffn(x, idx, w, gate_up, down)[0]
    s = x[0, 0] / (1 + math.exp(-x[0, 0])) * x[0, 0]
    ref = np.zeros(H)
    ref[1] = g["weights"][0] * a[1] * s
    ref[3] = g["weights"][1] * a[3] * s
    np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-16)


def pin_moe_all_experts_is_dense_softmax_sum(R):
    rng = _rng(16)
    E, H, Im, T = 5, 12, 6, 4
    h2 = rng.standard_normal((T, H)); router = rng.standard_normal((E, H))
    gate_up = rng.standard_normal((E, 2 * Im, H)); down = rng.standard_normal((E, H, Im))
    idx, w, p, _ = R.moe_route(h2, router, E, True)
    out = R.moe_ffn(h2, idx, w, gate_up, down)
    for t in range(T):
        lg = router @ h2[t]
        pr = np.exp(lg - lg.max()); pr /= pr.sum()
        ref = np.zeros(H)
        for e in range(E):
            g = gate_up[e, :Im] @ h2[t]; u = gate_up[e, Im:] @ h2[t]
            ref += pr[e] * (down[e] @ (g / (1 + np.exp(-g)) * u))
        np.testing.assert_allclose(out[t], ref, rtol=1e-10, atol=1e-12)


def pin_moe_sparse_equals_tokenwise(R):
    """The sparse per-expert evaluation equals a per-token loop over its own top-k."""
    rng = _rng(17)
    E, k, H, Im, T = 8, 3, 16, 5, 20
    h2 = rng.standard_normal((T, H)); router = rng.standard_normal((E, H))
    gate_up = rng.standard_normal((E, 2 * Im, H)); down = rng.standard_normal((E, H, Im))
    idx, w, p, _ = R.moe_route(h2, router, k, True)
    out = R.moe_ffn(h2, idx, w, gate_up, down)
    for t in range(T):
        lg = router @ h2[t]
        pr = np.exp(lg - lg.max()); pr /= pr.sum()
        top = sorted(range(E), key=lambda e: (-pr[e], e))[:k]
        assert list(idx[t]) == top
        ref = np.zeros(H)
        tot = sum(pr[e] for e in top)
        for e in top:
            g = gate_up[e, :Im] @ h2[t]; u = gate_up[e, Im:] @ h2[t]
            ref += pr[e] / tot * (down[e] @ (g / (1 + np.exp(-g)) * u))
        np.testing.assert_allclose(out[t], ref, rtol=1e-10, atol=1e-12)


def pin_moe_tie_break_and_margin(R):
    h2 = np.array([[1.0]])
    router = np.array([[0.5], [2.0], [2.0], [1.0], [2.0]])   # experts 1, 2, 4 tie
    idx, w, p, margin = R.moe_route(h2, router, 2, True)
    assert list(idx[0]) == [1, 2]
    assert margin[0] == 0.0
    np.testing.assert_allclose(w[0], [0.5, 0.5], rtol=1e-15)
    idx, w, p, margin = R.moe_route(h2, router, 3, False)
    assert list(idx[0]) == [1, 2, 4]
    np.testing.assert_allclose(w[0].sum(), 3 * math.e ** 2 / (math.e ** 0.5 + 3 * math.e ** 2 + math.e), rtol=1e-13)


def pin_moe_permutation(R):
    idx = np.array([[2, 0], [0, 1], [2, 1], [1, 0]])
    offsets, tok, slot = R.moe_permutation(idx, 4)
    assert list(offsets) == [0, 3, 6, 8, 8]
    assert list(tok) == [0, 1, 3, 1, 2, 3, 0, 2]
    assert list(slot) == [1, 0, 1, 1, 1, 0, 0, 0]
    for i in range(len(tok)):
        e = np.searchsorted(offsets, i, side="right") - 1
        assert idx[tok[i], slot[i]] == e


def _expert_closed(gate_up_e, down_e, r):
    """One SwiGLU expert on one row, restated: gate rows first, then up rows."""
    im = gate_up_e.shape[0] // 2
    g = gate_up_e[:im] @ r
    u = gate_up_e[im:] @ r
    return down_e @ (g / (1 + np.exp(-g)) * u)


def _moe_block_layer(R, rng, cfg):
    L = _layer(R, cfg, rng, moe=True)
    # norm weights far from 1, so that post- and pre-attention norms, and x1 versus
    # norm_2(x1), route differently
    L.in_norm = 1 + 0.6 * rng.standard_normal(cfg.hidden)
    L.post_norm = 1 + 0.6 * rng.standard_normal(cfg.hidden)
    return L


def pin_moe_block_worked_example(R):
    """The worked example at block level: with o_proj zero the attention half is the
    identity (x1 = x); a router built on the token's own norm_2(x) row gives the
    probabilities (0.05, 0.56, 0.15, 0.24), so top-2 picks E2 and E4 with weights 0.7
    and 0.3, and out = x + 0.7 E2(h2) + 0.3 E4(h2). With k = E the output is the dense
    sum over all experts weighted by the probabilities themselves."""
    g = json.load(open(os.path.join(GOLDEN, "moe_worked_example.json")))
    rng = _rng(24)
    cfg = _moe_cfg(R, E=g["n_experts"], k=g["top_k"], Im=6)
    L = _moe_block_layer(R, rng, cfg)
    L.wo = np.zeros_like(L.wo)
    x = 1.5 * rng.standard_normal((1, cfg.hidden))
    # norm_2 of x, restated: x / sqrt(mean x^2 + eps) * post_norm
    h2 = x[0] / math.sqrt(float(np.mean(x[0] ** 2)) + cfg.rms_eps) * L.post_norm
    probs = np.array([0.05, 0.56, 0.15, 0.24])
    L.router = np.log(probs)[:, None] * h2[None, :] / float(h2 @ h2)   # router . h2 = log p
    out, _, _, (idx, w, p, _) = R.moe_block_forward(x, L, cfg, np.array([3]))
    assert [int(i) + 1 for i in idx[0]] == g["selected_experts_1_based"], idx
    np.testing.assert_allclose(p[0], probs, rtol=1e-12)
    ref = x[0] + g["weights"][0] * _expert_closed(L.gate_up[1], L.down[1], h2) \
        + g["weights"][1] * _expert_closed(L.gate_up[3], L.down[3], h2)
    np.testing.assert_allclose(out[0], ref, rtol=1e-11, atol=1e-13)
    dense_cfg = _moe_cfg(R, E=g["n_experts"], k=g["n_experts"], Im=6)
    out_all, _, _, _ = R.moe_block_forward(x, L, dense_cfg, np.array([3]))
    ref_all = x[0] + sum(probs[e] * _expert_closed(L.gate_up[e], L.down[e], h2) for e in range(len(probs)))
    np.testing.assert_allclose(out_all[0], ref_all, rtol=1e-11, atol=1e-13)


def pin_moe_block_tokenwise(R):
    """The MoE block against a per-token loop that restates its second half: the
    post-attention RMSNorm of x1 (not x, not the input norm), the router's softmax on
    that row, top-k by descending probability (lower index first), renormalised
    weights, experts evaluated on the normed row, and the residual x1 added back. x1
    comes from the attention half, pinned on its own. The given-routing form of
    moe_ffn_half must reproduce the same rows from the same routing."""
    rng = _rng(25)
    cfg = _moe_cfg(R, E=8, k=3, Im=5)
    L = _moe_block_layer(R, rng, cfg)
    T = 9
    x = rng.standard_normal((T, cfg.hidden))
    pos = 5 + np.arange(T)
    out, _, _, (idx, w, _, _) = R.moe_block_forward(x, L, cfg, pos)
    x1, _, _ = R.attention_half(x, L, cfg, pos)
    for t in range(T):
        r = x1[t] / math.sqrt(float(np.mean(x1[t] ** 2)) + cfg.rms_eps) * L.post_norm
        lg = L.router @ r
        pr = np.exp(lg - lg.max()); pr /= pr.sum()
        top = sorted(range(cfg.n_experts), key=lambda e: (-pr[e], e))[:cfg.top_k]
        assert list(idx[t]) == top, (t, idx[t], top)
        tot = sum(pr[e] for e in top)
        ref = x1[t] + sum(pr[e] / tot * _expert_closed(L.gate_up[e], L.down[e], r) for e in top)
        np.testing.assert_allclose(out[t], ref, rtol=1e-11, atol=1e-12)
    given, _ = R.moe_ffn_half(x1, L, cfg, idx=idx, w=w)
    np.testing.assert_allclose(given, out, rtol=1e-13, atol=1e-14)
    # a different, valid routing is evaluated as given: every token on experts (0, 1, 2)
    # with equal weights
    idx2 = np.tile(np.arange(3, dtype=np.int32), (T, 1))
    w2 = np.full((T, 3), 1.0 / 3.0)
    given2, _ = R.moe_ffn_half(x1, L, cfg, idx=idx2, w=w2)
    for t in (0, T - 1):
        r = x1[t] / math.sqrt(float(np.mean(x1[t] ** 2)) + cfg.rms_eps) * L.post_norm
        ref = x1[t] + sum(_expert_closed(L.gate_up[e], L.down[e], r) for e in range(3)) / 3.0
        np.testing.assert_allclose(given2[t], ref, rtol=1e-11, atol=1e-12)


# ----------------------------------------------------------------------------- stack
def _stack_inputs(R, rng, cfg, n_layers):
    E = rng.standard_normal((cfg.vocab, cfg.hidden))
    layers = [_layer(R, cfg, rng) for _ in range(n_layers)]
    return E, layers


def pin_stack_zero_residual_closed_form(R):
    """All o_proj and down weights zero: every block is the identity, so
    logits[t] = norm(E[id_t]) . E^T. With unit final-norm weights and rows of equal
    norm r, logits[t][j] = E_id . E_j * sqrt(H) / r, maximal (= r sqrt(H)) at j = id_t."""
    rng = _rng(18)
    cfg = _cfg(R, rms_eps=0.0)
    E, layers = _stack_inputs(R, rng, cfg, 2)
    E = E / np.linalg.norm(E, axis=1, keepdims=True) * 2.5
    for L in layers:
        L.wo = np.zeros_like(L.wo); L.w_down = np.zeros_like(L.w_down)
    ids = rng.integers(0, cfg.vocab, 9)
    logits, _ = R.stack_forward(ids, E, layers, np.ones(cfg.hidden), cfg)
    assert logits.shape == (9, cfg.vocab)
    np.testing.assert_array_equal(np.argmax(logits, axis=1), ids)
    np.testing.assert_allclose(logits[np.arange(9), ids], 2.5 * math.sqrt(cfg.hidden), rtol=1e-12)


def pin_stack_last_only_and_causality(R):
    rng = _rng(19)
    cfg = _cfg(R)
    E, layers = _stack_inputs(R, rng, cfg, 2)
    E *= 0.3
    fn = 1 + 0.1 * rng.standard_normal(cfg.hidden)
    ids = rng.integers(0, cfg.vocab, 8)
    full, _ = R.stack_forward(ids, E, layers, fn, cfg)
    last, _ = R.stack_forward(ids, E, layers, fn, cfg, logit_rows=[7])
    np.testing.assert_allclose(last[0], full[7], rtol=1e-12, atol=1e-13)
    ids2 = ids.copy(); ids2[5:] = (ids2[5:] + 1) % cfg.vocab
    full2, _ = R.stack_forward(ids2, E, layers, fn, cfg)
    np.testing.assert_array_equal(full[:5], full2[:5])


def pin_stack_decode_equals_prefill(R):
    rng = _rng(20)
    cfg = _cfg(R)
    E, layers = _stack_inputs(R, rng, cfg, 2)
    E *= 0.3
    fn = np.ones(cfg.hidden)
    ids = rng.integers(0, cfg.vocab, 7)
    full, _ = R.stack_forward(ids, E, layers, fn, cfg)
    _, kv = R.stack_forward(ids[:6], E, layers, fn, cfg)
    caches = [(k, v, np.arange(6)) for (k, v) in kv]
    dec, _ = R.stack_forward(ids[6:], E, layers, fn, cfg, positions=np.array([6]), caches=caches)
    np.testing.assert_allclose(dec[0], full[6], rtol=1e-10, atol=1e-11)


# ----------------------------------------------------------------------------- sizes
def pin_model_sizes(R):
    g = json.load(open(os.path.join(GOLDEN, "model_sizes.json")))
    cfg = R.QWEN3_0_6B
    untied = R.param_count(cfg, tied=False)
    assert round(untied / 1e9, 3) == g["params_untied_billions_3dp"], untied
    assert round(untied * 4 / 1e9, 2) == g["fp32_weight_gb_2dp"]
    assert untied == 751_632_384
    assert R.param_count(cfg, tied=True) == untied - cfg.vocab * cfg.hidden
    assert R.kv_bytes_per_token_layer(cfg) == g["kv_bytes_per_token_layer"]
    assert R.kv_bytes_per_token_layer(cfg) * cfg.n_layers // 1024 == g["kv_kib_per_token_28_layers"]


def pin_printed_shapes(R):
    """Shapes the notebook prints for its 17-token prompt (2-expert variant)."""
    g = json.load(open(os.path.join(GOLDEN, "model_sizes.json")))
    cfg = R.QWEN3_0_6B
    rng = _rng(21)
    E = rng.standard_normal((64, cfg.hidden)) * 0.02
    x = E[rng.integers(0, 64, 17)]
    assert list(x.shape) == g["embed_shape_17"]
    wq = rng.standard_normal((cfg.n_q_heads * cfg.head_dim, cfg.hidden)) * 0.02
    q = (R.rms_norm(x, np.ones(cfg.hidden), cfg.rms_eps) @ wq.T).reshape(17, cfg.n_q_heads, cfg.head_dim)
    assert list(q[:, 0, :].shape) == g["q_head_shape_17"]
    idx, w, probs, _ = R.moe_route(x, rng.standard_normal((2, cfg.hidden)), 1, False)
    assert list(probs.shape) == g["router_logits_shape_17_2experts"]
    assert g["logits_shape"] == [cfg.vocab]


ALL_PINS = {name: fn for name, fn in globals().items() if name.startswith("pin_")}
