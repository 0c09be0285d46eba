"""Properties of the oracle over random small shapes (hypothesis, derandomised): the
fixed-shape pins of oracle_pins.py widened to head counts, group sizes, token counts,
start positions, chunkings and routing settings drawn at random. Each compares the
oracle with an independent computation, or with a second oracle call that must agree
by the definition (chunked prefill against one-shot prefill), never with a re-typed
copy of the function under test."""
import math

import numpy as np
import pytest

pytest.importorskip("hypothesis")
from hypothesis import HealthCheck, given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402

import oracle.qwen3_ref as R  # noqa: E402
from oracle_pins import _cfg, _layer  # noqa: E402

PROPS = settings(max_examples=30, deadline=None, derandomize=True, suppress_health_check=[HealthCheck.too_slow])
seeds = st.integers(0, 2 ** 31 - 1)


@PROPS
@given(hkv=st.sampled_from([1, 2, 4]), group=st.sampled_from([1, 2, 3, 4]), tk=st.integers(1, 12),
       tq=st.integers(1, 12), start=st.integers(0, 40000), d=st.sampled_from([4, 8, 16]), seed=seeds)
def test_attention_with_a_cache_offset_equals_mha_on_repeated_kv(hkv, group, tk, tq, start, d, seed):
    """Queries are the last tq of tk tokens at positions start.. (a chunk after a
    cache). Independent path: K/V repeated per query head, per-row log-sum-exp."""
    tq = min(tq, tk)
    rng = np.random.default_rng(seed)
    hq = hkv * group
    q = rng.standard_normal((tq, hq, d))
    k = rng.standard_normal((tk, hkv, d))
    v = rng.standard_normal((tk, hkv, d))
    k_pos = start + np.arange(tk)
    q_pos = k_pos[tk - tq:]
    out = R.causal_gqa_attention(q, k, v, q_pos, k_pos)
    kr, vr = np.repeat(k, group, axis=1), np.repeat(v, group, axis=1)
    for i in range(tq):
        n_vis = tk - tq + i + 1  # keys up to and including the query's own position
        for h in range(hq):
            s = kr[:n_vis, h] @ q[i, h] / math.sqrt(d)
            p = np.exp(s - np.logaddexp.reduce(s))
            np.testing.assert_allclose(out[i, h], p @ vr[:n_vis, h], rtol=1e-10, atol=1e-12)


@PROPS
@given(hkv=st.sampled_from([1, 2]), group=st.sampled_from([1, 2, 4]), T=st.integers(2, 10),
       split=st.integers(1, 9), start=st.integers(0, 30000), seed=seeds)
def test_chunked_prefill_equals_one_shot_prefill(hkv, group, T, split, start, seed):
    """A block over T tokens at positions start.. equals the same block run as two
    chunks, the second attending to the first's cached keys and values."""
    split = min(split, T - 1)
    rng = np.random.default_rng(seed)
    cfg = _cfg(R, n_q_heads=hkv * group, n_kv_heads=hkv)
    L = _layer(R, cfg, rng)
    x = rng.standard_normal((T, cfg.hidden))
    pos = start + np.arange(T)
    full, kf, vf = R.block_forward(x, L, cfg, pos)
    a, k1, v1 = R.block_forward(x[:split], L, cfg, pos[:split])
    b, k2, v2 = R.block_forward(x[split:], L, cfg, pos[split:], k1, v1, pos[:split])
    np.testing.assert_allclose(np.concatenate([a, b]), full, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(np.concatenate([k1, k2]), kf, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(np.concatenate([v1, v2]), vf, rtol=1e-12, atol=1e-13)


@PROPS
@given(d=st.sampled_from([8, 16, 64, 128]), m=st.integers(0, 40000), n=st.integers(0, 40000),
       shift=st.integers(0, 40000), seed=seeds)
def test_rope_keeps_pair_norms_and_depends_on_position_differences(d, m, n, shift, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, 1, d))
    k = rng.standard_normal((1, 1, d))
    rq = R.rope_rotate_half(q, np.array([m]), 1e6)
    h = d // 2
    np.testing.assert_allclose(rq[..., :h] ** 2 + rq[..., h:] ** 2, q[..., :h] ** 2 + q[..., h:] ** 2, rtol=1e-10)
    dot = lambda a, b: float(np.sum(R.rope_rotate_half(q, np.array([a]), 1e6) * R.rope_rotate_half(k, np.array([b]), 1e6)))
    scale = float(np.linalg.norm(q) * np.linalg.norm(k))
    assert abs(dot(m, n) - dot(m + shift, n + shift)) <= 1e-9 * scale


@PROPS
@given(E=st.integers(2, 8), k=st.integers(1, 8), T=st.integers(1, 6), renorm=st.booleans(), seed=seeds)
def test_moe_equals_a_tokenwise_loop_over_its_own_top_k(E, k, T, renorm, seed):
    """Independent per-token path: probabilities by exp/sum, top-k by Python's sort on
    (-p, index), the expert FFN written out, slots summed in order."""
    k = min(k, E)
    rng = np.random.default_rng(seed)
    H, Im = 12, 6
    h2 = rng.standard_normal((T, H))
    router = rng.standard_normal((E, H))
    gate_up = 0.3 * rng.standard_normal((E, 2 * Im, H))
    down = 0.3 * rng.standard_normal((E, H, Im))
    idx, w, probs, margin = R.moe_route(h2, router, k, renorm)
    out = R.moe_ffn(h2, idx, w, gate_up, down)
    for t in range(T):
        z = router @ h2[t]
        p = np.exp(z - z.max())
        p /= p.sum()
        np.testing.assert_allclose(probs[t], p, rtol=1e-12, atol=1e-15)
        top = sorted(range(E), key=lambda e: (-p[e], e))[:k]
        assert list(idx[t]) == top
        wt = p[top] / p[top].sum() if renorm else p[top]
        np.testing.assert_allclose(w[t], wt, rtol=1e-12)
        ref = np.zeros(H)
        for j, e in enumerate(top):
            g, u = gate_up[e, :Im] @ h2[t], gate_up[e, Im:] @ h2[t]
            ref += wt[j] * (down[e] @ (g / (1.0 + np.exp(-g)) * u))
        np.testing.assert_allclose(out[t], ref, rtol=1e-10, atol=1e-12)
        if k < E:
            assert margin[t] == pytest.approx(np.sort(p)[::-1][k - 1] - np.sort(p)[::-1][k], abs=1e-15)


@PROPS
@given(n_layers=st.integers(1, 3), T0=st.integers(1, 6), n_dec=st.integers(1, 4), hkv=st.sampled_from([1, 2]),
       group=st.sampled_from([1, 2, 4]), seed=seeds)
def test_stack_decode_steps_equal_the_rows_of_one_prefill(n_layers, T0, n_dec, hkv, group, seed):
    """A prompt of T0 tokens, then n_dec decode steps each appending its keys and
    values to every layer's cache, give the logits of rows T0..T0+n_dec-1 of a
    single prefill over all T0 + n_dec tokens (greedy feedback replaced by fixed ids)."""
    rng = np.random.default_rng(seed)
    cfg = _cfg(R, n_q_heads=hkv * group, n_kv_heads=hkv)
    E = 0.3 * rng.standard_normal((cfg.vocab, cfg.hidden))
    layers = [_layer(R, cfg, rng) for _ in range(n_layers)]
    fn = 1 + 0.1 * rng.standard_normal(cfg.hidden)
    ids = rng.integers(0, cfg.vocab, T0 + n_dec)
    full, _ = R.stack_forward(ids, E, layers, fn, cfg)
    _, kv = R.stack_forward(ids[:T0], E, layers, fn, cfg)
    caches = [(k, v, np.arange(T0)) for (k, v) in kv]
    for s in range(n_dec):
        pos = T0 + s
        dec, new = R.stack_forward(ids[pos:pos + 1], E, layers, fn, cfg, positions=np.array([pos]), caches=caches)
        np.testing.assert_allclose(dec[0], full[pos], rtol=1e-10, atol=1e-11)
        caches = [(np.concatenate([ck, k]), np.concatenate([cv, v]), np.append(cp, pos))
                  for (ck, cv, cp), (k, v) in zip(caches, new)]
