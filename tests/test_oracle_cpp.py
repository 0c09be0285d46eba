"""The fp64 C++ oracle (oracle/qwen3_ref.cpp, through oracle/cpp_ref.py): every pin the
numpy oracle answers to also holds for it, and the two oracles agree to about 1e-12 on
small shapes of every function (CPU only)."""
import numpy as np
import pytest

import oracle.cpp_ref as C
import oracle.qwen3_ref as R
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("name", sorted(ALL_PINS))
def test_pin_holds_for_the_cpp_oracle(name):
    ALL_PINS[name](C)


def _cfg(mod, **kw):
    base = dict(hidden=64, n_q_heads=4, n_kv_heads=2, head_dim=16, intermediate=96, vocab=50, n_layers=2,
                max_pos=4096, rope_theta=1.0e6, rms_eps=1.0e-6)
    base.update(kw)
    return mod.Config(**base)


def _layer(mod, cfg, rng, moe=False):
    H, d, hq, hkv, I = cfg.hidden, cfg.head_dim, cfg.n_q_heads, cfg.n_kv_heads, cfg.intermediate
    kw = dict(in_norm=1 + 0.1 * rng.standard_normal(H), wq=0.2 * rng.standard_normal((hq * d, H)),
              wk=0.2 * rng.standard_normal((hkv * d, H)), wv=0.2 * rng.standard_normal((hkv * d, H)),
              q_norm=1 + 0.1 * rng.standard_normal(d), k_norm=1 + 0.1 * rng.standard_normal(d),
              wo=0.2 * rng.standard_normal((H, hq * d)), post_norm=1 + 0.1 * rng.standard_normal(H))
    if moe:
        E, Im = cfg.n_experts, cfg.moe_intermediate
        kw.update(router=rng.standard_normal((E, H)), gate_up=0.2 * rng.standard_normal((E, 2 * Im, H)),
                  down=0.2 * rng.standard_normal((E, H, Im)))
    else:
        kw.update(w_gate=0.2 * rng.standard_normal((I, H)), w_up=0.2 * rng.standard_normal((I, H)),
                  w_down=0.2 * rng.standard_normal((H, I)))
    return kw


def _close(a, b, rtol=1e-12, atol=1e-13):
    np.testing.assert_allclose(a, b, rtol=rtol, atol=atol)


def test_primitives_agree():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((7, 64))
    w = 1 + 0.1 * rng.standard_normal(64)
    _close(C.rms_norm(x, w, 1e-6), R.rms_norm(x, w, 1e-6))
    u = rng.standard_normal((5, 3, 16))
    pos = np.array([0, 1, 17, 4000, 40959])
    _close(C.rope_rotate_half(u, pos, 1e6), R.rope_rotate_half(u, pos, 1e6))
    _close(C.rope_frequencies(128, 1e6), R.rope_frequencies(128, 1e6))
    z = rng.standard_normal(33) * 5
    _close(C.silu(z), R.silu(z))
    q, k, v = rng.standard_normal((6, 4, 16)), rng.standard_normal((9, 2, 16)), rng.standard_normal((9, 2, 16))
    qp, kp = np.arange(3, 9), np.arange(9)
    np.testing.assert_array_equal(C.causal_allowed(qp, kp), R.causal_allowed(qp, kp))
    _close(C.causal_gqa_attention(q, k, v, qp, kp), R.causal_gqa_attention(q, k, v, qp, kp))
    h = rng.standard_normal((4, 64))
    wg, wu, wd = rng.standard_normal((96, 64)), rng.standard_normal((96, 64)), rng.standard_normal((64, 96))
    _close(C.swiglu_ffn(h, wg, wu, wd), R.swiglu_ffn(h, wg, wu, wd), rtol=1e-11)


def test_block_and_cache_agree():
    rng = np.random.default_rng(2)
    cc, cr = _cfg(C), _cfg(R)
    kw = _layer(R, cr, rng)
    Lc, Lr = C.LayerWeights(**kw), R.LayerWeights(**kw)
    x = rng.standard_normal((11, 64))
    a = C.block_forward(x, Lc, cc, 20 + np.arange(11))
    b = R.block_forward(x, Lr, cr, 20 + np.arange(11))
    for ga, gb in zip(a, b):
        _close(ga, gb, rtol=1e-11, atol=1e-12)
    # with a cache and a row subset
    ck, cv = rng.standard_normal((20, 2, 16)), rng.standard_normal((20, 2, 16))
    rows = [0, 4, 10]
    a = C.block_forward(x, Lc, cc, 20 + np.arange(11), ck, cv, np.arange(20), rows=rows)
    b = R.block_forward(x, Lr, cr, 20 + np.arange(11), ck, cv, np.arange(20), rows=rows)
    for ga, gb in zip(a, b):
        _close(ga, gb, rtol=1e-11, atol=1e-12)


def test_moe_agrees():
    rng = np.random.default_rng(3)
    cc, cr = _cfg(C, n_experts=8, top_k=3, moe_intermediate=12), _cfg(R, n_experts=8, top_k=3, moe_intermediate=12)
    kw = _layer(R, cr, rng, moe=True)
    Lc, Lr = C.LayerWeights(**kw), R.LayerWeights(**kw)
    x = rng.standard_normal((13, 64))
    oc, _, _, rc = C.moe_block_forward(x, Lc, cc, np.arange(13))
    orr, _, _, rr = R.moe_block_forward(x, Lr, cr, np.arange(13))
    _close(oc, orr, rtol=1e-11, atol=1e-12)
    np.testing.assert_array_equal(rc[0], rr[0])
    for a, b in zip(rc[1:], rr[1:]):
        _close(a, b)
    for a, b in zip(C.moe_permutation(rr[0], 8), R.moe_permutation(rr[0], 8)):
        np.testing.assert_array_equal(a, b)


def test_stack_agrees_prefill_and_decode():
    rng = np.random.default_rng(4)
    cc, cr = _cfg(C, n_layers=3), _cfg(R, n_layers=3)
    kws = [_layer(R, cr, rng) for _ in range(3)]
    E = 0.3 * rng.standard_normal((50, 64))
    fn = 1 + 0.1 * rng.standard_normal(64)
    ids = rng.integers(0, 50, 9)
    lc, kvc = C.stack_forward(ids, E, [C.LayerWeights(**k) for k in kws], fn, cc)
    lr, kvr = R.stack_forward(ids, E, [R.LayerWeights(**k) for k in kws], fn, cr)
    _close(lc, lr, rtol=1e-11, atol=1e-12)
    caches = [(k, v, np.arange(9)) for k, v in kvr]
    dc, _ = C.stack_forward(ids[:1], E, [C.LayerWeights(**k) for k in kws], fn, cc, positions=np.array([9]),
                            caches=caches)
    dr, _ = R.stack_forward(ids[:1], E, [R.LayerWeights(**k) for k in kws], fn, cr, positions=np.array([9]),
                            caches=caches)
    _close(dc, dr, rtol=1e-11, atol=1e-12)
    assert C.param_count(C.QWEN3_0_6B, tied=False) == R.param_count(R.QWEN3_0_6B, tied=False)
