"""GPU edge cases: single-token prefill, device-side capacity and id checks, MoE
routing extremes (top-1 without renormalisation, every expert selected)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle.qwen3_ref as R  # noqa: E402
import qwen3_synth as synth  # noqa: E402
from helpers import (LAYER_MAX_ABS, LAYER_REL_FROB, Layer, Tensor, assert_device_ok, from_gpu_bf16,  # noqa: E402
                     kv_cache, max_abs, oracle_config, rel_frob, rope_gpu, workspace)


@pytest.fixture(scope="module")
def q3():
    import qwen3_decoder_block_b200 as m
    return m


def test_prefill_single_token(q3):
    """T = 1 per sequence, one sequence on an empty cache and one after 700 cached tokens."""
    cfg = q3.config_qwen3_0_6b()
    seed, B, T, starts = 1010, 2, 1, [0, 700]
    s_max = max(starts) + T + 3
    L = Layer(cfg, seed)
    x = Tensor(seed, synth.TID_X, (B * T, cfg.hidden))
    pk = Tensor(seed, 901, (B, cfg.n_kv_heads, s_max, cfg.head_dim))
    pv = Tensor(seed, 902, (B, cfg.n_kv_heads, s_max, cfg.head_dim))
    k, v, kv = kv_cache(cfg, B, s_max)
    for b in range(B):
        k[b, :, :starts[b]] = pk.gpu[b, :, :starts[b]]
        v[b, :, :starts[b]] = pv.gpu[b, :, :starts[b]]
    xg = x.gpu.clone()
    q3.block_prefill(cfg, L.c, xg, B, T, torch.tensor(starts, dtype=torch.int32, device="cuda"), kv,
                     rope_gpu(cfg), workspace(cfg, q3.OP_BLOCK_PREFILL, B, T, s_max))
    assert_device_ok()
    oc = oracle_config(cfg)
    got = from_gpu_bf16(xg)
    for b in range(B):
        ref, _, _ = R.block_forward(x.f[b:b + 1], L.oracle(), oc, np.array([starts[b]]),
                                    pk.f[b][:, :starts[b]].transpose(1, 0, 2),
                                    pv.f[b][:, :starts[b]].transpose(1, 0, 2), np.arange(starts[b]))
        assert rel_frob(got[b:b + 1], ref) <= LAYER_REL_FROB and max_abs(got[b:b + 1], ref) <= LAYER_MAX_ABS


def test_prefill_past_the_cache_is_reported_by_the_device(q3):
    """Start positions live on the device, so a prefill that runs past s_max is caught
    there: the kernels skip the out-of-range cache writes and record ECAPACITY, and the
    context stays usable."""
    cfg = q3.config_qwen3_0_6b()
    seed, B, T, s_max = 1011, 1, 16, 20
    L = Layer(cfg, seed)
    x = Tensor(seed, synth.TID_X, (B * T, cfg.hidden))
    k, v, kv = kv_cache(cfg, B, s_max)
    xg = x.gpu.clone()
    q3.block_prefill(cfg, L.c, xg, B, T, torch.tensor([10], dtype=torch.int32, device="cuda"), kv, rope_gpu(cfg),
                     workspace(cfg, q3.OP_BLOCK_PREFILL, B, T, s_max))
    assert q3.check_device_error() == q3.ECAPACITY
    # positions 20..25 were not written: they would land in rows 0..5 of the next
    # group's slab, and rows 0..9 of every group stay unwritten
    assert torch.isnan(k[0, :, :10].float()).all() and torch.isnan(v[0, :, :10].float()).all()
    # the error word was cleared and the next call runs normally
    xg2 = x.gpu.clone()
    q3.block_prefill(cfg, L.c, xg2, B, T, torch.tensor([0], dtype=torch.int32, device="cuda"), kv, rope_gpu(cfg),
                     workspace(cfg, q3.OP_BLOCK_PREFILL, B, T, s_max))
    assert_device_ok()
    assert np.isfinite(from_gpu_bf16(xg2)).all()


def test_decode_past_the_cache_is_reported_by_the_device(q3):
    cfg = q3.config_qwen3_0_6b()
    seed, B, s_max = 1012, 2, 64
    L = Layer(cfg, seed)
    x = Tensor(seed, synth.TID_X, (B, cfg.hidden))
    k, v, kv = kv_cache(cfg, B, s_max)
    k.zero_()
    v.zero_()
    lens = torch.tensor([10, s_max], dtype=torch.int32, device="cuda")  # sequence 1 has no free slot
    q3.block_decode(cfg, L.c, x.gpu.clone(), B, lens, kv, rope_gpu(cfg),
                    workspace(cfg, q3.OP_BLOCK_DECODE, B, 1, s_max))
    assert q3.check_device_error() == q3.ECAPACITY
    assert_device_ok()


def test_embed_rejects_out_of_range_ids_on_the_device(q3):
    V, H = 1000, 1024
    E = Tensor(1013, 81, (V, H), 0.0, 0.02)
    ids = torch.tensor([3, V, 7], dtype=torch.int32, device="cuda")
    out = torch.zeros((3, H), dtype=torch.float32, device="cuda")
    q3.op_embed(ids, 3, E.gpu, V, H, out)
    assert q3.check_device_error() == q3.EINVAL
    np.testing.assert_array_equal(out[0].cpu().double().numpy(), E.f[3])
    np.testing.assert_array_equal(out[2].cpu().double().numpy(), E.f[7])


def _moe_case(q3, cfg, seed, T):
    B, s_max = 1, T
    L = Layer(cfg, seed, moe=True, dense=False)
    x = Tensor(seed, synth.TID_X, (B * T, cfg.hidden))
    k, v, kv = kv_cache(cfg, B, s_max)
    xg = x.gpu.clone()
    kk = cfg.top_k
    idx = torch.empty((B * T, kk), dtype=torch.int32, device="cuda")
    w = torch.empty((B * T, kk), dtype=torch.float32, device="cuda")
    off = torch.empty(cfg.n_experts + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(B * T * kk, dtype=torch.int32, device="cuda")
    q3.moe_block(cfg, L.c, xg, B, T, torch.zeros(B, dtype=torch.int32, device="cuda"), kv, rope_gpu(cfg),
                 workspace(cfg, q3.OP_MOE_BLOCK, B, T, s_max), idx, w, off, perm)
    assert_device_ok()
    ref, _, _, (ridx, rw, rp, margin) = R.moe_block_forward(x.f, L.oracle(), oracle_config(cfg), np.arange(T))
    return from_gpu_bf16(xg), ref, idx.cpu().numpy(), w.cpu().numpy(), off.cpu().numpy(), ridx, rw, margin


def test_moe_top1_without_renormalisation(q3):
    """Top-1 routing weighted by the raw softmax probability (the two-expert form of the
    pages' MoE notebook is this setting)."""
    cfg = q3.make_config(hidden=512, n_q_heads=8, n_kv_heads=2, n_experts=32, top_k=1, moe_intermediate=128,
                         norm_topk_prob=0)
    got, ref, gi, gw, off, ridx, rw, margin = _moe_case(q3, cfg, 1014, 64)
    assert rel_frob(got, ref) <= LAYER_REL_FROB and max_abs(got, ref) <= LAYER_MAX_ABS
    sure = margin > 1e-3
    np.testing.assert_array_equal(gi[sure], ridx[sure])
    assert np.all(gw < 1.0) and np.all(gw > 0.0)  # raw probabilities, not renormalised to 1
    np.testing.assert_allclose(gw[sure], rw[sure], rtol=1e-2, atol=1e-3)
    assert off[0] == 0 and off[-1] == 64 and np.all(np.diff(off) >= 0)


def test_moe_every_expert_selected(q3):
    """top_k = n_experts: every token visits every expert; with renormalisation the
    weights are the full softmax and each expert gets every token."""
    E = 32
    cfg = q3.make_config(hidden=512, n_q_heads=8, n_kv_heads=2, n_experts=E, top_k=E, moe_intermediate=128)
    T = 40
    got, ref, gi, gw, off, ridx, rw, margin = _moe_case(q3, cfg, 1015, T)
    assert rel_frob(got, ref) <= LAYER_REL_FROB and max_abs(got, ref) <= LAYER_MAX_ABS
    np.testing.assert_array_equal(np.sort(gi, axis=1), np.tile(np.arange(E), (T, 1)))
    np.testing.assert_allclose(gw.sum(axis=1), 1.0, rtol=1e-5)
    np.testing.assert_array_equal(off, np.arange(E + 1) * T)


def test_moe_block_decode_step(q3):
    """One decode step per sequence through the MoE block (T = 1 at position cache_len[b],
    attending the cached positions and itself), against the oracle composed from its
    attention half with the cache, the router and the expert FFN."""
    cfg = q3.make_config(hidden=512, n_q_heads=8, n_kv_heads=2, n_experts=32, top_k=4, moe_intermediate=128)
    seed, lens = 1017, [0, 5, 130, 300]
    B, s_max = len(lens), max(lens) + 4
    D, hkv = cfg.head_dim, cfg.n_kv_heads
    L = Layer(cfg, seed, moe=True, dense=False)
    x = Tensor(seed, synth.TID_X, (B, cfg.hidden))
    pk = Tensor(seed, 905, (B, hkv, s_max, D))
    pv = Tensor(seed, 906, (B, hkv, s_max, D))
    k, v, kv = kv_cache(cfg, B, s_max)
    for b in range(B):
        k[b, :, :lens[b]] = pk.gpu[b, :, :lens[b]]
        v[b, :, :lens[b]] = pv.gpu[b, :, :lens[b]]
    xg = x.gpu.clone()
    kk = cfg.top_k
    idx = torch.empty((B, kk), dtype=torch.int32, device="cuda")
    w = torch.empty((B, kk), dtype=torch.float32, device="cuda")
    q3.moe_block(cfg, L.c, xg, B, 1, torch.tensor(lens, dtype=torch.int32, device="cuda"), kv, rope_gpu(cfg),
                 workspace(cfg, q3.OP_MOE_BLOCK, B, 1, s_max), idx, w)
    assert_device_ok()
    got, gi = from_gpu_bf16(xg), idx.cpu().numpy()
    oc, Lo = oracle_config(cfg), L.oracle()
    for b in range(B):
        x1, _, _ = R.attention_half(x.f[b:b + 1], Lo, oc, np.array([lens[b]]),
                                    pk.f[b][:, :lens[b]].transpose(1, 0, 2), pv.f[b][:, :lens[b]].transpose(1, 0, 2),
                                    np.arange(lens[b]))
        ref, (ridx, rw, _, margin) = R.moe_ffn_half(x1, Lo, oc)
        assert rel_frob(got[b:b + 1], ref) <= LAYER_REL_FROB and max_abs(got[b:b + 1], ref) <= LAYER_MAX_ABS
        if margin[0] > 1e-3:
            np.testing.assert_array_equal(np.sort(gi[b]), np.sort(ridx[0]))
