"""The decode-attention entry point that allocates nothing.

Some callers cannot allocate device memory (an application held to a fixed memory
budget, a plugin handed tensors but no allocator or workspace). For them the
library offers qwen3_op_attention_decode_noalloc, whose scratch is a static
device array of the library. This test calls it through the C ABI twice in a row
and checks each result against the workspace-taking qwen3_op_attention_decode, on
the decode workload's shapes (B 64, 4097 visible positions). The file is named so
that pytest collects it last.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from helpers import Tensor, assert_device_ok, from_gpu_bf16, kv_cache, workspace  # noqa: E402


def test_noalloc_decode_matches_workspace_decode_twice():
    import qwen3_decoder_block_b200 as q3
    cfg = q3.config_qwen3_0_6b()
    hq, hkv, D = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    B, L0 = 64, 4096
    s_max = L0 + 128
    k, v, kv = kv_cache(cfg, B, s_max)
    for step, seed in enumerate((501, 502)):
        lens = [L0 + step - (b % 7) * 300 for b in range(B)]  # ragged lengths
        kall = Tensor(seed, 1, (B, hkv, s_max, D))
        vall = Tensor(seed, 2, (B, hkv, s_max, D))
        k.copy_(kall.gpu)
        v.copy_(vall.gpu)
        qkv = Tensor(seed, 3, (B, (hq + 2 * hkv) * D))
        cl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        o_ref = torch.empty((B, hq * D), dtype=torch.bfloat16, device="cuda")
        o_new = torch.full((B, hq * D), float("nan"), dtype=torch.bfloat16, device="cuda")
        q3.op_attention_decode(cfg, qkv.gpu, B, cl, kv, o_ref, workspace(cfg, q3.OP_BLOCK_DECODE, B, 1, s_max))
        q3.op_attention_decode_noalloc(cfg, qkv.gpu, B, cl, kv, o_new)
        assert_device_ok()
        ref, got = from_gpu_bf16(o_ref), from_gpu_bf16(o_new)
        assert np.isfinite(got).all()
        # the same kernels with the same tile ranges and merge order: only the scratch's
        # address differs, so the outputs are identical bit for bit
        np.testing.assert_array_equal(o_new.view(torch.int16).cpu().numpy(), o_ref.view(torch.int16).cpu().numpy())


def test_noalloc_rejects_sizes_beyond_the_static_scratch():
    """The scratch of a call holds (B * Hkv + 256) partial slots of G heads x 130 floats,
    the tile plan (B + 1 ints, padded to 4) and B * Hkv merge counters. With 16 query
    heads that is 12,583,536 bytes for B 1251, above the 12 MiB static array, so the call
    is refused before launch; B 1250 (12,575,184 bytes) fits and runs. The cache is
    really allocated (s_max 8), so that the arguments describe valid memory whatever the
    order of the checks."""
    import qwen3_decoder_block_b200 as q3
    cfg = q3.config_qwen3_0_6b()
    B, s_max = 1251, 8
    k, v, kv = kv_cache(cfg, B, s_max)
    qkv = torch.zeros((B, 4096), dtype=torch.bfloat16, device="cuda")
    o = torch.zeros((B, 2048), dtype=torch.bfloat16, device="cuda")
    cl = torch.zeros(B, dtype=torch.int32, device="cuda")
    with pytest.raises(q3.Qwen3Error) as e:
        q3.op_attention_decode_noalloc(cfg, qkv, B, cl, kv, o)
    assert e.value.status == q3.EWORKSPACE
    assert "static scratch" in str(e.value)
    # one sequence less fits
    B2 = B - 1
    k.zero_()
    v.zero_()
    o.fill_(float("nan"))
    q3.op_attention_decode_noalloc(cfg, qkv[:B2], B2, cl[:B2], kv, o[:B2])
    assert_device_ok()
    assert bool((o[:B2] == 0).all())  # one visible key whose value row is zero
    assert bool(torch.isnan(o[B2:]).all())  # the refused row count is not exceeded
    del k, v
