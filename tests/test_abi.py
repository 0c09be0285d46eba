"""CPU-only checks of the boundary: the library loads, exports every symbol the
header declares, and host-side validation rejects bad arguments before any
launch (no GPU needed for these paths)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qwen3blk.h")


@pytest.fixture(scope="module")
def q3():
    import __graft_entry__
    __graft_entry__.build()
    import qwen3_decoder_block_b200 as m
    return m


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qwen3_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_four_block_calls():
    names = declared_functions()
    for n in ("qwen3_block_prefill", "qwen3_block_decode", "qwen3_moe_block", "qwen3_stack_forward"):
        assert n in names


def test_every_declared_symbol_is_exported(q3):
    lib = ctypes.CDLL(q3.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_every_declared_symbol(q3):
    assert set(declared_functions()) == set(q3.EXPORTED)


def test_synth_library_exports(q3):
    from qwen3_decoder_block_b200 import synth
    lib = synth.native()
    for n in ("qwen3synth_normal_bf16_host", "qwen3synth_normal_bf16_device", "qwen3synth_uniform_int_host",
              "qwen3synth_uniform_int_device"):
        assert hasattr(lib, n)


def test_default_config_is_qwen3_0_6b(q3):
    c = q3.config_qwen3_0_6b()
    assert (c.hidden, c.n_q_heads, c.n_kv_heads, c.head_dim, c.intermediate, c.vocab, c.n_layers, c.max_pos) == \
        (1024, 16, 8, 128, 3072, 151936, 28, 40960)
    assert abs(c.rope_theta - 1e6) == 0 and abs(c.rms_eps - 1e-6) < 1e-12
    assert q3.validate_config(c) == 0


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 64, -2), ("n_kv_heads", 3, -2), ("hidden", 1000, -2), ("hidden", 4096, -2),
    ("intermediate", 3000, -2), ("vocab", 151937, -2), ("n_q_heads", 0, -2)])
def test_validate_config_rejects(q3, field, value, status):
    c = q3.config_qwen3_0_6b()
    setattr(c, field, value)
    assert q3.validate_config(c) == status
    assert q3.lib.qwen3_last_error().decode()


def test_moe_config_checks(q3):
    c = q3.make_config(hidden=2048, n_q_heads=32, n_kv_heads=4, n_experts=128, top_k=8, moe_intermediate=768)
    assert q3.validate_config(c) == 0
    c.top_k = 129
    assert q3.validate_config(c) == -2
    c.top_k = 8
    c.moe_intermediate = 700
    assert q3.validate_config(c) == -2


def test_workspace_sizes_monotone(q3):
    c = q3.config_qwen3_0_6b()
    a = q3.workspace_size(c, q3.OP_BLOCK_PREFILL, 1, 16, 64)
    b = q3.workspace_size(c, q3.OP_BLOCK_PREFILL, 4, 2048, 2048)
    assert 0 < a < b
    # activations alone: h, qkv, o (bf16) + x1 (fp32) + act (bf16) for 8192 rows
    M = 4 * 2048
    assert b >= M * (1024 * 2 + 4096 * 2 + 2048 * 2 + 1024 * 4 + 3072 * 2)
    d = q3.workspace_size(c, q3.OP_BLOCK_DECODE, 64, 1, 4224)
    assert d >= 64 * 16 * 17 * 130 * 4  # split-KV partials (256-key chunks)
    assert q3.workspace_size(c, 99, 1, 1, 1) == 0
    assert q3.workspace_size(c, q3.OP_BLOCK_PREFILL, 0, 1, 1) == 0


def test_null_and_misaligned_arguments_rejected_without_launch(q3):
    c = q3.config_qwen3_0_6b()
    w = q3.LayerWeights()
    kv = q3.KVLayer(None, None, 16)
    st = q3.lib.qwen3_block_prefill(ctypes.byref(c), ctypes.byref(w), None, 1, 16, None, ctypes.byref(kv), None,
                                    None, 0, None)
    assert st == q3.EINVAL
    assert "NULL" in q3.lib.qwen3_last_error().decode()
    st = q3.lib.qwen3_op_gemm(8, 1024, 16, 1024, 32, 1024, 16, 1024, 1024, 0, None, 0, 0, 0, -1, None, 0, None)
    assert st == q3.EALIGN
    st = q3.lib.qwen3_op_gemm(16, 1024, 32, 1024, 48, 1024, 16, 1000, 1024, 0, None, 0, 0, 0, -1, None, 0, None)
    assert st == q3.ESHAPE  # N % 32
    st = q3.lib.qwen3_op_rmsnorm(16, 0, 1000, 32, 48, 1000, 4, 1000, 1e-6, None)
    assert st == q3.ESHAPE


def test_capacity_checked_on_host(q3):
    c = q3.config_qwen3_0_6b()
    kv = q3.KVLayer(16, 32, 8)
    st = q3.lib.qwen3_op_qk_norm_rope(ctypes.byref(c), 16, 4096, 1, 9, 16, 16, 16, ctypes.byref(kv), 16, None)
    assert st == q3.ECAPACITY


def test_workspace_too_small_rejected(q3):
    c = q3.config_qwen3_0_6b()
    fake = 1 << 20
    w = q3.layer_weights(in_norm=fake, w_qkv=fake, q_norm=fake, k_norm=fake, w_o=fake, post_norm=fake,
                         w_gate_up=fake, w_down=fake)
    kv = q3.KVLayer(fake, fake, 64)
    st = q3.lib.qwen3_block_prefill(ctypes.byref(c), ctypes.byref(w), fake, 1, 16, fake, ctypes.byref(kv), fake,
                                    fake, 1024, None)
    assert st == q3.EWORKSPACE
