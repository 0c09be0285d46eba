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
    import qwen3_synth as synth
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
    ("intermediate", 3000, -2), ("vocab", 151937, -2), ("n_q_heads", 0, -2), ("gemm_f16", 2, -2),
    ("gemm_f16", -1, -2)])
def test_validate_config_rejects(q3, field, value, status):
    c = q3.config_qwen3_0_6b()
    setattr(c, field, value)
    assert q3.validate_config(c) == status
    assert q3.lib.qwen3_last_error().decode()


@pytest.mark.parametrize("hq,hkv,ok", [(16, 16, True), (16, 8, True), (32, 8, True), (64, 8, True), (16, 1, True),
                                       (32, 1, False), (128, 1, False), (24, 8, False), (40, 8, False)])
def test_gqa_group_sizes(q3, hq, hkv, ok):
    """Query heads per KV group: 1, 2, 4, 8 or 16 (all the attention kernels handle);
    32 or more, and groups that do not divide a 128-row tile (3, or 5 as in 40/8), are
    rejected before anything runs."""
    c = q3.config_qwen3_0_6b()
    c.n_q_heads, c.n_kv_heads = hq, hkv
    st = q3.validate_config(c)
    assert (st == 0) if ok else (st == q3.ESHAPE), (hq, hkv, st)


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
    assert d >= (64 * 16 + 256 * 16) * 130 * 4  # decode partial slots: (rows + CTAs) x heads of a group
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
    st = q3.lib.qwen3_op_gemm(8, 1024, 16, 1024, 32, 1024, 16, 1024, 1024, 0, None, 0, 0, 0, -1, 0, None, 0, None)
    assert st == q3.EALIGN
    st = q3.lib.qwen3_op_gemm(16, 1024, 32, 1024, 48, 1024, 16, 1000, 1024, 0, None, 0, 0, 0, -1, 0, None, 0, None)
    assert st == q3.ESHAPE  # N % 32
    st = q3.lib.qwen3_op_rmsnorm(16, 0, 1000, 32, 48, 1000, 4, 1000, 1e-6, 0, None)
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


def _arena_layout(cfg, moe):
    """Byte offsets of one layer's members laid out back to back in one arena, sizes
    from the config (what a caller packing all weights into one buffer computes)."""
    H, D, hq, hkv = cfg.hidden, cfg.head_dim, cfg.n_q_heads, cfg.n_kv_heads
    sizes = dict(in_norm=H, w_qkv=(hq + 2 * hkv) * D * H, q_norm=D, k_norm=D, w_o=H * hq * D, post_norm=H)
    if moe:
        E, Im = cfg.n_experts, cfg.moe_intermediate
        sizes.update(router=E * H, moe_gate_up=E * 2 * Im * H, moe_down=E * H * Im)
    else:
        I = cfg.intermediate
        sizes.update(w_gate_up=2 * I * H, w_down=H * I)
    base, ptrs = 1 << 32, {}
    for name, n in sizes.items():
        ptrs[name] = base
        base += (2 * n + 255) // 256 * 256
    return ptrs, {k: 2 * v for k, v in sizes.items()}


def _status(q3, cfg, ptrs, kind):
    st = q3.lib.qwen3_check_layer_weights(ctypes.byref(cfg), ctypes.byref(q3.layer_weights(**ptrs)), kind)
    return st, q3.lib.qwen3_last_error().decode()


def test_layer_weights_two_way_check_accepts_correct_layouts(q3):
    cfg = q3.config_qwen3_0_6b()
    ptrs, _ = _arena_layout(cfg, moe=False)
    assert _status(q3, cfg, ptrs, q3.LAYER_DENSE) == (0, "")
    q3.check_layer_weights(cfg, q3.layer_weights(**ptrs))
    # one read-only buffer for both per-head norms (same pointer, same size) is allowed
    ptrs["k_norm"] = ptrs["q_norm"]
    assert _status(q3, cfg, ptrs, q3.LAYER_DENSE)[0] == 0
    moe = q3.make_config(hidden=2048, n_q_heads=32, n_kv_heads=4, n_experts=128, top_k=8, moe_intermediate=768)
    mptrs, _ = _arena_layout(moe, moe=True)
    assert _status(q3, moe, mptrs, q3.LAYER_MOE)[0] == 0


def test_layer_weights_forward_direction_every_read_member_present_and_aligned(q3):
    cfg = q3.config_qwen3_0_6b()
    ptrs, _ = _arena_layout(cfg, moe=False)
    for name in ptrs:
        bad = dict(ptrs)
        del bad[name]
        st, msg = _status(q3, cfg, bad, q3.LAYER_DENSE)
        assert st == q3.EINVAL and f"weights.{name} is NULL" in msg
    bad = dict(ptrs, w_o=ptrs["w_o"] + 8)
    st, msg = _status(q3, cfg, bad, q3.LAYER_DENSE)
    assert st == q3.EALIGN and "weights.w_o" in msg


def test_layer_weights_reverse_direction_no_member_of_the_other_kind(q3):
    cfg = q3.make_config(hidden=1024, n_q_heads=16, n_kv_heads=8, n_experts=32, top_k=4, moe_intermediate=256)
    dense, _ = _arena_layout(cfg, moe=False)
    moe, _ = _arena_layout(cfg, moe=True)
    far = 1 << 40
    st, msg = _status(q3, cfg, dict(dense, router=far), q3.LAYER_DENSE)
    assert st == q3.ESHAPE and "weights.router is set but a dense layer" in msg
    st, msg = _status(q3, cfg, dict(moe, w_down=far), q3.LAYER_MOE)
    assert st == q3.ESHAPE and "weights.w_down is set but a MoE layer" in msg
    # a dense layer checked as MoE: its FFN members are ones a MoE layer does not read,
    # and without them the expert members are missing
    st, msg = _status(q3, cfg, dense, q3.LAYER_MOE)
    assert st == q3.ESHAPE and "weights.w_gate_up is set but a MoE layer" in msg
    st, msg = _status(q3, cfg, {k: v for k, v in dense.items() if k not in ("w_gate_up", "w_down")}, q3.LAYER_MOE)
    assert st == q3.EINVAL and "weights.router is NULL" in msg
    st, _ = _status(q3, cfg, dense, 7)
    assert st == q3.EINVAL


def test_layer_weights_overlap_from_a_wrong_dimension_is_reported(q3):
    """An arena laid out with n_kv_heads taken as 4 instead of 8: w_qkv is then larger
    than the space left for it and runs into q_norm, the next member (the raw-pointer
    form of the pages' shape mismatch)."""
    cfg = q3.config_qwen3_0_6b()
    wrong = q3.config_qwen3_0_6b()
    wrong.n_kv_heads = 4
    ptrs, _ = _arena_layout(wrong, moe=False)
    st, msg = _status(q3, cfg, ptrs, q3.LAYER_DENSE)
    assert st == q3.EINVAL and "weights.w_qkv" in msg and "overlaps weights.q_norm" in msg
    # the same pointer for two members of different sizes is an overlap too
    good, _ = _arena_layout(cfg, moe=False)
    st, msg = _status(q3, cfg, dict(good, post_norm=good["w_o"]), q3.LAYER_DENSE)
    assert st == q3.EINVAL and "overlaps" in msg
    with pytest.raises(q3.Qwen3Error):
        q3.check_layer_weights(cfg, q3.layer_weights(**dict(good, post_norm=good["w_o"])))


def test_empty_batches_are_rejected_before_any_launch(q3):
    """B = 0 or T = 0: QWEN3_EINVAL from the host checks (nothing reaches a device, so
    this runs without a GPU), and no workspace."""
    c = q3.config_qwen3_0_6b()
    ptrs, _ = _arena_layout(c, moe=False)
    w = q3.layer_weights(**ptrs)
    fake = 1 << 44
    kv = q3.KVLayer(fake, fake + (1 << 36), 64)
    for B, T in [(0, 16), (2, 0), (-1, 4)]:
        st = q3.lib.qwen3_block_prefill(ctypes.byref(c), ctypes.byref(w), fake, B, T, fake, ctypes.byref(kv), fake,
                                        fake, 1 << 30, None)
        assert st == q3.EINVAL and "must be positive" in q3.lib.qwen3_last_error().decode(), (B, T)
        assert q3.workspace_size(c, q3.OP_BLOCK_PREFILL, B, T, 64) == 0
    st = q3.lib.qwen3_block_decode(ctypes.byref(c), ctypes.byref(w), fake, 0, fake, ctypes.byref(kv), fake, fake,
                                   1 << 30, None)
    assert st == q3.EINVAL
    kvs = (q3.KVLayer * c.n_layers)(*[q3.KVLayer(fake, fake + (1 << 36), 64)] * c.n_layers)
    layers = (q3.LayerWeights * c.n_layers)(*[w] * c.n_layers)
    st = q3.lib.qwen3_stack_forward(ctypes.byref(c), fake, layers, fake, fake, 0, 16, q3.MODE_PREFILL, fake, kvs,
                                    fake, fake, 0, fake, 1 << 30, None)
    assert st == q3.EINVAL
    st = q3.lib.qwen3_op_argmax(fake, 151936, 0, 151936, fake, 1, None)
    assert st == q3.EINVAL


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "qwen3blk.h"
int main(void) {
  qwen3_config c;
  if (qwen3_config_qwen3_0_6b(&c) != QWEN3_OK || c.hidden != 1024 || c.n_layers != 28) return 1;
  if (qwen3_validate_config(&c) != QWEN3_OK) return 2;
  if (qwen3_workspace_size(&c, QWEN3_OP_BLOCK_PREFILL, 1, 16, 64) == 0) return 3;
  qwen3_layer_weights w;
  memset(&w, 0, sizeof w);
  if (qwen3_check_layer_weights(&c, &w, QWEN3_LAYER_DENSE) != QWEN3_EINVAL) return 4;
  if (strstr(qwen3_last_error(), "in_norm") == NULL) return 5;
  c.head_dim = 64;
  if (qwen3_validate_config(&c) != QWEN3_ESHAPE) return 6;
  printf("%s\n", qwen3_status_string(QWEN3_ESHAPE));
  return 0;
}
"""


def test_header_is_plain_c_and_links(q3):
    """A C11 program (no C++) includes the header, links against the library and calls
    its host-only entry points."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(q3.LIB_PATH)
    src, exe = os.path.join(libdir, "abi_c_test.c"), os.path.join(libdir, "abi_c_test")
    with open(src, "w") as f:
        f.write(C_PROGRAM)
    cmd = [gcc, "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"), src,
           "-L", libdir, "-l:libqwen3blk.so", f"-Wl,-rpath,{libdir}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.strip() != ""


@pytest.mark.parametrize("ldo", [0, -2048, 2040, 2052, 1 << 3])
def test_decode_attention_rejects_bad_output_stride_before_launch(q3, ldo):
    """The decode attention writes o[b * ldo + h * 128 + d]: an ldo below n_q_heads * 128,
    not a multiple of 8, zero or negative is rejected on the host (QWEN3_EALIGN) by both
    entry points, before anything could be launched."""
    c = q3.config_qwen3_0_6b()
    fake = 1 << 44
    kv = q3.KVLayer(fake, fake + (1 << 36), 4224)
    st = q3.lib.qwen3_op_attention_decode(ctypes.byref(c), fake, 4096, 64, fake, ctypes.byref(kv), fake, ldo, fake,
                                          1 << 30, None)
    assert st == q3.EALIGN and "ldo" in q3.lib.qwen3_last_error().decode(), st
    st = q3.lib.qwen3_op_attention_decode_noalloc(ctypes.byref(c), fake, 4096, 64, fake, ctypes.byref(kv), fake, ldo,
                                                  None)
    assert st == q3.EALIGN and "ldo" in q3.lib.qwen3_last_error().decode(), st


def test_operand_mode_arguments_checked_before_launch(q3):
    """The gemm_f16 mode's host-side checks: the default configuration keeps the pages'
    bf16 operands; op_gemm takes ab_f16 0 or 1 only; the conversion refuses partly
    overlapping buffers (in place is allowed) and runs nothing on bad arguments."""
    c = q3.config_qwen3_0_6b()
    assert c.gemm_f16 == 0
    c.gemm_f16 = 1
    assert q3.validate_config(c) == 0
    st = q3.lib.qwen3_op_gemm(16, 1024, 32, 1024, 48, 1024, 16, 1024, 1024, 0, None, 0, 0, 0, -1, 2, None, 0, None)
    assert st == q3.EINVAL and "ab_f16" in q3.lib.qwen3_last_error().decode()
    base = 1 << 40
    assert q3.lib.qwen3_convert_to_f16(base, base + 16, 1024, None) == q3.EINVAL
    assert "overlap" in q3.lib.qwen3_last_error().decode()
    assert q3.lib.qwen3_convert_to_f16(base, base + 8, 4, None) == q3.EALIGN
    assert q3.lib.qwen3_convert_to_f16(None, base, 4, None) == q3.EINVAL
