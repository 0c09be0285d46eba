"""The algorithmic units behind the bench line's roofline figures (no GPU).

bench.py divides algorithmic FLOPs or bytes by measured time. These checks restate the
counts from the Qwen3-0.6B configuration in closed form, independently of bench.py's
own formulas, and compare both with the figures the design notes quote.
"""
import os
import sys
from types import SimpleNamespace

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

# "从零实现 Qwen3：拆解 mini-qwen3 的 0.6B Dense 架构", config table: hidden 1024,
# intermediate 3072, 16 query heads and 8 KV heads of 128 dims, 28 layers, vocabulary 151936
CFG = SimpleNamespace(hidden=1024, intermediate=3072, n_q_heads=16, n_kv_heads=8, head_dim=128, n_layers=28,
                      vocab=151936)


def linear_params_per_layer(c):
    """Weights of one layer's projections: QKV, o_proj, gate and up, down."""
    q = c.hidden * c.n_q_heads * c.head_dim
    kv = 2 * c.hidden * c.n_kv_heads * c.head_dim
    o = c.n_q_heads * c.head_dim * c.hidden
    ffn = 3 * c.hidden * c.intermediate
    return q + kv + o + ffn


def test_gemm_flops_are_two_per_weight_and_token():
    layers, lm = bench.gemm_flops_per_token(CFG)
    assert linear_params_per_layer(CFG) == 15_728_640
    assert layers == 2 * CFG.n_layers * linear_params_per_layer(CFG)
    assert lm == 2 * CFG.hidden * CFG.vocab  # the tied LM head: one product per vocabulary row
    # the B4 x T2048 prefill step: 9.76 TFLOP of projections and LM head
    step = 4 * 2048 * (layers + lm)
    assert abs(step / 1e12 - 9.76) < 0.005


def test_prefill_attention_flops_count_visible_pairs():
    def brute_pairs(T):
        return sum(1 for i in range(T) for j in range(T) if j <= i)

    for T in (1, 2, 7, 64):
        assert bench.attention_prefill_flops(CFG, 1, T) == CFG.n_layers * 4 * CFG.head_dim * CFG.n_q_heads * \
            brute_pairs(T)
    per_layer = bench.attention_prefill_flops(CFG, 4, 2048) / CFG.n_layers
    assert abs(per_layer / 1e9 - 68.75) < 0.01  # B4 x T2048: 68.75 GFLOP per layer
    assert abs(bench.attention_prefill_flops(CFG, 4, 2048) / 1e12 - 1.925) < 0.001
    long_layer = bench.attention_prefill_flops(CFG, 1, 32768) / CFG.n_layers
    assert abs(long_layer / 1e9 - 4398) < 1.0  # B1 x T32768: 4398 GFLOP per layer


def test_decode_attention_bytes_per_layer():
    """K and V of every visible position, bf16: 64 sequences x 8 KV heads x 4097
    positions x 128 dims x 2 tensors x 2 bytes = 1.074 GB per layer."""
    B, L = 64, 4096
    per_layer = B * CFG.n_kv_heads * (L + 1) * CFG.head_dim * 2 * 2
    assert per_layer == 1_074_003_968
    # the bench's traffic ratio divides measured DRAM bytes by exactly this figure
    assert abs(bench.DECODE_ATTN_TRAFFIC_RATIO * per_layer - per_layer) / per_layer < 0.02


def test_summarize_profile_shares():
    recs = [("a", 1.0), ("b", 3.0), ("a", 1.0), ("b", 3.0)]
    kern, per_step = bench.summarize_profile(recs, 2)
    assert list(kern) == ["b", "a"]
    assert kern["a"] == {"launches_per_step": 1.0, "ms_per_step": 1.0, "share": 0.25}
    assert kern["b"]["share"] == 0.75 and per_step == 4.0
