"""Error budget of bf16 intermediates in the 28-layer Qwen3-0.6B stack prefill.

Diagnostic script (not collected by pytest; it takes minutes). It answers one
question: how close to the exact (fp64) logits can ANY implementation get that keeps
some intermediate tensors of the block in bf16, as the pages' modules do ("从零实现
Qwen3：拆解 mini-qwen3 的 0.6B Dense 架构", sections RMSNorm, GQA, SwiGLU FFN: every
activation is a bf16 tensor between modules)?

It re-assembles the stack from the oracle's primitives (oracle/qwen3_ref.py) and
rounds a chosen set of intermediates to bf16 (round to nearest even), everything
else in fp64. Rounding points:

    h     RMSNorm output fed to the QKV projection
    qkv   q/k/v projection outputs before QK-norm
    v     value rows (the bf16 cache)
    qk    q and k after QK-norm + RoPE (the bf16 query operand and key cache)
    P     softmax probabilities fed to the P.V product
    o     attention output fed to o_proj
    h2    RMSNorm output fed to gate/up
    act   SwiGLU output fed to down
    hf    final RMSNorm output fed to the LM head

The residual stream stays unrounded (the library keeps it in fp32). Output: the
relative Frobenius error of the logits and the argmax agreement per variant, on one
sequence of the 28-layer prefill workload (random weights of seed 1001, T tokens).

    python tests/bf16_error_budget.py [T]
"""
import os
import sys
import time

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import oracle.qwen3_ref as R  # noqa: E402
from qwen3_decoder_block_b200 import synth  # noqa: E402

SEED = 1001


def to_bf16(x):
    return R.bf16_to_f64(synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32)))


def load(cfg, T):
    H, D, hq, hkv, I = cfg.hidden, cfg.head_dim, cfg.n_q_heads, cfg.n_kv_heads, cfg.intermediate

    def w(tid, shape, mean=0.0, std=synth.W_STD):
        return R.bf16_to_f64(synth.normal_bf16_fast(SEED, tid, shape, mean, std))

    layers = []
    for l in range(cfg.n_layers):
        t = lambda which: synth.layer_tid(l, which)  # noqa: E731
        layers.append(R.LayerWeights(
            in_norm=w(t(synth.L_IN_NORM), (H,), 1.0, 0.1), wq=w(t(synth.L_WQ), (hq * D, H)),
            wk=w(t(synth.L_WK), (hkv * D, H)), wv=w(t(synth.L_WV), (hkv * D, H)),
            q_norm=w(t(synth.L_Q_NORM), (D,), 1.0, 0.1), k_norm=w(t(synth.L_K_NORM), (D,), 1.0, 0.1),
            wo=w(t(synth.L_WO), (H, hq * D)), post_norm=w(t(synth.L_POST_NORM), (H,), 1.0, 0.1),
            w_gate=w(t(synth.L_WGATE), (I, H)), w_up=w(t(synth.L_WUP), (I, H)), w_down=w(t(synth.L_WDOWN), (H, I))))
    embed = w(synth.TID_EMBED, (cfg.vocab, H))
    final_norm = w(synth.TID_FINAL_NORM, (H,), 1.0, 0.1)
    ids = synth.uniform_int(SEED, synth.TID_IDS, (T,), cfg.vocab)
    return layers, embed, final_norm, ids


def logits(cfg, layers, embed, final_norm, ids, rounded):
    T = ids.shape[0]
    D, hq, hkv = cfg.head_dim, cfg.n_q_heads, cfg.n_kv_heads
    eps, theta = cfg.rms_eps, cfg.rope_theta
    rd = lambda name, x: to_bf16(x) if name in rounded else x  # noqa: E731
    pos = np.arange(T)
    allowed = R.causal_allowed(pos, pos)
    x = embed[ids]
    for L in layers:
        h = rd('h', R.rms_norm(x, L.in_norm, eps))
        q = rd('qkv', h @ L.wq.T).reshape(T, hq, D)
        k = rd('qkv', h @ L.wk.T).reshape(T, hkv, D)
        v = rd('v', rd('qkv', h @ L.wv.T)).reshape(T, hkv, D)
        q = rd('qk', R.rope_rotate_half(R.rms_norm(q, L.q_norm, eps), pos, theta))
        k = rd('qk', R.rope_rotate_half(R.rms_norm(k, L.k_norm, eps), pos, theta))
        if 'P' in rounded:
            # normalisation after the product, as a flash-style kernel does
            o = np.empty((T, hq, D))
            for head in range(hq):
                g = head // (hq // hkv)
                s = np.where(allowed, q[:, head] @ k[:, g].T / np.sqrt(D), -np.inf)
                p = np.exp(s - s.max(axis=1, keepdims=True))
                o[:, head] = (to_bf16(p) @ v[:, g]) / p.sum(axis=1, keepdims=True)
        else:
            o = R.causal_gqa_attention(q, k, v, pos, pos)
        x1 = x + rd('o', o.reshape(T, hq * D)) @ L.wo.T
        h2 = rd('h2', R.rms_norm(x1, L.post_norm, eps))
        a = rd('act', R.silu(h2 @ L.w_gate.T) * (h2 @ L.w_up.T))
        x = x1 + a @ L.w_down.T
    return rd('hf', R.rms_norm(x, final_norm, eps)) @ embed.T


def main():
    T = int(sys.argv[1]) if len(sys.argv) > 1 else 2048
    cfg = R.QWEN3_0_6B
    layers, embed, final_norm, ids = load(cfg, T)
    t0 = time.time()
    exact = logits(cfg, layers, embed, final_norm, ids, set())
    print(f"exact logits: {time.time() - t0:.1f} s", flush=True)
    library = {'h', 'v', 'qk', 'P', 'o', 'h2', 'act', 'hf'}  # what the GPU path keeps in bf16
    gemm_inputs = {'h', 'o', 'h2', 'act', 'hf'}
    variants = [
        ('every activation bf16', library | {'qkv'}),
        ('library rounding points', library),
        ('library, h and hf exact', library - {'h', 'hf'}),
        ('library, h, o and hf exact', library - {'h', 'o', 'hf'}),
        ('only the cache and P in bf16', library - gemm_inputs),
        ('only the cache in bf16', library - gemm_inputs - {'P'}),
    ]
    print(f"{'variant':32s} {'rel_frob':>10s} {'argmax':>8s}")
    for name, rounded in variants:
        lg = logits(cfg, layers, embed, final_norm, ids, rounded)
        rel = np.linalg.norm(lg - exact) / np.linalg.norm(exact)
        agree = np.mean(np.argmax(lg, axis=1) == np.argmax(exact, axis=1))
        print(f"{name:32s} {rel:10.3e} {agree:8.4f}", flush=True)


if __name__ == '__main__':
    main()
