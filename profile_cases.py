"""Single-kernel cases at the workloads' shapes, for timing and for ncu captures.

    python profile_cases.py <case> [--reps N]

Each case draws seeded inputs, runs the kernel once (warm-up), then N timed
repetitions with CUDA events, and prints one JSON line with the average device
time and the algorithmic throughput. For ncu, capture the second launch of the
kernel: ncu -k regex:<kernel> -s 1 -c 1 ...
"""
from __future__ import annotations

import argparse
import json

import torch

import qwen3_decoder_block_b200 as q3
import qwen3_synth as synth


def _bf16(shape, tid, std=1.0, seed=77):
    t = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    synth.normal_bf16_device(t.data_ptr(), 1, 1, t.numel(), 0, 0, seed, tid, 0.0, std)
    return t


GRAPH = False  # --graph: time `reps` launches captured in one CUDA graph (no host launch cost)


def _time(fn, reps):
    fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if GRAPH:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps):
                fn()
        g.replay()
        torch.cuda.synchronize()
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        del g
        return a.elapsed_time(b) / reps
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def case_attn_prefill(reps, B=4, T=2048, hq=16, hkv=8):
    """One layer's causal attention of the B4 x T2048 stack prefill, 16/8 heads."""
    cfg = q3.make_config(n_q_heads=hq, n_kv_heads=hkv, hidden=1024 if hq <= 16 else 2048)
    nqkv = (hq + 2 * hkv) * 128
    qkv = _bf16((B * T, nqkv), 1)
    k = _bf16((B, hkv, T, 128), 2)
    v = _bf16((B, hkv, T, 128), 3)
    kv = q3.kv_layer(k, v, T)
    o = torch.empty((B * T, hq * 128), dtype=torch.bfloat16, device="cuda")
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    ms = _time(lambda: q3.op_attention_prefill(cfg, qkv, B, T, pos, kv, o), reps)
    flops = 4 * 128 * hq * B * T * (T + 1) // 2
    return {"ms": ms, "tflops": flops / ms / 1e9, "flops": flops}


def case_attn_prefill_long(reps):
    """The B1 x T32768 layer's attention."""
    return case_attn_prefill(reps, B=1, T=32768)


def case_attn_decode(reps, B=64, L=4096):
    """One layer's decode attention of the B64 decode at 4096 cached tokens: 4097 visible positions each."""
    cfg = q3.config_qwen3_0_6b()
    s_max = L + 128
    nqkv = 32 * 128
    qkv = _bf16((B, nqkv), 4)
    k = _bf16((B, 8, s_max, 128), 5)
    v = _bf16((B, 8, s_max, 128), 6)
    kv = q3.kv_layer(k, v, s_max)
    o = torch.empty((B, 16 * 128), dtype=torch.bfloat16, device="cuda")
    lens = torch.full((B,), L, dtype=torch.int32, device="cuda")
    ws = torch.empty(q3.workspace_size(cfg, q3.OP_BLOCK_DECODE, B, 1, s_max), dtype=torch.uint8, device="cuda")
    ms = _time(lambda: q3.op_attention_decode(cfg, qkv, B, lens, kv, o, ws), reps)
    nbytes = B * 8 * (L + 1) * 128 * 2 * 2
    return {"ms": ms, "gbs": nbytes / ms / 1e6, "bytes": nbytes}


def _gemm(reps, M, N, K, epi=q3.EPI_STORE, swap=-1, out_f32=False, resid=False):
    A = _bf16((2 * M if swap == 3 else M, K), 7)  # swap 3: hi rows then lo rows
    W = _bf16((N, K), 8, 0.02)
    n_out = N // 2 if epi == q3.EPI_SWIGLU else N
    out = torch.empty((M, n_out), dtype=torch.float32 if out_f32 else torch.bfloat16, device="cuda")
    r = torch.zeros((M, N), dtype=torch.float32, device="cuda") if resid else None
    ws = torch.empty(48 << 20, dtype=torch.uint8, device="cuda")  # split-K scratch for small M
    ms = _time(lambda: q3.op_gemm(A, W, out, M, N, K, epilogue=epi, resid=r, swap=swap, ws=ws), reps)
    flops = 2 * M * N * K
    nbytes = 2 * (A.numel() + N * K) + out.numel() * out.element_size() + (r.numel() * 4 if resid else 0)
    return {"ms": ms, "tflops": flops / ms / 1e9, "gbs": nbytes / ms / 1e6, "flops": flops, "bytes": nbytes}


def case_gemm_gate_up(reps):
    """B4 x T2048 gate/up projection with the SwiGLU epilogue: M8192, N6144, K1024."""
    return _gemm(reps, 8192, 6144, 1024, epi=q3.EPI_SWIGLU)


def case_gemm_qkv(reps):
    """B4 x T2048 QKV projection: M8192, N4096, K1024."""
    return _gemm(reps, 8192, 4096, 1024)


def case_lm_head(reps):
    """B4 x T2048 tied LM head: M8192, N151936, K1024, fp32 logits."""
    return _gemm(reps, 8192, 151936, 1024, out_f32=True)


def case_gemm_qkv_fused(reps, B=4, T=2048):
    """B4 x T2048 QKV projection with the fused QK-norm + RoPE + KV-write epilogue (one block prefill
    minus the rest): M8192, N4096, K1024, measured through the block call's first GEMM."""
    cfg = q3.config_qwen3_0_6b()
    h = _bf16((B * T, 1024), 13)
    w = _bf16((4096, 1024), 14, 0.02)
    qkv = torch.empty((B * T, 4096), dtype=torch.bfloat16, device="cuda")
    qn, kn = _bf16((128,), 15), _bf16((128,), 16)
    k = torch.empty((B, 8, T, 128), dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    kv = q3.kv_layer(k, v, T)
    rope = torch.empty(q3.rope_table_bytes(cfg) // 4, dtype=torch.float32, device="cuda")
    q3.rope_table(cfg, rope)
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    ms = _time(lambda: q3.op_gemm_qkv_rope(cfg, h, w, qkv, B, T, pos, qn, kn, kv, rope), reps)
    flops = 2 * B * T * 4096 * 1024
    return {"ms": ms, "tflops": flops / ms / 1e9, "flops": flops}


def case_gemm_o(reps):
    """B4 x T2048 o_proj with the fp32 residual epilogue: M8192, N1024, K2048."""
    return _gemm(reps, 8192, 1024, 2048, epi=q3.EPI_RESID, out_f32=True, resid=True)


def case_gemm_down(reps):
    """B4 x T2048 down projection with the fp32 residual epilogue: M8192, N1024, K3072."""
    return _gemm(reps, 8192, 1024, 3072, epi=q3.EPI_RESID, out_f32=True, resid=True)


def case_gemm_o_decode(reps):
    """B64 decode o_proj: M64 (swap), N1024, K2048, fp32 residual epilogue."""
    return _gemm(reps, 64, 1024, 2048, epi=q3.EPI_RESID, out_f32=True, resid=True)


def case_gemm_gate_up_decode(reps):
    """B64 decode gate/up: M64 (swap), N6144, K1024, SwiGLU epilogue."""
    return _gemm(reps, 64, 6144, 1024, epi=q3.EPI_SWIGLU)


def case_gemm_qkv_decode(reps):
    """B64 decode QKV projection on the cluster split-K form: M64, N4096, K1024."""
    return _gemm(reps, 64, 4096, 1024, swap=2)


def case_gemm_down_decode(reps):
    """B64 decode down projection on the cluster split-K form: M64, N1024, K3072, fp32 residual."""
    return _gemm(reps, 64, 1024, 3072, epi=q3.EPI_RESID, out_f32=True, resid=True, swap=2)


def case_gemm_down_decode_splitk(reps):
    """As gemm_down_decode on the persistent GEMM with K split into fp32 partials in global
    memory and a separate completion launch (the form used for 65-256 tokens)."""
    return _gemm(reps, 64, 1024, 3072, epi=q3.EPI_RESID, out_f32=True, resid=True, swap=1)


def case_gemm_qkv_decode_splitk(reps):
    """As gemm_qkv_decode on the split-K partials form."""
    return _gemm(reps, 64, 4096, 1024, swap=1)


def case_gemm_down_decode_hilo(reps):
    """As gemm_down_decode with the activations as hi/lo rows (the decode path's form)."""
    return _gemm(reps, 64, 1024, 3072, epi=q3.EPI_RESID, out_f32=True, resid=True, swap=3)


def case_qk_norm_rope(reps, B=4, T=2048):
    """B4 x T2048 per-head QK-norm + RoPE + KV write: 8192 tokens x 32 head slots."""
    cfg = q3.config_qwen3_0_6b()
    qkv = _bf16((B * T, 4096), 9)
    qn, kn = _bf16((128,), 10), _bf16((128,), 11)
    k = torch.empty((B, 8, T, 128), dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    kv = q3.kv_layer(k, v, T)
    rope = torch.empty(q3.rope_table_bytes(cfg) // 4, dtype=torch.float32, device="cuda")
    q3.rope_table(cfg, rope)
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    ms = _time(lambda: q3.op_qk_norm_rope(cfg, qkv, B, T, pos, qn, kn, kv, rope), reps)
    nbytes = B * T * 4096 * 2 + B * T * (3072 * 2)  # read q,k,v; write q', k, v
    return {"ms": ms, "gbs": nbytes / ms / 1e6, "bytes": nbytes}


def case_rmsnorm(reps, rows=8192, n=1024):
    """B4 x T2048 RMSNorm of the fp32 residual stream: 8192 x 1024."""
    x = torch.randn((rows, n), dtype=torch.float32, device="cuda")
    w = _bf16((n,), 12)
    out = torch.empty((rows, n), dtype=torch.bfloat16, device="cuda")
    ms = _time(lambda: q3.op_rmsnorm(x, w, out, rows, n, 1e-6), reps)
    nbytes = rows * n * (4 + 2)
    return {"ms": ms, "gbs": nbytes / ms / 1e6, "bytes": nbytes}


CASES = {k[5:]: v for k, v in globals().items() if k.startswith("case_")}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=sorted(CASES) + ["all"])
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--graph", action="store_true", help="time the reps as one CUDA-graph replay")
    args = ap.parse_args()
    global GRAPH
    GRAPH = args.graph
    names = sorted(CASES) if args.case == "all" else [args.case]
    for n in names:
        r = CASES[n](args.reps)
        r["case"] = n
        print(json.dumps({k: (round(v, 4) if isinstance(v, float) else v) for k, v in r.items()}))
    assert q3.check_device_error() == 0


if __name__ == "__main__":
    main()
