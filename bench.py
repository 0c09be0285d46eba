"""Benchmark of libqwen3blk on the Qwen3-0.6B workloads (one process per GPU).

Headline (one JSON line on rank 0):
  value  = 28-layer Qwen3-0.6B stack prefill, B=4 x T=2048 (8192 tokens, all-position fp32
           logits through the tied LM head), tokens/s summed over all ranks (replicas).
  decode = 28-layer decode, B=64 sequences holding 4096 cached tokens, 128 successive steps
           (positions 4096..4223), tokens/s (rank 0's GPU).
Synthetic seeded inputs (random weights of the Qwen3-0.6B shapes, random token ids).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-decode]

--impl reference times the fp64 CPU oracle (the only reference this workload has) on a
bounded sample of the same prefill workload.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Qwen3-0.6B prefill & decode tokens/s on 1 B200; % of BF16/HBM roofline"
# measured DRAM bytes / algorithmic K/V bytes of one decode-attention launch (ncu
# dram__bytes_read.sum + dram__bytes_write.sum); None until captured for the current kernel
DECODE_ATTN_TRAFFIC_RATIO = (1078514176 + 7338240) / 1074003968
DECODE_ATTN_TRAFFIC_SOURCE = ("ncu capture of one attn_decode_tc_kernel launch at B64 x 4097 positions "
                              "(profiles/attn_decode_B64_ctx4096_layer.md), scaled by positions")

PREFILL_B, PREFILL_T = 4, 2048
DECODE_B, DECODE_CTX, DECODE_STEPS = 64, 4096, 128
SEED_PREFILL, SEED_DECODE = 1001, 1002


def max_over_ranks(dist, value: float, torch, device: str = "cuda") -> float:
    """The slowest rank's value: every rank times its own GPU, the job takes as long as
    the slowest (a no-op for one process)."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, units_per_rank_step: float, steps: int, ms: float) -> float:
    """Units per second of the whole job: every rank processes units_per_rank_step per
    step (replicas, weak scaling) and the job's time is the slowest rank's ms."""
    return world * units_per_rank_step * steps / (ms * 1e-3)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples every 50 ms; only the rows stamped inside the timed window
    (marked with begin()/end() around it) enter the summary."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def begin(self):
        self.t0 = datetime.datetime.now()

    def end(self):
        self.t1 = datetime.datetime.now()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        lines = open(self.path).read().splitlines()
        os.unlink(self.path)
        return self.summarize(lines, self.t0, self.t1)

    @classmethod
    def summarize(cls, lines, t0=None, t1=None):
        """Median SM clock, max clock and the throttle reasons seen, over the rows stamped
        in [t0, t1] (all rows when none is, with "window": "all samples")."""
        rows = []
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
            except ValueError:
                ts = None
            rows.append((ts, parts[1:]))
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        window = "timed region"
        inside = [r for ts, r in rows if ts is not None and t0 is not None and t1 is not None and t0 <= ts <= t1]
        if not inside:
            inside, window = [r for _, r in rows], "all samples"
        sm = [float(r[1]) for r in inside if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in inside if r[2].replace(".", "").isdigit()]
        reasons = sorted({cls.REASONS[i] for r in inside for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(inside), "window": window}


# --------------------------------------------------------------------------- model set-up
def _filler(seed):
    import qwen3_synth as synth

    def fill(t, tid, mean, std, n0=1, n1=1, n2=None, s0=0, s1=0, offset=0):
        n2 = t.numel() if n2 is None else n2
        synth.normal_bf16_device(t.data_ptr() + 2 * offset, n0, n1, n2, s0, s1, seed, tid, mean, std)
    return fill


def build_layer(q3, cfg, seed, l, torch, moe=False):
    """Random weights of one layer drawn on the device straight into the packed layouts
    (identical values to drawing the pages' layouts and calling the pack helpers)."""
    import qwen3_synth as synth
    H, D, hq, hkv, I = cfg.hidden, cfg.head_dim, cfg.n_q_heads, cfg.n_kv_heads, cfg.intermediate
    bf = dict(dtype=torch.bfloat16, device="cuda")
    fill = _filler(seed)
    tid = lambda w: synth.layer_tid(l, w)
    in_norm = torch.empty(H, **bf); fill(in_norm, tid(synth.L_IN_NORM), synth.NORM_MEAN, synth.NORM_STD)
    post_norm = torch.empty(H, **bf); fill(post_norm, tid(synth.L_POST_NORM), synth.NORM_MEAN, synth.NORM_STD)
    qn = torch.empty(D, **bf); fill(qn, tid(synth.L_Q_NORM), synth.NORM_MEAN, synth.NORM_STD)
    kn = torch.empty(D, **bf); fill(kn, tid(synth.L_K_NORM), synth.NORM_MEAN, synth.NORM_STD)
    wqkv = torch.empty(((hq + 2 * hkv) * D, H), **bf)
    fill(wqkv, tid(synth.L_WQ), 0.0, synth.W_STD, n2=hq * D * H)
    fill(wqkv, tid(synth.L_WK), 0.0, synth.W_STD, n2=hkv * D * H, offset=hq * D * H)
    fill(wqkv, tid(synth.L_WV), 0.0, synth.W_STD, n2=hkv * D * H, offset=(hq + hkv) * D * H)
    wo = torch.empty((H, hq * D), **bf); fill(wo, tid(synth.L_WO), 0.0, synth.W_STD)
    keep = [in_norm, post_norm, qn, kn, wqkv, wo]
    kw = dict(in_norm=in_norm, w_qkv=wqkv, q_norm=qn, k_norm=kn, w_o=wo, post_norm=post_norm)
    if moe:
        E, Im = cfg.n_experts, cfg.moe_intermediate
        router = torch.empty((E, H), **bf); fill(router, tid(synth.L_ROUTER), 0.0, synth.W_STD)
        gu_pages = torch.empty((E, 2 * Im, H), **bf); fill(gu_pages, tid(synth.L_MOE_GATE_UP), 0.0, synth.W_STD)
        gu = torch.empty_like(gu_pages)
        q3.pack_moe_gate_up(E, Im, H, gu_pages, gu)
        down = torch.empty((E, H, Im), **bf); fill(down, tid(synth.L_MOE_DOWN), 0.0, synth.W_STD)
        torch.cuda.synchronize()
        del gu_pages
        keep += [router, gu, down]
        kw.update(router=router, moe_gate_up=gu, moe_down=down)
    else:
        wgu = torch.empty((2 * I, H), **bf)
        fill(wgu, tid(synth.L_WGATE), 0.0, synth.W_STD, n0=I // 16, n1=16, n2=H, s0=32 * H, s1=H)
        fill(wgu, tid(synth.L_WUP), 0.0, synth.W_STD, n0=I // 16, n1=16, n2=H, s0=32 * H, s1=H, offset=16 * H)
        wd = torch.empty((H, I), **bf); fill(wd, tid(synth.L_WDOWN), 0.0, synth.W_STD)
        keep += [wgu, wd]
        kw.update(w_gate_up=wgu, w_down=wd)
    if cfg.gemm_f16:
        # the fp16 operand mode: the linear weights convert in place (exact at these magnitudes)
        for name in ("w_qkv", "w_o", "w_gate_up", "w_down", "router", "moe_gate_up", "moe_down"):
            if name in kw:
                kw[name] = q3.convert_to_f16(kw[name])
    w = q3.layer_weights(**kw)
    q3.check_layer_weights(cfg, w, q3.LAYER_MOE if moe else q3.LAYER_DENSE)
    return w, keep


def build_model(q3, cfg, seed, torch):
    import qwen3_synth as synth
    H = cfg.hidden
    bf = dict(dtype=torch.bfloat16, device="cuda")
    fill = _filler(seed)
    layers, keep = [], []
    for l in range(cfg.n_layers):
        w, k = build_layer(q3, cfg, seed, l, torch)
        layers.append(w)
        keep += k
    embed = torch.empty((cfg.vocab, H), **bf); fill(embed, synth.TID_EMBED, 0.0, synth.W_STD)
    fnorm = torch.empty(H, **bf); fill(fnorm, synth.TID_FINAL_NORM, synth.NORM_MEAN, synth.NORM_STD)
    if cfg.gemm_f16:
        embed = q3.convert_to_f16(embed)  # the tied embedding / LM head in the operand type
    keep += [embed, fnorm]
    return layers, embed, fnorm, keep


def gemm_flops_per_token(cfg):
    H, D, hq, hkv, I = cfg.hidden, cfg.head_dim, cfg.n_q_heads, cfg.n_kv_heads, cfg.intermediate
    per_layer = 2 * (H * (hq + 2 * hkv) * D + hq * D * H + H * 2 * I + I * H)
    return cfg.n_layers * per_layer, 2 * H * cfg.vocab


def attention_prefill_flops(cfg, B, T):
    pairs = B * T * (T + 1) // 2
    return cfg.n_layers * 4 * cfg.head_dim * cfg.n_q_heads * pairs


def summarize_profile(records, steps):
    by = {}
    for name, ms in records:
        n, t = by.get(name, (0, 0.0))
        by[name] = (n + 1, t + ms)
    total = sum(t for _, t in by.values())
    return {k: {"launches_per_step": n / steps, "ms_per_step": t / steps, "share": t / total if total else 0.0}
            for k, (n, t) in sorted(by.items(), key=lambda kv: -kv[1][1])}, total / steps


# --------------------------------------------------------------------------- workloads
def run_prefill(q3, torch, args, rank, world, dist, peaks, gemm_f16=1, light=False):
    """The headline prefill in the given operand mode. light: the timed window only
    (no clocks, per-launch profile or end-to-end leg), for the secondary mode."""
    cfg = q3.make_config(gemm_f16=gemm_f16)
    B, T = PREFILL_B, PREFILL_T
    M = B * T
    import qwen3_synth as synth
    layers, embed, fnorm, keep = build_model(q3, cfg, SEED_PREFILL, torch)
    s_max = T
    caches = []
    for _ in range(cfg.n_layers):
        k = torch.empty((B, cfg.n_kv_heads, s_max, cfg.head_dim), dtype=torch.bfloat16, device="cuda")
        v = torch.empty_like(k)
        caches.append((k, v))
    kvs = [q3.kv_layer(k, v, s_max) for k, v in caches]
    rope = torch.empty(q3.rope_table_bytes(cfg) // 4, dtype=torch.float32, device="cuda")
    q3.rope_table(cfg, rope)
    ids = torch.empty(M, dtype=torch.int32, device="cuda")
    synth.uniform_int_device(ids.data_ptr(), M, SEED_PREFILL, synth.TID_IDS, cfg.vocab)
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    ws = torch.empty(q3.workspace_size(cfg, q3.OP_STACK_PREFILL, B, T, s_max), dtype=torch.uint8, device="cuda")
    logits = torch.empty((M, cfg.vocab), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        q3.stack_forward(cfg, embed, layers, fnorm, ids, B, T, q3.MODE_PREFILL, pos, kvs, rope, logits, False, ws,
                         stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert q3.check_device_error() == 0

    if light:
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = max_over_ranks(dist, e0.elapsed_time(e1), torch)
        assert q3.check_device_error() == 0
        return {"value": job_throughput(world, M, args.steps, ms), "unit": "tokens/s",
                "ms_per_step": ms / args.steps, "gemm_f16": gemm_f16}

    clocks = ClockSampler(torch.cuda.current_device())
    if rank == 0:
        clocks.start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.begin()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.end()
    ms = max_over_ranks(dist, e0.elapsed_time(e1), torch)
    if dist:
        dist.barrier()
    clk = clocks.stop() if rank == 0 else None
    assert q3.check_device_error() == 0

    # end to end through the public call with host buffers: ids H2D, logits of each
    # sequence's last position D2H, inside the timed region (device events; the host's
    # own time to issue the steps is reported beside it)
    ids_host = ids.cpu().pin_memory()
    out_host = torch.empty((B, cfg.vocab), dtype=torch.float32).pin_memory()
    last_rows = logits.view(B, T, cfg.vocab)[:, T - 1]
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0 = time.perf_counter()
    f0.record(stream)
    for _ in range(args.steps):
        ids.copy_(ids_host, non_blocking=True)
        step()
        out_host.copy_(last_rows, non_blocking=True)
    f1.record(stream)
    h1 = time.perf_counter()
    torch.cuda.synchronize()
    h2 = time.perf_counter()
    e2e_ms = max_over_ranks(dist, f0.elapsed_time(f1), torch)
    e2e_host = {"issue_ms_per_step": (h1 - h0) * 1e3 / args.steps, "wall_ms_per_step": (h2 - h0) * 1e3 / args.steps}

    # per-kernel attribution: the same K steps again with CUDA events around every
    # launch (kept out of the timed value above, which they would slow slightly)
    q3.profile_begin(args.steps * 400 + 16)
    for _ in range(args.steps):
        step()
    records = q3.profile_end(stream)

    kernels, prof_ms = summarize_profile(records, args.steps)
    g_tok, lm_tok = gemm_flops_per_token(cfg)
    gemm_flops = M * (g_tok + lm_tok)
    gemm_names = ("gemm_qkv", "gemm_o", "gemm_gate_up", "gemm_down", "lm_head")
    gemm_ms = sum(kernels[n]["ms_per_step"] for n in gemm_names if n in kernels)
    gemm_launches = sum(kernels[n]["launches_per_step"] for n in gemm_names if n in kernels)
    attn_flops = attention_prefill_flops(cfg, B, T)
    attn = kernels.get("attn_prefill", {"ms_per_step": float("nan"), "launches_per_step": 0})
    # each launch is timed on its own (CUDA events around it): the burst peak applies
    peak = peaks["bf16_tflops"]
    achieved = gemm_flops / (gemm_ms * 1e-3) / 1e12
    attn_tf = attn_flops / (attn["ms_per_step"] * 1e-3) / 1e12
    per_step_ms = ms / args.steps
    n_launch = len(records) / args.steps
    return {
        "value": job_throughput(world, M, args.steps, ms),
        "gemm_f16": gemm_f16,
        "ms_per_step": per_step_ms,
        "e2e": {"value": job_throughput(world, M, args.steps, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": M * 4, "d2h_bytes_per_step": B * cfg.vocab * 4, "host": e2e_host},
        "roofline": {"bound": "tensor", "kernel": "gemm_tc_kernel (all projections + LM head)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{peaks['source']} bf16 burst (launches timed one by one)", "traffic": None,
                     "flops_per_launch": gemm_flops / gemm_launches,
                     "avg_launch_ms": gemm_ms / gemm_launches},
        "attention": {"achieved_tflops": attn_tf, "frac": attn_tf / peak, "ms_per_step": attn["ms_per_step"],
                      "flops_per_step": attn_flops},
        "kernels": {k: {kk: round(vv, 5) for kk, vv in v.items()} for k, v in kernels.items()},
        "gpu_launches": int(round(n_launch * args.steps)),
        "profiled_ms_per_step": prof_ms,
        "clocks": clk,
    }


def run_decode(q3, torch, args, peaks, gemm_f16=1):
    cfg = q3.make_config(gemm_f16=gemm_f16)
    B, L0, S = DECODE_B, DECODE_CTX, DECODE_STEPS
    import qwen3_synth as synth
    layers, embed, fnorm, keep = build_model(q3, cfg, SEED_DECODE, torch)
    s_max = L0 + S
    caches = []
    for l in range(cfg.n_layers):
        k = torch.empty((B, cfg.n_kv_heads, s_max, cfg.head_dim), dtype=torch.bfloat16, device="cuda")
        v = torch.empty_like(k)
        for t, which in ((k, synth.L_CACHE_K), (v, synth.L_CACHE_V)):
            synth.normal_bf16_device(t.data_ptr(), B * cfg.n_kv_heads, L0, cfg.head_dim, s_max * cfg.head_dim,
                                     cfg.head_dim, SEED_DECODE, synth.layer_tid(l, which), 0.0, 1.0)
        caches.append((k, v))
    kvs = [q3.kv_layer(k, v, s_max) for k, v in caches]
    rope = torch.empty(q3.rope_table_bytes(cfg) // 4, dtype=torch.float32, device="cuda")
    q3.rope_table(cfg, rope)
    all_ids = torch.empty((S, B), dtype=torch.int32, device="cuda")
    synth.uniform_int_device(all_ids.data_ptr(), S * B, SEED_DECODE, synth.TID_IDS_STEP, cfg.vocab)
    ids = torch.empty(B, dtype=torch.int32, device="cuda")
    lens = torch.full((B,), L0, dtype=torch.int32, device="cuda")
    ws = torch.empty(q3.workspace_size(cfg, q3.OP_STACK_DECODE, B, 1, s_max), dtype=torch.uint8, device="cuda")
    logits = torch.empty((B, cfg.vocab), dtype=torch.float32, device="cuda")
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()

    def step():
        q3.stack_forward(cfg, embed, layers, fnorm, ids, B, 1, q3.MODE_DECODE, lens, kvs, rope, logits, False, ws,
                         stream)

    with torch.cuda.stream(stream):
        ids.copy_(all_ids[0])
        step()  # eager step: one-time set-up outside capture
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream, capture_error_mode="thread_local"):
            step()
        for s in range(max(args.warmup, 3)):
            ids.copy_(all_ids[s % S])
            graph.replay()
        lens.fill_(L0)  # undo the warm-up steps
    torch.cuda.synchronize()
    assert q3.check_device_error(stream) == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for s in range(S):
            ids.copy_(all_ids[s])
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    assert q3.check_device_error(stream) == 0
    assert int(lens[0].item()) == L0 + S
    # per-kernel attribution: one profiled eager window (not part of the timed value)
    lens.fill_(L0)
    torch.cuda.synchronize()
    q3.profile_begin(8 * 300)
    with torch.cuda.stream(stream):
        for s in range(8):
            ids.copy_(all_ids[s])
            step()
    records = q3.profile_end(stream)
    kernels, _ = summarize_profile(records, 8)
    # algorithmic bytes of the decode attention: K and V of every visible position (8 prof steps)
    kv_bytes = sum(cfg.n_layers * B * (L0 + s + 1) * cfg.n_kv_heads * cfg.head_dim * 2 * 2 for s in range(8)) / 8
    attn_ms = kernels["attn_decode"]["ms_per_step"]
    achieved = kv_bytes / (attn_ms * 1e-3) / 1e9
    step_bytes = sum(cfg.n_layers * B * (L0 + s + 1) * cfg.n_kv_heads * cfg.head_dim * 4 for s in range(S)) / S
    w_bytes = 2 * (cfg.n_layers * (cfg.hidden * (cfg.n_q_heads + 2 * cfg.n_kv_heads) * cfg.head_dim +
                                   cfg.n_q_heads * cfg.head_dim * cfg.hidden + 3 * cfg.hidden * cfg.intermediate) +
                   cfg.vocab * cfg.hidden) + B * cfg.vocab * 4
    step_ms = ms / S
    hbm = peaks["hbm_gbs"]
    del graph
    gen = run_generate(q3, torch, cfg, layers, embed, fnorm, kvs, rope, B, s_max, stream)
    return {
        "value": B * S / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": step_ms, "gemm_f16": gemm_f16,
        "generate": gen,
        "workload": f"Qwen3-0.6B 28-layer decode, B{B}, {L0} cached tokens, {S} steps (positions {L0}..{L0 + S - 1}), "
                    "CUDA-graph replay per step",
        "step_roofline": {"bound": "hbm", "algorithmic_bytes_per_step": step_bytes + w_bytes,
                          "achieved_gbs": (step_bytes + w_bytes) / (step_ms * 1e-3) / 1e9,
                          "frac": (step_bytes + w_bytes) / (step_ms * 1e-3) / 1e9 / hbm},
        "roofline": {"bound": "hbm", "kernel": "attn_decode (plan + stream-K tiles, in-kernel merge)",
                     "achieved": achieved, "peak": hbm,
                     "unit": "GB/s", "frac": achieved / hbm, "peak_source": f"{peaks['source']} hbm copy",
                     "traffic": (kv_bytes / cfg.n_layers * DECODE_ATTN_TRAFFIC_RATIO
                                 if DECODE_ATTN_TRAFFIC_RATIO else None),
                     "traffic_source": DECODE_ATTN_TRAFFIC_SOURCE},
        "kernels": {k: {kk: round(vv, 5) for kk, vv in v.items()} for k, v in kernels.items()},
        "gpu_launches_per_step": len(records) / 8,
    }


def run_generate(q3, torch, cfg, layers, embed, fnorm, kvs, rope, B, s_max, stream, T=128, n_new=64):
    """The library's greedy loop (qwen3_generate_greedy): a T-token prompt per sequence,
    then n_new tokens (one stack prefill, n_new - 1 decode steps, an argmax after each),
    launched eagerly on one stream and timed with CUDA events around the call."""
    import qwen3_synth as synth
    prompt = torch.empty(B * T, dtype=torch.int32, device="cuda")
    synth.uniform_int_device(prompt.data_ptr(), B * T, SEED_DECODE, synth.TID_IDS, cfg.vocab)
    ws = torch.empty(q3.workspace_size(cfg, q3.OP_GENERATE, B, T, s_max), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, n_new), dtype=torch.int32, device="cuda")
    times = []
    with torch.cuda.stream(stream):
        for it in range(3):
            start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            start.record(stream)
            q3.generate_greedy(cfg, embed, layers, fnorm, prompt, B, T, n_new, kvs, rope, out, ws, stream)
            end.record(stream)
            end.synchronize()
            if it > 0:
                times.append(start.elapsed_time(end))
    if q3.check_device_error(stream) != 0:
        raise RuntimeError("generate: device error")
    ms = min(times)
    return {"value": B * n_new / (ms * 1e-3), "unit": "generated tokens/s", "ms_per_call": ms,
            "workload": f"Qwen3-0.6B greedy generation, B{B}, {T}-token prompt + {n_new} new tokens "
                        f"(one stack prefill, {n_new - 1} decode steps, device argmax), eager launches"}


def run_single_layer(q3, torch, args, name, B, T, seed, moe=False, reps=None):
    """One decoder block prefill (dense or MoE) timed with CUDA events: returns tokens/s,
    time per call and the algorithmic TFLOP/s of the whole block."""
    import qwen3_synth as synth
    if moe:
        cfg = q3.make_config(hidden=2048, n_q_heads=32, n_kv_heads=4, n_experts=128, top_k=8, moe_intermediate=768,
                             gemm_f16=1)
    else:
        cfg = q3.make_config(gemm_f16=1)
    H, D, hq, hkv = cfg.hidden, cfg.head_dim, cfg.n_q_heads, cfg.n_kv_heads
    w, keep = build_layer(q3, cfg, seed, 0, torch, moe=moe)
    x0 = torch.empty((B * T, H), dtype=torch.bfloat16, device="cuda")
    synth.normal_bf16_device(x0.data_ptr(), 1, 1, x0.numel(), 0, 0, seed, synth.TID_X, 0.0, 1.0)
    x = x0.clone()
    k = torch.empty((B, hkv, T, D), dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    kv = q3.kv_layer(k, v, T)
    rope = torch.empty(q3.rope_table_bytes(cfg) // 4, dtype=torch.float32, device="cuda")
    q3.rope_table(cfg, rope)
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    op = q3.OP_MOE_BLOCK if moe else q3.OP_BLOCK_PREFILL
    ws = torch.empty(q3.workspace_size(cfg, op, B, T, T), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    # the block updates x in place, so successive calls chain the layer (each call's input
    # is the previous call's output: the same work, no copy between calls)
    def call():
        if moe:
            q3.moe_block(cfg, w, x, B, T, pos, kv, rope, ws, stream=stream)
        else:
            q3.block_prefill(cfg, w, x, B, T, pos, kv, rope, ws, stream)

    reps = reps or max(3, args.steps)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0 = time.perf_counter()
    e0.record(stream)
    for _ in range(reps):
        call()
    e1.record(stream)
    h1 = time.perf_counter()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    host_issue_ms = (h1 - h0) * 1e3 / reps
    q3.profile_begin(400)
    call()
    recs = q3.profile_end(stream)
    assert q3.check_device_error() == 0
    M = B * T
    lin = 2 * M * (H * (hq + 2 * hkv) * D + hq * D * H)
    attn = 4 * D * hq * B * T * (T + 1) // 2
    if moe:
        ffn = 2 * M * (H * cfg.n_experts + cfg.top_k * 3 * H * cfg.moe_intermediate)
    else:
        ffn = 2 * M * 3 * H * cfg.intermediate
    flops = lin + attn + ffn
    kern, _ = summarize_profile(recs, 1)
    return {"workload": name, "tokens_per_s": M / (ms * 1e-3), "ms_per_call": ms, "host_issue_ms_per_call": host_issue_ms,
            "tflops": flops / (ms * 1e-3) / 1e12, "algorithmic_tflop": flops / 1e12,
            "kernels_ms": {kk: round(vv["ms_per_step"], 4) for kk, vv in kern.items()}}


def run_moe_decode(q3, torch, args, peaks, B=64, L0=4096, seed=1005):
    """One decode step of the MoE block (hidden 2048, 32/4 heads, 128 experts x 768,
    top-8; the block of the B1 x T4096 MoE workload) for B sequences holding L0 cached
    tokens: qwen3_moe_block with T = 1 at position L0. HBM-bound: the bytes are the K/V read, the attention and router weights,
    and the weights of every expert the step routes to (counted from the routing)."""
    import qwen3_synth as synth
    cfg = q3.make_config(hidden=2048, n_q_heads=32, n_kv_heads=4, n_experts=128, top_k=8, moe_intermediate=768,
                         gemm_f16=1)
    H, D, hq, hkv = cfg.hidden, cfg.head_dim, cfg.n_q_heads, cfg.n_kv_heads
    w, keep = build_layer(q3, cfg, seed, 0, torch, moe=True)
    s_max = L0 + 8
    k = torch.empty((B, hkv, s_max, D), dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    for t, which in ((k, synth.L_CACHE_K), (v, synth.L_CACHE_V)):
        synth.normal_bf16_device(t.data_ptr(), B * hkv, L0, D, s_max * D, D, seed, synth.layer_tid(0, which), 0.0, 1.0)
    kv = q3.kv_layer(k, v, s_max)
    x0 = torch.empty((B, H), dtype=torch.bfloat16, device="cuda")
    synth.normal_bf16_device(x0.data_ptr(), 1, 1, x0.numel(), 0, 0, seed, synth.TID_X, 0.0, 1.0)
    x = x0.clone()
    rope = torch.empty(q3.rope_table_bytes(cfg) // 4, dtype=torch.float32, device="cuda")
    q3.rope_table(cfg, rope)
    lens = torch.full((B,), L0, dtype=torch.int32, device="cuda")
    ws = torch.empty(q3.workspace_size(cfg, q3.OP_MOE_BLOCK, B, 1, s_max), dtype=torch.uint8, device="cuda")
    idx = torch.empty((B, cfg.top_k), dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()

    def call():
        x.copy_(x0)
        q3.moe_block(cfg, w, x, B, 1, lens, kv, rope, ws, idx, stream=stream)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    reps = max(10, args.steps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    q3.profile_begin(400)
    call()
    recs = q3.profile_end(stream)
    assert q3.check_device_error() == 0
    kern, _ = summarize_profile(recs, 1)
    experts_hit = int(torch.unique(idx).numel())
    Im, E = cfg.moe_intermediate, cfg.n_experts
    kv_bytes = B * hkv * (L0 + 1) * D * 2 * 2
    w_bytes = 2 * (H * (hq + 2 * hkv) * D + hq * D * H + E * H + experts_hit * 3 * H * Im)
    nbytes = kv_bytes + w_bytes
    return {"workload": f"MoE block decode step (hidden 2048, 32/4 heads, 128 experts x 768, top-8), B{B} at "
                        f"{L0} cached tokens", "tokens_per_s": B / (ms * 1e-3), "ms_per_call": ms,
            "experts_hit": experts_hit, "algorithmic_bytes": nbytes, "achieved_gbs": nbytes / (ms * 1e-3) / 1e9,
            "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "kernels_ms": {kk: round(vv["ms_per_step"], 4) for kk, vv in kern.items()}}


# --------------------------------------------------------------------------- oracle timing
def oracle_model(seed: int = SEED_PREFILL):
    """The prefill workload's random weights in the oracle's layouts (fp64), drawn once."""
    import oracle.qwen3_ref as R
    import qwen3_synth as synth
    cfg = R.QWEN3_0_6B
    H, D, hq, hkv, I = cfg.hidden, cfg.head_dim, cfg.n_q_heads, cfg.n_kv_heads, cfg.intermediate
    gen = lambda tid, shape, m=0.0, s=synth.W_STD: R.bf16_to_f64(synth.normal_bf16_fast(seed, tid, shape, m, s))
    layers = []
    for l in range(cfg.n_layers):
        t = lambda w: synth.layer_tid(l, w)
        layers.append(R.LayerWeights(
            in_norm=gen(t(synth.L_IN_NORM), (H,), synth.NORM_MEAN, synth.NORM_STD),
            wq=gen(t(synth.L_WQ), (hq * D, H)), wk=gen(t(synth.L_WK), (hkv * D, H)), wv=gen(t(synth.L_WV), (hkv * D, H)),
            q_norm=gen(t(synth.L_Q_NORM), (D,), synth.NORM_MEAN, synth.NORM_STD),
            k_norm=gen(t(synth.L_K_NORM), (D,), synth.NORM_MEAN, synth.NORM_STD),
            wo=gen(t(synth.L_WO), (H, hq * D)),
            post_norm=gen(t(synth.L_POST_NORM), (H,), synth.NORM_MEAN, synth.NORM_STD),
            w_gate=gen(t(synth.L_WGATE), (I, H)), w_up=gen(t(synth.L_WUP), (I, H)), w_down=gen(t(synth.L_WDOWN), (H, I))))
    embed = gen(synth.TID_EMBED, (cfg.vocab, H))
    fnorm = gen(synth.TID_FINAL_NORM, (H,), synth.NORM_MEAN, synth.NORM_STD)
    return cfg, layers, embed, fnorm


def oracle_sample(T_s: int, model=None, seed: int = SEED_PREFILL):
    """Times the fp64 oracle on one sequence of T_s tokens of the prefill workload
    (28 layers + final norm + tied LM head on all T_s positions)."""
    import oracle.qwen3_ref as R
    import qwen3_synth as synth
    cfg, layers, embed, fnorm = model if model is not None else oracle_model(seed)
    ids = synth.uniform_int(seed, synth.TID_IDS, (T_s,), cfg.vocab)
    t0 = time.perf_counter()
    R.stack_forward(ids, embed, layers, fnorm, cfg)
    return time.perf_counter() - t0


# The reference arm's whole run (warm-up and timed steps) is sized to about
# REF_BUDGET_S seconds at the oracle's measured rate on 8-16 host cores (66-87 tokens/s).
REF_BUDGET_S = 150.0
ORACLE_EST_TOKENS_S = 75.0


def reference_tokens_per_step(steps: int, warmup: int) -> int:
    """Tokens of the prefill workload per reference-arm step: the first n ids of one
    sequence, n a multiple of 64 in [64, 2048]."""
    n = int(REF_BUDGET_S * ORACLE_EST_TOKENS_S / max(1, steps + warmup)) // 64 * 64
    return max(64, min(PREFILL_T, n))


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(T_s: int = PREFILL_T):
    dt = oracle_sample(T_s)
    return {"value": T_s / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"one sequence of {T_s} tokens (prefill workload's first {T_s} ids) through the 28-layer "
                      f"stack + tied LM head in fp64 numpy, {dt:.1f} s"}


# --------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true")
    ap.add_argument("--workload", choices=["all", "prefill", "decode"], default="all",
                    help="prefill or decode alone (for profiler launch lists)")
    ap.add_argument("--oracle-tokens", type=int, default=None,
                    help="oracle tokens per sample (default: 2048 for cpu_baseline; sized to the run "
                         "for --impl reference)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    peaks = load_peaks()
    config = {"workload": f"Qwen3-0.6B 28-layer stack prefill, B{PREFILL_B} x T{PREFILL_T} "
                          "(positions 0..2047), final RMSNorm + tied LM head, fp32 logits for all positions",
              "global_batch": PREFILL_B * world, "seq_len": PREFILL_T,
              "parallelism": f"replicas x{world} (independent sequences, no collective)",
              "l2": "inputs larger than L2 (1.2 GB of weights and 5 GB of logits per step)"}

    if args.impl == "reference":
        if rank != 0:
            return
        # K timed steps after W warm-up steps, each the oracle on one bounded sample of
        # the prefill workload (the first n token ids of one sequence)
        n = args.oracle_tokens or reference_tokens_per_step(args.steps, args.warmup)
        model = oracle_model()
        times = [oracle_sample(n, model) for _ in range(args.warmup + args.steps)][args.warmup:]
        total = sum(times)
        v = n * args.steps / total
        # the oracle's rate depends on the sequence length (its attention is quadratic in
        # it): the config names the sample each step really processes
        ref_config = dict(config, sample=f"1 sequence x {n} tokens (the prefill workload's first {n} ids) per "
                                         f"step, 28 layers + final norm + tied LM head on all {n} positions")
        line = {"metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": ref_config,
                "impl": "reference",
                "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                                 "sample": f"one sequence of {n} tokens (the prefill workload's first {n} ids) "
                                           f"through the 28-layer stack + tied LM head in fp64 numpy, per step"},
                "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch
    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist_mod.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
        dist = dist_mod
    else:
        torch.cuda.set_device(local)
    import qwen3_decoder_block_b200 as q3

    if args.workload == "decode":
        dec = run_decode(q3, torch, args, peaks)
        print(json.dumps({"metric": METRIC, "workload": "decode only", "decode": dec}))
        return
    # the pages' bf16 operands first (timed window only), then the headline: fp16 operands,
    # the mode that meets the 28-layer logits bar at the same tensor-core rate
    pre_bf16 = run_prefill(q3, torch, args, rank, world, dist, peaks, gemm_f16=0, light=True)
    torch.cuda.empty_cache()
    pre = run_prefill(q3, torch, args, rank, world, dist, peaks, gemm_f16=1)
    dec = None
    if not args.no_decode and rank == 0 and args.workload == "all":
        torch.cuda.empty_cache()
        dec = run_decode(q3, torch, args, peaks)
    others = None
    if rank == 0 and not args.no_configs and args.workload == "all":
        torch.cuda.empty_cache()
        others = {
            "layer_B1xT16": run_single_layer(q3, torch, args, "1 Qwen3-0.6B layer prefill, B1 x T16", 1, 16, 1000,
                                   reps=200),
            "layer_B1xT32768": run_single_layer(q3, torch, args, "1 Qwen3-0.6B layer prefill, B1 x T32768", 1, 32768, 1003),
            "moe_block_B1xT4096": run_single_layer(q3, torch, args, "MoE block prefill (hidden 2048, 32/4 heads, 128 experts x "
                                   "768, top-8), B1 x T4096", 1, 4096, 1004, moe=True),
            "moe_decode_B64_ctx4096": run_moe_decode(q3, torch, args, peaks),
        }
        torch.cuda.empty_cache()
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.workload == "all":
        cpu = cpu_baseline(args.oracle_tokens or PREFILL_T)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {"metric": METRIC, "value": pre["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": pre["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16", "data": "synthetic (seeded random weights and token ids)",
            "config": config, "e2e": pre["e2e"], "roofline": pre["roofline"], "cpu_baseline": cpu,
            "gpu_launches": pre["gpu_launches"], "clocks": pre["clocks"], "attention": pre["attention"],
            "kernels": pre["kernels"], "operands": "fp16 projection operands (gemm_f16 = 1); KV cache, q and P bf16",
            "bf16_operands": pre_bf16, "decode": dec, "workloads": others}
    print(json.dumps(line))


if __name__ == "__main__":
    main()
