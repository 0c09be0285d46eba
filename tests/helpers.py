"""Shared helpers of the GPU parity tests: seeded inputs in both forms (torch
bf16 on the GPU for the CUDA path, float64 numpy for the oracle) and the error
metrics the tolerances are stated in."""
from __future__ import annotations

import numpy as np

import qwen3_synth as synth
import oracle.qwen3_ref as R

# Per-layer bar: relative Frobenius error <= 1e-2 and max abs error <= 3e-2.
LAYER_REL_FROB = 1e-2
LAYER_MAX_ABS = 3e-2
# 28-layer logits: relative Frobenius <= 3e-2 and argmax agreement >= 99%.
LOGITS_REL_FROB = 3e-2
LOGITS_ARGMAX = 0.99


def rel_frob(a, ref) -> float:
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(a - ref) / max(np.linalg.norm(ref), 1e-300))


def max_abs(a, ref) -> float:
    return float(np.max(np.abs(np.asarray(a, dtype=np.float64) - np.asarray(ref, dtype=np.float64))))


def to_gpu_bf16(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.uint16)).view(torch.bfloat16).cuda()


def from_gpu_bf16(t) -> np.ndarray:
    import torch
    return R.bf16_to_f64(t.detach().contiguous().cpu().view(torch.uint16).numpy())


def f64(bits) -> np.ndarray:
    return R.bf16_to_f64(bits)


class Tensor:
    """A seeded bf16 tensor available as host bits and float64."""

    def __init__(self, seed, tid, shape, mean=0.0, std=1.0):
        self.bits = synth.normal_bf16(seed, tid, shape, mean, std)
        self.f = R.bf16_to_f64(self.bits)
        self._gpu = None

    @property
    def gpu(self):
        if self._gpu is None:
            self._gpu = to_gpu_bf16(self.bits)
        return self._gpu


def oracle_config(cfg) -> "R.Config":
    return R.Config(hidden=cfg.hidden, n_q_heads=cfg.n_q_heads, n_kv_heads=cfg.n_kv_heads, head_dim=cfg.head_dim,
                    intermediate=cfg.intermediate, vocab=cfg.vocab, n_layers=cfg.n_layers, max_pos=cfg.max_pos,
                    rope_theta=cfg.rope_theta, rms_eps=float(np.float32(cfg.rms_eps)), n_experts=cfg.n_experts,
                    top_k=cfg.top_k, moe_intermediate=cfg.moe_intermediate,
                    norm_topk_prob=bool(cfg.norm_topk_prob))


class Layer:
    """Synthetic weights of one layer in the pages' layouts (host + GPU) and the
    library's packed layouts (GPU)."""

    def __init__(self, cfg, seed, layer=0, moe=False, dense=True):
        """With cfg.gemm_f16 set, the linear weights are converted to fp16 after packing
        (exact for these weights' magnitudes), the layout the fp16 operand mode reads."""
        import torch
        import qwen3_decoder_block_b200 as q3
        H, D, hq, hkv, I = cfg.hidden, cfg.head_dim, cfg.n_q_heads, cfg.n_kv_heads, cfg.intermediate
        t = lambda which, shape, mean=0.0, std=synth.W_STD: Tensor(seed, synth.layer_tid(layer, which), shape, mean, std)
        nm, ns = synth.NORM_MEAN, synth.NORM_STD
        self.in_norm = t(synth.L_IN_NORM, (H,), nm, ns)
        self.wq = t(synth.L_WQ, (hq * D, H))
        self.wk = t(synth.L_WK, (hkv * D, H))
        self.wv = t(synth.L_WV, (hkv * D, H))
        self.q_norm = t(synth.L_Q_NORM, (D,), nm, ns)
        self.k_norm = t(synth.L_K_NORM, (D,), nm, ns)
        self.wo = t(synth.L_WO, (H, hq * D))
        self.post_norm = t(synth.L_POST_NORM, (H,), nm, ns)
        self.dense = dense
        if dense:
            self.w_gate = t(synth.L_WGATE, (I, H))
            self.w_up = t(synth.L_WUP, (I, H))
            self.w_down = t(synth.L_WDOWN, (H, I))
        self.moe = moe
        if moe:
            E, Im = cfg.n_experts, cfg.moe_intermediate
            self.router = t(synth.L_ROUTER, (E, H))
            self.gate_up = t(synth.L_MOE_GATE_UP, (E, 2 * Im, H))
            self.down = t(synth.L_MOE_DOWN, (E, H, Im))
        # packed device layouts
        self.w_qkv = torch.empty(((hq + 2 * hkv) * D, H), dtype=torch.bfloat16, device="cuda")
        q3.pack_qkv(cfg, self.wq.gpu, self.wk.gpu, self.wv.gpu, self.w_qkv)
        kw = dict(in_norm=self.in_norm.gpu, w_qkv=self.w_qkv, q_norm=self.q_norm.gpu, k_norm=self.k_norm.gpu,
                  w_o=self.wo.gpu, post_norm=self.post_norm.gpu)
        if dense:
            self.w_gate_up = torch.empty((2 * I, H), dtype=torch.bfloat16, device="cuda")
            q3.pack_gate_up(I, H, self.w_gate.gpu, self.w_up.gpu, self.w_gate_up)
            kw.update(w_gate_up=self.w_gate_up, w_down=self.w_down.gpu)
        if moe:
            E, Im = cfg.n_experts, cfg.moe_intermediate
            self.moe_gate_up = torch.empty((E, 2 * Im, H), dtype=torch.bfloat16, device="cuda")
            q3.pack_moe_gate_up(E, Im, H, self.gate_up.gpu, self.moe_gate_up)
            kw.update(router=self.router.gpu, moe_gate_up=self.moe_gate_up, moe_down=self.down.gpu)
        if cfg.gemm_f16:
            self.f16 = {}
            for name in ("w_qkv", "w_o", "w_gate_up", "w_down", "router", "moe_gate_up", "moe_down"):
                if name in kw:
                    self.f16[name] = q3.convert_to_f16(kw[name], torch.empty(kw[name].shape, dtype=torch.float16,
                                                                              device="cuda"))
            kw.update(self.f16)
            torch.cuda.synchronize()
        self.c = q3.layer_weights(**kw)

    def oracle(self) -> "R.LayerWeights":
        kw = dict(in_norm=self.in_norm.f, wq=self.wq.f, wk=self.wk.f, wv=self.wv.f, q_norm=self.q_norm.f,
                  k_norm=self.k_norm.f, wo=self.wo.f, post_norm=self.post_norm.f)
        if self.dense:
            kw.update(w_gate=self.w_gate.f, w_up=self.w_up.f, w_down=self.w_down.f)
        if self.moe:
            kw.update(router=self.router.f, gate_up=self.gate_up.f, down=self.down.f)
        return R.LayerWeights(**kw)


def rope_gpu(cfg):
    import torch
    import qwen3_decoder_block_b200 as q3
    rope = torch.empty(q3.rope_table_bytes(cfg) // 4, dtype=torch.float32, device="cuda")
    q3.rope_table(cfg, rope)
    return rope


def workspace(cfg, op, B, T, s_max):
    import torch
    import qwen3_decoder_block_b200 as q3
    n = q3.workspace_size(cfg, op, B, T, s_max)
    assert n > 0
    return torch.empty(n, dtype=torch.uint8, device="cuda")


def to_f16(t):
    """An fp16 copy of a bf16 GPU tensor made by the library's conversion."""
    import torch
    import qwen3_decoder_block_b200 as q3
    return q3.convert_to_f16(t, torch.empty(t.shape, dtype=torch.float16, device="cuda"))


def kv_cache(cfg, B, s_max, fill=None):
    """KV cache for one layer. fill=None leaves the memory as NaN bit patterns so
    that reads of never-written slots show up."""
    import torch
    import qwen3_decoder_block_b200 as q3
    shape = (B, cfg.n_kv_heads, s_max, cfg.head_dim)
    k = torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    v = torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    return k, v, q3.kv_layer(k, v, s_max)


def assert_device_ok():
    import qwen3_decoder_block_b200 as q3
    rc = q3.check_device_error()
    assert rc == 0, f"device error word: {rc} ({q3.lib.qwen3_last_error().decode()})"
