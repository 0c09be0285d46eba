"""Python binding of libqwen3blk (argument marshalling only).

Every function here forwards to the C ABI declared in include/qwen3blk.h with
the same name (without the ``qwen3_`` prefix). Tensors are torch tensors on the
GPU; only their device pointers cross the boundary. There is no fallback: if the
compiled library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libqwen3blk.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with __graft_entry__.build() "
                      "(python -c 'import __graft_entry__ as g; g.build()')")

lib = ctypes.CDLL(LIB_PATH)

OK, EINVAL, ESHAPE, EALIGN, ECAPACITY, EWORKSPACE, ECUDA, ETIMEOUT, EDEVICE = 0, -1, -2, -3, -4, -5, -6, -7, -8
OP_BLOCK_PREFILL, OP_BLOCK_DECODE, OP_MOE_BLOCK, OP_STACK_PREFILL, OP_STACK_DECODE, OP_GENERATE = 1, 2, 3, 4, 5, 6
MODE_PREFILL, MODE_DECODE = 0, 1
EPI_STORE, EPI_RESID, EPI_SWIGLU = 0, 1, 2


class Config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("n_q_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("intermediate", ctypes.c_int), ("vocab", ctypes.c_int),
                ("n_layers", ctypes.c_int), ("max_pos", ctypes.c_int), ("n_experts", ctypes.c_int),
                ("top_k", ctypes.c_int), ("moe_intermediate", ctypes.c_int), ("norm_topk_prob", ctypes.c_int),
                ("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_double), ("gemm_f16", ctypes.c_int)]


class LayerWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("in_norm", "w_qkv", "q_norm", "k_norm", "w_o", "post_norm",
                                               "w_gate_up", "w_down", "router", "moe_gate_up", "moe_down")]


class KVLayer(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("s_max", ctypes.c_int)]


_vp, _i, _ll, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float, ctypes.c_size_t
_P = ctypes.POINTER

_SIGS = {
    "qwen3_last_error": ([], ctypes.c_char_p),
    "qwen3_status_string": ([_i], ctypes.c_char_p),
    "qwen3_config_qwen3_0_6b": ([_P(Config)], _i),
    "qwen3_validate_config": ([_P(Config)], _i),
    "qwen3_rope_table_bytes": ([_P(Config)], _sz),
    "qwen3_rope_table": ([_P(Config), _vp, _vp], _i),
    "qwen3_workspace_size": ([_P(Config), _i, _i, _i, _i], _sz),
    "qwen3_pack_qkv": ([_P(Config), _vp, _vp, _vp, _vp, _vp], _i),
    "qwen3_pack_gate_up": ([_i, _i, _vp, _vp, _vp, _vp], _i),
    "qwen3_pack_moe_gate_up": ([_i, _i, _i, _vp, _vp, _vp], _i),
    "qwen3_check_device_error": ([_vp], _i),
    "qwen3_check_layer_weights": ([_P(Config), _P(LayerWeights), _i], _i),
    "qwen3_block_prefill": ([_P(Config), _P(LayerWeights), _vp, _i, _i, _vp, _P(KVLayer), _vp, _vp, _sz, _vp], _i),
    "qwen3_block_decode": ([_P(Config), _P(LayerWeights), _vp, _i, _vp, _P(KVLayer), _vp, _vp, _sz, _vp], _i),
    "qwen3_moe_block": ([_P(Config), _P(LayerWeights), _vp, _i, _i, _vp, _P(KVLayer), _vp, _vp, _vp, _vp, _vp,
                         _vp, _sz, _vp], _i),
    "qwen3_stack_forward": ([_P(Config), _vp, _P(LayerWeights), _vp, _vp, _i, _i, _i, _vp, _P(KVLayer), _vp, _vp,
                             _i, _vp, _sz, _vp], _i),
    "qwen3_generate_greedy": ([_P(Config), _vp, _P(LayerWeights), _vp, _vp, _i, _i, _i, _P(KVLayer), _vp, _vp, _vp,
                               _sz, _vp], _i),
    "qwen3_profile_begin": ([_i], _i),
    "qwen3_profile_end": ([_vp], _i),
    "qwen3_profile_record": ([_i, ctypes.c_char_p, _i, _P(_f)], _i),
    "qwen3_op_rmsnorm": ([_vp, _i, _ll, _vp, _vp, _ll, _i, _i, _f, _i, _vp], _i),
    "qwen3_op_gemm": ([_vp, _ll, _vp, _ll, _vp, _ll, _i, _i, _i, _i, _vp, _ll, _i, _i, _i, _i, _vp, _sz, _vp], _i),
    "qwen3_op_qk_norm_rope": ([_P(Config), _vp, _ll, _i, _i, _vp, _vp, _vp, _P(KVLayer), _vp, _vp], _i),
    "qwen3_op_gemm_qkv_rope": ([_P(Config), _vp, _vp, _vp, _i, _i, _vp, _vp, _vp, _P(KVLayer), _vp, _vp], _i),
    "qwen3_op_attention_prefill": ([_P(Config), _vp, _ll, _i, _i, _vp, _P(KVLayer), _vp, _ll, _vp], _i),
    "qwen3_op_attention_decode": ([_P(Config), _vp, _ll, _i, _vp, _P(KVLayer), _vp, _ll, _vp, _sz, _vp], _i),
    "qwen3_op_attention_decode_noalloc": ([_P(Config), _vp, _ll, _i, _vp, _P(KVLayer), _vp, _ll, _vp], _i),
    "qwen3_op_embed": ([_vp, _i, _vp, _i, _i, _vp, _i, _i, _vp], _i),
    "qwen3_convert_to_f16": ([_vp, _vp, _sz, _vp], _i),
    "qwen3_op_argmax": ([_vp, _ll, _i, _i, _vp, _ll, _vp], _i),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res

EXPORTED = sorted(_SIGS)


class Qwen3Error(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lib.qwen3_last_error().decode()
        super().__init__(f"{where}: {lib.qwen3_status_string(status).decode()} ({status}): {msg}")
        self.status = status


def _check(status: int, where: str) -> None:
    if status != 0:
        raise Qwen3Error(status, where)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ------------------------------------------------------------------------- config
def config_qwen3_0_6b() -> Config:
    c = Config()
    _check(lib.qwen3_config_qwen3_0_6b(ctypes.byref(c)), "config_qwen3_0_6b")
    return c


def make_config(**kw) -> Config:
    c = config_qwen3_0_6b()
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def validate_config(cfg: Config) -> int:
    return lib.qwen3_validate_config(ctypes.byref(cfg))


def workspace_size(cfg: Config, op: int, B: int, T: int, s_max: int) -> int:
    return lib.qwen3_workspace_size(ctypes.byref(cfg), op, B, T, s_max)


def rope_table_bytes(cfg: Config) -> int:
    return lib.qwen3_rope_table_bytes(ctypes.byref(cfg))


def rope_table(cfg: Config, rope, stream=None) -> None:
    _check(lib.qwen3_rope_table(ctypes.byref(cfg), _ptr(rope), _stream(stream)), "rope_table")


def check_device_error(stream=None) -> int:
    return lib.qwen3_check_device_error(_stream(stream))


def profile_begin(max_records: int = 4096) -> None:
    _check(lib.qwen3_profile_begin(max_records), "profile_begin")


def profile_end(stream=None) -> list[tuple[str, float]]:
    n = lib.qwen3_profile_end(_stream(stream))
    if n < 0:
        _check(n, "profile_end")
    out = []
    buf = ctypes.create_string_buffer(64)
    ms = ctypes.c_float()
    for i in range(n):
        _check(lib.qwen3_profile_record(i, buf, 64, ctypes.byref(ms)), "profile_record")
        out.append((buf.value.decode(), ms.value))
    return out


# ------------------------------------------------------------------------- packing
def pack_qkv(cfg, wq, wk, wv, out, stream=None) -> None:
    _check(lib.qwen3_pack_qkv(ctypes.byref(cfg), _ptr(wq), _ptr(wk), _ptr(wv), _ptr(out), _stream(stream)), "pack_qkv")


def pack_gate_up(I, H, gate, up, out, stream=None) -> None:
    _check(lib.qwen3_pack_gate_up(I, H, _ptr(gate), _ptr(up), _ptr(out), _stream(stream)), "pack_gate_up")


def pack_moe_gate_up(E, Im, H, gate_up, out, stream=None) -> None:
    _check(lib.qwen3_pack_moe_gate_up(E, Im, H, _ptr(gate_up), _ptr(out), _stream(stream)), "pack_moe_gate_up")


def layer_weights(**tensors) -> LayerWeights:
    w = LayerWeights()
    for k, v in tensors.items():
        setattr(w, k, _ptr(v))
    return w


LAYER_DENSE, LAYER_MOE = 0, 1


def check_layer_weights(cfg: Config, w: LayerWeights, kind: int = LAYER_DENSE) -> None:
    """Two-way check of a layer's weight pointers (host only); raises Qwen3Error."""
    _check(lib.qwen3_check_layer_weights(ctypes.byref(cfg), ctypes.byref(w), kind), "check_layer_weights")


def kv_layer(k, v, s_max: int) -> KVLayer:
    return KVLayer(_ptr(k), _ptr(v), s_max)


# ------------------------------------------------------------------------- block calls
def block_prefill(cfg, w, x, B, T, start_pos, kv, rope, ws, stream=None) -> None:
    _check(lib.qwen3_block_prefill(ctypes.byref(cfg), ctypes.byref(w), _ptr(x), B, T, _ptr(start_pos),
                                   ctypes.byref(kv), _ptr(rope), _ptr(ws), ws.numel() * ws.element_size(),
                                   _stream(stream)), "block_prefill")


def block_decode(cfg, w, x, B, cache_len, kv, rope, ws, stream=None) -> None:
    _check(lib.qwen3_block_decode(ctypes.byref(cfg), ctypes.byref(w), _ptr(x), B, _ptr(cache_len), ctypes.byref(kv),
                                  _ptr(rope), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "block_decode")


def moe_block(cfg, w, x, B, T, start_pos, kv, rope, ws, topk_idx=None, topk_w=None, expert_offsets=None,
              perm_token=None, stream=None) -> None:
    _check(lib.qwen3_moe_block(ctypes.byref(cfg), ctypes.byref(w), _ptr(x), B, T, _ptr(start_pos), ctypes.byref(kv),
                               _ptr(rope), _ptr(topk_idx), _ptr(topk_w), _ptr(expert_offsets), _ptr(perm_token),
                               _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "moe_block")


def stack_forward(cfg, embed, layers, final_norm, ids, B, T, mode, pos_or_len, kvs, rope, logits, last_only, ws,
                  stream=None) -> None:
    """layers: list of LayerWeights; kvs: list of KVLayer (one per layer)."""
    n = len(layers)
    larr = (LayerWeights * n)(*layers)
    karr = (KVLayer * n)(*kvs)
    _check(lib.qwen3_stack_forward(ctypes.byref(cfg), _ptr(embed), larr, _ptr(final_norm), _ptr(ids), B, T, mode,
                                   _ptr(pos_or_len), karr, _ptr(rope), _ptr(logits), int(last_only), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)), "stack_forward")


def generate_greedy(cfg, embed, layers, final_norm, prompt_ids, B, T, n_new, kvs, rope, out_ids, ws,
                    stream=None) -> None:
    """Prefill the prompt, then n_new - 1 decode steps; out_ids [B, n_new] int32."""
    n = len(layers)
    larr = (LayerWeights * n)(*layers)
    karr = (KVLayer * n)(*kvs)
    _check(lib.qwen3_generate_greedy(ctypes.byref(cfg), _ptr(embed), larr, _ptr(final_norm), _ptr(prompt_ids), B, T,
                                     n_new, karr, _ptr(rope), _ptr(out_ids), _ptr(ws), ws.numel() * ws.element_size(),
                                     _stream(stream)), "generate_greedy")


# ------------------------------------------------------------------------- single kernels
def op_argmax(x, rows, V, out, ldx=None, ld_out=1, stream=None) -> None:
    _check(lib.qwen3_op_argmax(_ptr(x), ldx or V, rows, V, _ptr(out), ld_out, _stream(stream)), "op_argmax")


def op_rmsnorm(x, w, out, rows, n, eps, ldx=None, ldo=None, stream=None) -> None:
    """out: a bf16 tensor, or an fp16 one (the fp16 operand mode's projection input)."""
    import torch
    x_f32 = 1 if x.dtype == torch.float32 else 0
    out_f16 = 1 if out.dtype == torch.float16 else 0
    _check(lib.qwen3_op_rmsnorm(_ptr(x), x_f32, ldx or n, _ptr(w), _ptr(out), ldo or n, rows, n, eps, out_f16,
                                _stream(stream)), "op_rmsnorm")


def op_gemm(A, W, out, M, N, K, epilogue=EPI_STORE, resid=None, swap=-1, lda=None, ldw=None, ldo=None, ldr=None,
            ws=None, stream=None) -> None:
    """A and W both bf16 or both fp16 (torch dtypes decide the operand type)."""
    import torch
    out_f32 = 1 if out.dtype == torch.float32 else 0
    resid_f32 = 1 if (resid is not None and resid.dtype == torch.float32) else 0
    ab_f16 = 1 if A.dtype == torch.float16 else 0
    if (W.dtype == torch.float16) != bool(ab_f16):
        raise ValueError("op_gemm: A and W must share their type (bf16 or fp16)")
    if ldo is None:
        ldo = N // 2 if epilogue == EPI_SWIGLU else N
    _check(lib.qwen3_op_gemm(_ptr(A), lda or K, _ptr(W), ldw or K, _ptr(out), ldo, M, N, K, epilogue, _ptr(resid),
                             ldr or N, resid_f32, out_f32, swap, ab_f16, _ptr(ws),
                             0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)), "op_gemm")


def op_qk_norm_rope(cfg, qkv, B, T, pos_base, q_norm, k_norm, kv, rope, ldqkv=None, stream=None) -> None:
    ld = ldqkv or (cfg.n_q_heads + 2 * cfg.n_kv_heads) * cfg.head_dim
    _check(lib.qwen3_op_qk_norm_rope(ctypes.byref(cfg), _ptr(qkv), ld, B, T, _ptr(pos_base), _ptr(q_norm),
                                     _ptr(k_norm), ctypes.byref(kv), _ptr(rope), _stream(stream)), "op_qk_norm_rope")


def op_gemm_qkv_rope(cfg, h, w_qkv, qkv, B, T, pos_base, q_norm, k_norm, kv, rope, stream=None) -> None:
    _check(lib.qwen3_op_gemm_qkv_rope(ctypes.byref(cfg), _ptr(h), _ptr(w_qkv), _ptr(qkv), B, T, _ptr(pos_base),
                                      _ptr(q_norm), _ptr(k_norm), ctypes.byref(kv), _ptr(rope), _stream(stream)),
           "op_gemm_qkv_rope")


def op_attention_prefill(cfg, qkv, B, T, start_pos, kv, o, ldqkv=None, ldo=None, stream=None) -> None:
    ld = ldqkv or (cfg.n_q_heads + 2 * cfg.n_kv_heads) * cfg.head_dim
    _check(lib.qwen3_op_attention_prefill(ctypes.byref(cfg), _ptr(qkv), ld, B, T, _ptr(start_pos), ctypes.byref(kv),
                                          _ptr(o), ldo or cfg.n_q_heads * cfg.head_dim, _stream(stream)),
           "op_attention_prefill")


def op_attention_decode(cfg, qkv, B, cache_len, kv, o, ws, ldqkv=None, ldo=None, stream=None) -> None:
    ld = ldqkv or (cfg.n_q_heads + 2 * cfg.n_kv_heads) * cfg.head_dim
    _check(lib.qwen3_op_attention_decode(ctypes.byref(cfg), _ptr(qkv), ld, B, _ptr(cache_len), ctypes.byref(kv),
                                         _ptr(o), ldo or cfg.n_q_heads * cfg.head_dim, _ptr(ws),
                                         ws.numel() * ws.element_size(), _stream(stream)), "op_attention_decode")


def op_attention_decode_noalloc(cfg, qkv, B, cache_len, kv, o, ldqkv=None, ldo=None, stream=None) -> None:
    """Decode attention with the split scratch in the library's static device array
    (no caller workspace; see the header for the size limit and the sharing rules)."""
    ld = ldqkv or (cfg.n_q_heads + 2 * cfg.n_kv_heads) * cfg.head_dim
    _check(lib.qwen3_op_attention_decode_noalloc(ctypes.byref(cfg), _ptr(qkv), ld, B, _ptr(cache_len),
                                                 ctypes.byref(kv), _ptr(o), ldo or cfg.n_q_heads * cfg.head_dim,
                                                 _stream(stream)), "op_attention_decode_noalloc")


def op_embed(ids, n, embed, vocab, H, out, stream=None) -> None:
    import torch
    _check(lib.qwen3_op_embed(_ptr(ids), n, _ptr(embed), vocab, H, _ptr(out), 1 if out.dtype == torch.float32 else 0,
                              1 if embed.dtype == torch.float16 else 0, _stream(stream)), "op_embed")


def convert_to_f16(src, dst=None, stream=None):
    """bf16 -> fp16 (round to nearest even) into dst (a float16 tensor of the same size),
    or in place when dst is None; returns the fp16 view."""
    import torch
    n = src.numel()
    if dst is None:
        _check(lib.qwen3_convert_to_f16(_ptr(src), _ptr(src), n, _stream(stream)), "convert_to_f16")
        return src.view(torch.float16)
    if dst.numel() != n:
        raise ValueError("convert_to_f16: size mismatch")
    _check(lib.qwen3_convert_to_f16(_ptr(src), _ptr(dst), n, _stream(stream)), "convert_to_f16")
    return dst
