"""ctypes front of the fp64 C++ oracle (oracle/qwen3_ref.cpp) -- TEST INFRASTRUCTURE ONLY.

The same functions, signatures and return values as oracle/qwen3_ref.py, computed by
the C++ statement of the definitions, so that the pin suite (tests/oracle_pins.py) can
run against either oracle and the two can be checked against each other. This module
only marshals numpy arrays; it holds no arithmetic of the method. Only tests and the
benchmark's CPU-baseline leg may import it.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libqwen3ref.so")


# ---------------------------------------------------------------------------
# Configuration and weights (plain data, the pages' layouts as in qwen3_ref.py)
# ---------------------------------------------------------------------------
@dataclass
class Config:
    hidden: int = 1024
    n_q_heads: int = 16
    n_kv_heads: int = 8
    head_dim: int = 128
    intermediate: int = 3072
    vocab: int = 151936
    n_layers: int = 28
    max_pos: int = 40960
    rope_theta: float = 1.0e6
    rms_eps: float = 1.0e-6
    n_experts: int = 0
    top_k: int = 0
    moe_intermediate: int = 0
    norm_topk_prob: bool = True


QWEN3_0_6B = Config()


@dataclass
class LayerWeights:
    in_norm: np.ndarray
    wq: np.ndarray
    wk: np.ndarray
    wv: np.ndarray
    q_norm: np.ndarray
    k_norm: np.ndarray
    wo: np.ndarray
    post_norm: np.ndarray
    w_gate: Optional[np.ndarray] = None
    w_up: Optional[np.ndarray] = None
    w_down: Optional[np.ndarray] = None
    router: Optional[np.ndarray] = None
    gate_up: Optional[np.ndarray] = None
    down: Optional[np.ndarray] = None


class _Cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("hidden", "n_q_heads", "n_kv_heads", "head_dim", "intermediate",
                                              "vocab", "n_layers", "max_pos", "n_experts", "top_k",
                                              "moe_intermediate", "norm_topk_prob")] + \
               [("rope_theta", ctypes.c_double), ("rms_eps", ctypes.c_double)]


_LAYER_FIELDS = ("in_norm", "wq", "wk", "wv", "q_norm", "k_norm", "wo", "post_norm", "w_gate", "w_up", "w_down",
                 "router", "gate_up", "down")


class _Layer(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _LAYER_FIELDS]


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            from . import _build
            _build.build()
        _lib = ctypes.CDLL(LIB_PATH)
        _lib.q3ref_param_count.restype = ctypes.c_int64
        _lib.q3ref_kv_bytes_per_token_layer.restype = ctypes.c_int64
    return _lib


def _d(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _cfg(c: Config) -> _Cfg:
    return _Cfg(c.hidden, c.n_q_heads, c.n_kv_heads, c.head_dim, c.intermediate, c.vocab, c.n_layers, c.max_pos,
                c.n_experts, c.top_k, c.moe_intermediate, int(bool(c.norm_topk_prob)), float(c.rope_theta),
                float(c.rms_eps))


class _Pinned:
    """A layer's weights as contiguous float64 arrays kept alive with their struct."""

    def __init__(self, L: LayerWeights):
        self.arrays = {n: (None if getattr(L, n, None) is None else _d(getattr(L, n))) for n in _LAYER_FIELDS}
        self.s = _Layer(*[_p(self.arrays[n]) for n in _LAYER_FIELDS])


def bf16_to_f64(bits) -> np.ndarray:
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# The functions, as in qwen3_ref.py
# ---------------------------------------------------------------------------
def rms_norm(x, w, eps):
    x = _d(x)
    n = x.shape[-1]
    out = np.empty_like(x)
    lib().q3ref_rms_norm(_p(x), _p(_d(w)), ctypes.c_int64(x.size // n), ctypes.c_int64(n), ctypes.c_double(eps),
                         _p(out))
    return out


def rope_frequencies(head_dim, theta):
    out = np.empty(head_dim // 2)
    lib().q3ref_rope_frequencies(ctypes.c_int64(head_dim), ctypes.c_double(theta), _p(out))
    return out


def rope_rotate_half(u, positions, theta):
    u = _d(u)
    T, nh, d = u.shape
    out = np.empty_like(u)
    lib().q3ref_rope_rotate_half(_p(u), _p(_d(positions)), ctypes.c_int64(T), ctypes.c_int64(nh), ctypes.c_int64(d),
                                 ctypes.c_double(theta), _p(out))
    return out


def causal_allowed(q_pos, k_pos):
    qp, kp = _d(q_pos), _d(k_pos)
    out = np.empty((qp.size, kp.size), dtype=np.uint8)
    lib().q3ref_causal_allowed(_p(qp), _p(kp), ctypes.c_int64(qp.size), ctypes.c_int64(kp.size), _p(out))
    return out.astype(bool)


def causal_gqa_attention(q, k, v, q_pos, k_pos):
    q, k, v = _d(q), _d(k), _d(v)
    tq, hq, d = q.shape
    tk, hkv, _ = k.shape
    out = np.empty_like(q)
    lib().q3ref_causal_gqa_attention(_p(q), _p(k), _p(v), _p(_d(q_pos)), _p(_d(k_pos)), ctypes.c_int64(tq),
                                     ctypes.c_int64(tk), ctypes.c_int64(hq), ctypes.c_int64(hkv), ctypes.c_int64(d),
                                     _p(out))
    return out


def silu(z):
    z = _d(z)
    out = np.empty_like(z)
    lib().q3ref_silu(_p(z), ctypes.c_int64(z.size), _p(out))
    return out


def swiglu_ffn(h, w_gate, w_up, w_down):
    h = _d(h)
    T, H = h.shape
    I = w_gate.shape[0]
    out = np.empty((T, H))
    lib().q3ref_swiglu_ffn(_p(h), _p(_d(w_gate)), _p(_d(w_up)), _p(_d(w_down)), ctypes.c_int64(T), ctypes.c_int64(H),
                           ctypes.c_int64(I), _p(out))
    return out


def _rows(T, rows):
    if rows is None:
        return None, T
    r = np.ascontiguousarray(rows, dtype=np.int64)
    return r, r.size


def _cache(cfg, cache_k, cache_v, cache_pos):
    if cache_k is None or cache_k.shape[0] == 0:
        return None, None, None, 0
    return _d(cache_k), _d(cache_v), _d(cache_pos), cache_k.shape[0]


def attention_half(x, L, cfg, positions, cache_k=None, cache_v=None, cache_pos=None, rows=None):
    x = _d(x)
    T = x.shape[0]
    ck, cv, cp, S = _cache(cfg, cache_k, cache_v, cache_pos)
    r, n = _rows(T, rows)
    W = _Pinned(L)
    x1 = np.empty((n, cfg.hidden))
    kn = np.empty((T, cfg.n_kv_heads, cfg.head_dim))
    vn = np.empty_like(kn)
    c = _cfg(cfg)
    lib().q3ref_attention_half(ctypes.byref(c), ctypes.byref(W.s), _p(x), ctypes.c_int64(T), _p(_d(positions)), _p(ck),
                               _p(cv), _p(cp), ctypes.c_int64(S), _p(r), ctypes.c_int64(n), _p(x1), _p(kn), _p(vn))
    return x1, kn, vn


def dense_ffn_half(x1, L, cfg):
    x1 = _d(x1)
    out = np.empty_like(x1)
    W = _Pinned(L)
    c = _cfg(cfg)
    lib().q3ref_dense_ffn_half(ctypes.byref(c), ctypes.byref(W.s), _p(x1), ctypes.c_int64(x1.shape[0]), _p(out))
    return out


def block_forward(x, L, cfg, positions, cache_k=None, cache_v=None, cache_pos=None, rows=None):
    x = _d(x)
    T = x.shape[0]
    ck, cv, cp, S = _cache(cfg, cache_k, cache_v, cache_pos)
    r, n = _rows(T, rows)
    W = _Pinned(L)
    out = np.empty((n, cfg.hidden))
    kn = np.empty((T, cfg.n_kv_heads, cfg.head_dim))
    vn = np.empty_like(kn)
    c = _cfg(cfg)
    lib().q3ref_block_forward(ctypes.byref(c), ctypes.byref(W.s), _p(x), ctypes.c_int64(T), _p(_d(positions)), _p(ck),
                              _p(cv), _p(cp), ctypes.c_int64(S), _p(r), ctypes.c_int64(n), _p(out), _p(kn), _p(vn))
    return out, kn, vn


def moe_route(h2, router, top_k, norm_topk_prob=True):
    h2, router = _d(h2), _d(router)
    T, H = h2.shape
    E = router.shape[0]
    idx = np.empty((T, top_k), dtype=np.int32)
    w = np.empty((T, top_k))
    probs = np.empty((T, E))
    margin = np.empty(T)
    lib().q3ref_moe_route(_p(h2), _p(router), ctypes.c_int64(T), ctypes.c_int64(E), ctypes.c_int64(H),
                          ctypes.c_int64(top_k), ctypes.c_int(int(bool(norm_topk_prob))), _p(idx), _p(w), _p(probs),
                          _p(margin))
    return idx, w, probs, margin


def moe_permutation(idx, n_experts):
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    offsets = np.empty(n_experts + 1, dtype=np.int64)
    tok = np.empty(T * k, dtype=np.int64)
    slot = np.empty(T * k, dtype=np.int64)
    lib().q3ref_moe_permutation(_p(idx), ctypes.c_int64(T), ctypes.c_int64(k), ctypes.c_int64(n_experts), _p(offsets),
                                _p(tok), _p(slot))
    return offsets, tok, slot


def moe_ffn(h2, idx, w, gate_up, down):
    h2 = _d(h2)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    H = down.shape[1]
    Im = gate_up.shape[1] // 2
    out = np.empty((T, H))
    lib().q3ref_moe_ffn(_p(h2), _p(idx), _p(_d(w)), _p(_d(gate_up)), _p(_d(down)), ctypes.c_int64(T),
                        ctypes.c_int64(k), ctypes.c_int64(H), ctypes.c_int64(Im), _p(out))
    return out


def moe_ffn_half(x1, L, cfg, idx=None, w=None):
    x1 = _d(x1)
    T = x1.shape[0]
    k, E = cfg.top_k, cfg.n_experts
    W = _Pinned(L)
    c = _cfg(cfg)
    out = np.empty_like(x1)
    ri = np.empty((T, k), dtype=np.int32)
    rw = np.empty((T, k))
    given = idx is not None
    gi = np.ascontiguousarray(idx, dtype=np.int32) if given else None
    gw = _d(w) if given else None
    probs = None if given else np.empty((T, E))
    margin = None if given else np.empty(T)
    lib().q3ref_moe_ffn_half(ctypes.byref(c), ctypes.byref(W.s), _p(x1), ctypes.c_int64(T), _p(gi), _p(gw), _p(out),
                             _p(ri), _p(rw), _p(probs), _p(margin))
    return out, (ri, rw, probs, margin)


def moe_block_forward(x, L, cfg, positions, rows=None):
    x1, k, v = attention_half(x, L, cfg, positions, rows=rows)
    out, route = moe_ffn_half(x1, L, cfg)
    return out, k, v, route


def stack_forward(ids, embed, layers, final_norm, cfg, positions=None, caches=None, logit_rows=None):
    ids = np.ascontiguousarray(ids, dtype=np.int64)
    T = ids.size
    pos = _d(np.arange(T) if positions is None else positions)
    rows = np.ascontiguousarray(np.arange(T) if logit_rows is None else logit_rows, dtype=np.int64)
    nL = len(layers)
    pinned = [_Pinned(L) for L in layers]
    larr = (_Layer * nL)(*[p.s for p in pinned])
    keep = []
    PtrArr = ctypes.c_void_p * nL
    ck, cv, cp = PtrArr(), PtrArr(), PtrArr()
    clen = np.zeros(nL, dtype=np.int64)
    if caches is not None:
        for l, cache in enumerate(caches):
            if cache is None or cache[0].shape[0] == 0:
                continue
            a, b, p = _d(cache[0]), _d(cache[1]), _d(cache[2])
            keep += [a, b, p]
            ck[l], cv[l], cp[l] = a.ctypes.data, b.ctypes.data, p.ctypes.data
            clen[l] = a.shape[0]
    kn = [np.empty((T, cfg.n_kv_heads, cfg.head_dim)) for _ in range(nL)]
    vn = [np.empty_like(a) for a in kn]
    kp, vp = PtrArr(*[a.ctypes.data for a in kn]), PtrArr(*[a.ctypes.data for a in vn])
    logits = np.empty((rows.size, cfg.vocab))
    c = _cfg(cfg)
    E = _d(embed)
    lib().q3ref_stack_forward(ctypes.byref(c), _p(ids), ctypes.c_int64(T), _p(E), larr, _p(_d(final_norm)), _p(pos),
                              ck, cv, cp, _p(clen), _p(rows), ctypes.c_int64(rows.size), _p(logits), kp, vp)
    return logits, list(zip(kn, vn))


def param_count(cfg, tied):
    c = _cfg(cfg)
    return int(lib().q3ref_param_count(ctypes.byref(c), ctypes.c_int(int(bool(tied)))))


def kv_bytes_per_token_layer(cfg, bytes_per_elem=2):
    c = _cfg(cfg)
    return int(lib().q3ref_kv_bytes_per_token_layer(ctypes.byref(c), ctypes.c_int(bytes_per_elem)))
