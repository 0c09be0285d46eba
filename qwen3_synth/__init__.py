"""Seeded synthetic inputs shared by the CUDA path's tests, the oracle and the benchmark.

A package of its own, apart from the library: it holds no arithmetic of the decoder
block, imports nothing of the library or of the oracle, and neither imports it. It only defines how the
random weights, activations, token ids and cached keys/values of the synthetic
workloads are drawn, so that every consumer sees identical bits.

Definition (counter based, so any slice of any tensor can be regenerated alone):

    mix64(z)   = SplitMix64 finaliser:
                 z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
                 z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31   (mod 2^64)
    key        = mix64(mix64(seed) + tensor_id * GAMMA),  GAMMA = 0x9E3779B97F4A7C15
    word(i)    = mix64(key + (i + 1) * GAMMA)
    normal(i)  : u1 = ((word(2i) >> 11) + 1) * 2^-53         in (0, 1]
                 u2 =  (word(2i+1) >> 11)     * 2^-53         in [0, 1)
                 z  = sqrt(-2 ln u1) * cos(2 pi u2)            (Box-Muller, cosine branch)
                 value = mean + std * z, rounded to fp32 (nearest-even), then to bf16
                 (nearest-even)
    int(i, n)  = floor(word(i) * n / 2^64)                    uniform in [0, n)

`i` is the element's row-major index in the tensor's logical shape. The same
definition is implemented three times: vectorised numpy here (the reference),
host C++ with OpenMP and a CUDA kernel (``csrc/synth.cu``) for tensors too large
for numpy. Tests check that all three agree bit for bit.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK = (1 << 64) - 1


def _mix64_int(z: int) -> int:
    z &= _MASK
    z = ((z ^ (z >> 30)) * _M1) & _MASK
    z = ((z ^ (z >> 27)) * _M2) & _MASK
    return z ^ (z >> 31)


def stream_key(seed: int, tensor_id: int) -> int:
    return _mix64_int((_mix64_int(seed) + tensor_id * GAMMA) & _MASK)


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * np.uint64(_M1)
    z = z ^ (z >> np.uint64(27))
    z = z * np.uint64(_M2)
    return z ^ (z >> np.uint64(31))


def _words(key: int, idx: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return _mix64(np.uint64(key) + (idx.astype(np.uint64) + np.uint64(1)) * np.uint64(GAMMA))


def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest-even); NaN maps to the canonical quiet NaN."""
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    out = r.astype(np.uint16)
    nan = np.isnan(f)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    return (np.asarray(u, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(seed: int, tensor_id: int, shape, mean: float = 0.0, std: float = 1.0,
                index_base: int = 0) -> np.ndarray:
    """bf16 bits (uint16) of N(mean, std) draws for logical indices index_base + [0, prod(shape))."""
    n = int(np.prod(shape)) if len(shape) else 1
    key = stream_key(seed, tensor_id)
    out = np.empty(n, dtype=np.uint16)
    chunk = 1 << 22
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        i = np.arange(index_base + s, index_base + e, dtype=np.uint64)
        w1 = _words(key, i * np.uint64(2))
        w2 = _words(key, i * np.uint64(2) + np.uint64(1))
        u1 = ((w1 >> np.uint64(11)) + np.uint64(1)).astype(np.float64) * 2.0 ** -53
        u2 = (w2 >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
        z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
        v = (mean + std * z).astype(np.float32)
        out[s:e] = f32_to_bf16_bits(v)
    return out.reshape(shape)


def uniform_int(seed: int, tensor_id: int, shape, upper: int, index_base: int = 0) -> np.ndarray:
    """int32 draws uniform in [0, upper) (upper < 2^31)."""
    n = int(np.prod(shape)) if len(shape) else 1
    key = stream_key(seed, tensor_id)
    i = np.arange(index_base, index_base + n, dtype=np.uint64)
    w = _words(key, i)
    hi = w >> np.uint64(32)
    lo = w & np.uint64(0xFFFFFFFF)
    up = np.uint64(upper)
    with np.errstate(over="ignore"):
        t = hi * up + ((lo * up) >> np.uint64(32))
    return (t >> np.uint64(32)).astype(np.int32).reshape(shape)


# ---------------------------------------------------------------------------
# Tensor ids of the synthetic workloads (fixed; part of the input definition).
# ---------------------------------------------------------------------------
TID_EMBED = 1
TID_FINAL_NORM = 2
TID_X = 3
TID_IDS = 4
TID_IDS_STEP = 5          # decode step s draws its ids from tensor TID_IDS_STEP, index s*B + b
LAYER_BASE = 100
LAYER_STRIDE = 32
(L_IN_NORM, L_WQ, L_WK, L_WV, L_Q_NORM, L_K_NORM, L_WO, L_POST_NORM, L_WGATE, L_WUP, L_WDOWN,
 L_ROUTER, L_MOE_GATE_UP, L_MOE_DOWN, L_CACHE_K, L_CACHE_V) = range(16)


def layer_tid(layer: int, which: int) -> int:
    return LAYER_BASE + layer * LAYER_STRIDE + which


# Distributions of the synthetic workloads: projection and embedding weights
# N(0, 0.02); norm weights 1 + N(0, 0.1); activations N(0, 1); cached K/V N(0, 1).
W_STD = 0.02
NORM_MEAN, NORM_STD = 1.0, 0.1


# ---------------------------------------------------------------------------
# Native implementations (host OpenMP and CUDA) of the same definition.
# ---------------------------------------------------------------------------
_native = None


def native():
    """ctypes handle of libqwen3synth.so (host + device generators). Raises if not built."""
    global _native
    if _native is None:
        path = os.path.join(os.path.dirname(__file__), "lib", "libqwen3synth.so")
        if not os.path.exists(path):
            from . import _build
            _build.build()
        lib = ctypes.CDLL(path)
        i64, u64, dbl, vp = ctypes.c_int64, ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p
        lib.qwen3synth_normal_bf16_host.argtypes = [vp, i64, i64, i64, i64, i64, i64, u64, u64, dbl, dbl]
        lib.qwen3synth_normal_bf16_device.argtypes = [vp, i64, i64, i64, i64, i64, i64, u64, u64, dbl, dbl, vp]
        lib.qwen3synth_uniform_int_host.argtypes = [vp, i64, i64, u64, u64, i64]
        lib.qwen3synth_uniform_int_device.argtypes = [vp, i64, i64, u64, u64, i64, vp]
        for f in (lib.qwen3synth_normal_bf16_host, lib.qwen3synth_normal_bf16_device,
                  lib.qwen3synth_uniform_int_host, lib.qwen3synth_uniform_int_device):
            f.restype = ctypes.c_int
        _native = lib
    return _native


def normal_bf16_fast(seed: int, tensor_id: int, shape, mean: float = 0.0, std: float = 1.0,
                     index_base: int = 0) -> np.ndarray:
    """Same values as normal_bf16, drawn by the OpenMP host generator."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.uint16)
    rc = native().qwen3synth_normal_bf16_host(out.ctypes.data, 1, 1, n, 0, 0, index_base,
                                              seed, tensor_id, mean, std)
    if rc != 0:
        raise RuntimeError(f"qwen3synth_normal_bf16_host failed ({rc})")
    return out.reshape(shape)


def normal_bf16_device(dst_ptr: int, n0: int, n1: int, n2: int, s0: int, s1: int, seed: int,
                       tensor_id: int, mean: float, std: float, index_base: int = 0,
                       stream: int = 0) -> None:
    """Fill a strided device bf16 buffer: element (i0,i1,i2) with logical index
    index_base + (i0*n1 + i1)*n2 + i2 goes to dst[i0*s0 + i1*s1 + i2] (element units)."""
    rc = native().qwen3synth_normal_bf16_device(dst_ptr, n0, n1, n2, s0, s1, index_base, seed,
                                                tensor_id, mean, std, stream)
    if rc != 0:
        raise RuntimeError(f"qwen3synth_normal_bf16_device failed ({rc})")


def uniform_int_device(dst_ptr: int, n: int, seed: int, tensor_id: int, upper: int,
                       index_base: int = 0, stream: int = 0) -> None:
    rc = native().qwen3synth_uniform_int_device(dst_ptr, n, index_base, seed, tensor_id, upper, stream)
    if rc != 0:
        raise RuntimeError(f"qwen3synth_uniform_int_device failed ({rc})")
