"""Per-kernel GPU parity against the fp64 oracle, through the C ABI (ops)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle.qwen3_ref as R  # noqa: E402
from helpers import (Tensor, assert_device_ok, from_gpu_bf16, kv_cache, max_abs, oracle_config, rel_frob,  # noqa: E402
                     rope_gpu, to_f16, workspace)

SEED = 7


@pytest.fixture(scope="module")
def q3():
    import qwen3_decoder_block_b200 as m
    return m


def bf16_tol(ref, rel=2.0 ** -8, abs_=1e-6):
    return rel * np.abs(ref) + abs_


def f16_tol(ref, abs_=1e-6):
    """One rounding to fp16 (relative 2^-11) on top of fp32 accumulation."""
    return 2.0 ** -11 * np.abs(ref) + abs_


def f64_of(t):
    """float64 numpy copy of a bf16 / fp16 / fp32 GPU tensor (exact widening)."""
    return t.detach().cpu().double().numpy()


@pytest.mark.parametrize("n", [1024, 2048])
@pytest.mark.parametrize("f32_in", [False, True])
@pytest.mark.parametrize("rows", [1, 37, 1000])
def test_rmsnorm(q3, n, f32_in, rows):
    x = Tensor(SEED, 11, (rows, n))
    w = Tensor(SEED, 12, (n,), 1.0, 0.1)
    xin = x.gpu.float() if f32_in else x.gpu
    out = torch.empty((rows, n), dtype=torch.bfloat16, device="cuda")
    q3.op_rmsnorm(xin, w.gpu, out, rows, n, 1e-6)
    assert_device_ok()
    ref = R.rms_norm(x.f, w.f, 1e-6)
    got = from_gpu_bf16(out)
    assert np.all(np.abs(got - ref) <= bf16_tol(ref, abs_=1e-5))


GEMM_SHAPES = [(16, 4096, 1024), (64, 1024, 2048), (200, 512, 192), (300, 6144, 1024), (1000, 1024, 3072),
               (130, 96, 64), (257, 288, 128)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
@pytest.mark.parametrize("swap", [0, 1])
def test_gemm_store(q3, M, N, K, swap):
    A = Tensor(SEED, 21, (M, K))
    W = Tensor(SEED, 22, (N, K), 0.0, 0.02)
    ref = A.f @ W.f.T
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    q3.op_gemm(A.gpu, W.gpu, out, M, N, K, swap=swap)
    out32 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    q3.op_gemm(A.gpu, W.gpu, out32, M, N, K, swap=swap)
    assert_device_ok()
    got = from_gpu_bf16(out)
    assert np.all(np.abs(got - ref) <= bf16_tol(ref, abs_=1e-4 * np.sqrt(K / 1024))), max_abs(got, ref)
    got32 = out32.cpu().double().numpy()
    assert max_abs(got32, ref) <= 2e-5 * np.sqrt(K / 1024) * 8, max_abs(got32, ref)


@pytest.mark.parametrize("M,N,K", [(16, 1024, 2048), (77, 1024, 3072), (600, 2048, 1024)])
@pytest.mark.parametrize("swap", [0, 1])
@pytest.mark.parametrize("rt,ot", [("bf16", "f32"), ("f32", "bf16"), ("f32", "f32")])
def test_gemm_residual(q3, M, N, K, swap, rt, ot):
    A = Tensor(SEED, 31, (M, K))
    W = Tensor(SEED, 32, (N, K), 0.0, 0.02)
    Xr = Tensor(SEED, 33, (M, N))
    resid = Xr.gpu if rt == "bf16" else Xr.gpu.float()
    out = torch.empty((M, N), dtype=torch.float32 if ot == "f32" else torch.bfloat16, device="cuda")
    q3.op_gemm(A.gpu, W.gpu, out, M, N, K, epilogue=q3.EPI_RESID, resid=resid, swap=swap)
    assert_device_ok()
    ref = Xr.f + A.f @ W.f.T
    got = out.cpu().double().numpy() if ot == "f32" else from_gpu_bf16(out)
    tol = 1e-4 if ot == "f32" else bf16_tol(ref, abs_=1e-4)
    assert np.all(np.abs(got - ref) <= tol), max_abs(got, ref)


@pytest.mark.parametrize("M,N,K,epi", [(64, 1024, 2048, 1), (64, 6144, 1024, 2), (16, 4096, 1024, 0),
                                       (64, 1024, 3072, 1), (200, 512, 1024, 0), (3, 4736, 1024, 0)])
@pytest.mark.parametrize("out_f32", [0, 1])
@pytest.mark.parametrize("swap", [1, 0])
def test_gemm_split_k(q3, M, N, K, epi, out_f32, swap):
    """Small-M GEMMs split K across CTAs (fp32 partials + reduce with the epilogue),
    with tokens on the MMA's N side (swap) or on its 128-row side."""
    if epi == 2 and out_f32:
        pytest.skip("SwiGLU output is bf16")
    A = Tensor(SEED, 37, (M, K))
    W = Tensor(SEED, 38, (N, K), 0.0, 0.02)
    X = Tensor(SEED, 39, (M, N))
    n_out = N // 2 if epi == 2 else N
    out = torch.empty((M, n_out), dtype=torch.float32 if out_f32 else torch.bfloat16, device="cuda")
    ws = torch.empty(64 << 20, dtype=torch.uint8, device="cuda")
    resid = X.gpu.float() if epi == 1 else None
    packed = W.gpu
    if epi == 2:
        packed = torch.empty_like(W.gpu)
        q3.pack_gate_up(N // 2, K, W.gpu[:N // 2], W.gpu[N // 2:], packed)
    q3.op_gemm(A.gpu, packed, out, M, N, K, epilogue=epi, resid=resid, swap=swap, ws=ws)
    assert_device_ok()
    acc = A.f @ W.f.T
    if epi == 2:
        ref = R.silu(acc[:, :N // 2]) * acc[:, N // 2:]
    elif epi == 1:
        ref = X.f + acc
    else:
        ref = acc
    got = out.cpu().double().numpy() if out_f32 else from_gpu_bf16(out)
    tol = 1e-4 if out_f32 else bf16_tol(ref, abs_=2e-4)
    assert np.all(np.abs(got - ref) <= tol), max_abs(got, ref)


def test_gemm_residual_in_place(q3):
    M, N, K = 300, 1024, 1024
    A = Tensor(SEED, 34, (M, K))
    W = Tensor(SEED, 35, (N, K), 0.0, 0.02)
    X = Tensor(SEED, 36, (M, N))
    x = X.gpu.float().clone()
    q3.op_gemm(A.gpu, W.gpu, x, M, N, K, epilogue=q3.EPI_RESID, resid=x, swap=0)
    assert_device_ok()
    assert max_abs(x.cpu().double().numpy(), X.f + A.f @ W.f.T) < 1e-4


@pytest.mark.parametrize("M,I,K", [(16, 3072, 1024), (64, 768, 2048), (333, 3072, 1024), (129, 64, 128)])
@pytest.mark.parametrize("swap", [0, 1])
def test_gemm_swiglu(q3, M, I, K, swap):
    A = Tensor(SEED, 41, (M, K))
    Wg = Tensor(SEED, 42, (I, K), 0.0, 0.02)
    Wu = Tensor(SEED, 43, (I, K), 0.0, 0.02)
    packed = torch.empty((2 * I, K), dtype=torch.bfloat16, device="cuda")
    q3.pack_gate_up(I, K, Wg.gpu, Wu.gpu, packed)
    out = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
    q3.op_gemm(A.gpu, packed, out, M, 2 * I, K, epilogue=q3.EPI_SWIGLU, swap=swap)
    assert_device_ok()
    ref = R.silu(A.f @ Wg.f.T) * (A.f @ Wu.f.T)
    got = from_gpu_bf16(out)
    assert np.all(np.abs(got - ref) <= bf16_tol(ref, abs_=2e-4)), max_abs(got, ref)


def _rope_case(q3, cfg, B, T, starts, s_max):
    D, hq, hkv = cfg.head_dim, cfg.n_q_heads, cfg.n_kv_heads
    nqkv = (hq + 2 * hkv) * D
    qkv = Tensor(SEED, 51, (B * T, nqkv), 0.0, 0.6)
    qn = Tensor(SEED, 52, (D,), 1.0, 0.1)
    kn = Tensor(SEED, 53, (D,), 1.0, 0.1)
    k, v, kv = kv_cache(cfg, B, s_max)
    rope = rope_gpu(cfg)
    pos = torch.tensor(starts, dtype=torch.int32, device="cuda")
    buf = qkv.gpu.clone()
    q3.op_qk_norm_rope(cfg, buf, B, T, pos, qn.gpu, kn.gpu, kv, rope)
    assert_device_ok()
    return qkv, qn, kn, buf, k, v


def test_qk_norm_rope(q3):
    cfg = q3.config_qwen3_0_6b()
    B, T, s_max = 2, 37, 40000
    starts = [0, 39000]
    qkv, qn, kn, buf, k, v = _rope_case(q3, cfg, B, T, starts, s_max)
    D, hq, hkv = cfg.head_dim, cfg.n_q_heads, cfg.n_kv_heads
    got = from_gpu_bf16(buf)
    for b in range(B):
        rows = qkv.f[b * T:(b + 1) * T]
        pos = starts[b] + np.arange(T)
        q = R.rope_rotate_half(R.rms_norm(rows[:, :hq * D].reshape(T, hq, D), qn.f, 1e-6), pos, 1e6)
        kk = R.rope_rotate_half(R.rms_norm(rows[:, hq * D:(hq + hkv) * D].reshape(T, hkv, D), kn.f, 1e-6), pos, 1e6)
        vv = rows[:, (hq + hkv) * D:].reshape(T, hkv, D)
        gq = got[b * T:(b + 1) * T, :hq * D].reshape(T, hq, D)
        assert np.all(np.abs(gq - q) <= bf16_tol(q, abs_=2e-5)), max_abs(gq, q)
        gk = from_gpu_bf16(k[b][:, starts[b]:starts[b] + T]).transpose(1, 0, 2)
        gv = from_gpu_bf16(v[b][:, starts[b]:starts[b] + T]).transpose(1, 0, 2)
        assert np.all(np.abs(gk - kk) <= bf16_tol(kk, abs_=2e-5)), max_abs(gk, kk)
        np.testing.assert_array_equal(gv, vv)
        # positions outside [start, start+T) untouched (still NaN)
        assert bool(torch.isnan(k[b][:, :starts[b]].float()).all()) and bool(torch.isnan(k[b][:, starts[b] + T:].float()).all())


@pytest.mark.parametrize("B,T,starts", [(1, 300, [0]), (2, 200, [17, 3000]), (3, 129, [0, 1, 40000 - 140])])
def test_gemm_qkv_rope_fused(q3, B, T, starts):
    """QKV GEMM whose epilogue does QK-norm + RoPE + KV write on the fp32 accumulators."""
    cfg = q3.config_qwen3_0_6b()
    D, hq, hkv, H = cfg.head_dim, cfg.n_q_heads, cfg.n_kv_heads, cfg.hidden
    nqkv = (hq + 2 * hkv) * D
    s_max = max(starts) + T + 3
    h = Tensor(SEED, 91, (B * T, H))
    w = Tensor(SEED, 92, (nqkv, H), 0.0, 0.02)
    qn = Tensor(SEED, 93, (D,), 1.0, 0.1)
    kn = Tensor(SEED, 94, (D,), 1.0, 0.1)
    k, v, kv = kv_cache(cfg, B, s_max)
    qkv = torch.full((B * T, nqkv), float("nan"), dtype=torch.bfloat16, device="cuda")
    pos = torch.tensor(starts, dtype=torch.int32, device="cuda")
    q3.op_gemm_qkv_rope(cfg, h.gpu, w.gpu, qkv, B, T, pos, qn.gpu, kn.gpu, kv, rope_gpu(cfg))
    assert_device_ok()
    acc = h.f @ w.f.T
    got_q = from_gpu_bf16(qkv[:, :hq * D])
    for b in range(B):
        rows = acc[b * T:(b + 1) * T]
        p = starts[b] + np.arange(T)
        q = R.rope_rotate_half(R.rms_norm(rows[:, :hq * D].reshape(T, hq, D), qn.f, 1e-6), p, 1e6)
        kk = R.rope_rotate_half(R.rms_norm(rows[:, hq * D:(hq + hkv) * D].reshape(T, hkv, D), kn.f, 1e-6), p, 1e6)
        vv = rows[:, (hq + hkv) * D:].reshape(T, hkv, D)
        gq = got_q[b * T:(b + 1) * T].reshape(T, hq, D)
        gk = from_gpu_bf16(k[b][:, starts[b]:starts[b] + T]).transpose(1, 0, 2)
        gv = from_gpu_bf16(v[b][:, starts[b]:starts[b] + T]).transpose(1, 0, 2)
        for got, ref in ((gq, q), (gk, kk), (gv, vv)):
            assert np.all(np.abs(got - ref) <= bf16_tol(ref, abs_=1e-4)), max_abs(got, ref)


def _attention_oracle(cfg, qf, kf, vf, starts, B, T):
    """qf [B*T, Hq, D]; kf, vf [B, Hkv, S, D] cache contents; returns [B*T, Hq, D]."""
    out = []
    for b in range(B):
        L = starts[b] + T
        keys = kf[b][:, :L].transpose(1, 0, 2)
        vals = vf[b][:, :L].transpose(1, 0, 2)
        out.append(R.causal_gqa_attention(qf[b * T:(b + 1) * T], keys, vals, starts[b] + np.arange(T), np.arange(L)))
    return np.concatenate(out)


@pytest.mark.parametrize("hq,hkv", [(16, 8), (32, 4), (8, 8)])
@pytest.mark.parametrize("B,T,starts", [(1, 16, [0]), (2, 200, [0, 37]), (1, 300, [129]), (3, 1, [5, 0, 127]),
                                        (1, 1030, [0])])
def test_attention_prefill(q3, hq, hkv, B, T, starts):
    cfg = q3.make_config(n_q_heads=hq, n_kv_heads=hkv, hidden=2048 if hq == 32 else 1024)
    D = cfg.head_dim
    nqkv = (hq + 2 * hkv) * D
    s_max = max(starts) + T + 61
    qkv = Tensor(SEED, 61, (B * T, nqkv))
    kall = Tensor(SEED, 62, (B, hkv, s_max, D))
    vall = Tensor(SEED, 63, (B, hkv, s_max, D))
    k, v, kv = kv_cache(cfg, B, s_max)
    # cache: positions < start + T hold keys/values; the rest stays NaN
    for b in range(B):
        L = starts[b] + T
        k[b, :, :L] = kall.gpu[b, :, :L]
        v[b, :, :L] = vall.gpu[b, :, :L]
    o = torch.empty((B * T, hq * D), dtype=torch.bfloat16, device="cuda")
    pos = torch.tensor(starts, dtype=torch.int32, device="cuda")
    q3.op_attention_prefill(cfg, qkv.gpu, B, T, pos, kv, o)
    assert_device_ok()
    qf = qkv.f[:, :hq * D].reshape(B * T, hq, D)
    ref = _attention_oracle(cfg, qf, kall.f, vall.f, starts, B, T).reshape(B * T, hq * D)
    got = from_gpu_bf16(o)
    assert np.isfinite(got).all()
    # bound: bf16 rounding of the output (<= 2^-8 |o|) plus bf16 rounding of each softmax
    # weight in P.V (<= 2^-9 p_j |v_j|, summed: <= 2^-9 max|v|), plus fp32 slack
    vmax = np.abs(vall.f).max()
    tol = 2.0 ** -8 * np.abs(ref) + 2.0 ** -9 * vmax + 1e-4
    assert np.all(np.abs(got - ref) <= tol), (max_abs(got, ref), rel_frob(got, ref))
    assert rel_frob(got, ref) <= 1e-2


@pytest.mark.parametrize("hq,hkv", [(16, 8), (32, 4), (8, 8), (16, 4), (32, 2)])
@pytest.mark.parametrize("lens", [[0, 129, 598], [4095, 4096, 1, 200], [127, 255, 256]])
def test_attention_decode(q3, hq, hkv, lens):
    cfg = q3.make_config(n_q_heads=hq, n_kv_heads=hkv, hidden=2048 if hq == 32 else 1024)
    D = cfg.head_dim
    B = len(lens)
    s_max = max(lens) + 2
    nqkv = (hq + 2 * hkv) * D
    qkv = Tensor(SEED, 71, (B, nqkv))
    kall = Tensor(SEED, 72, (B, hkv, s_max, D))
    vall = Tensor(SEED, 73, (B, hkv, s_max, D))
    k, v, kv = kv_cache(cfg, B, s_max)
    for b in range(B):
        k[b, :, :lens[b] + 1] = kall.gpu[b, :, :lens[b] + 1]
        v[b, :, :lens[b] + 1] = vall.gpu[b, :, :lens[b] + 1]
    o = torch.empty((B, hq * D), dtype=torch.bfloat16, device="cuda")
    ws = workspace(cfg, q3.OP_BLOCK_DECODE, B, 1, s_max)
    cl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    q3.op_attention_decode(cfg, qkv.gpu, B, cl, kv, o, ws)
    assert_device_ok()
    got = from_gpu_bf16(o)
    for b in range(B):
        L = lens[b] + 1
        q = qkv.f[b, :hq * D].reshape(1, hq, D)
        ref = R.causal_gqa_attention(q, kall.f[b][:, :L].transpose(1, 0, 2), vall.f[b][:, :L].transpose(1, 0, 2),
                                     np.array([lens[b]]), np.arange(L)).reshape(-1)
        # fp32 scores, softmax and accumulation; P is rounded to bf16 for the P.V product
        # (relative 2^-9 per weight: at most 2^-9 max|v| on the normalised output) and the
        # output to bf16 (2^-8 |o|)
        vmax = np.abs(vall.f[b][:, :L]).max()
        tol = 2.0 ** -8 * np.abs(ref) + 2.0 ** -9 * vmax + 1e-4
        assert np.all(np.abs(got[b] - ref) <= tol), (b, max_abs(got[b], ref))


def test_embed(q3):
    V, H, n = 4096, 1024, 333
    E = Tensor(SEED, 81, (V, H), 0.0, 0.02)
    ids_np = np.random.default_rng(3).integers(0, V, n).astype(np.int32)
    ids = torch.from_numpy(ids_np).cuda()
    out = torch.empty((n, H), dtype=torch.float32, device="cuda")
    q3.op_embed(ids, n, E.gpu, V, H, out)
    outb = torch.empty((n, H), dtype=torch.bfloat16, device="cuda")
    q3.op_embed(ids, n, E.gpu, V, H, outb)
    assert_device_ok()
    np.testing.assert_array_equal(out.cpu().double().numpy(), E.f[ids_np])
    np.testing.assert_array_equal(from_gpu_bf16(outb), E.f[ids_np])


def test_synth_device_matches_host(q3):
    import qwen3_synth as synth
    n0, n1, n2, s1 = 3, 50, 128, 200 * 128
    buf = torch.zeros((n0, 200, n2), dtype=torch.bfloat16, device="cuda")
    synth.normal_bf16_device(buf.data_ptr(), n0, n1, n2, 200 * 128, 128, 11, 12, 0.0, 1.0, index_base=777)
    ids = torch.zeros(5000, dtype=torch.int32, device="cuda")
    synth.uniform_int_device(ids.data_ptr(), 5000, 11, 13, 151936)
    torch.cuda.synchronize()
    host = synth.normal_bf16(11, 12, (n0, n1, n2), 0.0, 1.0, index_base=777)
    got = buf[:, :n1].contiguous().cpu().view(torch.uint16).numpy()
    np.testing.assert_array_equal(got, host)
    assert bool((buf[:, n1:] == 0).all())
    np.testing.assert_array_equal(ids.cpu().numpy(), synth.uniform_int(11, 13, (5000,), 151936))


def test_convert_to_f16_rounds_like_torch(q3):
    """bf16 -> fp16 by the library equals torch's round-to-nearest-even conversion, in
    place and out of place, on normal, subnormal, overflowing and odd-length inputs."""
    x = Tensor(SEED, 91, (3001,)).gpu * 0.02
    x[:8] = torch.tensor([0.0, -0.0, 1e-7, -3e-6, 6.1e-5, 70000.0, -1e9, 2.0 ** -24], dtype=torch.bfloat16)
    ref = x.float().half()
    out = q3.convert_to_f16(x, torch.empty(x.shape, dtype=torch.float16, device="cuda"))
    y = x.clone()
    inplace = q3.convert_to_f16(y)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(inplace.view(torch.int16), ref.view(torch.int16))
    # bf16 values with |v| in [2^-17, 65504] are kept exactly
    keep = (x.float().abs() >= 2.0 ** -17) & (x.float().abs() <= 65504)
    assert torch.equal(out.float()[keep], x.float()[keep])


@pytest.mark.parametrize("rows", [1, 37, 1000])
def test_rmsnorm_f16_output(q3, rows):
    n = 1024
    x = Tensor(SEED, 11, (rows, n))
    w = Tensor(SEED, 12, (n,), 1.0, 0.1)
    out = torch.empty((rows, n), dtype=torch.float16, device="cuda")
    q3.op_rmsnorm(x.gpu.float(), w.gpu, out, rows, n, 1e-6)
    assert_device_ok()
    ref = R.rms_norm(x.f, w.f, 1e-6)
    assert np.all(np.abs(f64_of(out) - ref) <= f16_tol(ref, abs_=1e-5))


@pytest.mark.parametrize("M,N,K,epi,swap", [(16, 4096, 1024, 0, 2), (64, 1024, 2048, 1, 2), (64, 6144, 1024, 2, 2),
                                            (5, 1024, 3072, 1, 2), (200, 512, 192, 0, 1), (300, 6144, 1024, 2, 0),
                                            (1000, 1024, 3072, 1, 0), (600, 2048, 1024, 0, 0)])
def test_gemm_f16_operands(q3, M, N, K, epi, swap):
    """fp16 A and W (the gemm_f16 mode): the MMA's operand type switches, results within
    one rounding of the output (fp32 outputs: accumulation order only)."""
    A = Tensor(SEED, 51, (M, K))
    W = Tensor(SEED, 52, (N, K), 0.0, 0.02)
    X = Tensor(SEED, 53, (M, N))
    Wp = W.gpu
    if epi == 2:
        Wp = torch.empty_like(W.gpu)
        q3.pack_gate_up(N // 2, K, W.gpu[:N // 2], W.gpu[N // 2:], Wp)
    A16, W16 = to_f16(A.gpu), to_f16(Wp)
    torch.cuda.synchronize()
    a, w = f64_of(A16), f64_of(to_f16(W.gpu))
    acc = a @ w.T
    if epi == 2:
        out = torch.empty((M, N // 2), dtype=torch.float16, device="cuda")
        q3.op_gemm(A16, W16, out, M, N, K, epilogue=2, swap=swap)
        ref = R.silu(acc[:, :N // 2]) * acc[:, N // 2:]
        assert_device_ok()
        assert np.all(np.abs(f64_of(out) - ref) <= f16_tol(ref, abs_=2e-4)), max_abs(f64_of(out), ref)
        return
    out = torch.empty((M, N), dtype=torch.float32, device="cuda")
    resid = X.gpu.float() if epi == 1 else None
    q3.op_gemm(A16, W16, out, M, N, K, epilogue=epi, resid=resid, swap=swap)
    assert_device_ok()
    ref = acc + (X.f if epi == 1 else 0.0)
    assert max_abs(f64_of(out), ref) <= 2e-5 * np.sqrt(K / 1024) * 8, max_abs(f64_of(out), ref)


@pytest.mark.parametrize("M", [1, 3, 16, 37, 64])
@pytest.mark.parametrize("N,K,epi", [(4096, 1024, 0), (1024, 2048, 1), (6144, 1024, 2), (1024, 3072, 1), (128, 64, 0),
                                     (2048, 4096, 1)])
def test_gemm_cluster_split_k(q3, M, N, K, epi):
    """The decode-sized form (swap = 2): K split over the CTAs of a cluster and summed in
    shared memory across the cluster, in split order, with the epilogue in the same
    kernel; ragged token counts and a single K block."""
    A = Tensor(SEED, 61, (M, K))
    W = Tensor(SEED, 62, (N, K), 0.0, 0.02)
    X = Tensor(SEED, 63, (M, N))
    packed = W.gpu
    if epi == 2:
        packed = torch.empty_like(W.gpu)
        q3.pack_gate_up(N // 2, K, W.gpu[:N // 2], W.gpu[N // 2:], packed)
    acc = A.f @ W.f.T
    if epi == 2:
        out = torch.empty((M, N // 2), dtype=torch.bfloat16, device="cuda")
        q3.op_gemm(A.gpu, packed, out, M, N, K, epilogue=2, swap=2)
        assert_device_ok()
        ref = R.silu(acc[:, :N // 2]) * acc[:, N // 2:]
        assert np.all(np.abs(from_gpu_bf16(out) - ref) <= bf16_tol(ref, abs_=2e-4))
        return
    for out_dtype in (torch.float32, torch.bfloat16):
        out = torch.full((M, N), float("nan"), dtype=out_dtype, device="cuda")
        resid = X.gpu if epi == 1 else None
        q3.op_gemm(A.gpu, packed, out, M, N, K, epilogue=epi, resid=resid, swap=2)
        assert_device_ok()
        ref = acc + (X.f if epi == 1 else 0.0)
        got = f64_of(out)
        tol = 1e-4 if out_dtype == torch.float32 else bf16_tol(ref, abs_=1e-4)
        assert np.all(np.abs(got - ref) <= tol), (out_dtype, max_abs(got, ref))
    # deterministic: the same call twice gives the same bits
    again = torch.empty_like(out)
    q3.op_gemm(A.gpu, packed, again, M, N, K, epilogue=epi, resid=resid, swap=2)
    torch.cuda.synchronize()
    assert torch.equal(again.view(torch.int16), out.view(torch.int16))


def test_embed_f16_table(q3):
    V, H, n = 4096, 1024, 77
    E = Tensor(SEED, 81, (V, H), 0.0, 0.02)
    E16 = to_f16(E.gpu)
    ids_np = np.random.default_rng(5).integers(0, V, n).astype(np.int32)
    ids = torch.from_numpy(ids_np).cuda()
    out = torch.empty((n, H), dtype=torch.float32, device="cuda")
    q3.op_embed(ids, n, E16, V, H, out)
    assert_device_ok()
    np.testing.assert_array_equal(out.cpu().double().numpy(), f64_of(E16)[ids_np])


@pytest.mark.parametrize("M,N,K,epi,f16", [(64, 4096, 1024, 0, 0), (16, 1024, 2048, 1, 0), (37, 6144, 1024, 2, 0),
                                           (64, 1024, 3072, 1, 1), (5, 2048, 4096, 0, 1)])
def test_gemm_cluster_split_k_hilo_operand(q3, M, N, K, epi, f16):
    """swap = 3: the activation operand as hi/lo rows (hi = round(a), lo = round(a - hi) in
    the operand type). The product must carry the lo half: against the fp32 activations
    the error is far below one rounding of a (asserted 16x below the typical error of one
    bf16 rounding), which a kernel that dropped the lo rows could not reach."""
    rng = np.random.default_rng(M * 7 + K)
    a32 = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).cuda()
    dt = torch.float16 if f16 else torch.bfloat16
    hi = a32.to(dt)
    lo = (a32 - hi.float()).to(dt)
    A2 = torch.cat([hi, lo]).contiguous()
    W = Tensor(SEED, 72, (N, K), 0.0, 0.02)
    Wp = W.gpu
    if epi == 2:
        Wp = torch.empty_like(W.gpu)
        q3.pack_gate_up(N // 2, K, W.gpu[:N // 2], W.gpu[N // 2:], Wp)
    Wd = to_f16(Wp) if f16 else Wp
    a = a32.double().cpu().numpy()
    acc = a @ W.f.T
    # typical size of the product's error when a is rounded once to bf16 (independent
    # relative errors of 2^-9 / sqrt(3) per element)
    one_rounding = np.sqrt((a * a) @ (W.f.T * W.f.T)) * 2.0 ** -9 / np.sqrt(3.0)
    if epi == 2:
        out = torch.empty((M, N // 2), dtype=dt, device="cuda")
        q3.op_gemm(A2, Wd, out, M, N, K, epilogue=2, swap=3)
        assert_device_ok()
        ref = R.silu(acc[:, :N // 2]) * acc[:, N // 2:]
        assert np.all(np.abs(f64_of(out) - ref) <= 2.0 ** -7 * np.abs(ref) + 1e-3)
        return
    X = Tensor(SEED, 73, (M, N))
    out = torch.empty((M, N), dtype=torch.float32, device="cuda")
    q3.op_gemm(A2, Wd, out, M, N, K, epilogue=epi, resid=X.gpu.float() if epi == 1 else None, swap=3)
    assert_device_ok()
    ref = acc + (X.f if epi == 1 else 0.0)
    err = np.abs(f64_of(out) - ref)
    assert np.all(err <= one_rounding / 16 + 1e-6), float(np.max(err / (one_rounding + 1e-12)))
