"""Pins for the INT8 form of the SAGE-style comparison recipe in the oracle
("Accelerating Video Generation with GEMM Quantization, Attention Quantization
and Skip Softmax Attention in TensorRT-LLM", section "Quantized Attention": the
SAGE kernels take int8 or fp8 as qk_dtype, and the post runs int8).

The quantiser is pinned to what symmetric round-to-nearest INT8 coding fixes
(every code within half a step of its value, the group maximum on +-127,
sign and power-of-two symmetry, zero groups), the attention to exact softmax
on the dequantised operands, to the E4M3 form on values both types hold
exactly, and to closed forms."""
import math

import numpy as np
import pytest
import torch

import oracle

SC = 1.0 / math.sqrt(128)


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _f64(b):
    return torch.from_numpy(np.asarray(b, np.uint16).view(np.int16)).view(torch.bfloat16).double().numpy()


def _heads(N, seed, kshift=0.0):
    rng = np.random.default_rng(seed)
    Q = _bf16(rng.standard_normal((N, 128)))
    K = _bf16(rng.standard_normal((N, 128)) + kshift)
    V = _bf16(rng.standard_normal((N, 128)))
    return Q, K, V


def _smoothed_k(K, k_mean):
    # K' = K - k_mean, formed in fp32 as the recipe states (exact for bf16 values
    # of similar magnitude; fp32 rounding otherwise)
    return (_f64(K).astype(np.float32) - _f64(k_mean).astype(np.float32)).astype(np.float64)


def _check_groups(x, codes, scale):
    """x [n, m] values of n groups, codes [n, m] int8, scale [n]."""
    assert codes.dtype == np.int8
    assert np.all(np.abs(codes.astype(np.int32)) <= 127)
    amax = np.abs(x).max(1)
    live = amax > 0
    # a zero group: scale 1, codes 0
    assert np.all(scale[~live] == 1.0) and np.all(codes[~live] == 0)
    # the group's largest magnitude lands on +-127, with its sign
    i = np.abs(x).argmax(1)
    top = codes[np.arange(len(x)), i].astype(np.int32)
    assert np.all(np.abs(top[live]) == 127)
    assert np.all(np.sign(top[live]) == np.sign(x[np.arange(len(x)), i][live]))
    # scale = amax / 127 (the value the codes are multiplied by)
    assert np.allclose(scale[live], amax[live] / 127.0, rtol=2 ** -23, atol=0)
    # every code within half a step of its value (the fp32 product x * (127/amax)
    # is rounded once before the nearest-integer step: a 2^-16 slack covers it)
    if live.any():
        err = np.abs(x[live] / scale[live, None] - codes[live])
        assert err.max() <= 0.5 + 2 ** -16, err.max()


@pytest.mark.parametrize("N", [1, 16, 300, 1000])
def test_int8_quantiser_follows_its_definition(N):
    Q, K, V = _heads(N, 7 + N, kshift=2.0)
    ops = oracle.sage_quantize_head(Q, K, V, qk_dtype="int8")
    Np = (N + 127) // 128 * 128
    assert ops["Qq"].shape == (Np, 128) and ops["Kq"].shape == (Np, 128)
    _check_groups(_f64(Q), ops["Qq"][:N], ops["q_scale"][:N].astype(np.float64))
    kp = _smoothed_k(K, ops["k_mean"])
    ng = (N + 15) // 16
    pad = ng * 16 - N
    kg = np.concatenate([kp, np.zeros((pad, 128))]).reshape(ng, 16 * 128)
    cg = np.concatenate([ops["Kq"][:N], np.zeros((pad, 128), np.int8)]).reshape(ng, 16 * 128)
    _check_groups(kg, cg, ops["k_scale"][:ng].astype(np.float64))
    # padding rows and groups past the sequence
    assert np.all(ops["Qq"][N:] == 0) and np.all(ops["Kq"][N:] == 0)
    assert np.all(ops["q_scale"][N:] == 1.0) and np.all(ops["k_scale"][ng:] == 1.0)


def test_int8_and_fp8_recipes_share_v_and_k_mean():
    Q, K, V = _heads(500, 3, kshift=-1.5)
    a = oracle.sage_quantize_head(Q, K, V, qk_dtype="int8")
    b = oracle.sage_quantize_head(Q, K, V, qk_dtype="fp8")
    for key in ("VcT", "v_chscale", "k_mean"):
        assert np.array_equal(a[key], b[key]), key
    # the K mean: the exact channel mean of the bf16 keys, rounded once to bf16
    exact = _f64(K).mean(0)
    got = _f64(a["k_mean"])
    ulp = np.ldexp(1.0, np.floor(np.log2(np.abs(exact))).astype(int) - 7)
    assert np.all(np.abs(got - exact) <= ulp / 2 * (1 + 1e-9))


def test_int8_quantiser_symmetries():
    Q, K, V = _heads(260, 11)
    a = oracle.sage_quantize_head(Q, K, V, qk_dtype="int8")
    # negating Q negates its codes (round half to even is odd-symmetric)
    neg = oracle.sage_quantize_head(Q ^ np.uint16(0x8000), K, V, qk_dtype="int8")
    assert np.array_equal(neg["Qq"], -a["Qq"]) and np.array_equal(neg["q_scale"], a["q_scale"])
    # doubling every value doubles the scales and keeps the codes
    two = lambda b: _bf16(_f64(b) * 2.0)
    dbl = oracle.sage_quantize_head(two(Q), two(K), V, qk_dtype="int8")
    assert np.array_equal(dbl["Qq"], a["Qq"]) and np.array_equal(dbl["Kq"], a["Kq"])
    assert np.array_equal(dbl["q_scale"][:260], 2 * a["q_scale"][:260])
    assert np.array_equal(dbl["k_scale"][:17], 2 * a["k_scale"][:17])


def test_int8_codes_of_integer_rows_are_exact():
    # a row holding the integers -127..127 (with amax 127) codes to itself
    N = 2
    q = np.zeros((N, 128))
    q[0, :127] = np.arange(-63, 64)
    q[0, 127] = 127
    q[1, :] = np.linspace(-127, 127, 128).round()
    Q = _bf16(q)
    ops = oracle.sage_quantize_head(Q, Q, Q, qk_dtype="int8")
    assert np.array_equal(ops["Qq"][:N].astype(np.float64), _f64(Q))
    assert np.all(ops["q_scale"][:N] == 1.0)


def test_int8_attention_is_exact_softmax_on_its_dequantised_operands():
    N = 333
    Q, K, V = _heads(N, 21, kshift=1.0)
    ops = oracle.sage_quantize_head(Q, K, V, qk_dtype="int8")
    rows = np.arange(0, N, 7, dtype=np.int32)
    got, lse = oracle.attention_head_sage(ops, N, SC, rows=rows, flags=oracle.EXACT_EXP)
    e4 = np.array([oracle.lib().vo_e4m3_decode(i) for i in range(256)], np.float64)
    q = ops["Qq"][:N].astype(np.float64) * ops["q_scale"][:N, None]
    k = ops["Kq"][:N].astype(np.float64) * np.repeat(ops["k_scale"], 16)[:N, None]
    v = e4[ops["VcT"][:, :N].T] * ops["v_chscale"][None, :].astype(np.float64)
    s = q[rows] @ k.T * SC
    m = s.max(1, keepdims=True)
    p = np.exp(s - m)
    want = p @ v / p.sum(1, keepdims=True)
    assert np.abs(got - want).max() < 1e-10
    assert np.abs(lse - (m[:, 0] + np.log(p.sum(1)))).max() < 1e-9


def test_int8_attention_equals_fp8_form_on_shared_values():
    # codes in -16..16 are exact in both INT8 and E4M3: with the same scales the
    # two attentions must agree to the last bit (pins the INT8 decoding and its
    # indexing against the E4M3 path)
    rng = np.random.default_rng(5)
    N = 260
    Np = 384
    qi = np.zeros((Np, 128), np.int8)
    ki = np.zeros((Np, 128), np.int8)
    qi[:N] = rng.integers(-16, 17, (N, 128))
    ki[:N] = rng.integers(-16, 17, (N, 128))
    enc = lambda a: torch.from_numpy(a.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    base = oracle.sage_quantize_head(*_heads(N, 6), qk_dtype="fp8")
    qs = np.ones(Np, np.float32)
    qs[:N] = rng.uniform(0.001, 0.02, N)
    ks = np.ones(Np // 16, np.float32)
    ks[: (N + 15) // 16] = rng.uniform(0.001, 0.02, (N + 15) // 16)
    common = dict(q_scale=qs, k_scale=ks, VcT=base["VcT"], v_chscale=base["v_chscale"])
    o8, l8 = oracle.attention_head_sage(dict(common, Qq=enc(qi), Kq=enc(ki)), N, SC)
    oi, li = oracle.attention_head_sage(dict(common, Qq=qi, Kq=ki), N, SC)
    assert np.array_equal(o8, oi) and np.array_equal(l8, li)
    # a transposed or sign-flipped decoding would not
    oj, _ = oracle.attention_head_sage(dict(common, Qq=-qi, Kq=ki), N, SC)
    assert not np.array_equal(oj, oi)


def test_int8_attention_closed_forms():
    N = 200
    rng = np.random.default_rng(9)
    Q = _bf16(rng.standard_normal((N, 128)))
    # one key row repeated: K' = 0, every score 0, uniform weights
    K = np.tile(_bf16(rng.standard_normal((1, 128))), (N, 1))
    V = _bf16(rng.standard_normal((N, 128)))
    ops = oracle.sage_quantize_head(Q, K, V, qk_dtype="int8")
    assert np.all(ops["Kq"] == 0)
    O, lse = oracle.attention_head_sage(ops, N, SC, rows=np.arange(N, dtype=np.int32))
    e4 = np.array([oracle.lib().vo_e4m3_decode(i) for i in range(256)], np.float64)
    vmean = (e4[ops["VcT"][:, :N]] * ops["v_chscale"][:, None].astype(np.float64)).mean(1)
    assert np.abs(O - vmean[None, :]).max() < 1e-12
    # equal probabilities: lse = log N, off by at most the E4M3 step of the
    # one probability code every key shares (a factor within 2^(+-1/16))
    assert np.abs(lse - math.log(N)).max() <= math.log(2) / 16
    # one value row repeated: the output is that row, whatever the weights
    V1 = np.tile(_bf16(rng.standard_normal((1, 128))), (N, 1))
    ops1 = oracle.sage_quantize_head(Q, _heads(N, 2)[1], V1, qk_dtype="int8")
    O1, _ = oracle.attention_head_sage(ops1, N, SC, rows=np.arange(0, N, 9, dtype=np.int32))
    vrow = e4[ops1["VcT"][:, 0]] * ops1["v_chscale"].astype(np.float64)
    assert np.abs(O1 - vrow[None, :]).max() <= 1e-12 * np.abs(vrow).max()


def test_int8_attention_fidelity_against_exact():
    # the INT8 recipe keeps plain attention on the bf16 inputs (K smoothing is a
    # per-row shift of the scores): cosine >= 0.99 with ExpCast codes
    N = 700
    Q, K, V = _heads(N, 33, kshift=0.5)
    ops = oracle.sage_quantize_head(Q, K, V, qk_dtype="int8")
    rows = np.arange(0, N, 5, dtype=np.int32)
    got, _ = oracle.attention_head_sage(ops, N, SC, rows=rows)
    ex = oracle.exact_attention_head(Q, K, V, SC, rows=rows)
    cos = float((got * ex).sum() / np.sqrt((got * got).sum() * (ex * ex).sum()))
    assert cos >= 0.99, cos


def test_planted_scale_mistake_fails_the_pins():
    # a quantiser that divided by 128 instead of 127 (codes up to 128 would wrap)
    # or truncated instead of rounding fails the group checks
    Q, _, _ = _heads(64, 4)
    x = _f64(Q)
    amax = np.abs(x).max(1, keepdims=True).astype(np.float32)
    trunc = np.trunc(x.astype(np.float32) * (np.float32(127) / amax)).astype(np.int8)
    with pytest.raises(AssertionError):
        _check_groups(x, trunc, (amax[:, 0] / np.float32(127)).astype(np.float64))
    s128 = (amax[:, 0] / np.float32(128)).astype(np.float64)
    c128 = np.clip(np.rint(x / s128[:, None]), -128, 127).astype(np.int8)
    with pytest.raises(AssertionError):
        _check_groups(x, c128, s128)
