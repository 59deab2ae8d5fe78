"""Pins for the oracle of the 4-bit V-Smooth variant (CPU only).

NVFP4 is E2M1 elements with one E4M3 scale per 16 elements and one fp32 scale
per tensor ("Accelerating Video Generation with GEMM Quantization, Attention
Quantization and Skip Softmax Attention in TensorRT-LLM", table of
quantisation formats).  The 4-bit V-Smooth variant and the statement that
ExpCast is 8-bit only are from "Nunchux AI Introduces VC-Attention ..."
(abstract).  Each test checks the oracle against a library cast (ml_dtypes'
float4_e2m1fn, torch's float8_e4m3fn), brute force, a closed form or a bound
that the format fixes; several plant a mistake in the oracle (PLANT_*) and
check that the pin catches it.
"""
import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def bf16_bits_of(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bits_to_f32(b):
    return torch.from_numpy(np.asarray(b, np.uint16).view(np.int16)).view(torch.bfloat16).float().numpy()


def lib_e2m1_decode(codes):
    return np.asarray(codes, np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)


def lib_e4m3_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8).copy()).view(torch.float8_e4m3fn).double().numpy()


def half_gap(y):
    """Half the distance between the E2M1 magnitudes around |y| (|y| <= 6)."""
    a = np.abs(y)
    return np.where(a <= 2.0, 0.25, np.where(a <= 4.0, 0.5, 1.0))


# ----------------------------------------------------------------- E2M1
def test_e2m1_decode_matches_library_for_all_codes():
    ours = oracle.e2m1_decode_table()
    lib = lib_e2m1_decode(np.arange(16, dtype=np.uint8))
    assert np.array_equal(ours, lib)
    assert np.array_equal(ours[:8], E2M1_MAGNITUDES) and np.array_equal(ours[8:], -E2M1_MAGNITUDES)


def test_e2m1_encode_matches_library_cast_and_brute_force():
    rng = np.random.default_rng(1)
    mids = 0.5 * (E2M1_MAGNITUDES[1:] + E2M1_MAGNITUDES[:-1])
    x = np.concatenate([rng.uniform(-6.5, 6.5, 20000), mids, -mids, E2M1_MAGNITUDES, -E2M1_MAGNITUDES,
                        np.nextafter(mids, 0), np.nextafter(mids, 7)]).astype(np.float32)
    ours = oracle.e2m1_encode(x)
    assert np.array_equal(lib_e2m1_decode(ours), x.astype(ml_dtypes.float4_e2m1fn).astype(np.float64))
    # brute force: nearest magnitude, ties to the even code (codes 0..7 are the magnitudes in order)
    a = np.abs(x.astype(np.float64))[:, None]
    dist = np.abs(a - E2M1_MAGNITUDES[None, :])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    even = cand & (np.arange(8)[None, :] % 2 == 0)
    want = np.where(cand.sum(1) > 1, np.argmax(even, axis=1), np.argmax(cand, axis=1))
    assert np.array_equal(ours & 7, want)
    assert np.array_equal(ours >> 3, np.signbit(x).astype(np.uint8))


def test_e2m1_encode_saturates():
    x = np.array([6.0, 6.5, 7.0, 100.0, 3e38, -7.0, -1e9], np.float32)
    got = oracle.e2m1_encode(x)
    assert list(got) == [7, 7, 7, 7, 7, 15, 15]


# ----------------------------------------------------------------- NVFP4 groups
@pytest.mark.parametrize("n", [16, 160, 37])
def test_nvfp4_groups_meet_the_format_bound(n):
    rng = np.random.default_rng(n)
    x = (rng.standard_normal(n) * np.exp(rng.uniform(-3, 3, n))).astype(np.float32)
    G = float(np.float32(np.abs(x).max() / 2688.0))
    codes, scales = oracle.nvfp4_quantize(x, G)
    s = lib_e4m3_decode(scales)
    for g in range((n + 15) // 16):
        xs = x[16 * g:16 * g + 16].astype(np.float64)
        amax = np.abs(xs).max()
        # the scale is the E4M3 value nearest to amax / (6 G): within half an E4M3 step
        t = amax / (6.0 * G)
        assert abs(s[g] - t) <= t / 16 * (1 + 1e-6)
        xhat = G * s[g] * lib_e2m1_decode(codes[16 * g:16 * g + 16])
        y = xs / (s[g] * G)
        # unsaturated elements: within half a gap of the E2M1 grid; saturated ones at +-6
        sat = np.abs(y) > 6.0
        assert np.all(np.abs(xs - xhat)[~sat] <= (half_gap(y) * s[g] * G)[~sat] * (1 + 1e-6))
        assert np.all(np.abs(xhat[sat]) == 6.0 * s[g] * G)
        # the group maximum lands on +-6 up to the rounding of its scale
        k = np.argmax(np.abs(xs))
        assert abs(abs(xhat[k]) / amax - 1.0) <= 1.0 / 15
    # the tensor maximum: t = 448 exactly representable, so it comes back to fp32 accuracy
    k = np.argmax(np.abs(x))
    xhat_k = G * lib_e4m3_decode(scales[k // 16 : k // 16 + 1])[0] * lib_e2m1_decode(codes[k : k + 1])[0]
    assert xhat_k == pytest.approx(float(x[k]), rel=1e-6)


def test_nvfp4_all_zero_group_has_zero_scale_and_codes():
    x = np.zeros(32, np.float32)
    x[20] = 3.0
    codes, scales = oracle.nvfp4_quantize(x, 3.0 / 2688)
    assert scales[0] == 0 and not codes[:16].any()
    assert lib_e4m3_decode(scales[1:])[0] == 448.0 and codes[20] == 7


# ----------------------------------------------------------------- probabilities
def test_p_nvfp4_powers_of_two_closed_form():
    # p = 2^k for a whole group: t = 2^k / (6/8) = (4/3) 2^k rounds to 1.375 * 2^k in E4M3
    # (1.0101.. lies nearer 1.011 than 1.010); p / (s G) = 5.82 -> code 6; p_hat = 1.03125 * 2^k
    for k in (-6, 0, 3, 8):
        got = oracle.p_nvfp4(np.full(16, 2.0 ** k))
        assert np.all(got == 1.03125 * 2.0 ** k)


def test_p_nvfp4_groups_are_16_keys():
    rng = np.random.default_rng(3)
    p = 2.0 ** rng.uniform(-12, 8, 128)
    base = oracle.p_nvfp4(p)
    for g in range(8):
        q = p.copy()
        q[16 * g:16 * g + 16] *= 0.37
        got = oracle.p_nvfp4(q)
        outside = np.ones(128, bool)
        outside[16 * g:16 * g + 16] = False
        assert np.array_equal(got[outside], base[outside])
        assert not np.array_equal(got[~outside], base[~outside])
    # planted: 32-key groups -- scaling one 16-key half moves the other half's values
    bad0 = oracle.p_nvfp4(p, flags=oracle.PLANT_P_GROUP32)
    q = p.copy()
    q[16:32] *= 64.0
    bad1 = oracle.p_nvfp4(q, flags=oracle.PLANT_P_GROUP32)
    assert not np.array_equal(bad0[:16], bad1[:16])


def test_p_nvfp4_bound_and_ragged_block():
    rng = np.random.default_rng(4)
    for n in (128, 75, 3):
        p = 2.0 ** rng.uniform(-10, 8, n)
        got = oracle.p_nvfp4(p)
        for g in range((n + 15) // 16):
            ps, gs = p[16 * g:16 * g + 16], got[16 * g:16 * g + 16]
            amax = ps.max()
            # largest E2M1 half-gap is 1 unit of s*G, and s*G <= (amax/6)(1 + 1/16)
            assert np.all(np.abs(ps - gs) <= amax / 6 * (1 + 1 / 16) * (1 + 1e-6))
            assert abs(gs[np.argmax(ps)] / amax - 1.0) <= 1.0 / 15


# ----------------------------------------------------------------- V-Smooth 4-bit prep
def _head(N, d=128, seed=0):
    rng = np.random.default_rng(seed)
    Q = bf16_bits_of(rng.standard_normal((N, d)))
    K = bf16_bits_of(rng.standard_normal((N, d)))
    V = bf16_bits_of(rng.standard_normal((N, d)) * np.exp(rng.uniform(-1, 1, (N, 1))) + rng.standard_normal(d))
    perm = rng.permutation(N).astype(np.int32)
    return Q, K, V, perm


def _dequant_v_residual(ops, N):
    """Residual of permuted token j, channel c, from the documented layout:
    byte c*Np/2 + j/2, low nibble for even j; group scale c*Np/16 + j/16."""
    d, half = ops["VrT4"].shape
    j = np.arange(N)
    byte = ops["VrT4"][:, j // 2]
    nib = np.where(j % 2 == 0, byte & 15, byte >> 4).astype(np.uint8)
    s = lib_e4m3_decode(ops["v_sc"][:, j // 16])
    return (float(ops["v_gscale"][0]) * s * lib_e2m1_decode(nib)).T   # [N][d]


@pytest.mark.parametrize("N", [700, 256, 1])
def test_fp4_prep_shares_q_k_and_means_and_bounds_the_residual(N):
    Q, K, V, perm = _head(N, seed=N)
    o4 = oracle.smooth_quantize_head_fp4(Q, K, V, perm)
    o8 = oracle.smooth_quantize_head(Q, K, V, perm)
    for key in ("Qq", "q_scale", "Kq", "k_scale", "v_mean"):
        assert np.array_equal(o4[key], o8[key]), key
    Vp = bits_to_f32(V[perm]).astype(np.float64)
    mu = bits_to_f32(o4["v_mean"]).astype(np.float64)[np.arange(N) // 128]
    r = Vp - mu
    G = float(o4["v_gscale"][0])
    # G = amax / (6 * 448); an all-zero residual (a single token is its own mean) keeps G = 1
    assert G == (pytest.approx(np.abs(r).max() / 2688.0, rel=1e-6) if np.abs(r).max() > 0 else 1.0)
    rhat = _dequant_v_residual(o4, N)
    # every group: error within half an E2M1 gap of its own (s G) after the E4M3 scale rounding
    ng = (N + 15) // 16
    for g in range(ng):
        rs, hs = r[16 * g:16 * g + 16], rhat[16 * g:16 * g + 16]
        amax = np.abs(rs).max(axis=0)
        assert np.all(np.abs(rs - hs) <= amax / 6 * (1 + 1 / 16) * (1 + 1e-6) + 1e-30)
    # padding: no codes past N, no scales for groups wholly past N
    Np = o4["VrT4"].shape[1] * 2
    if N % 2:
        assert not (o4["VrT4"][:, N // 2] >> 4).any()
    assert not o4["VrT4"][:, (N + 1) // 2:].any()
    assert not o4["v_sc"][:, ng:].any()
    assert Np == ((N + 127) // 128) * 128


def test_fp4_planted_nibble_order_fails_the_layout_pin():
    # a row whose weight sits on one key reads that key's residual back: the
    # pin catches a swapped nibble order (VO_PLANT_NIBBLE)
    N = 300
    Q, K, V, perm = _head(N, seed=11)
    inv = np.argsort(perm)
    rows = np.array([0, 5, 6, 131, 299], np.int32)
    Qone = Q.copy()
    Qone[rows] = K[rows]          # query i equals key i: its own key dominates by ~100 octaves
    ops_one = oracle.smooth_quantize_head_fp4(Qone, K, V, perm)
    O, _ = oracle.attention_head_fp4(ops_one, N, 1.0, rows)
    rhat = _dequant_v_residual(ops_one, N)
    mu = bits_to_f32(ops_one["v_mean"]).astype(np.float64)
    jp = inv[rows]
    want = mu[jp // 128] + rhat[jp]
    assert np.array_equal(O, want)
    bad, _ = oracle.attention_head_fp4(ops_one, N, 1.0, rows, flags=oracle.PLANT_NIBBLE)
    assert not np.allclose(bad, want)


# ----------------------------------------------------------------- attention
@pytest.mark.parametrize("N", [300, 129])
def test_fp4_attention_reduces_to_exact_with_identity_quantisers(N):
    Q, K, V, perm = _head(N, seed=20 + N)
    sc = 1 / np.sqrt(128)
    got = oracle.attention_head_fp4_bf16(Q, K, V, perm, sc, flags=oracle.IDENTITY_QUANT)
    ex = oracle.exact_attention_head(Q, K, V, sc)
    assert np.abs(got - ex).max() < 1e-12
    bad = oracle.attention_head_fp4_bf16(Q, K, V, perm, sc, flags=oracle.IDENTITY_QUANT | oracle.PLANT_NO_MEAN)
    assert np.abs(bad - ex).max() > 1e-3


def test_fp4_attention_uniform_row_is_the_mean_of_the_dequantised_values():
    # q = 0: every key has the same probability, so every full or ragged group
    # gets the same NVFP4 value and the output is the plain mean over the N keys
    N = 300
    Q, K, V, perm = _head(N, seed=31)
    Q[7] = 0
    ops = oracle.smooth_quantize_head_fp4(Q, K, V, perm)
    O, _ = oracle.attention_head_fp4(ops, N, 1 / np.sqrt(128), np.array([7], np.int32))
    mu = bits_to_f32(ops["v_mean"]).astype(np.float64)[np.arange(N) // 128]
    want = (mu + _dequant_v_residual(ops, N)).mean(axis=0)
    assert np.abs(O[0] - want).max() < 1e-12
    bad, _ = oracle.attention_head_fp4(ops, N, 1 / np.sqrt(128), np.array([7], np.int32),
                                       flags=oracle.PLANT_NO_MEAN)
    assert np.abs(bad[0] - want).max() > 1e-2


def test_fp4_attention_fidelity_between_the_bounds():
    # NVFP4 P and V cost more fidelity than the 8-bit variant, and stay close to exact
    N = 700
    Q, K, V, perm = _head(N, seed=41)
    sc = 1 / np.sqrt(128)
    rows = np.arange(0, N, 13, dtype=np.int32)
    ex = oracle.exact_attention_head(Q, K, V, sc, rows)
    e4 = np.linalg.norm(oracle.attention_head_fp4_bf16(Q, K, V, perm, sc, rows) - ex) / np.linalg.norm(ex)
    e8 = np.linalg.norm(oracle.attention_head_bf16(Q, K, V, perm, sc, rows) - ex) / np.linalg.norm(ex)
    assert e8 < e4 < 0.05
