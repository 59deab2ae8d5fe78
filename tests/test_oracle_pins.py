"""Pins the CPU oracle to things other than itself (CPU only).

Each test checks the oracle against a number the pages print
(tests/golden/pages_constants.json), a closed form, an invariant, a library
routine (torch's float8_e4m3fn cast, numpy argsort/argmin), or brute force on
tiny inputs.  Several tests also plant a mistake in the oracle (flags
PLANT_*) and check that the pin catches it.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_constants.json")))


def torch_e4m3(x):
    """Library RNE cast to E4M3 (valid for |x| < 464)."""
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def bf16_bits_of(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bits_to_f32(b):
    return torch.from_numpy(np.asarray(b, np.uint16).view(np.int16)).view(torch.bfloat16).float().numpy()


# ----------------------------------------------------------------- E4M3
def test_e4m3_decode_matches_library_for_all_bytes():
    ours = oracle.e4m3_decode_table()
    lib = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], lib[~nan])
    assert ours[0x38] == 1.0 and ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9
    assert np.all(np.diff(ours[:127]) > 0)


def test_e4m3_encode_matches_library_cast():
    rng = np.random.default_rng(0)
    vals = oracle.e4m3_decode_table()[:127]
    mids = (vals[:-1] + vals[1:]) / 2                      # exact ties -> even code
    x = np.concatenate([
        rng.standard_normal(200000) * 30,
        rng.uniform(-460, 460, 100000),
        np.exp2(rng.uniform(-14, 8.8, 100000)) * rng.choice([-1, 1], 100000),
        mids, -mids, vals, -vals, np.nextafter(mids, 0), np.nextafter(mids, 1000),
        [0.0, -0.0, 2.0 ** -10, -(2.0 ** -10), 2.0 ** -10 * 1.0001, 1e-30, -1e-30],
    ]).astype(np.float32)
    x = x[np.abs(x) < 460]
    assert np.array_equal(oracle.e4m3_encode(x), torch_e4m3(x))


def test_e4m3_encode_saturates_and_nan():
    out = oracle.e4m3_encode(np.array([448, 463.9, 464, 1e9, np.inf, -np.inf, -1e9, np.nan], np.float32))
    assert list(out) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x7F]


# ----------------------------------------------------------------- ExpCast
def test_expcast_byte_at_probability_one():
    assert int(oracle.expcast([0.0])[0]) == GOLD["byte_at_p_one"]["value"] == 0x38
    assert oracle.e4m3_decode(0x38) == 1.0


def test_expcast_slope_and_offset_on_exact_octaves():
    # at z = -k (p = 2^-k) the byte is 56 - 8k exactly: slope 8, offset 56
    z = -np.arange(0, 7, dtype=np.float32)
    codes = oracle.expcast(z).astype(int)
    assert list(codes) == [GOLD["expcast_byte_offset"]["value"] - GOLD["expcast_byte_slope"]["value"] * k
                           for k in range(7)]


@pytest.mark.parametrize("octave", [0, 1, 2, 3, 4, 5])
def test_expcast_agreement_with_exp2_then_cast(octave):
    g = GOLD["same_byte_fraction_per_doubling"]
    z = ((np.arange(2 ** 18, dtype=np.float64) + 0.5) / 2 ** 18 - 1.0 - octave).astype(np.float32)
    ours = oracle.expcast(z).astype(int)
    ref = torch_e4m3(np.exp2(z)).astype(int)       # fp32 exponent, then the library cast
    frac = float(np.mean(ours == ref))
    assert abs(frac - g["value"]) <= g["tol"], frac
    assert np.abs(ours - ref).max() == GOLD["max_code_difference"]["value"]


def test_expcast_planted_mistakes_fail_agreement_pin():
    g = GOLD["same_byte_fraction_per_doubling"]
    z = ((np.arange(2 ** 16, dtype=np.float64) + 0.5) / 2 ** 16 - 1.0).astype(np.float32)
    ref = torch_e4m3(np.exp2(z))
    for flag in (oracle.PLANT_TRUNC, oracle.PLANT_BETA0):
        frac = float(np.mean(oracle.expcast(z, flag) == ref))
        assert abs(frac - g["value"]) > 0.02, (flag, frac)


def test_expcast_underflow_tail_and_specials():
    # codes 1..7 (E4M3 subnormals) are kept as computed; below that, zero
    z = np.array([-6.1, -6.5, -6.9, -7.5, -20.0, -np.inf, np.inf, 100.0, np.nan], np.float32)
    c = oracle.expcast(z)
    assert list(c[:6]) == [7, 4, 0, 0, 0, 0]
    assert oracle.e4m3_decode(4) == 4 * 2.0 ** -9
    assert c[6] == 126 and c[7] == 126 and c[8] == 0x7F


def _tv(z, codes):
    p = np.exp2(z.astype(np.float64))
    ph = np.array([oracle.e4m3_decode(int(c)) for c in codes])
    return 0.5 * np.abs(ph / ph.sum() - p / p.sum()).sum()


def test_expcast_row_tv_bound_random_rows():
    bound = GOLD["per_row_tv_bound"]["value"]
    rng = np.random.default_rng(1)
    worst = 0.0
    for _ in range(300):
        n = int(rng.integers(2, 300))
        z = rng.uniform(-5.9, 0.0, n).astype(np.float32)   # codes >= 8: no underflow tail
        codes = oracle.expcast(z)
        assert codes.min() >= 8
        worst = max(worst, _tv(z, codes))
    assert worst <= bound


def test_expcast_row_tv_bound_is_attained_by_two_level_rows():
    # The decoded/true ratio r(z) ranges over [a, b]; a row that puts mass
    # sqrt(b)/(sqrt(a)+sqrt(b)) at the low extreme and the rest at the high
    # extreme has TV (sqrt(b)-sqrt(a))/(sqrt(b)+sqrt(a)) -- the 3.64% of the pages.
    g = GOLD["per_row_tv_bound"]
    z = ((np.arange(2 ** 16) + 0.5) / 2 ** 16 - 1.0).astype(np.float32)
    codes = oracle.expcast(z)
    dec = oracle.e4m3_decode_table()[codes]
    ratio = dec / np.exp2(z.astype(np.float64))
    ia, ib = int(np.argmin(ratio)), int(np.argmax(ratio))
    a, b = ratio[ia], ratio[ib]
    closed = (math.sqrt(b) - math.sqrt(a)) / (math.sqrt(b) + math.sqrt(a))
    assert abs(closed - g["value"]) <= g["tol"], closed
    # build the row: n_a copies of z_a and n_b copies of z_b
    wa = math.sqrt(b) / (math.sqrt(a) + math.sqrt(b))
    pa, pb = 2.0 ** float(z[ia]), 2.0 ** float(z[ib])
    n_tot = 4000
    best = 0.0
    for na in range(1, n_tot):
        nb = n_tot - na
        ma = na * pa / (na * pa + nb * pb)
        if abs(ma - wa) < 2e-3:
            row = np.array([z[ia]] * na + [z[ib]] * nb, np.float32)
            best = max(best, _tv(row, oracle.expcast(row)))
    assert g["value"] - 2e-4 <= best <= g["value"] + 1e-9, best


# ----------------------------------------------------------------- bf16
def test_double_to_bf16_direct_rounding():
    assert oracle.double_to_bf16(1.0 + 2 ** -8) == 0x3F80              # tie -> even
    assert oracle.double_to_bf16(1.0 + 2 ** -8 + 2 ** -40) == 0x3F81   # no double rounding
    assert oracle.double_to_bf16(1.0 + 3 * 2 ** -8) == 0x3F82          # tie -> even (up)
    assert oracle.double_to_bf16(-2.5) == 0xC020
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(20000) * 10.0 ** rng.uniform(-30, 30, 20000)).astype(np.float32)
    ours = np.array([oracle.double_to_bf16(float(v)) for v in x], np.uint16)
    assert np.array_equal(ours, bf16_bits_of(x))


# ----------------------------------------------------------------- k-means
def test_kmeans_two_separated_groups_split_exactly():
    rng = np.random.default_rng(3)
    N, d = 64, 128
    v = np.where(np.arange(N)[:, None] < 24, 5.0, -5.0) + 0.1 * rng.standard_normal((N, d))
    Vb = bf16_bits_of(v)
    cent, assign, counts = oracle.kmeans_head(Vb, k=2, iters=3, init=np.stack([bits_to_f32(Vb[0]), bits_to_f32(Vb[-1])]))
    assert list(assign[:24]) == [0] * 24 and list(assign[24:]) == [1] * 40
    assert list(counts) == [24, 40]
    vf = bits_to_f32(Vb).astype(np.float64)
    assert np.allclose(cent[0], vf[:24].mean(0), rtol=0, atol=1e-6)
    assert np.allclose(cent[1], vf[24:].mean(0), rtol=0, atol=1e-6)


def test_kmeans_assign_is_argmin_brute_force():
    rng = np.random.default_rng(4)
    for trial in range(5):
        N, k = 12, 4
        v = bits_to_f32(bf16_bits_of(rng.standard_normal((N, 128)))).astype(np.float32)
        cent = rng.standard_normal((k, 128)).astype(np.float32)
        a = oracle.kmeans_assign(v, cent)
        dist = ((v[:, None, :].astype(np.float64) - cent[None].astype(np.float64)) ** 2).sum(-1)
        assert np.array_equal(a, np.argmin(dist, axis=1))


def test_kmeans_ties_go_to_lowest_index_and_empty_keeps_centroid():
    v = np.ones((5, 128), np.float32)
    cent = np.stack([np.zeros(128), np.zeros(128), np.full(128, 7.0)]).astype(np.float32)
    a = oracle.kmeans_assign(v, cent)
    assert list(a) == [0] * 5
    new, counts = oracle.kmeans_update(v, a, cent)
    assert list(counts) == [5, 0, 0]
    assert np.array_equal(new[0], np.ones(128, np.float32))
    assert np.array_equal(new[1:], cent[1:])


def test_kmeans_update_is_exact_mean():
    rng = np.random.default_rng(5)
    v = bits_to_f32(bf16_bits_of(rng.standard_normal((300, 128)) * 3)).astype(np.float32)
    a = rng.integers(0, 7, 300).astype(np.int32)
    cent, counts = oracle.kmeans_update(v, a, np.zeros((7, 128), np.float32))
    for c in range(7):
        m = v[a == c].astype(np.float64)
        exact = [float(sum(Fraction(float(x)) for x in m[:, ch]) / len(m)) for ch in range(0, 128, 17)]
        assert np.array_equal(cent[c, ::17], np.array(exact, np.float32))   # one rounding to fp32


def test_kmeans_invariants_on_mixture():
    rng = np.random.default_rng(6)
    cents = rng.standard_normal((8, 128))
    v = cents[rng.integers(0, 8, 700)] + 0.3 * rng.standard_normal((700, 128))
    Vb = bf16_bits_of(v)
    vf = bits_to_f32(Vb).astype(np.float32)
    prev_obj = np.inf
    for T in range(1, 6):
        c_prev, _, _ = oracle.kmeans_head(Vb, 8, T - 1) if T > 1 else (None, None, None)
        cent, assign, counts = oracle.kmeans_head(Vb, 8, T)
        if c_prev is None:
            c_prev = vf[(np.arange(8) * 700) // 8]
        d = ((vf[:, None, :].astype(np.float64) - c_prev[None].astype(np.float64)) ** 2).sum(-1)
        assert np.array_equal(assign, np.argmin(d, axis=1))          # every token at its argmin
        for c in range(8):                                            # centroid = mean of members
            if counts[c]:
                assert np.allclose(cent[c], vf[assign == c].astype(np.float64).mean(0), atol=1e-6)
        obj = sum(((vf[assign == c] - cent[c]) ** 2).sum() for c in range(8))
        assert obj <= prev_obj + 1e-3
        prev_obj = obj


def test_stable_perm_matches_library_stable_argsort():
    rng = np.random.default_rng(7)
    for N, k in [(1, 1), (7, 3), (1000, 32), (1024, 8)]:
        a = rng.integers(0, k, N).astype(np.int32)
        p = oracle.stable_perm(a, k)
        assert np.array_equal(p, np.argsort(a, kind="stable"))
        assert np.array_equal(np.sort(p), np.arange(N))


# ----------------------------------------------------------------- quantise
def test_v_exponent_is_smallest_power():
    rng = np.random.default_rng(8)
    xs = list(np.exp2(rng.uniform(-140, 25, 3000)).astype(np.float32))
    xs += [np.float32(448 * 2.0 ** e) for e in range(-20, 20)]
    xs += [np.nextafter(np.float32(448 * 2.0 ** e), np.float32(1e30)) for e in range(-20, 20)]
    for x in xs:
        e = oracle.v_exponent(float(x))
        brute = next(e2 for e2 in range(-200, 200) if float(x) <= 448.0 * 2.0 ** e2)
        assert e == max(-127, brute), (x, e, brute)
    assert oracle.v_exponent(0.0) == 0


def _head(N, seed=9, scale=1.0, integer=False):
    rng = np.random.default_rng(seed)
    mk = (lambda: rng.integers(-8, 9, (N, 128)).astype(np.float64)) if integer else \
         (lambda: rng.standard_normal((N, 128)) * scale)
    return bf16_bits_of(mk()), bf16_bits_of(mk()), bf16_bits_of(mk())


@pytest.mark.parametrize("N", [1, 128, 200, 1000])
def test_quantize_q_and_k_against_library_cast(N):
    Q, K, V = _head(N)
    perm = np.random.default_rng(N).permutation(N).astype(np.int32)
    ops = oracle.smooth_quantize_head(Q, K, V, perm)
    nb = (N + 127) // 128
    for name, src, order in (("Q", Q, np.arange(N)), ("K", K, perm)):
        x = bits_to_f32(src)[order]
        codes = ops[name + "q"]
        sc = ops[name.lower() + "_scale"]
        for b in range(nb):
            blk = x[b * 128:(b + 1) * 128]
            amax = np.float32(np.abs(blk).max())
            assert sc[b] == np.float32(amax / np.float32(448.0))
            inv = np.float32(448.0) / amax
            assert np.array_equal(codes[b * 128:b * 128 + len(blk)], torch_e4m3(blk * inv))
        assert not codes[N:].any()


@pytest.mark.parametrize("N", [128, 200, 1000])
def test_quantize_v_mean_exact_on_integer_inputs(N):
    Q, K, V = _head(N, integer=True)
    perm = np.arange(N, dtype=np.int32)[::-1].copy()
    ops = oracle.smooth_quantize_head(Q, K, V, perm)
    vf = bits_to_f32(V)[perm]
    for b in range((N + 127) // 128):
        blk = vf[b * 128:(b + 1) * 128]
        for ch in (0, 5, 127):
            exact = Fraction(int(blk[:, ch].sum()), len(blk))
            # exact rational mean, rounded once to bf16 (RNE)
            assert ops["v_mean"][b, ch] == oracle.double_to_bf16(float(exact)) or \
                abs(float(exact) - bits_to_f32(ops["v_mean"][b:b + 1, ch:ch + 1])[0, 0]) <= abs(float(exact)) * 2 ** -9


def test_mean_costs_an_eighth_bit_per_element():
    N = 1000
    ops = oracle.smooth_quantize_head(*_head(N), np.arange(N, dtype=np.int32))
    bits = ops["v_mean"].size * 16
    assert bits / (ops["v_mean"].shape[0] * 128 * 128) == GOLD["mean_bits_per_value_element"]["value"]


@pytest.mark.parametrize("N", [200, 1000])
def test_quantize_v_reconstruction_bound(N):
    Q, K, V = _head(N, scale=2.0)
    perm = np.random.default_rng(1).permutation(N).astype(np.int32)
    ops = oracle.smooth_quantize_head(Q, K, V, perm)
    vf = bits_to_f32(V)[perm].astype(np.float64)
    dec = oracle.e4m3_decode_table()
    Np = ops["VrT"].shape[1]
    assert not ops["VrT"][:, N:].any()
    for b in range((N + 127) // 128):
        e = int(ops["v_exp"][b])
        mu = bits_to_f32(ops["v_mean"][b]).astype(np.float64)
        blk = vf[b * 128:(b + 1) * 128]
        r = blk - mu
        amax = np.abs(r).max()
        assert amax <= 448 * 2.0 ** e and (amax > 448 * 2.0 ** (e - 1) or e == -127)
        rh = dec[ops["VrT"][:, b * 128:b * 128 + len(blk)].T] * 2.0 ** e
        # E4M3 RNE: error <= half a step, step = 2^(floor(log2|x|)-3), >= 2^-9 (subnormal)
        y = np.abs(r) / 2.0 ** e
        step = np.exp2(np.maximum(np.floor(np.log2(np.maximum(y, 1e-300))), -6) - 3)
        assert np.all(np.abs(rh - r) <= 0.5 * step * 2.0 ** e + 1e-12)
        # the mean is the bf16 rounding of the exact block mean
        exact = blk.mean(0)
        assert np.all(np.abs(mu - exact) <= np.abs(exact) * 2 ** -8 + 1e-30)


@pytest.mark.parametrize("N", [1, 700])
def test_quantize_v_per_head_exponent_reading(N):
    # the second reading: one V exponent per head.  Q, K and the means are the
    # per-block prep's; the head exponent is the largest block exponent (the
    # exponent rule is monotone in max|r|); every residual is within half an
    # E4M3 step of the head's scale
    rng = np.random.default_rng(N)
    Q, K, _ = _head(N, scale=2.0)
    # blocks whose residuals differ by octaves
    V = bf16_bits_of(rng.standard_normal((N, 128)) * np.exp2(np.arange(N) // 128 % 5 - 2)[:, None])
    perm = np.arange(N, dtype=np.int32)
    blk = oracle.smooth_quantize_head(Q, K, V, perm)
    hd = oracle.smooth_quantize_head(Q, K, V, perm, v_scale="head")
    for key in ("Qq", "q_scale", "Kq", "k_scale", "v_mean"):
        assert np.array_equal(blk[key], hd[key]), key
    e = int(blk["v_exp"].max())
    assert np.all(hd["v_exp"] == e)
    vf = bits_to_f32(V).astype(np.float64)
    mu = bits_to_f32(hd["v_mean"]).astype(np.float64)[np.arange(N) // 128]
    r = vf - mu
    rh = oracle.e4m3_decode_table()[hd["VrT"][:, :N].T] * 2.0 ** e
    y = np.abs(r) / 2.0 ** e
    step = np.exp2(np.maximum(np.floor(np.log2(np.maximum(y, 1e-300))), -6) - 3)
    assert np.all(np.abs(rh - r) <= 0.5 * step * 2.0 ** e + 1e-12)
    # the blocks that already had the head's exponent are coded identically
    nb = (N + 127) // 128
    for b in range(nb):
        if blk["v_exp"][b] == e:
            assert np.array_equal(blk["VrT"][:, b * 128:(b + 1) * 128], hd["VrT"][:, b * 128:(b + 1) * 128])


def test_per_head_exponent_changes_attention_little():
    # the two readings of the V scale give nearly the same attention: E4M3's own
    # exponent absorbs the spread of the block exponents (measured 3e-7 .. 2e-6
    # relative on the synthetic workloads; bounded here at 1e-4)
    from bit_attention_video_02_b200 import workloads as W
    w = W.shrink(W.WORKLOADS[1], H=1)
    Q, K, V = W.make_qkv(w, "cpu")
    q, k, v = (W.bf16_bits(t[0, 0]) for t in (Q, K, V))
    ops = oracle.prep_head(q, k, v, w.k, 3)
    hd = oracle.smooth_quantize_head(q, k, v, ops["perm"], v_scale="head")
    rows = np.arange(0, w.N, 7, dtype=np.int32)
    sc = 1 / np.sqrt(128)
    o_blk, _, _ = oracle.attention_head(ops, w.N, sc, rows)
    o_hd, _, _ = oracle.attention_head(hd, w.N, sc, rows)
    assert np.linalg.norm(o_hd - o_blk) / np.linalg.norm(o_blk) < 1e-4
    assert not np.array_equal(hd["VrT"], ops["VrT"])


# ----------------------------------------------------------------- attention
def _bits(rng, N, s=1.0):
    return bf16_bits_of(rng.standard_normal((N, 128)) * s)


def test_exact_attention_closed_forms():
    rng = np.random.default_rng(10)
    N = 50
    Q, K = _bits(rng, N), _bits(rng, N)
    row = bf16_bits_of(rng.standard_normal((1, 128)))
    V = np.repeat(row, N, axis=0)
    O = oracle.exact_attention_head(Q, K, V, 0.3)
    assert np.allclose(O, np.repeat(bits_to_f32(row), N, 0), atol=1e-12, rtol=0)   # constant V
    Vr = _bits(rng, N)
    O0 = oracle.exact_attention_head(np.zeros_like(Q), K, Vr, 0.3)
    assert np.allclose(O0, bits_to_f32(Vr).astype(np.float64).mean(0)[None], atol=1e-12)  # Q = 0
    # two keys: softmax is a logistic function of the score difference
    q = bf16_bits_of(np.full((1, 128), 0.25))
    k2 = bf16_bits_of(np.stack([np.full(128, 0.5), np.full(128, -0.25)]))
    v2 = bf16_bits_of(np.stack([np.full(128, 3.0), np.full(128, -1.0)]))
    O2 = oracle.exact_attention_head(np.repeat(q, 2, 0), k2, v2, 0.1)
    ds = 0.1 * 128 * 0.25 * (0.5 + 0.25)
    w = 1.0 / (1.0 + math.exp(-ds))
    assert abs(O2[0, 0] - (3.0 * w - (1 - w))) < 1e-13
    # very large scale: O -> V[argmax]
    Oh = oracle.exact_attention_head(Q, K, Vr, 1e4, rows=[3])
    s = bits_to_f32(Q)[3].astype(np.float64) @ bits_to_f32(K).astype(np.float64).T
    assert np.allclose(Oh[0], bits_to_f32(Vr)[int(np.argmax(s))], atol=1e-9)


def test_exact_attention_brute_force_and_permutation_invariance():
    rng = np.random.default_rng(11)
    N = 40
    Q, K, V = _bits(rng, N), _bits(rng, N), _bits(rng, N)
    q, k, v = (bits_to_f32(a).astype(np.longdouble) for a in (Q, K, V))
    s = (q @ k.T) * np.longdouble(0.088)
    p = np.exp(s - s.max(1, keepdims=True))
    ref = (p @ v) / p.sum(1, keepdims=True)
    O = oracle.exact_attention_head(Q, K, V, 0.088)
    assert np.abs(O - ref.astype(np.float64)).max() < 1e-13
    perm = rng.permutation(N)
    Op = oracle.exact_attention_head(Q, K[perm], V[perm], 0.088)
    assert np.abs(O - Op).max() < 1e-13


@pytest.mark.parametrize("N", [128, 200, 700])
def test_same_algorithm_reduces_to_exact(N):
    rng = np.random.default_rng(12 + N)
    Q, K, V = _bits(rng, N), _bits(rng, N), _bits(rng, N, 2.0)
    V[rng.integers(0, N, 5)] = bf16_bits_of(rng.standard_normal((5, 128)) * 40)
    perm = rng.permutation(N).astype(np.int32)
    sc = 1 / math.sqrt(128)
    exact = oracle.exact_attention_head(Q, K, V, sc)
    red = oracle.attention_head_bf16(Q, K, V, perm, sc, flags=oracle.EXACT_EXP | oracle.IDENTITY_QUANT)
    assert np.abs(red - exact).max() < 1e-12
    bad = oracle.attention_head_bf16(Q, K, V, perm, sc,
                                     flags=oracle.EXACT_EXP | oracle.IDENTITY_QUANT | oracle.PLANT_NO_MEAN)
    assert np.abs(bad - exact).max() > 1e-3


def test_online_rescale_reduces_to_exact():
    # later key blocks score much higher, so the running reference moves up by
    # more than 4 octaves several times; with exact exponentials and identity
    # quantisers the online result must still equal exact attention
    rng = np.random.default_rng(21)
    N = 900
    kf = rng.standard_normal((N, 128))
    kf *= (1.0 + np.arange(N) // 128)[:, None] * 1.5
    qf = np.abs(rng.standard_normal((N, 128))) * 0.5
    Q, K, V = bf16_bits_of(qf), bf16_bits_of(np.abs(kf)), _bits(rng, N)
    perm = np.arange(N, dtype=np.int32)
    sc = 1 / math.sqrt(128)
    exact = oracle.exact_attention_head(Q, K, V, sc)
    fl = oracle.EXACT_EXP | oracle.IDENTITY_QUANT
    red = oracle.attention_head_bf16(Q, K, V, perm, sc, flags=fl)
    assert np.abs(red - exact).max() < 1e-12
    bad = oracle.attention_head_bf16(Q, K, V, perm, sc, flags=fl | oracle.PLANT_NO_RESCALE)
    assert np.abs(bad - exact).max() > 1e-2
    # with ExpCast codes the largest code stays <= 120 (never the 126 clamp)
    ops = oracle.smooth_quantize_head(Q, K, V, perm)
    O, _, lblk = oracle.attention_head(ops, N, sc, rows=np.arange(0, N, 50, dtype=np.int32), want_lblk=True)
    assert np.all(np.isfinite(O)) and np.all(lblk <= 128 * 256.0)


@pytest.mark.parametrize("N", [200, 1000])
def test_same_algorithm_fidelity_and_row_sums(N):
    rng = np.random.default_rng(13)
    Q, K, V = _bits(rng, N), _bits(rng, N), _bits(rng, N)
    perm = rng.permutation(N).astype(np.int32)
    sc = 1 / math.sqrt(128)
    ops = oracle.smooth_quantize_head(Q, K, V, perm)
    rows = np.arange(0, N, 7, dtype=np.int32)
    O, lse, lblk = oracle.attention_head(ops, N, sc, rows=rows, want_lblk=True)
    exact = oracle.exact_attention_head(Q, K, V, sc, rows=rows)
    cos = (O * exact).sum() / np.sqrt((O * O).sum() * (exact * exact).sum())
    assert cos >= 0.99
    # lse: log of the sum of decoded probabilities, relative to the snapped max
    s = bits_to_f32(Q)[rows].astype(np.float64) @ bits_to_f32(K).astype(np.float64).T * sc
    true_lse = np.log(np.exp(s - s.max(1, keepdims=True)).sum(1)) + s.max(1)
    assert np.abs(lse - true_lse).max() < 0.06        # quantised scores + ExpCast, ~ln(1.05)
    assert lblk.shape == (len(rows), (N + 127) // 128) and np.all(lblk >= 0)
    # the snapped max keeps the largest decoded probability in [0.5, 1]... so sum >= 0.5
    assert np.all(lblk.sum(1) >= 0.5)


def test_same_algorithm_invariant_to_key_order_within_rounding():
    # Exact attention does not depend on the permutation; the quantised one
    # changes only through block statistics, so two different permutations
    # agree to the quantisation error, and identical permutations bit-for-bit.
    rng = np.random.default_rng(14)
    N = 300
    Q, K, V = _bits(rng, N), _bits(rng, N), _bits(rng, N)
    sc = 1 / math.sqrt(128)
    p1 = rng.permutation(N).astype(np.int32)
    a = oracle.attention_head_bf16(Q, K, V, p1, sc)
    b = oracle.attention_head_bf16(Q, K, V, p1.copy(), sc)
    assert np.array_equal(a, b)
    c = oracle.attention_head_bf16(Q, K, V, np.arange(N, dtype=np.int32), sc)
    ex = oracle.exact_attention_head(Q, K, V, sc)
    for o in (a, c):
        assert np.linalg.norm(o - ex) / np.linalg.norm(ex) < 0.08


# ------------------------------------------------------------------ Skip Softmax (BLASST)
def _skip_case(seed=31, N=700):
    # strong and weak key blocks alternate: the weak ones sit ~6 natural-log
    # units below the running maximum (rejected at lambda = 2^-6), the strong
    # ones within ~1 unit of it (kept)
    rng = np.random.default_rng(seed)
    qf = np.abs(rng.standard_normal((N, 128))) * 0.4
    kf = np.abs(rng.standard_normal((N, 128))) * 0.2
    blk = np.arange(N) // 128
    factor = np.array([12.0, 1.0, 11.5, 1.5, 12.0, 0.5, 11.0, 1.0])
    kf *= factor[blk % len(factor)][:, None]
    return bf16_bits_of(qf), bf16_bits_of(kf), _bits(rng, N)


def _survivors(Q, K, sc, lam, rows):
    # rejection decided from fp64 logits: block max vs the running max (which
    # includes the block), natural-log units
    q = bits_to_f32(Q).astype(np.float64)[rows]
    k = bits_to_f32(K).astype(np.float64)
    s = q @ k.T * sc
    N = k.shape[0]
    keep = np.ones_like(s, dtype=bool)
    for r in range(len(rows)):
        run = -np.inf
        for b in range(0, N, 128):
            m = s[r, b:b + 128].max()
            run = max(run, m)
            if b > 0 and np.exp(m - run) < lam:
                keep[r, b:b + 128] = False
    return keep


def test_skip_softmax_equals_exact_attention_over_the_kept_blocks():
    Q, K, V = _skip_case()
    N = Q.shape[0]
    perm = np.arange(N, dtype=np.int32)
    sc = 1 / math.sqrt(128)
    rows = np.arange(0, N, 23, dtype=np.int32)
    lam = 2.0 ** -6
    keep = _survivors(Q, K, sc, lam, rows)
    assert 0.05 < 1 - keep.mean() < 0.95           # the case really rejects blocks, not all
    fl = oracle.EXACT_EXP | oracle.IDENTITY_QUANT
    got = oracle.attention_head_bf16(Q, K, V, perm, sc, rows=rows, flags=fl, skip_lambda=lam)
    vf = bits_to_f32(V).astype(np.float64)
    q = bits_to_f32(Q).astype(np.float64)[rows]
    k = bits_to_f32(K).astype(np.float64)
    s = q @ k.T * sc
    for r in range(len(rows)):
        kk = keep[r]
        p = np.exp(s[r, kk] - s[r, kk].max())
        want = p @ vf[kk] / p.sum()
        assert np.abs(got[r] - want).max() < 1e-10
    # without the rule it is plain exact attention, which differs
    full = oracle.attention_head_bf16(Q, K, V, perm, sc, rows=rows, flags=fl)
    assert np.abs(full - got).max() > 1e-6


def test_skip_softmax_zero_lambda_is_the_plain_algorithm():
    Q, K, V = _skip_case(seed=32, N=400)
    perm = np.arange(Q.shape[0], dtype=np.int32)
    ops = oracle.smooth_quantize_head(Q, K, V, perm)
    a, la, _ = oracle.attention_head(ops, Q.shape[0], 1 / math.sqrt(128))
    b, lb, _ = oracle.attention_head(ops, Q.shape[0], 1 / math.sqrt(128), skip_lambda=0.0)
    assert np.array_equal(a, b) and np.array_equal(la, lb)
    # rejected blocks contribute a zero row sum
    rows = np.arange(0, Q.shape[0], 9, dtype=np.int32)
    _, _, lblk = oracle.attention_head(ops, Q.shape[0], 1 / math.sqrt(128), rows=rows, want_lblk=True,
                                       skip_lambda=2.0 ** -6)
    keep = _survivors(Q, K, 1 / math.sqrt(128), 2.0 ** -6, rows)[:, ::128]
    assert np.all(lblk[~keep] == 0.0) and np.all(lblk[keep] > 0.0)


# ------------------------------------------------------------------ SAGE-style comparison recipe
def _e4m3_table():
    return np.array([oracle.lib().vo_e4m3_decode(i) for i in range(256)], np.float64)


def _e4m3_err_bound(x_scaled):
    # round-to-nearest E4M3: half an ulp, i.e. 2^(e-4) for normal values and
    # 2^-10 in the subnormal range (scaled units); the 1e-4 slack covers the
    # fp32 scale product (x * (448/amax) is rounded in fp32 before encoding,
    # so a value the fp64 check places just past a midpoint may sit on it)
    e = np.floor(np.log2(np.maximum(np.abs(x_scaled), 2.0 ** -6)))
    return np.ldexp(1.0, (e - 4).astype(int)) * (1.0 + 1e-4)


def test_sage_quantisers_follow_their_definition():
    rng = np.random.default_rng(41)
    N = 300
    Q, K, V = _bits(rng, N), _bits(rng, N), _bits(rng, N)
    ops = oracle.sage_quantize_head(Q, K, V)
    dec = _e4m3_table()
    qf, kf, vf = (bits_to_f32(a).astype(np.float64) for a in (Q, K, V))
    # K mean: exact mean over all tokens, rounded once to bf16
    want_mean = bf16_bits_of(kf.mean(0).astype(np.float64))
    assert np.array_equal(ops["k_mean"], want_mean)
    km = bits_to_f32(ops["k_mean"]).astype(np.float64)
    # Q: one scale per token
    assert np.allclose(ops["q_scale"][:N], np.abs(qf).max(1).astype(np.float32) / np.float32(448), rtol=0, atol=0)
    qrec = dec[ops["Qq"][:N]] * ops["q_scale"][:N, None]
    assert np.all(np.abs(qrec - qf) <= _e4m3_err_bound(qf / ops["q_scale"][:N, None]) * ops["q_scale"][:N, None])
    # K: smoothed, one scale per 16 tokens
    ks = np.repeat(ops["k_scale"], 16)[:N, None].astype(np.float64)
    kp = (kf.astype(np.float32) - km.astype(np.float32)).astype(np.float64)
    krec = dec[ops["Kq"][:N]] * ks
    assert np.all(np.abs(krec - kp) <= _e4m3_err_bound(kp / ks) * ks)
    # V: one scale per channel over all tokens
    vs = ops["v_chscale"].astype(np.float64)
    assert np.allclose(vs, (np.abs(vf).max(0).astype(np.float32) / np.float32(448)), rtol=0, atol=0)
    vrec = dec[ops["VcT"][:, :N].T] * vs[None, :]
    assert np.all(np.abs(vrec - vf) <= _e4m3_err_bound(vf / vs[None, :]) * vs[None, :])


def test_sage_attention_is_exact_softmax_on_its_dequantised_operands():
    # with exact exponentials the row algorithm must equal plain softmax
    # attention on Q^, K'^ (the smoothed keys) and V^ * channel scale
    rng = np.random.default_rng(42)
    N = 350
    Q, K, V = _bits(rng, N), _bits(rng, N), _bits(rng, N)
    ops = oracle.sage_quantize_head(Q, K, V)
    dec = _e4m3_table()
    sc = 1 / math.sqrt(128)
    rows = np.arange(0, N, 11, dtype=np.int32)
    got, _ = oracle.attention_head_sage(ops, N, sc, rows=rows, flags=oracle.EXACT_EXP)
    q = dec[ops["Qq"][:N]] * ops["q_scale"][:N, None]
    k = dec[ops["Kq"][:N]] * np.repeat(ops["k_scale"], 16)[:N, None]
    v = dec[ops["VcT"][:, :N].T] * ops["v_chscale"][None, :].astype(np.float64)
    s = q[rows] @ k.T * sc
    p = np.exp(s - s.max(1, keepdims=True))
    want = p @ v / p.sum(1, keepdims=True)
    assert np.abs(got - want).max() < 1e-10


def test_k_mean_smoothing_leaves_softmax_attention_unchanged():
    # the identity the recipe relies on: q.(k - mu) = q.k - q.mu, a per-row shift
    rng = np.random.default_rng(43)
    q, k, v = rng.standard_normal((40, 128)), rng.standard_normal((90, 128)) + 3.0, rng.standard_normal((90, 128))
    def att(kk):
        s = q @ kk.T / math.sqrt(128)
        p = np.exp(s - s.max(1, keepdims=True))
        return p @ v / p.sum(1, keepdims=True)
    assert np.abs(att(k) - att(k - k.mean(0))).max() < 1e-12
