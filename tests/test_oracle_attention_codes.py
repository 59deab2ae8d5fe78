"""Pins of the oracle's in-attention ExpCast step and its reference rule.

The oracle's attention writes, for every key, the byte
    code = clamp(rne(8 z + 55 - 8 n + 8 * 4), 0, 126)
(the ExpCast byte of z - m + 4 with m = n + 0.65/8 the reference maximum on the
phi grid, four octaves of headroom), computed in fp64.  Here that step is tied
to the separately pinned encoder ``oracle.expcast`` (the pages' 0x38 at p = 1,
79.6 % per-octave agreement, 3.64 % TV bound): z is recomputed in numpy from
operands decoded by the library's float8_e4m3fn, the reference from the block
maxima, and every code must equal expcast(float32(z - n - phi + 4)) except at
near-ties, where the fp32 argument of expcast and the oracle's fp64 sum may round
apart.  The per-block row sums must be the exact sums of the decoded codes.

Sources: "VC-Attention: Training-Free Low-Bit Attention Speeds Video Diffusion
Up to 3.6x" (ExpCast-FP8 bullet); "Nunchux AI Introduces VC-Attention..."
(abstract: byte ~ 8 log2 p + 56 + beta, one FMA).
"""
import math

import numpy as np
import pytest
import torch

import oracle

from helpers import PHI, e4m3_lib
from helpers import scores_log2 as _scores_log2

HEADROOM = 4
LAG = 4
SCALE = 1 / math.sqrt(128)


def bf16_bits_of(x):
    return (torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
            .view(torch.int16).numpy().view(np.uint16))


def scores_log2(ops, N, rows, scale=SCALE):
    return _scores_log2(ops, N, rows, scale)


def reference_per_block(z, N, global_max=False):
    """The integer n of the reference each key block is coded against:
    n_b = ceil(block max - phi); online, the first block sets it and it moves
    to n_b only when n_b exceeds it by more than 4; global, it is the snapped
    maximum of the whole row."""
    nb = -(-N // 128)
    zb = np.stack([z[:, b * 128:min(N, (b + 1) * 128)].max(1) for b in range(nb)], 1)
    nblk = np.ceil(zb - PHI)
    # rows whose block maxima sit on a grid point are ambiguous at fp64 rounding
    tie = (np.abs(zb - PHI - np.round(zb - PHI)) < 1e-9).any(1)
    if global_max:
        n = np.repeat(np.ceil(z.max(1) - PHI)[:, None], nb, 1)
        return n, tie
    n = np.empty_like(nblk)
    n[:, 0] = nblk[:, 0]
    for b in range(1, nb):
        n[:, b] = np.where(nblk[:, b] > n[:, b - 1] + LAG, nblk[:, b], n[:, b - 1])
    return n, tie


def code_pin(ops, N, rows, flags=0, headroom=HEADROOM, global_max=False):
    """Runs the oracle's attention and checks its codes, references and row
    sums.  Returns (mismatch fraction of the codes, compared count, details)."""
    O, lse, lblk, codes, nref = oracle.attention_head_codes(ops, N, SCALE, rows=rows, flags=flags)
    z = scores_log2(ops, N, rows)
    n, tie_rows = reference_per_block(z, N, global_max)
    keep = ~tie_rows
    assert keep.mean() > 0.9
    assert np.array_equal(nref[keep], n[keep].astype(np.int32)), "reference rule differs"
    nk = n[:, np.arange(N) // 128]
    want = oracle.expcast((z - nk - PHI + headroom).astype(np.float32))
    x = 8.0 * z + 55.0 - 8.0 * nk + 8.0 * headroom
    near_tie = np.abs(x - np.floor(x) - 0.5) < 1e-4
    cmp = keep[:, None] & ~near_tie
    mism = float((codes != want)[cmp].mean())
    # per-block row sums = exact sums of the decoded codes, in the final frame
    dec = e4m3_lib(codes)
    nb = nref.shape[1]
    sums = np.stack([dec[:, b * 128:min(N, (b + 1) * 128)].sum(1) for b in range(nb)], 1)
    frame = np.ldexp(1.0, (nref - nref[:, -1:]).astype(np.int64))
    assert np.array_equal(lblk, sums * frame), "row sums are not the sums of the decoded codes"
    return mism, int(cmp.sum()), dict(codes=codes, nref=nref, O=O, lse=lse)


def _random_case(N, seed):
    rng = np.random.default_rng(seed)
    Q, K, V = (bf16_bits_of(rng.standard_normal((N, 128)).astype(np.float32)) for _ in range(3))
    perm = rng.permutation(N).astype(np.int32)
    return oracle.smooth_quantize_head(Q, K, V, perm)


def _climbing_case(N=900, seed=21):
    # later key blocks score much higher: the online reference moves up by more
    # than 4 octaves several times
    rng = np.random.default_rng(seed)
    kf = rng.standard_normal((N, 128))
    kf = np.abs(kf * (1.0 + np.arange(N) // 128)[:, None] * 1.5)
    qf = np.abs(rng.standard_normal((N, 128))) * 0.5
    V = bf16_bits_of(rng.standard_normal((N, 128)).astype(np.float32))
    return oracle.smooth_quantize_head(bf16_bits_of(qf), bf16_bits_of(kf), V, np.arange(N, dtype=np.int32))


CASES = {"random-N1000": lambda: (_random_case(1000, 13), 1000),
         "random-N200": lambda: (_random_case(200, 5), 200),
         "climbing-N900": lambda: (_climbing_case(), 900)}


@pytest.mark.parametrize("name", sorted(CASES))
def test_attention_codes_are_expcast_of_the_referenced_score(name):
    ops, N = CASES[name]()
    rows = np.arange(0, N, 3, dtype=np.int32)
    mism, n, _ = code_pin(ops, N, rows)
    assert n > 0.95 * len(rows) * N
    assert mism == 0.0


def test_reference_moves_on_the_climbing_case():
    ops, N = CASES["climbing-N900"]()
    rows = np.arange(0, N, 3, dtype=np.int32)
    _, _, det = code_pin(ops, N, rows)
    moves = (np.diff(det["nref"], axis=1) > 0).sum(1)
    assert moves.max() >= 2          # the lag rule is exercised, not just the first block
    assert det["codes"].max() <= 120  # four octaves of lag + four of headroom stay below 126


@pytest.mark.parametrize("plant", [oracle.PLANT_TRUNC, oracle.PLANT_BETA0])
@pytest.mark.parametrize("name", ["random-N1000", "climbing-N900"])
def test_planted_code_mistakes_fail_the_code_pin(name, plant):
    ops, N = CASES[name]()
    rows = np.arange(0, N, 5, dtype=np.int32)
    mism, _, _ = code_pin(ops, N, rows, flags=plant)
    assert mism > 0.2   # truncation moves ~1/2 of the codes, beta = 0 ~0.35 of them


@pytest.mark.parametrize("name", sorted(CASES))
def test_global_max_reading_codes_and_reduction(name):
    ops, N = CASES[name]()
    rows = np.arange(0, N, 3, dtype=np.int32)
    mism, _, det = code_pin(ops, N, rows, flags=oracle.GLOBAL_MAX, global_max=True)
    assert mism == 0.0
    # the row maximum lands on codes 80..88 (4 octaves above 0x38's octave)
    assert det["codes"].max(1).min() >= 80 and det["codes"].max() <= 88
    # without the 4-octave headroom it lands on 48..56, 0x38 = p 1 at the top
    mism0, _, det0 = code_pin(ops, N, rows, flags=oracle.GLOBAL_MAX | oracle.NO_HEADROOM, headroom=0,
                              global_max=True)
    assert mism0 == 0.0
    assert det0["codes"].max(1).min() >= 48 and det0["codes"].max() <= 0x38
    # with exact exponentials every reference rule is the same softmax
    a, la, _ = oracle.attention_head(ops, N, SCALE, rows=rows, flags=oracle.EXACT_EXP)
    b, lb, _ = oracle.attention_head(ops, N, SCALE, rows=rows, flags=oracle.EXACT_EXP | oracle.GLOBAL_MAX)
    c, lc, _ = oracle.attention_head(ops, N, SCALE, rows=rows,
                                     flags=oracle.EXACT_EXP | oracle.GLOBAL_MAX | oracle.NO_HEADROOM)
    assert np.abs(a - b).max() < 1e-12 and np.abs(a - c).max() < 1e-12
    assert np.abs(la - lb).max() < 1e-12 and np.abs(la - lc).max() < 1e-12


def test_online_and_global_codes_differ_by_whole_octaves_above_the_tail():
    # against a lagging reference the codes are the global-max codes shifted by
    # 8 per octave of lag, wherever neither side is in the underflow tail
    ops, N = CASES["climbing-N900"]()
    rows = np.arange(0, N, 3, dtype=np.int32)
    _, _, on = code_pin(ops, N, rows)
    _, _, gl = code_pin(ops, N, rows, flags=oracle.GLOBAL_MAX, global_max=True)
    z = scores_log2(ops, N, rows)
    nglob = np.ceil(z.max(1) - PHI)
    lag = (nglob[:, None] - on["nref"])[:, np.arange(N) // 128].astype(np.int64)
    c_on, c_gl = on["codes"].astype(np.int64), gl["codes"].astype(np.int64)
    normal = (c_gl >= 8) & (c_on >= 8)
    assert normal.sum() > 5000 and (lag[normal] > 0).any()
    assert np.array_equal(c_on[normal], c_gl[normal] + 8 * lag[normal])
