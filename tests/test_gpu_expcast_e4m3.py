"""GPU vs oracle, bit for bit: the ExpCast-FP8 byte map and the E4M3 encoder."""
import numpy as np
import pytest
import torch

import oracle
from bit_attention_video_02_b200 import vca

pytestmark = pytest.mark.gpu


def _gpu_expcast(z: np.ndarray) -> np.ndarray:
    return vca.expcast_ref(torch.from_numpy(np.ascontiguousarray(z)).cuda()).cpu().numpy()


def _gpu_e4m3(x: np.ndarray) -> np.ndarray:
    return vca.e4m3_encode(torch.from_numpy(np.ascontiguousarray(x)).cuda()).cpu().numpy()


def test_expcast_boundaries_and_specials():
    k = np.arange(-60, 140, dtype=np.float64)
    edges = ((k + 0.5 - 55.65) / 8.0).astype(np.float32)        # rounding boundaries of 8z+55.65
    near = np.concatenate([edges, *[np.nextafter(edges, np.float32(s * np.inf)) for s in (-1, 1)]])
    for _ in range(3):
        near = np.concatenate([near, np.nextafter(near, np.float32(np.inf)), np.nextafter(near, np.float32(-np.inf))])
    special = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, -np.nan, 1e-45, -1e-45, 3.4e38, -3.4e38,
                        -6.9, -6.89375, -6.95625, 8.79375, 8.8, 9.0], np.float32)
    z = np.concatenate([near, special]).astype(np.float32)
    assert np.array_equal(_gpu_expcast(z), oracle.expcast(z))


def test_expcast_exhaustive_all_fp32_patterns():
    # every fp32 bit pattern, in chunks of 2^28
    step = 1 << 28
    for start in range(0, 1 << 32, step):
        u = np.arange(start, start + step, dtype=np.uint32)
        z = u.view(np.float32)
        g = _gpu_expcast(z)
        o = oracle.expcast(z)
        bad = np.nonzero(g != o)[0]
        assert bad.size == 0, (hex(int(u[bad[0]])), int(g[bad[0]]), int(o[bad[0]]))


def test_e4m3_encoder_exhaustive_over_the_finite_range():
    # every fp32 pattern with |x| in [2^-12, 2^10) (all of E4M3's rounding
    # decisions), both signs, plus the extremes
    lo = int(np.float32(2.0 ** -12).view(np.uint32))
    hi = int(np.float32(2.0 ** 10).view(np.uint32))
    for sign in (0, 0x80000000):
        for i in range(lo, hi, 1 << 27):
            xs = (np.arange(i, min(hi, i + (1 << 27)), dtype=np.uint32) | np.uint32(sign)).view(np.float32)
            g, o = _gpu_e4m3(xs), oracle.e4m3_encode(xs)
            bad = np.nonzero(g != o)[0]
            assert bad.size == 0, (float(xs[bad[0]]), int(g[bad[0]]), int(o[bad[0]]))
    extremes = np.array([0.0, -0.0, 1e-45, -1e-45, 1e-30, -1e-30, 2.0 ** -11, 2.0 ** -10, -(2.0 ** -10),
                         448.0, 464.0, 465.0, 1e9, -1e9, np.inf, -np.inf], np.float32)
    assert np.array_equal(_gpu_e4m3(extremes), oracle.e4m3_encode(extremes))


def test_expcast_odd_lengths():
    rng = np.random.default_rng(0)
    for n in (1, 3, 4, 5, 1023, 4097):
        z = (rng.standard_normal(n) * 8).astype(np.float32)
        assert np.array_equal(_gpu_expcast(z), oracle.expcast(z))
