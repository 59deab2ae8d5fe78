"""The error bound behind the k-means assignment's candidate filter, checked on
the CPU.

The assignment ("VC-Attention" (aikraft.ru), section "Решение": a lightweight
k-means groups similar tokens) keeps the defined fp32 distance; the kernel only
skips centroids that a tensor-core estimate rules out.  The estimate is
d_c = |v|^2 + |mu_c|^2 - 2 v.mu_c with mu split into bf16 hi + lo, and the bound
it relies on is |d_c - D_c| < 2^-10 (|v|^2 + |mu_c|^2) + 2^-90, D_c the defined
fp32 distance.  Here the estimate is emulated in numpy with two summation orders
(sequential and pairwise fp32) and compared with the exact distance, whose own
fp32 rounding is at most 131 units of 2^-24; the bound must hold with a wide
margin, and on the workload recipe it must leave about one candidate per token
(else the filter would save nothing)."""
import numpy as np
import pytest
import torch

from bit_attention_video_02_b200 import workloads as W

REL, ABS = 2.0 ** -10, 2.0 ** -90
U = 2.0 ** -24


def _bf16(x32: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def _fp32_sum(terms: np.ndarray, pairwise: bool) -> np.ndarray:
    # sum over the last axis in fp32, sequentially or as a pairwise tree
    t = terms.astype(np.float32)
    if not pairwise:
        acc = np.zeros(t.shape[:-1], np.float32)
        for i in range(t.shape[-1]):
            acc = (acc + t[..., i]).astype(np.float32)
        return acc
    while t.shape[-1] > 1:
        t = (t[..., 0::2] + t[..., 1::2]).astype(np.float32)
    return t[..., 0]


def _estimate(v: np.ndarray, mu: np.ndarray, pairwise: bool) -> np.ndarray:
    hi = _bf16(mu)
    lo = _bf16((mu - hi).astype(np.float32))
    prods = np.concatenate([v[:, None, :] * hi[None], v[:, None, :] * lo[None]], axis=-1)   # exact in fp32
    dot = _fp32_sum(prods, pairwise)
    nv = _fp32_sum(v * v, pairwise)
    nc = _fp32_sum(mu * mu, pairwise)
    sn = (nv[:, None] + nc[None, :]).astype(np.float32)
    return (sn - np.float32(2.0) * dot).astype(np.float32), nv.astype(np.float64), nc.astype(np.float64)


def _check(v32: np.ndarray, mu32: np.ndarray):
    exact = ((v32.astype(np.float64)[:, None, :] - mu32.astype(np.float64)[None]) ** 2).sum(-1)
    worst = 0.0
    for pairwise in (False, True):
        d, nv, nc = _estimate(v32, mu32, pairwise)
        bound = REL * (nv[:, None] + nc[None, :]) + ABS
        # the defined fp32 distance is within 131 u of the exact one
        err = np.abs(d.astype(np.float64) - exact) + 131 * U * exact
        worst = max(worst, float((err / bound).max()))
    return worst, exact, d, nv, nc


@pytest.mark.parametrize("kind", ["workload", "common_mean", "tiny"])
def test_filter_bound_holds_with_margin(kind):
    rng = np.random.default_rng(5)
    if kind == "workload":
        w = W.shrink(W.WORKLOADS[3], H=1, N=2048)
        _, _, V = W.make_qkv(w, "cpu")
        v = V[0, 0].float().numpy()
    elif kind == "common_mean":
        # a large shared offset makes |v|^2 + |mu|^2 much larger than the distances
        v = _bf16(rng.normal(0, 1, (1024, 128)).astype(np.float32) + np.float32(300.0))
    else:
        v = _bf16(rng.normal(0, 1e-30, (1024, 128)).astype(np.float32))
    mu = v[rng.choice(len(v), 32, replace=False)].astype(np.float32)
    mu = (mu + rng.normal(0, 0.01, mu.shape).astype(np.float32) * np.abs(mu).max()).astype(np.float32)
    worst, *_ = _check(v.astype(np.float32), mu)
    # the kernel's bound is at least ten times the emulated error
    assert worst < 0.1, worst


def test_filter_keeps_about_one_candidate_on_the_workload():
    w = W.shrink(W.WORKLOADS[3], H=1, N=4096)
    _, _, V = W.make_qkv(w, "cpu")
    v = V[0, 0].float().numpy().astype(np.float32)
    mu = v[:: len(v) // w.k][: w.k].copy()          # the kernel's first-round centroids
    _, exact, d, nv, nc = _check(v, mu)
    e = REL * (nv[:, None] + nc[None, :]) + ABS
    ub = (d + e).min(1)
    cand = (d - e <= ub[:, None])
    # every exact argmin survives, and the filter drops nearly everything else
    assert cand[np.arange(len(v)), exact.argmin(1)].all()
    assert cand.sum(1).mean() < 1.2
