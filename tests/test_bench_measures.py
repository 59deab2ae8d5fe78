"""CPU checks of measurements bench.py reports: the block-mean energy share
(the share of a head's value energy that its 128-token block means carry, in
sequence order, in static cubes of the latent grid and in k-means order;
"Nunchux AI Introduces VC-Attention ...", abstract: 8 % / 12 % / 36 % on
Wan2.2 heads) and the algorithmic byte counts behind the roofline fractions."""
import os
import sys

import numpy as np
import pytest
import torch

import oracle

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def brute_share(v, groups):
    """1 - sum |v - mean_g|^2 / sum |v|^2 with explicit loops over the groups."""
    total = float((v.astype(np.float64) ** 2).sum())
    resid = 0.0
    for g in groups:
        x = v[g].astype(np.float64)
        resid += float(((x - x.mean(axis=0)) ** 2).sum())
    return 1.0 - resid / total


def test_constant_and_zero_mean_blocks():
    rng = np.random.default_rng(0)
    N, d = 300, 16
    base = rng.standard_normal((3, d))
    v = np.repeat(base, [128, 128, 44], axis=0)      # every block constant
    seq = torch.arange(N) // 128
    assert bench.group_mean_energy(torch.from_numpy(v), seq, 3) == pytest.approx(1.0, abs=1e-12)
    x = rng.standard_normal((150, d))
    v0 = np.concatenate([x[:64], -x[:64], x[64:128], -x[64:128], x[128:150], -x[128:150]])
    assert bench.group_mean_energy(torch.from_numpy(v0), seq, 3) == pytest.approx(0.0, abs=1e-12)


def test_share_matches_brute_force_for_every_grouping():
    rng = np.random.default_rng(1)
    T, Hg, Wg = 3, 10, 12
    N, d = T * Hg * Wg, 8
    v = rng.standard_normal((N, d)) + rng.standard_normal(d)
    vt = torch.from_numpy(v)
    seq = torch.arange(N) // 128
    nb = (N + 127) // 128
    want = brute_share(v, [np.arange(N)[np.arange(N) // 128 == b] for b in range(nb)])
    assert bench.group_mean_energy(vt, seq, nb) == pytest.approx(want, rel=1e-12)
    gid, ng = bench.cube_groups((T, Hg, Wg), N, "cpu")
    # brute force cube membership from the coordinates
    idx = np.arange(N)
    t, h, w = idx // (Hg * Wg), (idx // Wg) % Hg, idx % Wg
    key = (t // 2) * 1000000 + (h // 8) * 1000 + (w // 8)
    groups = [idx[key == k] for k in np.unique(key)]
    assert len(groups) == len(np.unique(gid.numpy())) and ng >= len(groups)
    assert max(len(g) for g in groups) <= 128
    for g in groups:
        assert len(np.unique(gid.numpy()[g])) == 1
    assert bench.group_mean_energy(vt, gid, ng) == pytest.approx(brute_share(v, groups), rel=1e-12)


def test_full_cubes_hold_128_tokens_on_the_wan_grid():
    gid, ng = bench.cube_groups((21, 45, 80), 75600, "cpu")
    cnt = torch.bincount(gid, minlength=ng)
    assert int(cnt.sum()) == 75600
    # 10 x 6 x 10 cubes of up to 2 x 8 x 8; t = 20 and h = 40..44 are ragged
    assert ng == 11 * 6 * 10 and int(cnt.max()) == 128
    assert int((cnt == 128).sum()) == 10 * 5 * 10


def test_sorting_by_clusters_raises_the_share():
    # a head whose values come from a few centroids in shuffled sequence order:
    # after the k-means order most blocks hold one centroid
    rng = np.random.default_rng(2)
    N, d, k = 1024, 128, 8
    cent = rng.standard_normal((k, d)) * 3
    lab = rng.integers(0, k, N)
    v = (cent[lab] + 0.1 * rng.standard_normal((N, d))).astype(np.float32)
    bits = torch.from_numpy(v).to(torch.bfloat16)
    ops = oracle.prep_head(bits.view(torch.int16).numpy().view(np.uint16),
                           bits.view(torch.int16).numpy().view(np.uint16),
                           bits.view(torch.int16).numpy().view(np.uint16), k=k, iters=3)
    perm = torch.from_numpy(ops["perm"].astype(np.int64))
    V = bits.float().reshape(1, 1, N, d)
    got = bench.block_mean_energy(V, perm.reshape(1, 1, N), None)
    assert set(got) == {"sequence", "sorted"}
    # blocks straddle cluster boundaries (no padding), so the sorted share stays below 1
    assert got["sorted"] > 0.6 and got["sequence"] < 0.3
    # the sorted share is the sequence share of the permuted tokens
    Vp = V[:, :, perm]
    same = bench.block_mean_energy(Vp, torch.arange(N).reshape(1, 1, N), None)
    assert same["sequence"] == pytest.approx(got["sorted"], abs=1e-4)


def test_kmeans_order_reaches_the_between_cluster_share_on_a_separable_mixture():
    # 8 well-separated clusters of exactly 128 tokens in shuffled order, one of
    # them at each k-means seed position (token c*N/k): the grouping must recover
    # the clusters, every sorted block is one cluster, and the share equals the
    # between-cluster energy fraction sum_c n_c |mean_c|^2 / sum |v|^2
    rng = np.random.default_rng(5)
    N, d, k = 1024, 128, 8
    lab = rng.permutation(np.repeat(np.arange(k), N // k))
    for c in range(k):                      # cluster c at seed position c * 128
        j = np.flatnonzero(lab == c)[0]
        lab[[j, c * 128]] = lab[[c * 128, j]]
    cent = rng.standard_normal((k, d)) * 4
    v = (cent[lab] + 0.05 * rng.standard_normal((N, d))).astype(np.float32)
    vb = torch.from_numpy(v).to(torch.bfloat16)
    vbits = vb.view(torch.int16).numpy().view(np.uint16)
    cents, assign, counts = oracle.kmeans_head(vbits, k, 3)
    perm = oracle.stable_perm(assign, k)
    # the partition is recovered (cluster ids may be relabelled)
    assert sorted(counts.tolist()) == [128] * k
    for c in range(k):
        assert len(np.unique(assign[lab == c])) == 1
    vf = vb.float().numpy().astype(np.float64)
    between = sum(128 * float((vf[lab == c].mean(axis=0) ** 2).sum()) for c in range(k)) / float((vf ** 2).sum())
    got = bench.block_mean_energy(vb.float().reshape(1, 1, N, d), torch.from_numpy(perm.astype(np.int64)).reshape(1, 1, N),
                                  None)
    assert got["sorted"] == pytest.approx(between, abs=1e-4)
    assert got["sequence"] < 0.5 * between


def test_roofline_byte_counts_match_their_closed_forms():
    # the algorithmic bytes the bench divides by, per (b, h), as stated beside the kernels
    from bit_attention_video_02_b200 import workloads as W
    w = W.WORKLOADS[3]
    N, d, nb = w.N, w.d, (w.N + 127) // 128
    Np = 128 * nb
    per_head = 3 * N * d * 2 + 4 * N + 2 * Np * d + Np * 64 + Np * 8 + 2 * nb * 4 + nb * d * 2 + 4
    assert bench.fp4_prep_algorithmic_bytes(w) == w.B * w.H * per_head == 3_333_270_880
    # 8-bit prep: Q, K, V in once and Qq, Kq, VrT out (9 B per element), V once more per
    # k-means round, the block means
    assert bench.prep_algorithmic_bytes(w) == 9.0 * w.B * w.H * N * d + 3 * 2.0 * w.B * w.H * N * d \
        + 2.0 * w.B * w.H * nb * d
    assert bench.whole_job_value(2, w.flops, 0.1) == pytest.approx(2 * w.flops / 0.1 / 1e12)
