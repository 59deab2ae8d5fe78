"""GPU vs oracle, bit for bit: k-means assignment and centroids, the cluster
permutation, and every V-Smooth quantised operand (E4M3 Q/K/V-residual
bytes, block scales, V exponents, block means)."""
import numpy as np
import pytest
import torch

import oracle
from bit_attention_video_02_b200 import vca
from bit_attention_video_02_b200 import workloads as W
from helpers import bits

pytestmark = pytest.mark.gpu

# (workload, heads, tokens): the small workloads at full size, the others at
# reduced sizes with ragged tails, and degenerate sizes
CASES = [(1, None, None), (2, None, None), (3, 2, 1000), (4, 2, 640), (5, 2, 200),
         (1, 1, 1), (1, 1, 129), (2, 3, 128), (3, 1, 4097)]


def _ids(c):
    return f"cfg{c[0]}-H{c[1] or 'full'}-N{c[2] or 'full'}"


def _gpu_prep(w, Q, K, V, init=None):
    cent, assign, perm = vca.cluster_permute(V, w.k, iters=3, init=init)
    ops = vca.smooth_quantize(Q, K, V, perm)
    torch.cuda.synchronize()
    return cent, assign, perm, ops


def _compare_head(w, Q, K, V, cent, assign, perm, ops, b, h, init=None):
    Qb, Kb, Vb = (bits(t[b, h]) for t in (Q, K, V))
    ref = oracle.prep_head(Qb, Kb, Vb, w.k, 3, init)
    assert np.array_equal(assign[b, h].cpu().numpy(), ref["assign"]), "k-means assignment"
    assert np.array_equal(cent[b, h].cpu().numpy().view(np.uint32), ref["centroids"].view(np.uint32)), "centroids"
    assert np.array_equal(perm[b, h].cpu().numpy(), ref["perm"]), "permutation"
    for name in ("Qq", "Kq", "VrT"):
        g = ops[name][b, h].cpu().numpy()
        bad = np.argwhere(g != ref[name])
        assert bad.size == 0, (name, bad[:3].tolist())
    for name in ("q_scale", "k_scale"):
        assert np.array_equal(ops[name][b, h].cpu().numpy().view(np.uint32), ref[name].view(np.uint32)), name
    assert np.array_equal(ops["v_exp"][b, h].cpu().numpy(), ref["v_exp"]), "v_exp"
    assert np.array_equal(ops["v_mean"][b, h].cpu().view(torch.int16).numpy().view(np.uint16), ref["v_mean"]), "v_mean"


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_prep_bit_exact(case):
    cid, H, N = case
    w = W.shrink(W.WORKLOADS[cid], H=H, N=N)
    Q, K, V = W.make_qkv(w, "cuda")
    cent, assign, perm, ops = _gpu_prep(w, Q, K, V)
    for h in range(w.H):
        _compare_head(w, Q, K, V, cent, assign, perm, ops, 0, h)


def test_prep_warm_start_and_reused_permutation():
    # denoising steps: centroids of step 0 warm-start a later step; the step-0
    # permutation is reused to quantise steps 1..3
    w = W.shrink(W.WORKLOADS[4], H=2, N=1024)
    Q0, K0, V0 = W.make_qkv(w, "cuda", step=0)
    cent0, _, perm0, _ = _gpu_prep(w, Q0, K0, V0)
    for step in (1, 3):
        Q, K, V = W.make_qkv(w, "cuda", step=step)
        cent, assign, perm, ops = _gpu_prep(w, Q, K, V, init=cent0)
        for h in range(w.H):
            _compare_head(w, Q, K, V, cent, assign, perm, ops, 0, h, init=cent0[0, h].cpu().numpy())
        ops_r = vca.smooth_quantize(Q, K, V, perm0)
        for h in range(w.H):
            ref = oracle.smooth_quantize_head(*(bits(t[0, h]) for t in (Q, K, V)), perm0[0, h].cpu().numpy())
            for name in ("Qq", "Kq", "VrT", "v_exp"):
                assert np.array_equal(ops_r[name][0, h].cpu().numpy(), ref[name]), name


@pytest.mark.parametrize("cid", [3, 4, 5])
def test_prep_full_size_sampled_heads(cid):
    w = W.WORKLOADS[cid]
    Q, K, V = W.make_qkv(w, "cuda")
    cent, assign, perm, ops = _gpu_prep(w, Q, K, V)
    for h in (0, w.H - 1):
        _compare_head(w, Q, K, V, cent, assign, perm, ops, 0, h)
    # padding of the last block is zero, the permutation is a bijection everywhere
    nb = (w.N + 127) // 128
    assert not ops["Kq"][:, :, w.N:].any() and not ops["VrT"][:, :, :, w.N:].any()
    ps = torch.sort(perm.long(), dim=-1).values
    assert torch.equal(ps, torch.arange(w.N, device=ps.device).expand_as(ps))
    assert ops["v_exp"].shape[-1] == nb


def test_nonfinite_input_is_reported():
    w = W.shrink(W.WORKLOADS[1], H=1, N=256)
    Q, K, V = W.make_qkv(w, "cuda")
    V[0, 0, 5, 7] = float("nan")
    perm = torch.arange(256, dtype=torch.int32, device="cuda").view(1, 1, 256).contiguous()
    ws = vca.Workspace(256)
    vca.smooth_quantize(Q, K, V, perm, ws=ws)
    with pytest.raises(vca.VcaError) as e:
        ws.check()
    assert e.value.code == vca.ERR_NONFINITE
    ws.check()   # cleared after reading


@pytest.mark.parametrize("bad,code", [(2.0 ** 21, "ERR_INVALID"), (float("inf"), "ERR_NONFINITE")])
def test_grouping_reports_values_outside_its_exact_range(bad, code):
    # the k-means sums are exact only for |v| < 2^20: a larger or non-finite
    # value is recorded in the workspace status word
    w = W.shrink(W.WORKLOADS[1], H=2, N=600)
    _, _, V = W.make_qkv(w, "cuda")
    V[0, 1, 77, 5] = bad
    ws = vca.Workspace(vca.lib().vca_cluster_permute_workspace_size(1, w.H, w.N, w.k))
    vca.cluster_permute(V, w.k, 3, ws=ws)
    with pytest.raises(vca.VcaError) as e:
        ws.check()
    assert e.value.code == getattr(vca, code)
    # in range: no error
    V[0, 1, 77, 5] = 2.0 ** 19
    vca.cluster_permute(V, w.k, 3, ws=ws)
    ws.check()


@pytest.mark.parametrize("k", [1, 5, 32, 33, 64])
def test_assignment_ties_and_near_ties(k):
    # the assignment evaluates the defined distance only for the centroids a
    # tensor-core estimate cannot rule out: centroids that tie exactly (the
    # lower index must win), differ by one unit in the last place, or sit on
    # either side of a token at the same distance must all reach the exact
    # comparison, and the result must equal the oracle's full scan
    w = W.shrink(W.WORKLOADS[2], H=2, N=777)
    _, _, V = W.make_qkv(w, "cuda")
    Vf = V.float().cpu().numpy()
    rng = np.random.default_rng(11 + k)
    init = np.empty((1, w.H, k, 128), dtype=np.float32)
    for h in range(w.H):
        idx = rng.choice(w.N, size=k, replace=False)
        c = Vf[0, h, idx].copy()
        if k >= 2:
            c[1] = c[0]                                   # exact tie with centroid 0
        if k >= 4:
            c[3] = c[2]
            c[3, 17] = np.nextafter(c[2, 17], np.float32(np.inf))   # one ulp apart
        if k >= 6:
            t = Vf[0, h, idx[4]]                          # a token between 4 and 5
            c[4] = t
            c[5] = t
            c[4, 9] = t[9] + np.float32(0.25)
            c[5, 9] = t[9] - np.float32(0.25)
        init[0, h] = c
    _, assign, _ = vca.cluster_permute(V, k, iters=1, init=torch.from_numpy(init).cuda())
    torch.cuda.synchronize()
    for h in range(w.H):
        want = oracle.kmeans_assign(Vf[0, h], init[0, h])
        got = assign[0, h].cpu().numpy()
        assert np.array_equal(got, want), (h, np.argwhere(got != want)[:5].tolist())
