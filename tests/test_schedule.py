"""Denoising-schedule reuse of the grouping ("Nunchux AI Introduces
VC-Attention...", abstract and section "V-Smooth 與 ExpCast-FP8": grouping only
in the first 25 % of the denoising steps, each permutation reused across 4
adjacent steps).  The rule lives in the library (vca_schedule_regroup, a host
function); the per-layer state in vca.VCAttentionLayer."""
import numpy as np
import pytest
import torch

from bit_attention_video_02_b200 import vca
from bit_attention_video_02_b200 import workloads as W


def regroup_steps(total, reuse=4, frac=0.25):
    return [s for s in range(total) if vca.schedule_regroup(s, total, reuse, frac)]


def test_schedule_first_quarter_every_fourth_step():
    # 50 steps: the first quarter is steps 0..12 (12 < 12.5), regroup every 4th
    assert regroup_steps(50) == [0, 4, 8, 12]
    assert regroup_steps(40) == [0, 4, 8]
    assert regroup_steps(8) == [0]            # first quarter is steps 0, 1
    assert regroup_steps(1) == [0]
    assert regroup_steps(16, reuse=1) == [0, 1, 2, 3]
    assert regroup_steps(10, reuse=4, frac=1.0) == [0, 4, 8]


def test_schedule_amortisation_counts():
    # the grouping runs on ceil(frac * S / reuse) steps: ~S/16 with the pages' numbers
    for S in (16, 30, 50, 64, 100):
        n = len(regroup_steps(S))
        assert n == -(-int(np.ceil(0.25 * S)) // 4)
        assert n <= S / 16 + 1


@pytest.mark.parametrize("args", [(-1, 10, 4, 0.25), (10, 10, 4, 0.25), (0, 0, 4, 0.25), (0, 10, 0, 0.25),
                                  (0, 10, 4, 0.0), (0, 10, 4, 1.5), (0, 10, 4, float("nan"))])
def test_schedule_rejects_bad_arguments(args):
    assert vca.lib().vca_schedule_regroup(*args) == vca.ERR_INVALID
    assert b"vca_schedule_regroup" in vca.lib().vca_last_error()


@pytest.mark.gpu
def test_layer_reuses_and_warm_starts_the_grouping():
    import oracle
    from helpers import bf16_to_f64, bits, rel_l2, sample_rows
    w = W.shrink(W.WORKLOADS[4], H=2, N=3000)
    total = 20                                  # first quarter: steps 0..4 -> regroup at 0 and 4
    layer = vca.VCAttentionLayer(total, k=w.k, iters=3)
    perms, cents = {}, {}
    outs = {}
    for step in range(6):
        Q, K, V = W.make_qkv(w, "cuda", step=step)
        outs[step] = layer(Q, K, V, step)
        perms[step] = layer.perm.clone()
        cents[step] = layer.centroids.clone()
    torch.cuda.synchronize()
    assert layer.regrouped_at == [0, 4]
    for s in (1, 2, 3):
        assert torch.equal(perms[s], perms[0])
    assert torch.equal(perms[5], perms[4])
    # step 4 regrouped from step 0's centroids: the same as a direct warm-started call
    Q4, K4, V4 = W.make_qkv(w, "cuda", step=4)
    c4, _, p4 = vca.cluster_permute(V4, w.k, 3, init=cents[0])
    assert torch.equal(p4, perms[4]) and torch.equal(c4, cents[4])
    # step 5 output = the plain path with the reused permutation (bit for bit),
    # and within the attention tolerance of the oracle on sampled rows
    Q5, K5, V5 = W.make_qkv(w, "cuda", step=5)
    ref = vca.vc_attention(Q5, K5, V5, k=w.k, perm=perms[4])
    assert torch.equal(ref, outs[5])
    scale = 1.0 / np.sqrt(w.d)
    for h in range(w.H):
        Qb, Kb, Vb = (bits(t[0, h]) for t in (Q5, K5, V5))
        ops = oracle.smooth_quantize_head(Qb, Kb, Vb, perms[4][0, h].cpu().numpy())
        rows = sample_rows(w.N, 128, 500 + h)
        o_ref, _, _ = oracle.attention_head(ops, w.N, scale, rows=rows)
        assert rel_l2(bf16_to_f64(outs[5][0, h])[rows], o_ref) <= 1e-2
