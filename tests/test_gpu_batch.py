"""Batch > 1: every kernel flattens (batch, head); each (b, h) must match the
oracle exactly as with B = 1 (prep and SAGE quantisation bit for bit, attention
within the tolerance)."""
import math

import numpy as np
import pytest
import torch

import oracle
from bit_attention_video_02_b200 import vca
from bit_attention_video_02_b200 import workloads as W
from helpers import bf16_to_f64, bits, rel_l2, sample_rows

pytestmark = pytest.mark.gpu


def _batch2(w):
    # two different layers' inputs (denoising steps 0 and 1) as batch entries
    a, b = W.make_qkv(w, "cuda", step=0), W.make_qkv(w, "cuda", step=1)
    return tuple(torch.cat([x, y], 0).contiguous() for x, y in zip(a, b))


def test_vsmooth_path_batch2():
    w = W.shrink(W.WORKLOADS[4], H=2, N=900)
    Q, K, V = _batch2(w)
    scale = 1.0 / math.sqrt(w.d)
    cent, assign, perm = vca.cluster_permute(V, w.k, 3)
    ops = vca.smooth_quantize(Q, K, V, perm)
    O = vca.attention_fwd(ops, w.N, scale)
    torch.cuda.synchronize()
    for b in range(2):
        for h in range(w.H):
            Qb, Kb, Vb = (bits(t[b, h]) for t in (Q, K, V))
            ref = oracle.prep_head(Qb, Kb, Vb, w.k, 3)
            assert np.array_equal(perm[b, h].cpu().numpy(), ref["perm"])
            for key in ("Qq", "Kq", "VrT", "q_scale", "k_scale", "v_exp"):
                assert np.array_equal(ops[key][b, h].cpu().numpy(), ref[key]), (key, b, h)
            rows = sample_rows(w.N, 128, 10 * b + h)
            o_ref, _, _ = oracle.attention_head(ref, w.N, scale, rows=rows)
            assert rel_l2(bf16_to_f64(O[b, h])[rows], o_ref) <= 1e-2


def test_sage_path_batch2():
    w = W.shrink(W.WORKLOADS[2], H=2, N=700)
    Q, K, V = _batch2(w)
    scale = 1.0 / math.sqrt(w.d)
    ops = vca.sage_quantize(Q, K, V)
    O = vca.attention_fwd_sage(ops, w.N, scale)
    torch.cuda.synchronize()
    for b in range(2):
        for h in range(w.H):
            ref = oracle.sage_quantize_head(bits(Q[b, h]), bits(K[b, h]), bits(V[b, h]))
            for key in ("Qq", "Kq", "VcT", "q_scale", "k_scale", "v_chscale"):
                assert np.array_equal(ops[key][b, h].cpu().numpy(), ref[key]), (key, b, h)
            rows = sample_rows(w.N, 128, 20 + 10 * b + h)
            o_ref, _ = oracle.attention_head_sage(ref, w.N, scale, rows=rows)
            assert rel_l2(bf16_to_f64(O[b, h])[rows], o_ref) <= 1e-2


def test_host_pipeline_batch2():
    w = W.shrink(W.WORKLOADS[1], H=2, N=600)
    Q, K, V = _batch2(w)
    _, _, perm = vca.cluster_permute(V, w.k, 3)
    ref = vca.attention_fwd(vca.smooth_quantize(Q, K, V, perm), w.N).cpu()
    hQ, hK, hV = (t.cpu().pin_memory() for t in (Q, K, V))
    for hpc in (0, 1, 3):
        assert torch.equal(vca.vc_attention_host(hQ, hK, hV, k=w.k, iters=3, heads_per_chunk=hpc), ref)
