"""SAGE-style comparison recipe ("Accelerating Video Generation with GEMM
Quantization, Attention Quantization and Skip Softmax Attention in
TensorRT-LLM", section "Quantized Attention") on the GPU, with Q/K coded as
E4M3 or as INT8 (the post's two qk_dtype choices): the quantisation bit for bit
against the oracle, the attention on its operands (QK^T as kind::f8f6f4 or
kind::i8) within the attention tolerance, and its fidelity beside V-Smooth's on
the same inputs."""
import math

import numpy as np
import pytest
import torch

import oracle
from bit_attention_video_02_b200 import vca
from bit_attention_video_02_b200 import workloads as W
from helpers import bf16_to_f64, bits, cosine, rel_l2, sample_rows

pytestmark = pytest.mark.gpu
CASES = [(1, None, None), (2, 2, 1500), (3, 2, 1000), (5, 1, 700)]


def _ids(c):
    return f"cfg{c[0]}" + (f"_H{c[1]}_N{c[2]}" if c[1] else "")


QK = ["fp8", "int8"]


@pytest.mark.parametrize("qk", QK)
@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_sage_quantisation_bit_exact(case, qk):
    cid, H, N = case
    w = W.WORKLOADS[cid] if H is None else W.shrink(W.WORKLOADS[cid], H=H, N=N)
    Q, K, V = W.make_qkv(w, "cuda")
    ops = vca.sage_quantize(Q, K, V, qk_dtype=qk)
    torch.cuda.synchronize()
    for h in range(w.H):
        ref = oracle.sage_quantize_head(bits(Q[0, h]), bits(K[0, h]), bits(V[0, h]), qk_dtype=qk)
        for key in ("Qq", "Kq", "VcT", "q_scale", "k_scale", "v_chscale"):
            got = ops[key][0, h].cpu().numpy()
            assert np.array_equal(got, ref[key]), (key, h)
        assert np.array_equal(bits(ops["k_mean"][0, h]), ref["k_mean"])


@pytest.mark.parametrize("qk", QK)
@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_sage_attention_matches_oracle(case, qk):
    cid, H, N = case
    w = W.WORKLOADS[cid] if H is None else W.shrink(W.WORKLOADS[cid], H=H, N=N)
    Q, K, V = W.make_qkv(w, "cuda")
    scale = 1.0 / math.sqrt(w.d)
    ops = vca.sage_quantize(Q, K, V, qk_dtype=qk)
    O, lse = vca.attention_fwd_sage(ops, w.N, scale, want_lse=True)
    torch.cuda.synchronize()
    for h in range(w.H):
        # the oracle quantises the same bf16 inputs itself (its operands equal
        # the GPU's bit for bit: test_sage_quantisation_bit_exact)
        ref = oracle.sage_quantize_head(bits(Q[0, h]), bits(K[0, h]), bits(V[0, h]), qk_dtype=qk)
        rows = sample_rows(w.N, 200, 900 + h)
        o_ref, lse_ref = oracle.attention_head_sage(ref, w.N, scale, rows=rows)
        g = bf16_to_f64(O[0, h])[rows]
        gl = lse[0, h].cpu().numpy().astype(np.float64)[rows]
        ex = oracle.exact_attention_head(bits(Q[0, h]), bits(K[0, h]), bits(V[0, h]), scale, rows=rows)
        line = dict(case=_ids(case), qk=qk, head=h, rel_l2=rel_l2(g, o_ref), cos=cosine(g, ex),
                    lse_maxdiff=float(np.abs(gl - lse_ref).max()))
        print(line)
        assert np.all(np.isfinite(g))
        assert line["rel_l2"] <= 1e-2, line
        # a score near an ExpCast rounding boundary may take the neighbouring
        # code between fp32 and fp64: one E4M3 step of one probability at most
        assert line["lse_maxdiff"] <= 1e-2, line
        assert line["cos"] >= 0.99, line


def test_sage_int8_full_size_sampled_rows():
    # the Wan-shaped layer at full size (40 heads, 75,600 tokens), INT8 Q/K;
    # first and last head on sampled rows
    w = W.WORKLOADS[3]
    Q, K, V = W.make_qkv(w, "cuda")
    scale = 1.0 / math.sqrt(w.d)
    ops = vca.sage_quantize(Q, K, V, qk_dtype="int8")
    O = vca.attention_fwd_sage(ops, w.N, scale)
    torch.cuda.synchronize()
    for h in (0, w.H - 1):
        ref = oracle.sage_quantize_head(bits(Q[0, h]), bits(K[0, h]), bits(V[0, h]), qk_dtype="int8")
        for key in ("Qq", "Kq", "q_scale", "k_scale"):
            assert np.array_equal(ops[key][0, h].cpu().numpy(), ref[key]), (key, h)
        rows = sample_rows(w.N, 128, 70 + h)
        o_ref, _ = oracle.attention_head_sage(ref, w.N, scale, rows=rows)
        g = bf16_to_f64(O[0, h])[rows]
        print(dict(head=h, rel_l2=rel_l2(g, o_ref)))
        assert rel_l2(g, o_ref) <= 1e-2


@pytest.mark.parametrize("cid", [2, 3])
def test_fidelity_vsmooth_beside_sage(cid):
    # same inputs, both recipes, error against exact attention; reported, and
    # both must stay inside the fidelity bar
    w = W.shrink(W.WORKLOADS[cid], H=2, N=3000)
    Q, K, V = W.make_qkv(w, "cuda")
    scale = 1.0 / math.sqrt(w.d)
    O_vc = vca.vc_attention(Q, K, V, k=w.k, iters=3)
    O_sg = vca.attention_fwd_sage(vca.sage_quantize(Q, K, V), w.N, scale)
    torch.cuda.synchronize()
    for h in range(w.H):
        rows = sample_rows(w.N, 256, 50 + h)
        ex = oracle.exact_attention_head(bits(Q[0, h]), bits(K[0, h]), bits(V[0, h]), scale, rows=rows)
        e_vc = rel_l2(bf16_to_f64(O_vc[0, h])[rows], ex)
        e_sg = rel_l2(bf16_to_f64(O_sg[0, h])[rows], ex)
        print(dict(cfg=cid, head=h, rel_l2_vsmooth=e_vc, rel_l2_sage=e_sg))
        assert cosine(bf16_to_f64(O_vc[0, h])[rows], ex) >= 0.99
        assert cosine(bf16_to_f64(O_sg[0, h])[rows], ex) >= 0.99
