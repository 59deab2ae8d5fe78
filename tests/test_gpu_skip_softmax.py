"""Skip Softmax (BLASST) block rejection in the FP8 kernel
("Accelerating Video Generation with GEMM Quantization, Attention Quantization
and Skip Softmax Attention in TensorRT-LLM", section "Sparse Attention with Skip
Softmax") against the oracle's rule, row by row."""
import math

import numpy as np
import pytest
import torch

import oracle
from bit_attention_video_02_b200 import vca
from bit_attention_video_02_b200 import workloads as W
from helpers import bf16_to_f64, bits, rel_l2, sample_rows

pytestmark = pytest.mark.gpu
TOL_REL_L2 = 1e-2


def _strong_weak(N, H, seed):
    # key blocks alternate strong / weak (x12 / x1 scale on |K|): every query
    # row sits ~6 natural-log units higher on the strong blocks, so at
    # lambda = 2^-6 whole query tiles drop the weak blocks
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(1, H, N, 128, generator=g).abs() * 0.4
    k = torch.randn(1, H, N, 128, generator=g).abs() * 0.2
    blk = torch.arange(N) // 128
    k *= torch.where(blk % 2 == 0, 12.0, 1.0)[None, None, :, None]
    v = torch.randn(1, H, N, 128, generator=g)
    return (t.to(torch.bfloat16).cuda() for t in (q, k, v))


def _check(Q, K, V, lam, rows_per_head=128, expect_skips=None):
    B, H, N, d = Q.shape
    scale = 1.0 / math.sqrt(d)
    perm = torch.arange(N, dtype=torch.int32, device="cuda").expand(B, H, N).contiguous()
    ops = vca.smooth_quantize(Q, K, V, perm)
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    O = vca.attention_fwd_skip(ops, N, lam, skipped=cnt)
    torch.cuda.synchronize()
    for h in range(H):
        Qb, Kb, Vb = (bits(t[0, h]) for t in (Q, K, V))
        ref = oracle.smooth_quantize_head(Qb, Kb, Vb, np.arange(N, dtype=np.int32))
        rows = sample_rows(N, rows_per_head, 77 + h)
        o_ref, _, _ = oracle.attention_head(ref, N, scale, rows=rows, skip_lambda=lam)
        err = rel_l2(bf16_to_f64(O[0, h])[rows], o_ref)
        print(dict(head=h, lam=lam, rel_l2=err, skipped=int(cnt.item())))
        assert err <= TOL_REL_L2
    if expect_skips is not None:
        assert expect_skips(int(cnt.item()))
    return O, int(cnt.item())


def test_zero_lambda_is_the_plain_kernel():
    w = W.shrink(W.WORKLOADS[2], H=2, N=1500)
    Q, K, V = W.make_qkv(w, "cuda")
    _, _, perm = vca.cluster_permute(V, w.k, 3)
    ops = vca.smooth_quantize(Q, K, V, perm)
    a, la = vca.attention_fwd(ops, w.N, want_lse=True)
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    b, lb = vca.attention_fwd_skip(ops, w.N, 0.0, want_lse=True, skipped=cnt)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(la, lb) and cnt.item() == 0


@pytest.mark.parametrize("N", [1000, 2200])
def test_whole_tiles_skip_and_match_the_oracle(N):
    Q, K, V = _strong_weak(N, 2, seed=N)
    nb = (N + 127) // 128
    ntiles = (nb + 1) // 2 * 2          # query tiles the kernel runs (odd counts pad one)
    _check(Q, K, V, 2.0 ** -6, expect_skips=lambda c: c >= (nb // 2 - 1) * (nb // 2))


def test_lambda_on_the_video_recipe():
    # the sinusoid video recipe with a large lambda: rows drop different
    # blocks (few whole-tile skips); each row must still match the oracle
    w = W.shrink(W.WORKLOADS[3], H=2, N=2500)
    Q, K, V = W.make_qkv(w, "cuda")
    _check(Q, K, V, 0.25)


def test_skip_rejects_bad_lambda():
    w = W.shrink(W.WORKLOADS[1], H=1, N=256)
    Q, K, V = W.make_qkv(w, "cuda")
    perm = torch.arange(w.N, dtype=torch.int32, device="cuda").expand(1, 1, w.N).contiguous()
    ops = vca.smooth_quantize(Q, K, V, perm)
    for lam in (1.0, -0.5, float("nan")):
        with pytest.raises(vca.VcaError):
            vca.attention_fwd_skip(ops, w.N, lam)
