"""GPU vs oracle, bit for bit: the 4-bit V-Smooth prep (vca_smooth_quantize_qkv_fp4).

Q/K codes and scales and the block means must equal the 8-bit prep's; the NVFP4
V residual (packed E2M1 codes, E4M3 group scales, the head's fp32 tensor scale)
must equal the oracle's vo_smooth_quantize_head_fp4 on the same permutation."""
import numpy as np
import pytest
import torch

import oracle
from bit_attention_video_02_b200 import vca
from bit_attention_video_02_b200 import workloads as W
from helpers import bits

pytestmark = pytest.mark.gpu

# small workloads at full size, reduced ones with ragged tails (odd token
# counts leave half a code byte and part of a 16-token group), degenerate sizes
CASES = [(1, None, None), (2, 2, None), (3, 2, 1000), (5, 2, 301), (1, 1, 1), (1, 1, 129), (4, 1, 4097)]


def _ids(c):
    return f"cfg{c[0]}-H{c[1] or 'full'}-N{c[2] or 'full'}"


def _compare(w, Q, K, V, perm, o4, o8, heads):
    for h in heads:
        ref = oracle.smooth_quantize_head_fp4(*(bits(t[0, h]) for t in (Q, K, V)), perm[0, h].cpu().numpy())
        for name in ("Qq", "Kq", "VrT4", "v_sc"):
            g = o4[name][0, h].cpu().numpy()
            bad = np.argwhere(g != ref[name])
            assert bad.size == 0, (name, h, bad[:3].tolist())
        for name in ("q_scale", "k_scale"):
            assert np.array_equal(o4[name][0, h].cpu().numpy().view(np.uint32), ref[name].view(np.uint32)), name
        assert np.array_equal(o4["v_mean"][0, h].cpu().view(torch.int16).numpy().view(np.uint16), ref["v_mean"])
        assert o4["v_gscale"][0, h].cpu().numpy().view(np.uint32) == ref["v_gscale"].view(np.uint32)[0]
        # the operands the two variants share are the 8-bit prep's, byte for byte
        for name in ("Qq", "Kq", "q_scale", "k_scale", "v_mean"):
            assert torch.equal(o4[name][0, h], o8[name][0, h]), name


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_fp4_prep_bit_exact(case):
    cid, H, N = case
    w = W.shrink(W.WORKLOADS[cid], H=H, N=N)
    Q, K, V = W.make_qkv(w, "cuda")
    _, _, perm = vca.cluster_permute(V, w.k, iters=3)
    ws = vca.Workspace(vca.lib().vca_smooth_quantize_fp4_workspace_size(w.B, w.H, w.N))
    o4 = vca.smooth_quantize_fp4(Q, K, V, perm, ws=ws)
    o8 = vca.smooth_quantize(Q, K, V, perm)
    torch.cuda.synchronize()
    ws.check()
    _compare(w, Q, K, V, perm, o4, o8, range(w.H))


def test_fp4_prep_full_size_sampled_heads():
    # the Wan-shaped layer at full size (N = 75,600: the last block holds 80
    # tokens, so its last three 16-token groups are padding); first and last
    # head against the oracle
    w = W.WORKLOADS[3]
    Q, K, V = W.make_qkv(w, "cuda")
    _, _, perm = vca.cluster_permute(V, w.k, iters=3)
    ws = vca.Workspace(vca.lib().vca_smooth_quantize_fp4_workspace_size(w.B, w.H, w.N))
    o4 = vca.smooth_quantize_fp4(Q, K, V, perm, ws=ws)
    o8 = vca.smooth_quantize(Q, K, V, perm)
    torch.cuda.synchronize()
    ws.check()
    _compare(w, Q, K, V, perm, o4, o8, [0, w.H - 1])
    assert torch.all(o4["v_gscale"] > 0)
    # groups wholly past N have zero scales and codes in every head
    assert not o4["v_sc"][..., 75600 // 16:].any() and not o4["VrT4"][..., 75600 // 2:].any()


def test_fp4_prep_nonfinite_input_is_reported():
    w = W.shrink(W.WORKLOADS[1], H=1, N=256)
    Q, K, V = W.make_qkv(w, "cuda")
    perm = torch.arange(w.N, dtype=torch.int32, device="cuda").reshape(1, 1, w.N).contiguous()
    V[0, 0, 7, 3] = float("inf")
    ws = vca.Workspace(vca.lib().vca_smooth_quantize_fp4_workspace_size(w.B, w.H, w.N))
    vca.smooth_quantize_fp4(Q, K, V, perm, ws=ws)
    with pytest.raises(vca.VcaError) as e:
        ws.check()
    assert e.value.code == vca.ERR_NONFINITE
