"""The in-repo BF16 comparator against exact fp64 attention, and the device
status paths (bounded-wait timeout, argument errors) on the GPU."""
import math

import numpy as np
import pytest
import torch

import oracle
from bit_attention_video_02_b200 import vca
from bit_attention_video_02_b200 import workloads as W
from helpers import bf16_to_f64, bits, cosine, rel_l2, sample_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("case", [(1, None, None), (3, 2, 1000), (2, 1, 129), (1, 1, 1), (5, 2, 4100)])
def test_bf16_comparator_matches_exact(case):
    cid, H, N = case
    w = W.shrink(W.WORKLOADS[cid], H=H, N=N)
    Q, K, V = W.make_qkv(w, "cuda")
    scale = 1.0 / math.sqrt(w.d)
    O, lse = vca.bf16_attention_fwd(Q, K, V, scale, want_lse=True)
    torch.cuda.synchronize()
    for h in range(w.H):
        rows = sample_rows(w.N, 300, h)
        Qb, Kb, Vb = (bits(t[0, h]) for t in (Q, K, V))
        ex = oracle.exact_attention_head(Qb, Kb, Vb, scale, rows=rows)
        g = bf16_to_f64(O[0, h])[rows]
        r = rel_l2(g, ex)
        print(dict(head=h, rel_l2=r, cos=cosine(g, ex)))
        assert r <= 1e-2
        q = bf16_to_f64(Q[0, h])[rows]
        s = q @ bf16_to_f64(K[0, h]).T * scale
        true_lse = np.log(np.exp(s - s.max(1, keepdims=True)).sum(1)) + s.max(1)
        assert np.abs(lse[0, h].cpu().numpy()[rows] - true_lse).max() < 1e-2


def test_bf16_comparator_full_size_sampled_rows():
    w = W.WORKLOADS[3]
    Q, K, V = W.make_qkv(w, "cuda")
    scale = 1.0 / math.sqrt(w.d)
    O = vca.bf16_attention_fwd(Q, K, V, scale)
    torch.cuda.synchronize()
    for h in (0, w.H - 1):
        rows = sample_rows(w.N, 32, h)
        Qb, Kb, Vb = (bits(t[0, h]) for t in (Q, K, V))
        ex = oracle.exact_attention_head(Qb, Kb, Vb, scale, rows=rows)
        assert rel_l2(bf16_to_f64(O[0, h])[rows], ex) <= 1e-2


def test_bounded_wait_times_out_and_reports():
    ws = vca.Workspace(256)
    vca.debug_wait_timeout(ws, 20_000_000)     # 20 ms on an mbarrier nobody arrives on
    with pytest.raises(vca.VcaError) as e:
        ws.check()
    assert e.value.code == vca.ERR_TIMEOUT
    ws.check()                                  # the status word was cleared
    # the context is still usable afterwards
    x = torch.zeros(16, device="cuda", dtype=torch.float32)
    assert vca.expcast_ref(x).cpu().tolist() == [56] * 16


def test_argument_errors_on_device_pointers():
    x = torch.zeros(64, device="cuda", dtype=torch.float32)
    with pytest.raises(vca.VcaError) as e:
        rc = vca.lib().vca_expcast_ref(x.data_ptr() + 4, x.data_ptr(), 8, None)   # misaligned input
        vca._check(rc)
    assert e.value.code == vca.ERR_INVALID
    w = W.shrink(W.WORKLOADS[1], H=1, N=256)
    Q, K, V = W.make_qkv(w, "cuda")
    with pytest.raises(vca.VcaError) as e:
        vca.cluster_permute(V, k=65)
    assert e.value.code == vca.ERR_UNSUPPORTED
    ws_small = vca.Workspace(256)
    need = vca.lib().vca_cluster_permute_workspace_size(1, 1, 256, 8)
    rc = vca.lib().vca_cluster_permute(V.data_ptr(), 1, 1, 256, 128, 8, 3, None,
                                       torch.empty(8, 128, device="cuda").data_ptr(),
                                       torch.empty(256, dtype=torch.int32, device="cuda").data_ptr(),
                                       torch.empty(256, dtype=torch.int32, device="cuda").data_ptr(),
                                       ws_small.buf.data_ptr(), 16, None)
    assert need > 16 and rc == vca.ERR_WORKSPACE
