"""The no-allocation grouping entry point, for callers that cannot allocate
device memory when they call the library (an engine plugin that owns the whole
GPU memory budget, or an enqueue path that must not risk cudaMalloc's device
synchronisation).  It must give exactly what the workspace entry point gives,
call after call, although its scratch array keeps the previous call's contents.

Kept in a file that pytest collects last; it passes alone in a fresh process
and after the rest of the suite."""
import ctypes

import pytest
import torch

from bit_attention_video_02_b200 import vca
from bit_attention_video_02_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _noalloc_raw(V, k, iters):
    """Calls vca_cluster_permute_noalloc straight through the C ABI."""
    B, H, N, d = V.shape
    cent = torch.full((B, H, k, d), float("nan"), dtype=torch.float32, device=V.device)
    assign = torch.full((B, H, N), -1, dtype=torch.int32, device=V.device)
    perm = torch.full((B, H, N), -1, dtype=torch.int32, device=V.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = vca.lib().vca_cluster_permute_noalloc(
        ctypes.c_void_p(V.data_ptr()), B, H, N, d, k, iters, None, ctypes.c_void_p(cent.data_ptr()),
        ctypes.c_void_p(assign.data_ptr()), ctypes.c_void_p(perm.data_ptr()), stream)
    assert rc == vca.OK, vca.lib().vca_last_error()
    return cent, assign, perm


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    # two different inputs back to back: the second call must not see the
    # first call's leftovers in the shared scratch array
    cases = [W.shrink(W.WORKLOADS[3], H=3, N=2000), W.shrink(W.WORKLOADS[2], H=2, N=1500)]
    for w in cases:
        _, _, V = W.make_qkv(w, "cuda")
        got = _noalloc_raw(V, w.k, 3)
        ref = vca.cluster_permute(V, w.k, 3)
        torch.cuda.synchronize()
        for a, b, name in zip(got, ref, ("centroids", "assign", "perm")):
            assert torch.equal(a, b), name     # bit-exact, the tolerance of the grouping tests


def test_noalloc_rejects_shapes_beyond_its_fixed_scratch():
    V = torch.zeros(16, dtype=torch.bfloat16, device="cuda")      # never read: rejected first
    out = torch.zeros(16, dtype=torch.int32, device="cuda")
    B, H, N, k = 1, 2000, 4096, 64
    need = vca.lib().vca_cluster_permute_workspace_size(B, H, N, k)
    assert need > (8 << 20)
    rc = vca.lib().vca_cluster_permute_noalloc(
        ctypes.c_void_p(V.data_ptr()), B, H, N, 128, k, 3, None, ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(out.data_ptr()), None)
    assert rc == vca.ERR_UNSUPPORTED
    assert b"scratch" in vca.lib().vca_last_error()


def test_noalloc_python_wrapper_matches_and_checks_its_outputs():
    # the binding's wrapper: the same results as the workspace entry point,
    # into caller-provided outputs; outputs of the wrong shape, dtype or device
    # are refused before anything reaches the library
    w = W.shrink(W.WORKLOADS[2], H=2, N=900)
    _, _, V = W.make_qkv(w, "cuda")
    cent = torch.empty(1, w.H, w.k, 128, dtype=torch.float32, device="cuda")
    got = vca.cluster_permute_noalloc(V, w.k, 3, centroids=cent)
    ref = vca.cluster_permute(V, w.k, 3)
    torch.cuda.synchronize()
    assert got[0] is cent
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
    bad = torch.empty(1, w.H, w.N + 1, dtype=torch.int32, device="cuda")
    with pytest.raises(AssertionError):
        vca.cluster_permute_noalloc(V, w.k, 3, perm=bad)
    with pytest.raises(AssertionError):
        vca.cluster_permute_noalloc(V, w.k, 3, assign=torch.empty(1, w.H, w.N, dtype=torch.int64, device="cuda"))
    with pytest.raises(AssertionError):
        vca.cluster_permute_noalloc(V, w.k, 3, init=torch.empty(1, w.H, w.k, 128, dtype=torch.float32))
