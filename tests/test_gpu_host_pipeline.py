"""vca_vc_attention_host: host buffers in, host buffer out, copies overlapped
with the kernels over two device slots.  Heads are independent, so the chunked
pipeline must give the whole-layer device path's output bit for bit."""
import pytest
import torch

from bit_attention_video_02_b200 import vca
from bit_attention_video_02_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _device_path(Q, K, V, k, iters):
    _, _, perm = vca.cluster_permute(V, k, iters)
    ops = vca.smooth_quantize(Q, K, V, perm)
    return vca.attention_fwd(ops, Q.shape[2])


@pytest.mark.parametrize("heads_per_chunk", [0, 1, 2, 5])
def test_host_pipeline_equals_device_path(heads_per_chunk):
    w = W.shrink(W.WORKLOADS[2], H=5, N=1500)
    Q, K, V = W.make_qkv(w, "cuda")
    ref = _device_path(Q, K, V, w.k, 3).cpu()
    hQ, hK, hV = (t.cpu().pin_memory() for t in (Q, K, V))
    O = vca.vc_attention_host(hQ, hK, hV, k=w.k, iters=3, heads_per_chunk=heads_per_chunk)
    assert O.device.type == "cpu"
    assert torch.equal(O, ref)


@pytest.mark.parametrize("heads_per_chunk", [0, 4])
def test_host_pipeline_ramp_and_tail(heads_per_chunk):
    # 13 heads: chunks of 1, 2, 3 (ramp), the middle, then 3 and 1 (tail); the
    # slots are reused while the previous chunk's attention or output copy runs
    w = W.shrink(W.WORKLOADS[2], H=13, N=900)
    Q, K, V = W.make_qkv(w, "cuda")
    ref = _device_path(Q, K, V, w.k, 3).cpu()
    hQ, hK, hV = (t.cpu().pin_memory() for t in (Q, K, V))
    for _ in range(2):
        assert torch.equal(vca.vc_attention_host(hQ, hK, hV, k=w.k, iters=3, heads_per_chunk=heads_per_chunk), ref)


def test_host_pipeline_pageable_memory_and_repeat_calls():
    w = W.shrink(W.WORKLOADS[1], H=2, N=700)
    Q, K, V = W.make_qkv(w, "cuda")
    ref = _device_path(Q, K, V, w.k, 3).cpu()
    hQ, hK, hV = (t.cpu() for t in (Q, K, V))          # not page-locked
    for _ in range(2):
        O = vca.vc_attention_host(hQ, hK, hV, k=w.k, iters=3, heads_per_chunk=1)
        assert torch.equal(O, ref)


def test_host_pipeline_rejects_small_buffer():
    w = W.shrink(W.WORKLOADS[1], H=2, N=300)
    Q, K, V = (t.cpu() for t in W.make_qkv(w, "cuda"))
    O = torch.empty_like(Q)
    need = vca.lib().vca_vc_attention_host_buffer_size(1, 2, 300, 128, w.k, 1)
    buf = torch.empty(need // 2, dtype=torch.uint8, device="cuda")
    import ctypes
    rc = vca.lib().vca_vc_attention_host(vca._ptr(Q), vca._ptr(K), vca._ptr(V), 1, 2, 300, 128, w.k, 3,
                                         0.0883883, vca._ptr(O), 1, ctypes.c_void_p(buf.data_ptr()),
                                         buf.numel(), None)
    assert rc == vca.ERR_WORKSPACE
