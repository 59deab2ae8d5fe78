"""CPU checks of the C-ABI library: it loads and exports every declared symbol;
argument validation runs on the host and needs no GPU."""
import ctypes
import os
import re

import pytest

from bit_attention_video_02_b200 import build, vca

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "vca.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(vca_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return vca.lib()


def test_library_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 16
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing
    assert sorted(vca.EXPORTED) == sorted(n for n in names if n in vca.EXPORTED)


def test_workspace_queries(L):
    assert L.vca_status_bytes() == 16
    assert L.vca_smooth_quantize_workspace_size(1, 2, 1024) >= 16
    small = L.vca_cluster_permute_workspace_size(1, 2, 1024, 8)
    big = L.vca_cluster_permute_workspace_size(1, 40, 75600, 32)
    assert small >= 16 and big > small
    assert L.vca_cluster_permute_workspace_size(0, 1, 1, 1) == 0


def test_host_argument_validation_needs_no_gpu(L):
    # d != 128 and bad k are rejected before anything touches the device
    rc = L.vca_cluster_permute(None, 1, 1, 16, 64, 4, 3, None, None, None, None, None, 0, None)
    assert rc == vca.ERR_UNSUPPORTED
    rc = L.vca_cluster_permute(None, 1, 1, 16, 128, 0, 3, None, None, None, None, None, 0, None)
    assert rc == vca.ERR_UNSUPPORTED
    rc = L.vca_smooth_quantize_qkv(None, None, None, None, 1, 1, 16, 128, 64, *([None] * 7), None, 0, None)
    assert rc == vca.ERR_UNSUPPORTED
    rc = L.vca_attention_fwd(*([None] * 7), 1, 1, 16, 128, 0.1, None, None, None, 0, None)
    assert rc == vca.ERR_INVALID
    rc = L.vca_expcast_ref(None, None, -1, None)
    assert rc == vca.ERR_INVALID
    assert b"n < 0" in L.vca_last_error()
    rc = L.vca_bf16_attention_fwd(None, None, None, 1, 1, 16, 96, 0.1, None, None, None, 0, None)
    assert rc == vca.ERR_UNSUPPORTED


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "bit_attention_video_02_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "vca_oracle" not in txt and "liboracle" not in txt, f


FAKE = ctypes.c_void_p(0x10000)       # a 16-byte-aligned address that is never dereferenced
FAKE_ODD = ctypes.c_void_p(0x10001)


def test_attention_variants_validate_on_the_host(L):
    ops = [FAKE] * 7
    # skip_lambda must lie in [0, 1)
    rc = L.vca_attention_fwd_skip(*ops, 1, 1, 300, 128, 0.1, 1.0, FAKE, None, None, FAKE, 256, None)
    assert rc == vca.ERR_INVALID and b"skip_lambda" in L.vca_last_error()
    rc = L.vca_attention_fwd_skip(*ops, 1, 1, 300, 128, 0.1, -0.5, FAKE, None, None, FAKE, 256, None)
    assert rc == vca.ERR_INVALID
    # alignment of the TMA-fed tensors, softmax scale, grid limit, workspace
    rc = L.vca_attention_fwd(FAKE_ODD, *ops[1:], 1, 1, 300, 128, 0.1, FAKE, None, FAKE, 256, None)
    assert rc == vca.ERR_INVALID and b"aligned" in L.vca_last_error()
    rc = L.vca_attention_fwd(*ops, 1, 1, 300, 128, 0.0, FAKE, None, FAKE, 256, None)
    assert rc == vca.ERR_INVALID and b"softmax_scale" in L.vca_last_error()
    rc = L.vca_attention_fwd(*ops, 256, 256, 300, 128, 0.1, FAKE, None, FAKE, 256, None)
    assert rc == vca.ERR_INVALID
    rc = L.vca_attention_fwd(*ops, 1, 1, 300, 128, 0.1, FAKE, None, FAKE, 16, None)
    assert rc == vca.ERR_WORKSPACE
    # SAGE operands: the per-channel V scale is required; d must be 128
    rc = L.vca_attention_fwd_sage(*[FAKE] * 5, None, 1, 1, 300, 128, 0.1, FAKE, None, FAKE, 256, None)
    assert rc == vca.ERR_INVALID
    rc = L.vca_attention_fwd_sage(*[FAKE] * 6, 1, 1, 300, 64, 0.1, FAKE, None, FAKE, 256, None)
    assert rc == vca.ERR_UNSUPPORTED
    rc = L.vca_sage_quantize_qkv(FAKE, FAKE, FAKE, 1, 1, 300, 96, *[FAKE] * 7, FAKE, 1 << 20, None)
    assert rc == vca.ERR_UNSUPPORTED


def test_host_pipeline_validates_and_sizes_on_the_host(L):
    B, H, N, k = 1, 8, 1000, 32
    full = L.vca_vc_attention_host_buffer_size(B, H, N, 128, k, 0)
    one = L.vca_vc_attention_host_buffer_size(B, H, N, 128, k, 1)
    all8 = L.vca_vc_attention_host_buffer_size(B, H, N, 128, k, 8)
    # two slots, each sized for one chunk: more heads per chunk, more memory
    assert 0 < one < full <= all8
    assert L.vca_vc_attention_host_buffer_size(B, H, N, 128, k, 100) == all8
    # at least Q, K, V, O in bf16 and the three FP8 operands per slot
    assert one >= 2 * (4 * N * 128 * 2 + 3 * N * 128)
    for bad in ((0, H, N, 128, k, 0), (B, H, N, 64, k, 0), (B, H, N, 128, 0, 0), (B, H, N, 128, 1000, 0)):
        assert L.vca_vc_attention_host_buffer_size(*bad) == 0
    host = [FAKE] * 3
    rc = L.vca_vc_attention_host(None, FAKE, FAKE, B, H, N, 128, k, 3, 0.1, FAKE, 0, FAKE, full, None)
    assert rc == vca.ERR_INVALID
    rc = L.vca_vc_attention_host(*host, B, H, N, 64, k, 3, 0.1, FAKE, 0, FAKE, full, None)
    assert rc == vca.ERR_UNSUPPORTED
    rc = L.vca_vc_attention_host(*host, B, H, N, 128, k, 0, 0.1, FAKE, 0, FAKE, full, None)
    assert rc == vca.ERR_INVALID
    rc = L.vca_vc_attention_host(*host, B, H, N, 128, k, 3, 0.1, FAKE, -1, FAKE, full, None)
    assert rc == vca.ERR_INVALID
    rc = L.vca_vc_attention_host(*host, B, H, N, 128, k, 3, 0.1, FAKE, 0, FAKE, full - 1, None)
    assert rc == vca.ERR_WORKSPACE and b"too small" in L.vca_last_error()


def test_fp4_prep_validates_on_the_host(L):
    assert L.vca_smooth_quantize_fp4_workspace_size(1, 40, 75600) == 256 + 256
    assert L.vca_smooth_quantize_fp4_workspace_size(2, 100, 10) == 256 + 1024
    assert L.vca_smooth_quantize_fp4_workspace_size(0, 1, 1) == 0
    outs = [FAKE] * 8
    rc = L.vca_smooth_quantize_qkv_fp4(FAKE, FAKE, FAKE, FAKE, 1, 1, 300, 64, *outs, FAKE, 1 << 20, None)
    assert rc == vca.ERR_UNSUPPORTED
    rc = L.vca_smooth_quantize_qkv_fp4(FAKE, FAKE, FAKE, FAKE, 1, 1, 300, 128, *outs[:6], None, outs[7],
                                       FAKE, 1 << 20, None)
    assert rc == vca.ERR_INVALID and b"null" in L.vca_last_error()
    rc = L.vca_smooth_quantize_qkv_fp4(FAKE, FAKE, FAKE, FAKE, 1, 1, 300, 128, *outs[:5], FAKE_ODD, *outs[6:],
                                       FAKE, 1 << 20, None)
    assert rc == vca.ERR_INVALID and b"aligned" in L.vca_last_error()
    rc = L.vca_smooth_quantize_qkv_fp4(FAKE, FAKE, FAKE, FAKE, 1, 1, 300, 128, *outs, FAKE, 300, None)
    assert rc == vca.ERR_WORKSPACE
