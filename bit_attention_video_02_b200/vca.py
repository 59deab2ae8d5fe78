"""Thin ctypes binding of libvca.so (argument marshalling only).

Every computation runs in the library's CUDA kernels; this module allocates the
caller-owned device buffers with PyTorch, passes their pointers and the current
CUDA stream, and turns non-zero status codes into exceptions.  It fails loudly
when the library has not been built: there is no CPU fallback.

Names follow the C ABI in include/vca.h.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libvca.so")
HEAD_DIM = 128
BLOCK = 128

OK, ERR_INVALID, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_NONFINITE, ERR_WORKSPACE = 0, -1, -2, -3, -4, -5, -6
_NAMES = {0: "VCA_OK", -1: "VCA_ERR_INVALID", -2: "VCA_ERR_UNSUPPORTED", -3: "VCA_ERR_CUDA",
          -4: "VCA_ERR_TIMEOUT", -5: "VCA_ERR_NONFINITE", -6: "VCA_ERR_WORKSPACE"}

_lib = None

EXPORTED = [
    "vca_status_bytes", "vca_reset_status", "vca_check_status", "vca_last_error",
    "vca_set_wait_limit_ns", "vca_debug_wait_timeout", "vca_expcast_ref", "vca_e4m3_encode",
    "vca_cluster_permute_workspace_size", "vca_cluster_permute", "vca_cluster_permute_noalloc",
    "vca_smooth_quantize_workspace_size", "vca_smooth_quantize_qkv",
    "vca_attention_workspace_size", "vca_attention_fwd",
    "vca_bf16_attention_workspace_size", "vca_bf16_attention_fwd", "vca_schedule_regroup",
    "vca_attention_fwd_skip", "vca_vc_attention_host_buffer_size", "vca_vc_attention_host",
    "vca_sage_quantize_workspace_size", "vca_sage_quantize_qkv", "vca_attention_fwd_sage",
    "vca_sage_quantize_qkv_i8", "vca_attention_fwd_sage_i8",
    "vca_smooth_quantize_fp4_workspace_size", "vca_smooth_quantize_qkv_fp4",
    "vca_attention_fwd_fp4", "vca_debug_fp4_mma",
]


class VcaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{_NAMES.get(code, code)}: {msg}")
        self.code = code


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run `python -m bit_attention_video_02_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
        L.vca_status_bytes.restype = sz
        L.vca_reset_status.argtypes = [vp, vp]
        L.vca_check_status.argtypes = [vp, vp, ctypes.POINTER(i32), ctypes.POINTER(i32)]
        L.vca_last_error.restype = ctypes.c_char_p
        L.vca_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        L.vca_debug_wait_timeout.argtypes = [vp, ctypes.c_uint64, vp]
        L.vca_expcast_ref.argtypes = [vp, vp, i64, vp]
        L.vca_e4m3_encode.argtypes = [vp, vp, i64, vp]
        L.vca_cluster_permute_workspace_size.restype = sz
        L.vca_cluster_permute_workspace_size.argtypes = [i32, i32, i32, i32]
        L.vca_cluster_permute.argtypes = [vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, sz, vp]
        L.vca_cluster_permute_noalloc.argtypes = [vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp]
        L.vca_smooth_quantize_workspace_size.restype = sz
        L.vca_smooth_quantize_workspace_size.argtypes = [i32, i32, i32]
        L.vca_smooth_quantize_qkv.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32] + [vp] * 7 + [vp, sz, vp]
        L.vca_attention_workspace_size.restype = sz
        L.vca_attention_workspace_size.argtypes = [i32, i32, i32]
        L.vca_attention_fwd.argtypes = [vp] * 7 + [i32, i32, i32, i32, f32, vp, vp, vp, sz, vp]
        L.vca_bf16_attention_workspace_size.restype = sz
        L.vca_bf16_attention_workspace_size.argtypes = [i32, i32, i32]
        L.vca_bf16_attention_fwd.argtypes = [vp, vp, vp, i32, i32, i32, i32, f32, vp, vp, vp, sz, vp]
        L.vca_schedule_regroup.argtypes = [i32, i32, i32, f32]
        L.vca_attention_fwd_skip.argtypes = [vp] * 7 + [i32, i32, i32, i32, f32, f32, vp, vp, vp, vp, sz, vp]
        L.vca_sage_quantize_workspace_size.restype = sz
        L.vca_sage_quantize_workspace_size.argtypes = [i32, i32, i32]
        L.vca_sage_quantize_qkv.argtypes = [vp, vp, vp] + [i32] * 4 + [vp] * 7 + [vp, sz, vp]
        L.vca_attention_fwd_sage.argtypes = [vp] * 6 + [i32] * 4 + [f32, vp, vp, vp, sz, vp]
        L.vca_sage_quantize_qkv_i8.argtypes = L.vca_sage_quantize_qkv.argtypes
        L.vca_attention_fwd_sage_i8.argtypes = L.vca_attention_fwd_sage.argtypes
        L.vca_smooth_quantize_fp4_workspace_size.restype = sz
        L.vca_smooth_quantize_fp4_workspace_size.argtypes = [i32, i32, i32]
        L.vca_smooth_quantize_qkv_fp4.argtypes = [vp] * 4 + [i32] * 4 + [vp] * 8 + [vp, sz, vp]
        L.vca_attention_fwd_fp4.argtypes = [vp] * 8 + [i32, i32, i32, i32, f32, vp, vp, vp, sz, vp]
        L.vca_debug_fp4_mma.argtypes = [vp] * 6
        L.vca_vc_attention_host_buffer_size.restype = sz
        L.vca_vc_attention_host_buffer_size.argtypes = [i32] * 6
        L.vca_vc_attention_host.argtypes = [vp, vp, vp] + [i32] * 6 + [f32, vp, i32, vp, sz, vp]
        for fn in ("vca_reset_status", "vca_check_status", "vca_debug_wait_timeout", "vca_expcast_ref",
                   "vca_e4m3_encode", "vca_cluster_permute", "vca_cluster_permute_noalloc",
                   "vca_smooth_quantize_qkv",
                   "vca_attention_fwd", "vca_bf16_attention_fwd", "vca_schedule_regroup",
                   "vca_attention_fwd_skip", "vca_vc_attention_host", "vca_sage_quantize_qkv",
                   "vca_attention_fwd_sage", "vca_sage_quantize_qkv_i8", "vca_attention_fwd_sage_i8"):
            getattr(L, fn).restype = i32
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int):
    if rc != OK:
        raise VcaError(rc, lib().vca_last_error().decode(errors="replace"))


class Workspace:
    """Caller-owned device scratch; its first bytes hold the device status word."""

    def __init__(self, nbytes: int, device="cuda"):
        self.nbytes = max(int(nbytes), 256)
        self.buf = torch.zeros(self.nbytes, dtype=torch.uint8, device=device)

    def ensure(self, nbytes: int):
        if nbytes > self.nbytes:
            self.__init__(nbytes, self.buf.device)
        return self

    @property
    def ptr(self):
        return ctypes.c_void_p(self.buf.data_ptr())

    def check(self, stream=None):
        where, info = ctypes.c_int(0), ctypes.c_int(0)
        rc = lib().vca_check_status(self.ptr, _stream(stream), ctypes.byref(where), ctypes.byref(info))
        if rc != OK:
            raise VcaError(rc, lib().vca_last_error().decode(errors="replace"))


def set_wait_limit_ns(ns: int):
    lib().vca_set_wait_limit_ns(int(ns))


def debug_wait_timeout(ws: Workspace, limit_ns: int, stream=None):
    _check(lib().vca_debug_wait_timeout(ws.ptr, int(limit_ns), _stream(stream)))


# ------------------------------------------------------------------ ExpCast / E4M3
def expcast_ref(z: torch.Tensor, stream=None) -> torch.Tensor:
    assert z.is_cuda and z.dtype == torch.float32 and z.is_contiguous()
    out = torch.empty(z.shape, dtype=torch.uint8, device=z.device)
    _check(lib().vca_expcast_ref(_ptr(z), _ptr(out), z.numel(), _stream(stream)))
    return out


def e4m3_encode(x: torch.Tensor, stream=None) -> torch.Tensor:
    assert x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(lib().vca_e4m3_encode(_ptr(x), _ptr(out), x.numel(), _stream(stream)))
    return out


# ------------------------------------------------------------------ V-Smooth
def _bhnd(x):
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 4, \
        "expected contiguous bf16 CUDA tensor [B, H, N, d]"
    return x.shape


def cluster_permute(V: torch.Tensor, k: int, iters: int = 3, init=None, ws: Workspace | None = None,
                    stream=None):
    B, H, N, d = _bhnd(V)
    dev = V.device
    cent = torch.empty(B, H, k, d, dtype=torch.float32, device=dev)
    assign = torch.empty(B, H, N, dtype=torch.int32, device=dev)
    perm = torch.empty(B, H, N, dtype=torch.int32, device=dev)
    need = lib().vca_cluster_permute_workspace_size(B, H, N, k)
    ws = (ws or Workspace(need, dev)).ensure(need)
    if init is not None:
        assert init.shape == (B, H, k, d) and init.dtype == torch.float32 and init.is_contiguous()
    _check(lib().vca_cluster_permute(_ptr(V), B, H, N, d, k, iters, _ptr(init), _ptr(cent), _ptr(assign),
                                     _ptr(perm), ws.ptr, ws.nbytes, _stream(stream)))
    return cent, assign, perm


def cluster_permute_noalloc(V: torch.Tensor, k: int, iters: int = 3, init=None, centroids=None, assign=None,
                            perm=None, stream=None):
    """vca_cluster_permute_noalloc: the library allocates nothing (scratch is a
    fixed array inside the library); the output tensors may be passed in."""
    B, H, N, d = _bhnd(V)
    dev = V.device

    def _out(t, shape, dtype, what):
        if t is None:
            return torch.empty(shape, dtype=dtype, device=dev)
        assert tuple(t.shape) == shape and t.dtype == dtype and t.device == dev and t.is_contiguous(), \
            f"{what} must be a contiguous {dtype} tensor of shape {shape} on {dev}"
        return t

    cent = _out(centroids, (B, H, k, d), torch.float32, "centroids")
    assign = _out(assign, (B, H, N), torch.int32, "assign")
    perm = _out(perm, (B, H, N), torch.int32, "perm")
    if init is not None:
        _out(init, (B, H, k, d), torch.float32, "init")
    _check(lib().vca_cluster_permute_noalloc(_ptr(V), B, H, N, d, k, iters, _ptr(init), _ptr(cent),
                                             _ptr(assign), _ptr(perm), _stream(stream)))
    return cent, assign, perm


def alloc_quantized(B, H, N, device="cuda"):
    nb = (N + BLOCK - 1) // BLOCK
    Np = nb * BLOCK
    u8, f32 = torch.uint8, torch.float32
    return dict(
        Qq=torch.empty(B, H, Np, HEAD_DIM, dtype=u8, device=device),
        q_scale=torch.empty(B, H, nb, dtype=f32, device=device),
        Kq=torch.empty(B, H, Np, HEAD_DIM, dtype=u8, device=device),
        k_scale=torch.empty(B, H, nb, dtype=f32, device=device),
        VrT=torch.empty(B, H, HEAD_DIM, Np, dtype=u8, device=device),
        v_exp=torch.empty(B, H, nb, dtype=torch.int8, device=device),
        v_mean=torch.empty(B, H, nb, HEAD_DIM, dtype=torch.bfloat16, device=device))


def smooth_quantize(Q, K, V, perm, out=None, ws: Workspace | None = None, stream=None):
    B, H, N, d = _bhnd(Q)
    assert K.shape == Q.shape and V.shape == Q.shape
    assert perm.is_cuda and perm.dtype == torch.int32 and perm.shape == (B, H, N) and perm.is_contiguous()
    o = out or alloc_quantized(B, H, N, Q.device)
    need = lib().vca_smooth_quantize_workspace_size(B, H, N)
    ws = (ws or Workspace(need, Q.device)).ensure(need)
    _check(lib().vca_smooth_quantize_qkv(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(perm), B, H, N, d, BLOCK, _ptr(o["Qq"]), _ptr(o["q_scale"]),
        _ptr(o["Kq"]), _ptr(o["k_scale"]), _ptr(o["VrT"]), _ptr(o["v_exp"]), _ptr(o["v_mean"]),
        ws.ptr, ws.nbytes, _stream(stream)))
    return o


def smooth_quantize_fp4(Q, K, V, perm, out=None, ws: Workspace | None = None, stream=None) -> dict:
    """4-bit V-Smooth prep: Q/K and block means as ``smooth_quantize``, the V
    residual in NVFP4 (VrT4 [B,H,d,Np/2] packed codes, v_sc [B,H,d,Np/16] E4M3
    group scales, v_gscale [B,H] fp32 head scales)."""
    B, H, N, d = _bhnd(Q)
    assert K.shape == Q.shape and V.shape == Q.shape
    assert perm.is_cuda and perm.dtype == torch.int32 and perm.shape == (B, H, N) and perm.is_contiguous()
    nb = (N + BLOCK - 1) // BLOCK
    Np = nb * BLOCK
    dev = Q.device
    u8, f32 = torch.uint8, torch.float32
    o = out or dict(
        Qq=torch.empty(B, H, Np, d, dtype=u8, device=dev), q_scale=torch.empty(B, H, nb, dtype=f32, device=dev),
        Kq=torch.empty(B, H, Np, d, dtype=u8, device=dev), k_scale=torch.empty(B, H, nb, dtype=f32, device=dev),
        VrT4=torch.empty(B, H, d, Np // 2, dtype=u8, device=dev),
        v_sc=torch.empty(B, H, d, Np // 16, dtype=u8, device=dev),
        v_gscale=torch.empty(B, H, dtype=f32, device=dev),
        v_mean=torch.empty(B, H, nb, d, dtype=torch.bfloat16, device=dev))
    need = lib().vca_smooth_quantize_fp4_workspace_size(B, H, N)
    ws = (ws or Workspace(need, dev)).ensure(need)
    _check(lib().vca_smooth_quantize_qkv_fp4(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(perm), B, H, N, d, _ptr(o["Qq"]), _ptr(o["q_scale"]),
        _ptr(o["Kq"]), _ptr(o["k_scale"]), _ptr(o["VrT4"]), _ptr(o["v_sc"]), _ptr(o["v_gscale"]),
        _ptr(o["v_mean"]), ws.ptr, ws.nbytes, _stream(stream)))
    return o


# ------------------------------------------------------------------ attention
def attention_fwd(ops: dict, N: int, softmax_scale: float | None = None, O=None, lse=None,
                  want_lse: bool = False, ws: Workspace | None = None, stream=None):
    B, H, Np, d = ops["Qq"].shape
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    dev = ops["Qq"].device
    if O is None:
        O = torch.empty(B, H, N, d, dtype=torch.bfloat16, device=dev)
    if want_lse and lse is None:
        lse = torch.empty(B, H, N, dtype=torch.float32, device=dev)
    need = lib().vca_attention_workspace_size(B, H, N)
    ws = (ws or Workspace(need, dev)).ensure(need)
    _check(lib().vca_attention_fwd(
        _ptr(ops["Qq"]), _ptr(ops["q_scale"]), _ptr(ops["Kq"]), _ptr(ops["k_scale"]), _ptr(ops["VrT"]),
        _ptr(ops["v_exp"]), _ptr(ops["v_mean"]), B, H, N, d, scale, _ptr(O), _ptr(lse), ws.ptr, ws.nbytes,
        _stream(stream)))
    return (O, lse) if want_lse else O


def attention_fwd_skip(ops: dict, N: int, skip_lambda: float, softmax_scale: float | None = None, O=None,
                       lse=None, want_lse: bool = False, skipped=None, ws: Workspace | None = None, stream=None):
    """vca_attention_fwd_skip: attention with Skip Softmax block rejection.
    `skipped`, if given, is a one-element int64 device tensor the number of
    skipped (query tile, key block) pairs is added to."""
    B, H, Np, d = ops["Qq"].shape
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    dev = ops["Qq"].device
    if O is None:
        O = torch.empty(B, H, N, d, dtype=torch.bfloat16, device=dev)
    if want_lse and lse is None:
        lse = torch.empty(B, H, N, dtype=torch.float32, device=dev)
    if skipped is not None:
        assert skipped.dtype == torch.int64 and skipped.numel() == 1
    need = lib().vca_attention_workspace_size(B, H, N)
    ws = (ws or Workspace(need, dev)).ensure(need)
    _check(lib().vca_attention_fwd_skip(
        _ptr(ops["Qq"]), _ptr(ops["q_scale"]), _ptr(ops["Kq"]), _ptr(ops["k_scale"]), _ptr(ops["VrT"]),
        _ptr(ops["v_exp"]), _ptr(ops["v_mean"]), B, H, N, d, scale, float(skip_lambda), _ptr(O), _ptr(lse),
        _ptr(skipped), ws.ptr, ws.nbytes, _stream(stream)))
    return (O, lse) if want_lse else O


def bf16_attention_fwd(Q, K, V, softmax_scale: float | None = None, O=None, lse=None, want_lse=False,
                       ws: Workspace | None = None, stream=None):
    B, H, N, d = _bhnd(Q)
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    if O is None:
        O = torch.empty_like(Q)
    if want_lse and lse is None:
        lse = torch.empty(B, H, N, dtype=torch.float32, device=Q.device)
    need = lib().vca_bf16_attention_workspace_size(B, H, N)
    ws = (ws or Workspace(need, Q.device)).ensure(need)
    _check(lib().vca_bf16_attention_fwd(_ptr(Q), _ptr(K), _ptr(V), B, H, N, d, scale, _ptr(O), _ptr(lse),
                                        ws.ptr, ws.nbytes, _stream(stream)))
    return (O, lse) if want_lse else O


def vc_attention(Q, K, V, k: int = 32, iters: int = 3, softmax_scale=None, perm=None, ws=None, stream=None):
    """Whole path: cluster/permute (unless `perm` is given), quantise, attend."""
    if perm is None:
        _, _, perm = cluster_permute(V, k, iters, ws=ws, stream=stream)
    ops = smooth_quantize(Q, K, V, perm, ws=ws, stream=stream)
    return attention_fwd(ops, Q.shape[2], softmax_scale, ws=ws, stream=stream)


def schedule_regroup(step: int, total_steps: int, reuse: int = 4, group_fraction: float = 0.25) -> bool:
    """vca_schedule_regroup: does this denoising step regroup (k-means + sort)?"""
    rc = lib().vca_schedule_regroup(step, total_steps, reuse, group_fraction)
    if rc < 0:
        _check(rc)
    return rc == 1


class VCAttentionLayer:
    """One attention layer across a denoising run: keeps the layer's permutation
    and centroids between steps, regroups (warm-started from the last
    centroids) when vca_schedule_regroup says so, quantises and attends every
    step.  Holds state only; every step of the path runs in the library."""

    def __init__(self, total_steps: int, k: int = 32, iters: int = 3, reuse: int = 4,
                 group_fraction: float = 0.25, ws: Workspace | None = None):
        self.total_steps, self.k, self.iters = total_steps, k, iters
        self.reuse, self.group_fraction = reuse, group_fraction
        self.ws = ws
        self.centroids = None
        self.perm = None
        self.regrouped_at = []

    def __call__(self, Q, K, V, step: int, softmax_scale=None, stream=None):
        if self.ws is None:
            self.ws = Workspace(lib().vca_status_bytes(), V.device)
        if self.perm is None or schedule_regroup(step, self.total_steps, self.reuse, self.group_fraction):
            self.centroids, _, self.perm = cluster_permute(V, self.k, self.iters, init=self.centroids,
                                                           ws=self.ws, stream=stream)
            self.regrouped_at.append(step)
        ops = smooth_quantize(Q, K, V, self.perm, ws=self.ws, stream=stream)
        return attention_fwd(ops, Q.shape[2], softmax_scale, ws=self.ws, stream=stream)


_host_bufs = {}


def vc_attention_host(Q, K, V, k: int = 32, iters: int = 3, softmax_scale=None, O=None, heads_per_chunk: int = 0,
                      device=None, stream=None):
    """vca_vc_attention_host: the whole path from host (CPU) bf16 tensors to a
    host bf16 output, copies overlapped with the kernels.  Pass page-locked
    tensors (tensor.pin_memory()) for the overlap.  The device scratch is kept
    per (device, size) between calls."""
    assert Q.device.type == "cpu" and Q.dtype == torch.bfloat16 and Q.is_contiguous()
    assert K.shape == Q.shape == V.shape and K.is_contiguous() and V.is_contiguous()
    B, H, N, d = Q.shape
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    if O is None:
        O = torch.empty(Q.shape, dtype=torch.bfloat16, pin_memory=Q.is_pinned())
    need = lib().vca_vc_attention_host_buffer_size(B, H, N, d, k, heads_per_chunk)
    if need == 0:
        raise VcaError(ERR_INVALID, "vc_attention_host: unsupported shape")
    key = (dev.index, need)
    if key not in _host_bufs:
        _host_bufs.clear()
        _host_bufs[key] = torch.empty(need, dtype=torch.uint8, device=dev)
    buf = _host_bufs[key]
    with torch.cuda.device(dev):
        _check(lib().vca_vc_attention_host(_ptr(Q), _ptr(K), _ptr(V), B, H, N, d, k, iters, scale, _ptr(O),
                                           heads_per_chunk, ctypes.c_void_p(buf.data_ptr()), need,
                                           _stream(stream)))
    return O


def sage_quantize(Q, K, V, ws: Workspace | None = None, stream=None, qk_dtype: str = "fp8") -> dict:
    """vca_sage_quantize_qkv (qk_dtype "fp8": E4M3 Q and K') or
    vca_sage_quantize_qkv_i8 ("int8": signed-byte Q and K'): the SAGE-style
    comparison quantisation."""
    if qk_dtype not in ("fp8", "int8"):
        raise ValueError(f"qk_dtype must be 'fp8' or 'int8', not {qk_dtype!r}")
    B, H, N, d = _bhnd(Q)
    dev = Q.device
    nb = (N + 127) // 128
    Np = nb * 128
    ct = torch.int8 if qk_dtype == "int8" else torch.uint8
    out = dict(Qq=torch.empty(B, H, Np, d, dtype=ct, device=dev),
               q_scale=torch.empty(B, H, Np, dtype=torch.float32, device=dev),
               Kq=torch.empty(B, H, Np, d, dtype=ct, device=dev),
               k_scale=torch.empty(B, H, Np // 16, dtype=torch.float32, device=dev),
               VcT=torch.empty(B, H, d, Np, dtype=torch.uint8, device=dev),
               v_chscale=torch.empty(B, H, d, dtype=torch.float32, device=dev),
               k_mean=torch.empty(B, H, d, dtype=torch.bfloat16, device=dev))
    need = lib().vca_sage_quantize_workspace_size(B, H, N)
    ws = (ws or Workspace(need, dev)).ensure(need)
    fn = lib().vca_sage_quantize_qkv_i8 if qk_dtype == "int8" else lib().vca_sage_quantize_qkv
    _check(fn(
        _ptr(Q), _ptr(K), _ptr(V), B, H, N, d, _ptr(out["Qq"]), _ptr(out["q_scale"]), _ptr(out["Kq"]),
        _ptr(out["k_scale"]), _ptr(out["VcT"]), _ptr(out["v_chscale"]), _ptr(out["k_mean"]), ws.ptr, ws.nbytes,
        _stream(stream)))
    return out


def attention_fwd_fp4(ops: dict, N: int, softmax_scale: float | None = None, O=None, lse=None,
                      want_lse: bool = False, ws: Workspace | None = None, stream=None):
    """vca_attention_fwd_fp4: attention of the 4-bit variant on the operands of
    ``smooth_quantize_fp4`` (NVFP4 probabilities and V residual in PV)."""
    B, H, Np, d = ops["Qq"].shape
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    dev = ops["Qq"].device
    if O is None:
        O = torch.empty(B, H, N, d, dtype=torch.bfloat16, device=dev)
    if want_lse and lse is None:
        lse = torch.empty(B, H, N, dtype=torch.float32, device=dev)
    need = lib().vca_attention_workspace_size(B, H, N)
    ws = (ws or Workspace(need, dev)).ensure(need)
    _check(lib().vca_attention_fwd_fp4(
        _ptr(ops["Qq"]), _ptr(ops["q_scale"]), _ptr(ops["Kq"]), _ptr(ops["k_scale"]), _ptr(ops["VrT4"]),
        _ptr(ops["v_sc"]), _ptr(ops["v_gscale"]), _ptr(ops["v_mean"]), B, H, N, d, scale, _ptr(O), _ptr(lse),
        ws.ptr, ws.nbytes, _stream(stream)))
    return (O, lse) if want_lse else O


def debug_fp4_mma(a_codes, sf_cols, b_codes, ws: Workspace | None = None, stream=None) -> torch.Tensor:
    """vca_debug_fp4_mma: one 128x128x128 block-scaled FP4 product with known
    operands (uint8 device tensors [128, 64] A codes, [128, 64] the 16 scale
    columns of every tensor-memory lane, [128, 64] B^T codes)."""
    for t in (a_codes, sf_cols, b_codes):
        assert t.is_cuda and t.dtype == torch.uint8 and tuple(t.shape) == (128, 64) and t.is_contiguous()
    D = torch.empty(128, 128, dtype=torch.float32, device=a_codes.device)
    ws = ws or Workspace(256, a_codes.device)
    _check(lib().vca_debug_fp4_mma(_ptr(a_codes), _ptr(sf_cols), _ptr(b_codes), _ptr(D), ws.ptr, _stream(stream)))
    ws.check(stream)
    return D


def attention_fwd_sage(ops: dict, N: int, softmax_scale: float | None = None, O=None, lse=None,
                       want_lse: bool = False, ws: Workspace | None = None, stream=None):
    """vca_attention_fwd_sage (E4M3 Q/K) or vca_attention_fwd_sage_i8 (int8 Q/K,
    picked by the operands' dtype): attention on SAGE-style operands."""
    B, H, Np, d = ops["Qq"].shape
    if ops["Qq"].dtype != ops["Kq"].dtype or ops["Qq"].dtype not in (torch.uint8, torch.int8):
        raise ValueError("Qq and Kq must both be uint8 (E4M3) or both int8")
    fn = lib().vca_attention_fwd_sage_i8 if ops["Qq"].dtype == torch.int8 else lib().vca_attention_fwd_sage
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    dev = ops["Qq"].device
    if O is None:
        O = torch.empty(B, H, N, d, dtype=torch.bfloat16, device=dev)
    if want_lse and lse is None:
        lse = torch.empty(B, H, N, dtype=torch.float32, device=dev)
    need = lib().vca_attention_workspace_size(B, H, N)
    ws = (ws or Workspace(need, dev)).ensure(need)
    _check(fn(
        _ptr(ops["Qq"]), _ptr(ops["q_scale"]), _ptr(ops["Kq"]), _ptr(ops["k_scale"]), _ptr(ops["VcT"]),
        _ptr(ops["v_chscale"]), B, H, N, d, scale, _ptr(O), _ptr(lse), ws.ptr, ws.nbytes, _stream(stream)))
    return (O, lse) if want_lse else O
