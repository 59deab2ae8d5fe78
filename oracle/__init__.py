"""Plain, slow CPU oracle for VC-Attention-style FP8 attention (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (``bit_attention_video_02_b200``)
never does, and the two share no code: this package wraps ``liboracle.so``,
built from ``vca_oracle.c`` with gcc, in fp64 (fp32 with explicit ``fmaf`` where
the method fixes fp32).

Sources are the pages describing the method:
  * "VC-Attention: Training-Free Low-Bit Attention Speeds Video Diffusion Up to
    3.6x" (agihunt.info) -- V-Smooth and ExpCast-FP8 bullets;
  * "Nunchux AI Introduces VC-Attention: A Training-Free Low-Bit Attention Kernel
    That Speeds Up Video Diffusion Transformers" (MarkTechPost abstract and its
    Chinese summary, section "V-Smooth 與 ExpCast-FP8");
  * "VC-Attention" (aikraft.ru), section "Решение".

Each wrapper below follows one step of the method; the C source states the
passage and the reading taken where the pages are silent.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

EXACT_EXP = 1
IDENTITY_QUANT = 2
PLANT_TRUNC = 64
PLANT_NO_MEAN = 128
PLANT_BETA0 = 256
PLANT_NO_RESCALE = 512
PLANT_NIBBLE = 1024
PLANT_P_GROUP32 = 2048
GLOBAL_MAX = 4096      # second reading: the reference is the snapped row maximum, fixed
NO_HEADROOM = 8192     # codes written at the reference instead of 4 octaves above it
P_GSCALE = 0.125   # NVFP4 tensor scale of the 4-bit variant's probabilities
BLOCK = 128

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = ctypes.CDLL(path)
        _declare(_lib)
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _declare(L):
    vp, i32, i64, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
    L.vo_e4m3_decode.restype = f64
    L.vo_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.vo_e4m3_encode.restype = ctypes.c_uint8
    L.vo_e4m3_encode.argtypes = [ctypes.c_float]
    L.vo_e4m3_encode_array.argtypes = [vp, vp, i64]
    L.vo_expcast.restype = ctypes.c_uint8
    L.vo_expcast.argtypes = [ctypes.c_float, i32]
    L.vo_expcast_array.argtypes = [vp, vp, i64, i32]
    L.vo_double_to_bf16_rne.restype = ctypes.c_uint16
    L.vo_double_to_bf16_rne.argtypes = [f64]
    L.vo_kmeans_assign.argtypes = [vp, i32, i32, vp, i32, vp]
    L.vo_kmeans_update.argtypes = [vp, i32, i32, vp, i32, vp, vp]
    L.vo_kmeans_head.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp]
    L.vo_stable_perm.argtypes = [vp, i32, i32, vp]
    L.vo_v_exponent.restype = i32
    L.vo_v_exponent.argtypes = [ctypes.c_float]
    L.vo_smooth_quantize_head.argtypes = [vp] * 4 + [i32, i32] + [vp] * 7
    L.vo_attention_head.argtypes = [vp] * 7 + [i32, i32, f64, vp, i32, i32, vp, vp, vp]
    L.vo_attention_head_bf16.argtypes = [vp] * 4 + [i32, i32, f64, vp, i32, i32, vp]
    L.vo_smooth_quantize_head_vhead.argtypes = [vp] * 4 + [i32, i32] + [vp] * 7
    L.vo_sage_quantize_head.argtypes = [vp] * 3 + [i32, i32] + [vp] * 7
    L.vo_attention_head_sage.argtypes = [vp] * 6 + [i32, i32, f64, vp, i32, i32, vp, vp]
    L.vo_sage_quantize_head_i8.argtypes = [vp] * 3 + [i32, i32] + [vp] * 7
    L.vo_attention_head_sage_i8.argtypes = [vp] * 6 + [i32, i32, f64, vp, i32, i32, vp, vp]
    L.vo_attention_head_skip.argtypes = [vp] * 7 + [i32, i32, f64, vp, i32, i32, f64, vp, vp, vp]
    L.vo_attention_head_ex.argtypes = [vp] * 7 + [i32, i32, f64, vp, i32, i32, f64, vp, vp, vp, vp, vp]
    L.vo_attention_head_bf16_skip.argtypes = [vp] * 4 + [i32, i32, f64, vp, i32, i32, f64, vp]
    L.vo_e2m1_decode.restype = f64
    L.vo_e2m1_decode.argtypes = [ctypes.c_uint8]
    L.vo_e2m1_encode.restype = ctypes.c_uint8
    L.vo_e2m1_encode.argtypes = [ctypes.c_float]
    L.vo_nvfp4_quantize.argtypes = [vp, i64, ctypes.c_float, vp, vp]
    L.vo_smooth_quantize_head_fp4.argtypes = [vp] * 4 + [i32, i32] + [vp] * 8
    L.vo_attention_head_fp4.argtypes = [vp] * 6 + [ctypes.c_float, vp, i32, i32, f64, vp, i32, i32, vp, vp]
    L.vo_p_nvfp4.argtypes = [vp, i32, i32, vp]
    L.vo_attention_head_fp4_bf16.argtypes = [vp] * 4 + [i32, i32, f64, vp, i32, i32, vp]
    L.vo_exact_attention_head.argtypes = [vp] * 3 + [i32, i32, f64, vp, i32, vp]
    L.vo_num_threads.restype = i32


def num_threads() -> int:
    return int(lib().vo_num_threads())


# ------------------------------------------------------------------ E4M3
def e4m3_decode(code: int) -> float:
    return float(lib().vo_e4m3_decode(int(code) & 0xFF))


def e4m3_decode_table() -> np.ndarray:
    return np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)


def e4m3_encode(x) -> np.ndarray:
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    out = np.empty(x.shape, dtype=np.uint8)
    lib().vo_e4m3_encode_array(_p(x), _p(out), x.size)
    return out


# ------------------------------------------------------------------ E2M1 / NVFP4
def e2m1_decode_table() -> np.ndarray:
    return np.array([lib().vo_e2m1_decode(c) for c in range(16)], np.float64)


def e2m1_encode(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32)
    return np.array([lib().vo_e2m1_encode(float(v)) for v in x.ravel()], np.uint8).reshape(x.shape)


def nvfp4_quantize(x, G: float):
    """NVFP4 codes (one nibble per byte) and E4M3 group scales of x[n] in
    groups of 16 consecutive elements, tensor scale G."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32).ravel())
    codes = np.empty(x.size, np.uint8)
    scales = np.empty((x.size + 15) // 16, np.uint8)
    lib().vo_nvfp4_quantize(_p(x), x.size, float(G), _p(codes), _p(scales))
    return codes, scales


# ------------------------------------------------------------------ ExpCast
def expcast(z, flags: int = 0) -> np.ndarray:
    z = np.ascontiguousarray(np.asarray(z, dtype=np.float32))
    out = np.empty(z.shape, dtype=np.uint8)
    lib().vo_expcast_array(_p(z), _p(out), z.size, int(flags))
    return out


def double_to_bf16(x: float) -> int:
    return int(lib().vo_double_to_bf16_rne(float(x)))


# ------------------------------------------------------------------ k-means
def kmeans_assign(v: np.ndarray, cent: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    cent = np.ascontiguousarray(cent, dtype=np.float32)
    N, d = v.shape
    out = np.empty(N, dtype=np.int32)
    lib().vo_kmeans_assign(_p(v), N, d, _p(cent), cent.shape[0], _p(out))
    return out


def kmeans_update(v: np.ndarray, assign: np.ndarray, cent: np.ndarray):
    v = np.ascontiguousarray(v, dtype=np.float32)
    assign = np.ascontiguousarray(assign, dtype=np.int32)
    cent = np.array(cent, dtype=np.float32, copy=True)
    k = cent.shape[0]
    counts = np.empty(k, dtype=np.int32)
    lib().vo_kmeans_update(_p(v), v.shape[0], v.shape[1], _p(assign), k, _p(cent), _p(counts))
    return cent, counts


def kmeans_head(V_bits: np.ndarray, k: int, iters: int, init=None):
    """One head. ``V_bits``: [N, d] uint16 bf16 bit patterns."""
    V_bits = np.ascontiguousarray(V_bits, dtype=np.uint16)
    N, d = V_bits.shape
    cent = np.empty((k, d), dtype=np.float32)
    assign = np.empty(N, dtype=np.int32)
    counts = np.empty(k, dtype=np.int32)
    initp = None
    if init is not None:
        init = np.ascontiguousarray(init, dtype=np.float32)
        initp = _p(init)
    lib().vo_kmeans_head(_p(V_bits), N, d, k, iters, initp, _p(cent), _p(assign), _p(counts))
    return cent, assign, counts


def stable_perm(assign: np.ndarray, k: int) -> np.ndarray:
    assign = np.ascontiguousarray(assign, dtype=np.int32)
    perm = np.empty(assign.shape[0], dtype=np.int32)
    lib().vo_stable_perm(_p(assign), assign.shape[0], k, _p(perm))
    return perm


# ------------------------------------------------------------------ quantise
def v_exponent(amax: float) -> int:
    return int(lib().vo_v_exponent(float(amax)))


def smooth_quantize_head(Q, K, V, perm, v_scale: str = "block"):
    """One head of V-Smooth prep; inputs [N, d] uint16 bf16 bits, perm [N] int32.
    v_scale "block" (one V residual exponent per block) or "head" (one per head)."""
    Q, K, V = (np.ascontiguousarray(a, dtype=np.uint16) for a in (Q, K, V))
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    N, d = Q.shape
    nb = (N + BLOCK - 1) // BLOCK
    Np = nb * BLOCK
    out = dict(
        Qq=np.zeros((Np, d), np.uint8), q_scale=np.empty(nb, np.float32),
        Kq=np.zeros((Np, d), np.uint8), k_scale=np.empty(nb, np.float32),
        VrT=np.zeros((d, Np), np.uint8), v_exp=np.empty(nb, np.int8),
        v_mean=np.empty((nb, d), np.uint16))
    assert v_scale in ("block", "head")
    fn = lib().vo_smooth_quantize_head if v_scale == "block" else lib().vo_smooth_quantize_head_vhead
    fn(
        _p(Q), _p(K), _p(V), _p(perm), N, d, _p(out["Qq"]), _p(out["q_scale"]),
        _p(out["Kq"]), _p(out["k_scale"]), _p(out["VrT"]), _p(out["v_exp"]),
        _p(out["v_mean"]))
    return out


def smooth_quantize_head_fp4(Q, K, V, perm):
    """One head of the 4-bit V-Smooth variant: Q/K and block means as the 8-bit
    prep, the V residual in NVFP4 (VrT4 [d, Np/2] packed, v_sc [d, Np/16],
    v_gscale)."""
    Q, K, V = (np.ascontiguousarray(a, dtype=np.uint16) for a in (Q, K, V))
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    N, d = Q.shape
    nb = (N + BLOCK - 1) // BLOCK
    Np = nb * BLOCK
    out = dict(
        Qq=np.zeros((Np, d), np.uint8), q_scale=np.empty(nb, np.float32),
        Kq=np.zeros((Np, d), np.uint8), k_scale=np.empty(nb, np.float32),
        VrT4=np.zeros((d, Np // 2), np.uint8), v_sc=np.zeros((d, Np // 16), np.uint8),
        v_gscale=np.empty(1, np.float32), v_mean=np.empty((nb, d), np.uint16))
    lib().vo_smooth_quantize_head_fp4(
        _p(Q), _p(K), _p(V), _p(perm), N, d, _p(out["Qq"]), _p(out["q_scale"]),
        _p(out["Kq"]), _p(out["k_scale"]), _p(out["VrT4"]), _p(out["v_sc"]),
        _p(out["v_gscale"]), _p(out["v_mean"]))
    return out


def sage_quantize_head(Q, K, V, qk_dtype: str = "fp8"):
    """One head of the SAGE-style comparison quantisation (per-token Q,
    per-16-token K after K-mean smoothing, per-channel V; no reordering).
    qk_dtype "fp8" codes Q and K' as E4M3 (uint8), "int8" as signed bytes."""
    if qk_dtype not in ("fp8", "int8"):
        raise ValueError(f"qk_dtype must be 'fp8' or 'int8', not {qk_dtype!r}")
    Q, K, V = (np.ascontiguousarray(a, dtype=np.uint16) for a in (Q, K, V))
    N, d = Q.shape
    Np = (N + BLOCK - 1) // BLOCK * BLOCK
    ct = np.int8 if qk_dtype == "int8" else np.uint8
    out = dict(
        Qq=np.zeros((Np, d), ct), q_scale=np.empty(Np, np.float32),
        Kq=np.zeros((Np, d), ct), k_scale=np.empty(Np // 16, np.float32),
        VcT=np.zeros((d, Np), np.uint8), v_chscale=np.empty(d, np.float32),
        k_mean=np.empty(d, np.uint16))
    fn = lib().vo_sage_quantize_head_i8 if qk_dtype == "int8" else lib().vo_sage_quantize_head
    fn(_p(Q), _p(K), _p(V), N, d, _p(out["Qq"]), _p(out["q_scale"]), _p(out["Kq"]), _p(out["k_scale"]),
       _p(out["VcT"]), _p(out["v_chscale"]), _p(out["k_mean"]))
    return out


# ------------------------------------------------------------------ attention
def _rows(rows, N):
    if rows is None:
        rows = np.arange(N, dtype=np.int32)
    return np.ascontiguousarray(rows, dtype=np.int32)


def attention_head(ops: dict, N: int, softmax_scale: float, rows=None, flags: int = 0,
                   want_lblk: bool = False, skip_lambda: float = 0.0):
    """Same-algorithm attention from quantised operands (dict as returned by
    ``smooth_quantize_head``).  Returns (O [nrows, d] fp64, lse [nrows], lblk).
    skip_lambda > 0 applies the Skip Softmax block rejection."""
    rows = _rows(rows, N)
    d = ops["Qq"].shape[1]
    nb = ops["q_scale"].shape[0]
    O = np.empty((rows.shape[0], d), np.float64)
    lse = np.empty(rows.shape[0], np.float64)
    lblk = np.empty((rows.shape[0], nb), np.float64) if want_lblk else None
    c = {k: np.ascontiguousarray(v) for k, v in ops.items()}
    lib().vo_attention_head_skip(
        _p(c["Qq"]), _p(c["q_scale"]), _p(c["Kq"]), _p(c["k_scale"]), _p(c["VrT"]),
        _p(c["v_exp"]), _p(c["v_mean"]), N, d, float(softmax_scale), _p(rows),
        rows.shape[0], int(flags), float(skip_lambda), _p(O), _p(lse), _p(lblk) if lblk is not None else None)
    return O, lse, lblk


def attention_head_codes(ops: dict, N: int, softmax_scale: float, rows=None, flags: int = 0,
                         skip_lambda: float = 0.0):
    """As ``attention_head``, also returning what each row coded.  Returns
    (O, lse, lblk [nrows, nb], codes [nrows, N] uint8 in permuted key order,
    nref [nrows, nb] int32: the reference n each block was coded against)."""
    rows = _rows(rows, N)
    d = ops["Qq"].shape[1]
    nb = ops["q_scale"].shape[0]
    O = np.empty((rows.shape[0], d), np.float64)
    lse = np.empty(rows.shape[0], np.float64)
    lblk = np.empty((rows.shape[0], nb), np.float64)
    codes = np.empty((rows.shape[0], N), np.uint8)
    nref = np.empty((rows.shape[0], nb), np.int32)
    c = {k: np.ascontiguousarray(v) for k, v in ops.items()}
    lib().vo_attention_head_ex(
        _p(c["Qq"]), _p(c["q_scale"]), _p(c["Kq"]), _p(c["k_scale"]), _p(c["VrT"]),
        _p(c["v_exp"]), _p(c["v_mean"]), N, d, float(softmax_scale), _p(rows),
        rows.shape[0], int(flags), float(skip_lambda), _p(O), _p(lse), _p(lblk), _p(codes), _p(nref))
    return O, lse, lblk, codes, nref


def attention_head_bf16(Q, K, V, perm, softmax_scale: float, rows=None, flags: int = 0, skip_lambda: float = 0.0):
    Q, K, V = (np.ascontiguousarray(a, dtype=np.uint16) for a in (Q, K, V))
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    N, d = Q.shape
    rows = _rows(rows, N)
    O = np.empty((rows.shape[0], d), np.float64)
    lib().vo_attention_head_bf16_skip(_p(Q), _p(K), _p(V), _p(perm), N, d, float(softmax_scale),
                                      _p(rows), rows.shape[0], int(flags), float(skip_lambda), _p(O))
    return O


def attention_head_sage(ops: dict, N: int, softmax_scale: float, rows=None, flags: int = 0):
    """Attention on SAGE-style operands (dict from ``sage_quantize_head``; the
    Q/K code dtype, uint8 E4M3 or int8, picks the decoding).
    Returns (O [nrows, d] fp64, lse [nrows])."""
    rows = _rows(rows, N)
    d = ops["Qq"].shape[1]
    O = np.empty((rows.shape[0], d), np.float64)
    lse = np.empty(rows.shape[0], np.float64)
    c = {k: np.ascontiguousarray(v) for k, v in ops.items()}
    if c["Qq"].dtype != c["Kq"].dtype or c["Qq"].dtype not in (np.uint8, np.int8):
        raise ValueError("Qq and Kq must both be uint8 (E4M3) or both int8")
    fn = lib().vo_attention_head_sage_i8 if c["Qq"].dtype == np.int8 else lib().vo_attention_head_sage
    fn(_p(c["Qq"]), _p(c["q_scale"]), _p(c["Kq"]), _p(c["k_scale"]), _p(c["VcT"]), _p(c["v_chscale"]),
       N, d, float(softmax_scale), _p(rows), rows.shape[0], int(flags), _p(O), _p(lse))
    return O, lse


def attention_head_fp4(ops: dict, N: int, softmax_scale: float, rows=None, flags: int = 0):
    """Attention of the 4-bit variant (dict from ``smooth_quantize_head_fp4``).
    Returns (O [nrows, d] fp64, lse [nrows])."""
    rows = _rows(rows, N)
    d = ops["Qq"].shape[1]
    O = np.empty((rows.shape[0], d), np.float64)
    lse = np.empty(rows.shape[0], np.float64)
    c = {k: np.ascontiguousarray(v) for k, v in ops.items()}
    lib().vo_attention_head_fp4(
        _p(c["Qq"]), _p(c["q_scale"]), _p(c["Kq"]), _p(c["k_scale"]), _p(c["VrT4"]), _p(c["v_sc"]),
        float(c["v_gscale"].ravel()[0]), _p(c["v_mean"]), N, d, float(softmax_scale), _p(rows),
        rows.shape[0], int(flags), _p(O), _p(lse))
    return O, lse


def p_nvfp4(p, flags: int = 0) -> np.ndarray:
    """The 4-bit variant's probability quantisation of one key block (n <= 128)."""
    p = np.ascontiguousarray(np.asarray(p, np.float64).ravel())
    assert p.size <= BLOCK
    out = np.empty_like(p)
    lib().vo_p_nvfp4(_p(p), p.size, int(flags), _p(out))
    return out


def attention_head_fp4_bf16(Q, K, V, perm, softmax_scale: float, rows=None, flags: int = 0):
    Q, K, V = (np.ascontiguousarray(a, dtype=np.uint16) for a in (Q, K, V))
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    N, d = Q.shape
    rows = _rows(rows, N)
    O = np.empty((rows.shape[0], d), np.float64)
    lib().vo_attention_head_fp4_bf16(_p(Q), _p(K), _p(V), _p(perm), N, d, float(softmax_scale),
                                     _p(rows), rows.shape[0], int(flags), _p(O))
    return O


def exact_attention_head(Q, K, V, softmax_scale: float, rows=None):
    Q, K, V = (np.ascontiguousarray(a, dtype=np.uint16) for a in (Q, K, V))
    N, d = Q.shape
    rows = _rows(rows, N)
    O = np.empty((rows.shape[0], d), np.float64)
    lib().vo_exact_attention_head(_p(Q), _p(K), _p(V), N, d, float(softmax_scale),
                                  _p(rows), rows.shape[0], _p(O))
    return O


# ------------------------------------------------------------------ whole prep
def prep_head(Q, K, V, k: int, iters: int = 3, init=None):
    """k-means -> stable permutation -> V-Smooth quantisation for one head."""
    cent, assign, counts = kmeans_head(V, k, iters, init)
    perm = stable_perm(assign, k)
    ops = smooth_quantize_head(Q, K, V, perm)
    ops.update(centroids=cent, assign=assign, counts=counts, perm=perm)
    return ops
