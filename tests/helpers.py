"""Shared helpers for the parity tests: bf16 bit patterns, row sampling, metrics,
scores recomputed from library-decoded operands, and the lse tolerance that
codes rounding the other way at an fp32/fp64 boundary allow."""
from __future__ import annotations

import math

import numpy as np
import torch

from bit_attention_video_02_b200 import workloads as W


def bits(t: torch.Tensor) -> np.ndarray:
    """uint16 numpy copy of a bf16 tensor's bit patterns."""
    return W.bf16_bits(t)


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def cosine(a, b) -> float:
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / max(np.linalg.norm(a) * np.linalg.norm(b), 1e-300))


def psnr(test, ref) -> float:
    """10 log10(max|ref|^2 / MSE), peak = largest magnitude of the reference."""
    test = np.asarray(test, np.float64)
    ref = np.asarray(ref, np.float64)
    mse = float(np.mean((test - ref) ** 2))
    peak = float(np.max(np.abs(ref)))
    return float("inf") if mse == 0 else 10.0 * math.log10(peak * peak / mse)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def sample_rows(N: int, n: int, seed: int) -> np.ndarray:
    """Seeded query rows, always including the first and last rows (ragged tail)."""
    if n >= N:
        return np.arange(N, dtype=np.int32)
    rng = np.random.default_rng(seed)
    r = rng.choice(N, size=n - 2, replace=False)
    return np.unique(np.concatenate([r, [0, N - 1]])).astype(np.int32)


PHI = 0.65 / 8          # the ExpCast maximum grid: m = n + 0.65/8
LOG2E = 1.4426950408889634


def e4m3_lib(codes) -> np.ndarray:
    """Library decode of E4M3 bytes (torch float8_e4m3fn), as fp64."""
    a = np.ascontiguousarray(codes, dtype=np.uint8)
    return torch.from_numpy(a).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def scores_log2(ops, N, rows, scale, with_abs=False):
    """z[i, j] = (q_i . k_j) sq sk scale log2(e) in fp64 for query rows `rows`
    over the N permuted keys (E4M3 dot products are exact in fp64); with_abs
    also returns sum_c |q_ic k_jc| (the accumulation error scale)."""
    q = e4m3_lib(ops["Qq"][rows])
    k = e4m3_lib(ops["Kq"][:N])
    qs = ops["q_scale"].astype(np.float64)[np.asarray(rows) // 128]
    ks = ops["k_scale"].astype(np.float64)[np.arange(N) // 128]
    cz = qs[:, None] * ks[None, :] * scale * LOG2E
    z = (q @ k.T) * cz
    if not with_abs:
        return z
    return z, (np.abs(q) @ np.abs(k).T) * cz


def lse_tolerance(ops, N, rows, scale, codes, nref, lblk, lse_ref) -> np.ndarray:
    """Per-row bound on |lse_gpu - lse_oracle| derived from the code rounding.

    The kernel forms 8 z + 87 - 8 n in fp32 (scale products rounded three
    times, tensor-core sums) where the oracle uses fp64, so a code can round
    the other way only where the fp64 value lies within the fp32 error of a
    half-integer: eps = 2^-20 (8 |z| + 8 sum|q k| cz).  Such a flip moves that
    key's decoded probability by at most one E4M3 step (the larger of the steps
    to its neighbours, in the frame of the final reference).  The row's
    log-sum then moves by at most ln(1 + sum of those steps / sum of the row's
    probabilities); the kernel's fp32 sums over (nb + 64) terms and its fp32
    log add (nb + 64) 2^-24 and 2^-17 (|lse| + 1)."""
    rows = np.asarray(rows)
    table = e4m3_lib(np.arange(128, dtype=np.uint8))
    nb = lblk.shape[1]
    delta = np.empty(len(rows))
    for r0 in range(0, len(rows), 32):          # bounded memory at full N
        sl = slice(r0, r0 + 32)
        z, zabs = scores_log2(ops, N, rows[sl], scale, with_abs=True)
        nk = nref[sl][:, np.arange(N) // 128].astype(np.float64)
        x = 8.0 * z + 87.0 - 8.0 * nk
        eps = 2.0 ** -20 * (8.0 * np.abs(z) + 8.0 * zabs) + 1e-6
        near = np.abs(x - np.floor(x) - 0.5) <= eps
        c = codes[sl].astype(np.int64)
        up = table[np.minimum(c + 1, 126)] - table[c]
        dn = table[c] - table[np.maximum(c - 1, 0)]
        frame = np.ldexp(1.0, (nk - nref[sl][:, -1:]).astype(np.int64))
        delta[sl] = np.where(near, np.maximum(up, dn) * frame, 0.0).sum(1)
    L = lblk.sum(1)
    return np.log1p(delta / L) + (nb + 64) * 2.0 ** -24 + 2.0 ** -17 * (np.abs(lse_ref) + 1.0)
