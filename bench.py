"""Benchmark: V-Smooth prep + ExpCast-FP8 attention on one B200 per rank.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload 3] [--no-cpu-baseline] [--no-e2e]

One step is one pass of the whole hot path over one synthetic layer input:
k-means over V + stable permutation (vca_cluster_permute), V-Smooth
quantisation of Q/K/V (vca_smooth_quantize_qkv) and ExpCast-FP8 attention
(vca_attention_fwd).  `value` is 4*B*H*N^2*d / (step time), i.e. attention
TFLOP/s counting the prep inside the step, summed over ranks (each rank runs
its own layer: weak scaling, no collective on the data path).

Rank 0 prints one JSON line.  Multi-GPU runs are launched with
torch.distributed.run (one rank per GPU); the timed region is bracketed by a
barrier and synchronize, and the time is the max over ranks.

--impl reference times the plain CPU oracle on the host cores (the method has
no other reference implementation) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_attention_video_02_b200 import build as vca_build  # noqa: E402
from bit_attention_video_02_b200 import vca  # noqa: E402
from bit_attention_video_02_b200 import workloads as W  # noqa: E402

METRIC = "FP8 attention TFLOP/s (4*B*H*N^2*d/t) & % of B200 FP8 peak; V-Smooth prep ms"
KMEANS_ITERS = 3
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_PER_BF16 = 2.0          # nominal dense FP8 / BF16 tensor throughput ratio (4.5 / 2.25 PFLOP/s)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def whole_job_value(world: int, flops_per_rank: float, seconds_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank runs its own layer of `flops_per_rank`
    (weak scaling) and the step time is the slowest rank's."""
    return world * flops_per_rank / seconds_per_step / 1e12


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.25)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ our arm
def run_ours(args, world, rank, local):
    vca_build.build()
    w = W.shrink(W.WORKLOADS[args.workload], H=args.heads)
    dev = torch.device("cuda", local)
    scale = 1.0 / math.sqrt(w.d)
    Q, K, V = W.make_qkv(w, dev)
    B, H, N, d = w.B, w.H, w.N, w.d
    ws = vca.Workspace(vca.lib().vca_cluster_permute_workspace_size(B, H, N, w.k), dev)
    ops = vca.alloc_quantized(B, H, N, dev)
    O = torch.empty(B, H, N, d, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    # init, T x (assign, sort count, sort scan, sort scatter, accumulate, update), quantise, attention
    launches_per_step = 1 + 6 * KMEANS_ITERS + 1 + 1

    def step(t_attn=None):
        _, _, perm = vca.cluster_permute(V, w.k, KMEANS_ITERS, ws=ws)
        vca.smooth_quantize(Q, K, V, perm, out=ops, ws=ws)
        if t_attn is not None:
            t_attn[0].record(stream)
        vca.attention_fwd(ops, N, scale, O=O, ws=ws)
        if t_attn is not None:
            t_attn[1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ws.check()

    # ---- timed: whole step, device resident inputs (inputs exceed L2: no flush needed)
    ev_a = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        e0.record(stream)
        for i in range(args.steps):
            step(ev_a[i])
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ws.check()
    t_total = e0.elapsed_time(e1) / 1e3
    t_attn = statistics.mean(a.elapsed_time(b) for a, b in ev_a) / 1e3
    t_total = max_over_ranks(t_total, world)
    t_attn = max_over_ranks(t_attn, world)

    # ---- prep alone (cluster + quantise) and the reuse path (quantise only)
    _, _, perm = vca.cluster_permute(V, w.k, KMEANS_ITERS, ws=ws)
    reps = max(3, args.steps)
    p0, p1, q1 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    torch.cuda.synchronize()
    p0.record(stream)
    for _ in range(reps):
        _, _, perm = vca.cluster_permute(V, w.k, KMEANS_ITERS, ws=ws)
        vca.smooth_quantize(Q, K, V, perm, out=ops, ws=ws)
    p1.record(stream)
    for _ in range(reps):
        vca.smooth_quantize(Q, K, V, perm, out=ops, ws=ws)
    q1.record(stream)
    torch.cuda.synchronize()
    prep_ms = p0.elapsed_time(p1) / reps
    quant_ms = p1.elapsed_time(q1) / reps

    # ---- 4-bit V-Smooth prep (NVFP4 V residual) on the same inputs and permutation
    ws4 = vca.Workspace(vca.lib().vca_smooth_quantize_fp4_workspace_size(B, H, N), dev)
    ops4 = vca.smooth_quantize_fp4(Q, K, V, perm, ws=ws4)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    f0.record(stream)
    for _ in range(reps):
        vca.smooth_quantize_fp4(Q, K, V, perm, out=ops4, ws=ws4)
    f1.record(stream)
    torch.cuda.synchronize()
    ws4.check()
    fp4_ms = f0.elapsed_time(f1) / reps
    # ---- attention of the 4-bit variant (NVFP4 P and V residual in PV) on those operands
    O4 = vca.attention_fwd_fp4(ops4, N, scale, ws=ws4)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a0.record(stream)
    for _ in range(3):
        vca.attention_fwd_fp4(ops4, N, scale, O=O4, ws=ws4)
    a1.record(stream)
    torch.cuda.synchronize()
    ws4.check()
    fp4_attn_ms = a0.elapsed_time(a1) / 3
    del ops4, O4

    # ---- in-repo BF16 comparator on the same shapes
    bf16_ms = None
    if not args.no_bf16:
        for _ in range(2):
            vca.bf16_attention_fwd(Q, K, V, scale, O=O, ws=ws)
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        b0.record(stream)
        for _ in range(3):
            vca.bf16_attention_fwd(Q, K, V, scale, O=O, ws=ws)
        b1.record(stream)
        torch.cuda.synchronize()
        bf16_ms = b0.elapsed_time(b1) / 3
    ws.check()

    # ---- Skip Softmax (BLASST) variant: on the workload itself, and on a
    # block-sparse version of it (K scaled x12 on every other key block, identity
    # order) where whole query tiles drop the weak blocks
    skip = None
    if not args.no_skip:
        lam = args.skip_lambda
        nb = (N + 127) // 128
        pairs = B * H * ((nb + 1) // 2 * 2) * nb

        def time_skip(o, reps=3):
            cnt = torch.zeros(1, dtype=torch.int64, device=dev)
            vca.attention_fwd_skip(o, N, lam, O=O, skipped=cnt, ws=ws)
            torch.cuda.synchronize()
            cnt.zero_()
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            for _ in range(reps):
                vca.attention_fwd_skip(o, N, lam, O=O, skipped=cnt, ws=ws)
            s1.record(stream)
            torch.cuda.synchronize()
            return s0.elapsed_time(s1) / reps, cnt.item() / reps / pairs

        ms_w, frac_w = time_skip(ops)
        ident = torch.arange(N, dtype=torch.int32, device=dev).expand(B, H, N).contiguous()
        blk = torch.arange(N, device=dev) // 128
        K2 = K * torch.where(blk % 2 == 0, 12.0, 1.0).to(K.dtype)[None, None, :, None]
        ops2 = vca.alloc_quantized(B, H, N, dev)
        vca.smooth_quantize(Q, K2, V, ident, out=ops2, ws=ws)
        del K2
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        vca.attention_fwd(ops2, N, scale, O=O, ws=ws)
        d0.record(stream)
        for _ in range(3):
            vca.attention_fwd(ops2, N, scale, O=O, ws=ws)
        d1.record(stream)
        torch.cuda.synchronize()
        dense_ms = d0.elapsed_time(d1) / 3
        ms_s, frac_s = time_skip(ops2)
        del ops2
        skip = {"lambda": lam,
                "workload": {"attn_ms": round(ms_w, 3), "skipped_tile_frac": round(frac_w, 4)},
                "block_sparse_case": {"dense_attn_ms": round(dense_ms, 3), "skip_attn_ms": round(ms_s, 3),
                                      "skipped_tile_frac": round(frac_s, 4),
                                      "what": "workload Q, V; K x12 on even key blocks; identity order"}}
        ws.check()

    # ---- SAGE-style comparison recipe on the same inputs: prep and attention
    # time, and the fidelity of both recipes against the exact-softmax BF16
    # kernel's output (over the whole layer, on the GPU)
    sage = None
    if not args.no_sage:
        sops = vca.sage_quantize(Q, K, V, ws=ws)
        O_sg = vca.attention_fwd_sage(sops, N, scale, ws=ws)
        g0, g1, g2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        torch.cuda.synchronize()
        g0.record(stream)
        for _ in range(3):
            vca.sage_quantize(Q, K, V, ws=ws)
        g1.record(stream)
        for _ in range(3):
            vca.attention_fwd_sage(sops, N, scale, O=O_sg, ws=ws)
        g2.record(stream)
        torch.cuda.synchronize()
        O_vc = vca.attention_fwd(ops, N, scale, ws=ws)
        O_ex = vca.bf16_attention_fwd(Q, K, V, scale, ws=ws)
        torch.cuda.synchronize()

        def fid(a):
            a, b = a.float(), O_ex.float()
            return {"rel_l2": round((torch.linalg.vector_norm(a - b) / torch.linalg.vector_norm(b)).item(), 5),
                    "cosine": round((torch.sum(a * b) / (torch.linalg.vector_norm(a) *
                                                         torch.linalg.vector_norm(b))).item(), 6)}

        sage = {"prep_ms": round(g0.elapsed_time(g1) / 3, 3), "attn_ms": round(g1.elapsed_time(g2) / 3, 3),
                "fidelity_vs_bf16_exact_softmax": {"v_smooth": fid(O_vc), "sage": fid(O_sg)}}
        del sops, O_sg
        # the post's INT8 qk_dtype: Q/K as signed bytes, QK^T as kind::i8
        iops = vca.sage_quantize(Q, K, V, ws=ws, qk_dtype="int8")
        O_si = vca.attention_fwd_sage(iops, N, scale, ws=ws)
        torch.cuda.synchronize()
        g0.record(stream)
        for _ in range(3):
            vca.sage_quantize(Q, K, V, ws=ws, qk_dtype="int8")
        g1.record(stream)
        for _ in range(3):
            vca.attention_fwd_sage(iops, N, scale, O=O_si, ws=ws)
        g2.record(stream)
        torch.cuda.synchronize()
        sage["int8_qk"] = {"prep_ms": round(g0.elapsed_time(g1) / 3, 3), "attn_ms": round(g1.elapsed_time(g2) / 3, 3),
                           "fidelity_vs_bf16_exact_softmax": fid(O_si)}
        del iops, O_si, O_vc, O_ex
        ws.check()

    # ---- end to end through the C ABI with host buffers: vca_vc_attention_host
    # takes page-locked host Q, K, V and returns the host O, its copies
    # overlapped with the kernels (each step copies all inputs in and O out)
    e2e = None
    if not args.no_e2e:
        hQ, hK, hV = (t.cpu().pin_memory() for t in (Q, K, V))
        hO = torch.empty(O.shape, dtype=O.dtype).pin_memory()

        def e2e_step():
            vca.vc_attention_host(hQ, hK, hV, k=w.k, iters=KMEANS_ITERS, softmax_scale=scale, O=hO)

        e2e_step()
        n_e2e = max(2, min(args.steps, 5))
        barrier(world)
        torch.cuda.synchronize()
        x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        x0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        x1.record(stream)
        torch.cuda.synchronize()
        t_e2e = max_over_ranks(x0.elapsed_time(x1) / 1e3 / n_e2e, world)
        e2e = {"value": whole_job_value(world, w.flops, t_e2e), "unit": "TFLOP/s",
               "h2d_bytes_per_step": 3 * Q.numel() * 2, "d2h_bytes_per_step": O.numel() * 2,
               "ms_per_step": t_e2e * 1e3, "api": "vca_vc_attention_host (pinned host buffers)"}

    gemm_tflops, gemm_err = fp8_gemm_ceiling(dev)
    peaks, peak_kind = load_peaks()
    fp8_peak_sust = peaks["bf16_tflops_sustained"] * FP8_PER_BF16
    fp8_peak_burst = peaks["bf16_tflops"] * FP8_PER_BF16
    achieved = w.flops / t_attn / 1e12
    traffic = None
    tfile = os.path.join(ROOT, "profiles", "attn_fp8_traffic.json")
    if os.path.exists(tfile):
        with open(tfile) as f:
            tj = json.load(f)
        if tj.get("workload") == args.workload and tj.get("kernel_rev") == kernel_revision():
            traffic = tj.get("dram_bytes_per_launch")
    ms_step = t_total / args.steps * 1e3
    value = whole_job_value(world, w.flops, t_total / args.steps)
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3 (fp32 accumulate)",
        "data": "synthetic (seeded sinusoid video-DiT recipe; see workloads.py)",
        "config": {"workload": f"cfg{w.cid} {w.name}", "B": B, "H": H, "N": N, "d": d,
                   "grid": list(w.grid) if w.grid else None, "k": w.k, "kmeans_iters": KMEANS_ITERS,
                   "step": "cluster_permute + smooth_quantize + attention_fwd",
                   "l2": "inputs (2.3 GB bf16) exceed the 126 MB L2; no flush",
                   "parallelism": f"replicas x{world} (independent layers, no collective)"},
        "attn_ms": round(t_attn * 1e3, 3),
        "attn_tflops": round(achieved, 2),
        "prep_ms": round(prep_ms, 3),
        "quant_only_ms": round(quant_ms, 3),
        "bf16_attn_ms": round(bf16_ms, 3) if bf16_ms else None,
        "skip_softmax": skip,
        "sage_comparison": sage,
        "fp8_over_bf16": round(bf16_ms / (t_attn * 1e3), 3) if bf16_ms else None,
        # the kernel runs at the full SM clock (see clocks), so its peak is the
        # burst figure; the sustained one was measured at a lower clock under the
        # power cap and is kept only as a labelled extra
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": round(fp8_peak_burst, 1),
                     "unit": "TFLOP/s", "frac": round(achieved / fp8_peak_burst, 4), "traffic": traffic,
                     "peak_source": f"{peak_kind}: bf16 burst {peaks['bf16_tflops']} x "
                                    f"{FP8_PER_BF16} nominal FP8/BF16 (of measured)",
                     "frac_of_sustained": round(achieved / fp8_peak_sust, 4),
                     "frac_of_spec_4500": round(achieved / 4500.0, 4)},
        "e2e": e2e,
        "gpu_launches": launches_per_step * (args.steps),
        "clocks": clk.summary(),
    }
    clocks = line["clocks"]
    if clocks.get("sm_mhz"):
        # 148 SMs x 16,384 dense E4M3 FLOP per SM per clock at the clock seen under load
        cpk = 148 * 16384 * clocks["sm_mhz"] * 1e6 / 1e12
        line["clock_adjusted_peak"] = {"peak_tflops": round(cpk, 1), "frac": round(achieved / cpk, 4)}
    line["fp8_gemm_ceiling"] = {"tflops": round(gemm_tflops, 1) if gemm_tflops else None,
                                "frac": round(achieved / gemm_tflops, 4) if gemm_tflops else None,
                                "what": "torch._scaled_mm E4M3 8192^3, bf16 out", "error": gemm_err}
    # denoising-schedule reuse: grouping on the first quarter of a 50-step run,
    # every 4th step; quantisation every step (vca_schedule_regroup)
    S = 50
    n_regroup = sum(vca.schedule_regroup(st, S) for st in range(S))
    group_ms = max(prep_ms - quant_ms, 0.0)
    line["schedule"] = {"total_steps": S, "regroup_steps": n_regroup, "grouping_ms": round(group_ms, 3),
                        "quantise_ms": round(quant_ms, 3),
                        "grouping_frac_of_attention": round(n_regroup * group_ms / (S * t_attn * 1e3), 4),
                        "prep_frac_of_attention": round((n_regroup * group_ms + S * quant_ms) / (S * t_attn * 1e3), 4)}
    # share of block energy the V block mean carries (what V-Smooth removes before
    # quantising), in three token orders; perm is the product path's grouping
    line["block_mean_energy"] = dict(block_mean_energy(V, perm, w.grid), heads=B * H,
                                     cube="2x8x8 tokens of the (t, h, w) latent grid")
    fb = fp4_prep_algorithmic_bytes(w)
    line["fp4_prep"] = {"ms": round(fp4_ms, 3), "bound": "hbm", "algorithmic_bytes": fb,
                        "achieved": round(fb / (fp4_ms / 1e3) / 1e9, 1), "unit": "GB/s", "peak": peaks["hbm_gbs"],
                        "frac": round(fb / (fp4_ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
                        "launches": 2, "what": "vca_smooth_quantize_qkv_fp4: one streaming launch for Q/K "
                                              "(E4M3 as the 8-bit prep) and the first pass over V (means, head "
                                              "maxima), one launch coding the NVFP4 V residual"}
    line["fp4_attention"] = {"ms": round(fp4_attn_ms, 3), "tflops": round(w.flops / (fp4_attn_ms / 1e3) / 1e12, 1),
                             "what": "vca_attention_fwd_fp4: QK^T E4M3, PV kind::mxf4nvf4 with NVFP4 probabilities "
                                     "(exp2 on the MUFU pipe) and NVFP4 V residual"}
    pb = prep_algorithmic_bytes(w)
    line["prep_roofline"] = {"bound": "hbm", "algorithmic_bytes": pb,
                             "achieved": round(pb / (prep_ms / 1e3) / 1e9, 1), "unit": "GB/s",
                             "peak": peaks["hbm_gbs"], "frac": round(pb / (prep_ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4)}
    # the FP8 output of the workload, for the fidelity check on the host
    O_fp8 = vca.attention_fwd(ops, N, scale, ws=ws)
    torch.cuda.synchronize()
    return line, (Q, K, V, w, O_fp8)


def group_mean_energy(v: torch.Tensor, gid: torch.Tensor, ngroups: int) -> float:
    """Share of the energy of one head's value tokens v [N, d] that their group
    means carry, sum_g n_g |mean_g|^2 / sum_j |v_j|^2: what subtracting the
    means removes, since sum |v|^2 = sum_g n_g |mean_g|^2 + sum |v - mean|^2."""
    v = v.double()
    sums = torch.zeros(ngroups, v.shape[1], dtype=torch.float64, device=v.device).index_add_(0, gid, v)
    cnt = torch.bincount(gid, minlength=ngroups).double()
    keep = cnt > 0
    carried = ((sums[keep] ** 2).sum(1) / cnt[keep]).sum()
    return float(carried / (v * v).sum())


def cube_groups(grid, N: int, device, cube=(2, 8, 8)):
    """Static spatiotemporal cubes of the latent grid (tokens flattened t-major):
    2 x 8 x 8 = 128 tokens, ragged at the grid's edges.  Returns (gid, ngroups)."""
    T, Hg, Wg = grid
    n = torch.arange(N, device=device)
    t, rem = n // (Hg * Wg), n % (Hg * Wg)
    h, w = rem // Wg, rem % Wg
    ct, ch, cw = cube
    nh, nw = -(-Hg // ch), -(-Wg // cw)
    gid = ((t // ct) * nh + h // ch) * nw + w // cw
    return gid, -(-T // ct) * nh * nw


def block_mean_energy(V: torch.Tensor, perm: torch.Tensor, grid, block: int = 128) -> dict:
    """Energy share of the 128-token block means of V, averaged over heads, with
    the tokens in sequence order, in static cubes of the latent grid, and in
    the k-means order of perm ("Nunchux AI Introduces VC-Attention ...",
    abstract: 8 % / 12 % / 36 % over 100 Wan2.2 heads)."""
    N = V.shape[-2]
    Vh = V.reshape(-1, N, V.shape[-1])
    P = perm.reshape(-1, N)
    nb = -(-N // block)
    seq = torch.arange(N, device=V.device) // block
    cube = cube_groups(grid, N, V.device) if grid else None
    out = {"sequence": [], "static_cube": [], "sorted": []}
    for h in range(Vh.shape[0]):
        out["sequence"].append(group_mean_energy(Vh[h], seq, nb))
        if cube is not None:
            out["static_cube"].append(group_mean_energy(Vh[h], *cube))
        srt = torch.empty(N, dtype=torch.long, device=V.device)
        srt[P[h].long()] = seq          # token perm[i] sits at sorted position i
        out["sorted"].append(group_mean_energy(Vh[h], srt, nb))
    return {k: round(statistics.mean(x), 4) for k, x in out.items() if x}


def fp8_gemm_ceiling(dev, n=8192, reps=10):
    """Dense E4M3 GEMM throughput of the library path (torch._scaled_mm, a
    cuBLASLt call) on this GPU in this run: a practical FP8 ceiling the
    attention kernel is compared against (measurement only)."""
    try:
        a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()
        one = torch.ones((), device=dev, dtype=torch.float32)
        for _ in range(3):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        e1.record()
        torch.cuda.synchronize()
        return 2.0 * n ** 3 / (e0.elapsed_time(e1) / reps / 1e3) / 1e12, None
    except Exception as ex:  # reported, not fatal: the ceiling is context only
        return None, f"{type(ex).__name__}: {ex}"[:200]


def prep_algorithmic_bytes(w) -> float:
    """Bytes the prep must move at minimum: Q, K, V read once and Qq, Kq, VrT
    written once (2 + 2 + 2 read, 1 + 1 + 1 written per element), V read once
    more per k-means pass, plus the block means (2 bytes per channel per block)."""
    elems = w.B * w.H * w.N * w.d
    nb = (w.N + 127) // 128
    return 9.0 * elems + KMEANS_ITERS * 2.0 * elems + 2.0 * w.B * w.H * nb * w.d


def fp4_prep_algorithmic_bytes(w) -> float:
    """Bytes the 4-bit prep must move once: Q, K, V and the permutation in;
    Qq, Kq (1 B/element), the NVFP4 residual (0.5 B/element + one scale byte per
    16), scales and block means out."""
    BH, N, d = w.B * w.H, w.N, w.d
    nb = (N + 127) // 128
    Np = nb * 128
    return float(BH * (3 * N * d * 2 + N * 4 + 2 * Np * d + Np * d // 2 + Np * d // 16
                       + 2 * nb * 4 + nb * d * 2 + 4))


def kernel_revision() -> str:
    import hashlib
    p = os.path.join(ROOT, "bit_attention_video_02_b200", "csrc", "vca_attn_fp8.cu")
    with open(p, "rb") as f:
        return hashlib.sha1(f.read()).hexdigest()[:12]


# ------------------------------------------------------------------ oracle timing
def _bits(t):
    return W.bf16_bits(t)


def run_oracle_baseline(w, Q, K, V, rows=8192):
    """Times the oracle as it stands on a bounded sample of the workload: head
    0's full prep and `rows` of its query rows, extrapolated linearly to a full
    step.  Returns (TFLOP/s, threads used, sample description, step seconds)."""
    import numpy as np
    import oracle
    scale = 1.0 / math.sqrt(w.d)
    Qb, Kb, Vb = (_bits(t[0, 0]) for t in (Q, K, V))
    t0 = time.perf_counter()
    ops = oracle.prep_head(Qb, Kb, Vb, w.k, KMEANS_ITERS)
    t1 = time.perf_counter()
    rng = np.random.default_rng(7)
    rsel = np.sort(rng.choice(w.N, size=min(rows, w.N), replace=False)).astype(np.int32)
    oracle.attention_head(ops, w.N, scale, rows=rsel)
    t2 = time.perf_counter()
    per_head = (t1 - t0) + (t2 - t1) * (w.N / len(rsel))
    step_s = per_head * w.B * w.H
    desc = (f"head 0 of cfg{w.cid}: full prep (k-means x{KMEANS_ITERS}, permutation, quantisation) "
            f"{t1 - t0:.2f}s + attention for {len(rsel)} of {w.N} query rows {t2 - t1:.2f}s; "
            f"extrapolated linearly to {w.B * w.H} heads x {w.N} rows")
    return w.flops / step_s / 1e12, oracle.num_threads(), desc, step_s


def fidelity_vs_exact(w, Q, K, V, O, nrows=256):
    """Cosine, PSNR and relative L2 of the FP8 path's output against exact fp64
    softmax attention (the oracle's) on seeded sampled rows of the first and
    last head, outside the timed region."""
    import numpy as np
    import oracle
    scale = 1.0 / math.sqrt(w.d)
    out = {}
    for h in sorted({0, w.H - 1}):
        rng = np.random.default_rng(500 + h)
        rows = np.sort(rng.choice(w.N, size=min(nrows, w.N), replace=False)).astype(np.int32)
        ex = oracle.exact_attention_head(_bits(Q[0, h]), _bits(K[0, h]), _bits(V[0, h]), scale, rows=rows)
        g = O[0, h].float().cpu().numpy().astype(np.float64)[rows]
        cos = float((g * ex).sum() / np.sqrt((g * g).sum() * (ex * ex).sum()))
        mse = float(np.mean((g - ex) ** 2))
        out[f"head{h}"] = {"rows": int(len(rows)), "cosine": round(cos, 6),
                           "psnr_db": round(10 * math.log10(float(np.abs(ex).max()) ** 2 / mse), 2),
                           "rel_l2": round(float(np.linalg.norm(g - ex) / np.linalg.norm(ex)), 6)}
    return out


# ------------------------------------------------------------------ reference arm
def run_reference(args, world, rank):
    if rank != 0:
        return None
    w = W.shrink(W.WORKLOADS[args.workload], H=args.heads)
    Q, K, V = W.make_qkv(w, "cuda" if torch.cuda.is_available() else "cpu")
    vals = []
    for i in range(args.warmup + args.steps):
        v, cores, desc, step_s = run_oracle_baseline(w, Q, K, V, rows=2048)
        if i >= args.warmup:
            vals.append((v, step_s))
    value = statistics.mean(v for v, _ in vals)
    step_ms = statistics.mean(s for _, s in vals) * 1e3
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
        "data": "synthetic (seeded sinusoid video-DiT recipe)",
        "config": {"workload": f"cfg{w.cid} {w.name}", "B": w.B, "H": w.H, "N": w.N, "d": w.d, "k": w.k},
        "cpu_baseline": {"kind": "oracle", "cores": cores, "sample": desc, "value": value},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", type=int, default=3)
    ap.add_argument("--heads", type=int, default=None, help="run the workload with fewer heads (profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-bf16", action="store_true")
    ap.add_argument("--no-skip", action="store_true")
    ap.add_argument("--no-sage", action="store_true")
    ap.add_argument("--skip-lambda", type=float, default=2.0 ** -6)
    args = ap.parse_args()
    world, rank, local = dist_setup(args)
    if args.gpus != world and rank == 0:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; reporting {world} rank(s)", file=sys.stderr)
    try:
        if args.impl == "reference":
            line = run_reference(args, world, rank)
        else:
            line, (Q, K, V, w, O_fp8) = run_ours(args, world, rank, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                v, cores, desc, _ = run_oracle_baseline(w, Q, K, V)
                line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                        "sample": desc}
                line["fidelity_vs_exact_fp64"] = fidelity_vs_exact(w, Q, K, V, O_fp8)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
