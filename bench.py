"""Benchmark: MXFP4 attention with UOS + PNQ (MXAttention) on B200.

One step = the whole hot path on one batch: Q/K and V^T quantize/pack
(mxattn_prepare) + the fused attention kernel (mxattn_attend), i.e.
mxattn_forward, on the video-DiT self-attention workload B=1, H=40,
N=32760 (21 frames x 30 x 52 tokens), d=128, kv_tile=128, UOS + PNQ, with
synthetic seeded inputs already resident in HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Under torchrun (N > 1) every rank runs its own batch (seed = rank): weak
scaling with no data-path collective; the timed region is bracketed by a
barrier and synchronize, and the slowest rank's time counts.  Rank 0 prints
one JSON line.  `--impl reference` times the CPU oracle (fp64, plain loops) on
a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mxfp4_microscaled_quantization_b200 import workloads as wl  # noqa: E402

METRIC = "MXFP4 attention TFLOPS (4BHN²d) and % of B200 FP4 peak at N=32760,d=128"
UNIT = "TFLOP/s"
WORKLOAD = wl.WORKLOADS["video_dit"]
FP4_PER_BF16 = 4.0  # nominal dense FP4 : BF16 tensor ratio (9 : 2.25 PFLOP/s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ATTN_PROFILE = os.path.join(ROOT, "profiles", "attention_video_dit.md")
# the attention kernel's source: attention.cu and the device functions it inlines from ptx.cuh
ATTN_SOURCES = tuple(os.path.join(ROOT, "mxfp4_microscaled_quantization_b200", "csrc", f)
                     for f in ("attention.cu", "ptx.cuh"))


PARALLELISM = {
    "heads": "heads sharded over {world} ranks (one problem, no exchange)",
    "sequence": "tokens sharded over {world} ranks (one problem; all-to-all to heads and back, NCCL)",
    "replicas": "{world} independent replicas (one batch per rank)"}


def config_dict(w=WORKLOAD, world=1, shard="replicas"):
    """The workload the line is quoted on; both arms (ours and the reference) print the same dict."""
    gb = 3 * w.B * w.H * w.N * w.d * 2 / 1e9
    return {"workload": f"{w.name}: B={w.B} H={w.H} N={w.N} ({w.frames}x{w.rows}x{w.cols} tokens) d={w.d} "
                        f"kv_tile={w.kv_tile}, UOS + PNQ, smooth low-rank + noise bf16 inputs",
            "B": w.B, "H": w.H, "N": w.N, "d": w.d, "kv_tile": w.kv_tile, "rule": "uos", "pnq": True,
            "step": "mxattn_prepare (Q/K + V^T quantize) + mxattn_attend (fused attention)",
            "l2": f"inputs larger than L2: {gb:.1f} GB of bf16 Q/K/V per step (no flush)",
            "parallelism": PARALLELISM[shard].format(world=world)}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def profiled_traffic():
    """Per-launch DRAM bytes of the attention kernel from the committed ncu
    summary, if it was taken on the current kernel source (attention.cu then
    ptx.cuh, hashed together); else None."""
    try:
        with open(ATTN_PROFILE) as f:
            text = f.read()
        h = hashlib.sha256()
        for path in ATTN_SOURCES:
            with open(path, "rb") as f:
                h.update(f.read())
        digest = h.hexdigest()[:16]
    except OSError:
        return None
    src = [ln for ln in text.splitlines() if ln.startswith("source_sha256_16:")]
    tr = [ln for ln in text.splitlines() if ln.startswith("dram_bytes_per_full_launch:")]
    if not src or not tr or src[0].split(":", 1)[1].split()[0] != digest:
        return None
    return float(tr[0].split(":", 1)[1].strip())


class ClockSampler:
    """SM clock, its maximum and the clock-event (throttle) reasons of this
    rank's GPU during the timed region: read every 10 ms by NVML in a
    background thread (read only; the device is matched by PCI bus id), or
    polled with nvidia-smi every 100 ms when NVML is unavailable."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.thread = None
        self.samples = []  # (sm MHz, max sm MHz, reason names)
        self.path = os.path.join("/tmp", f"mxattn_clocks_{os.getpid()}.csv")

    def _nvml_handle(self):
        import pynvml
        import torch

        pynvml.nvmlInit()
        try:
            pr = torch.cuda.get_device_properties(self.gpu)
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(
                f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0".encode())
        except Exception:  # noqa: BLE001 - older properties or bus-id formats: fall back to the index
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def __enter__(self):
        import threading

        try:
            nv, h = self._nvml_handle()
            smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            bits = [(name, getattr(nv, attr)) for name, attr in self.REASONS]
            self.stop = threading.Event()

            def run():
                while not self.stop.is_set():
                    try:
                        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                        mask = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    except Exception:  # noqa: BLE001 - a failed read is skipped, not fatal
                        sm, mask = None, 0
                    if sm is not None:
                        self.samples.append((float(sm), float(smax), [n for n, bit in bits if mask & bit]))
                    self.stop.wait(0.01)

            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            return self
        except Exception:  # noqa: BLE001 - no NVML: poll nvidia-smi instead
            self.thread = None
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "100"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        source = "nvml"
        rows = list(self.samples)
        if self.thread is None:
            if self.proc is None:
                return None
            source = "nvidia-smi"
            names = [n for n, _ in self.REASONS]
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9 and parts[1].replace(".", "").isdigit() and parts[2].replace(".", "").isdigit():
                        rows.append((float(parts[1]), float(parts[2]),
                                     [names[i] for i in range(4) if parts[5 + i].lower().startswith("active")]))
            try:
                os.remove(self.path)
            except OSError:
                pass
        if not rows:
            return None
        smax = max(r[1] for r in rows)
        loaded = [r[0] for r in rows if r[0] >= 0.3 * smax] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax,
                "reasons": sorted({n for r in rows for n in r[2]}), "samples": len(rows), "source": source}


def oracle_sample(Q, K, V, w, rows, nthreads=0):
    """The CPU oracle on `rows` query rows of head 0 (plus its K/V quantization)."""
    import oracle

    t0 = time.perf_counter()
    oracle.attention(Q[:, :1], K[:, :1], V[:, :1], w.kv_tile, rule="uos", pnq=True, rows=rows, nthreads=nthreads)
    return time.perf_counter() - t0


def sized_oracle_rows(Q, K, V, w, budget_s, threads):
    """Grow a seeded row sample until one oracle call takes about `budget_s` (or all rows)."""
    n = 2 * threads
    for _ in range(4):
        rows = np.linspace(0, w.N - 1, n).astype(np.int64)
        t = oracle_sample(Q, K, V, w, rows, threads)
        if t >= 0.5 * budget_s or n >= w.N:
            return rows, t
        n = int(min(w.N, max(n + 1, n * budget_s / max(t, 1e-3))))
    return rows, t


def cpu_baseline(Q, K, V, w, budget_s=15.0):
    """Time the oracle as it stands on a bounded sample: query rows of head 0 sized to
    about `budget_s` of CPU work, converted to the same unit (4*N*d flops per row)."""
    import oracle

    threads = oracle.max_threads()
    rows, t = sized_oracle_rows(Q, K, V, w, budget_s, threads)
    flops = 4.0 * len(rows) * w.N * w.d
    return {"value": flops / t / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{len(rows)} evenly spaced query rows of head 0 of {w.name} (that head's K/V quantization "
                      f"included), {t:.1f} s on {threads} OpenMP threads"}


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle on the host cores (rank 0 only)."""
    if rank != 0:
        return 0
    import oracle

    w = WORKLOAD
    Q, K, V = wl.make_qkv(w, seed=0)
    threads = oracle.max_threads()
    # size one step to a bounded sample so warmup + steps stay within a few minutes
    step_budget_s = args.ref_step_budget or max(2.0, 120.0 / (args.warmup + args.steps))
    rows0, _ = sized_oracle_rows(Q, K, V, w, step_budget_s, threads)
    n = len(rows0)
    times = []
    for i in range(args.warmup + args.steps):
        rng = np.random.default_rng(i)
        rows = np.sort(rng.choice(w.N, n, replace=False))
        t = oracle_sample(Q, K, V, w, rows, threads)
        if i >= args.warmup:
            times.append(t)
    t_step = sum(times) / len(times)
    value = 4.0 * n * w.N * w.d / t_step / 1e12
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_step * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": config_dict(w, world, args.shard),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"per step {n} seeded query rows of head 0 (with that head's K/V "
                                       f"quantization) on {threads} OpenMP threads"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


QUANT_SWEEP_LOG2 = (20, 24, 27, 30)


def quantize_sweep(torch, mx, peaks, peak_kind, iters=10):
    """The standalone quantize kernel (mxattn_quantize) on the config-5 sweep:
    0.5 * StudentT(3) bf16 [2^k / 4096, 4096] for k in 20, 24, 27, 30 (the first
    2^k elements of one seeded 2^30-element draw), OCP and UOS.  Every launch is
    timed on its own with CUDA events, after a 512 MB write that flushes L2
    (the smaller sizes fit in L2); GB/s counts 2.53125 bytes per element."""
    big = max(QUANT_SWEEP_LOG2)
    x = wl.student_t_matrix(1 << big, 4096, seed=0)
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    del x
    codes = torch.empty((xd.shape[0], 2048), dtype=torch.uint8, device="cuda")
    scales = torch.empty((xd.shape[0], 128), dtype=torch.uint8, device="cuda")
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    points = []
    for k in QUANT_SWEEP_LOG2:
        rows = (1 << k) // 4096
        xs, cs, ss = xd[:rows], codes[:rows], scales[:rows]
        for rule in ("ocp", "uos"):
            for _ in range(3):
                mx.mxattn_quantize(xs, rule, cs, ss)
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
            for e0, e1 in ev:
                flush.fill_(k & 0xFF)
                e0.record()
                mx.mxattn_quantize(xs, rule, cs, ss)
                e1.record()
            torch.cuda.synchronize()
            t = sum(e0.elapsed_time(e1) for e0, e1 in ev) / iters / 1e3
            gbs = (1 << k) * 2.53125 / t / 1e9
            points.append({"log2_elements": k, "rule": rule, "us_per_launch": t * 1e6, "achieved_gbs": gbs,
                           "frac": gbs / peaks["hbm_gbs"], "frac_of_8tbs_spec": gbs / 8000.0})
    del xd, codes, scales, flush
    torch.cuda.empty_cache()
    return {"points": points, "bytes_per_element": 2.53125, "peak_gbs": peaks["hbm_gbs"], "peak_kind": peak_kind,
            "shape": "[2^k / 4096, 4096] bf16, 0.5 * StudentT(3), seed 0", "l2": "512 MB written before every launch"}


def long_video_leg(torch, mx, steps=3):
    """The long video-DiT workload (B=1, H=24, N=75600, d=128, kv_tile=128, UOS +
    PNQ): the same step (prepare + attend), attention and step times from CUDA
    events, inputs generated by the same recipe (seed 0)."""
    w = wl.WORKLOADS["long_video_dit"]
    Q, K, V = wl.make_qkv(w, seed=0)
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)  # noqa: E731
    q, k, v = to_dev(Q), to_dev(K), to_dev(V)
    del Q, K, V
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    ws = mx.new_workspace(w.B, w.H, w.N, w.d)
    for _ in range(2):
        mx.mxattn_prepare(q, k, v, "uos", ws)
        mx.mxattn_attend(ws, w.B, w.H, w.N, w.d, w.kv_tile, True, "uos", 0.0, out)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for e in ev:
        e[0].record()
        mx.mxattn_prepare(q, k, v, "uos", ws)
        e[1].record()
        mx.mxattn_attend(ws, w.B, w.H, w.N, w.d, w.kv_tile, True, "uos", 0.0, out)
        e[2].record()
    torch.cuda.synchronize()
    if mx.mxattn_workspace_status(ws) != 0:
        raise RuntimeError("attention kernel reported a timeout (long video-DiT)")
    attn = sum(e[1].elapsed_time(e[2]) for e in ev) / steps
    step = sum(e[0].elapsed_time(e[2]) for e in ev) / steps
    del q, k, v, out, ws
    torch.cuda.empty_cache()
    return {"workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d={w.d} kv_tile={w.kv_tile}, UOS + PNQ",
            "attn_ms": attn, "step_ms": step, "attn_tflops": w.flops / (attn / 1e3) / 1e12,
            "step_tflops": w.flops / (step / 1e3) / 1e12, "steps": steps}


# MUFU exponentials per S element in mxattn_fwd_kernel with MXFP4 and PNQ: 9 of
# every 16 pairs on the MUFU (ex2.approx), 7 on the FMA pipe; plus the rescale
# factor, one per row and 128-column key tile.  Block exponents take no exponential.
MUFU_EX2_PER_ELEMENT = 9.0 / 16 + 1.0 / 128


def mufu_roofline(w, attn_ms, clocks, sms=148, ex2_per_clk_per_sm=16):
    """The unit that actually bounds the attention kernel: ex2.approx issue on the
    MUFU (16 per clock per SM, measured), at the SM clock seen during the run."""
    mhz = (clocks or {}).get("sm_mhz") or 1965.0
    elements = float(w.B * w.H) * w.N * w.N
    achieved = elements * MUFU_EX2_PER_ELEMENT / (attn_ms / 1e3)
    peak = sms * ex2_per_clk_per_sm * mhz * 1e6
    return {"bound": "mufu", "unit": "ex2/s", "achieved": achieved, "peak": peak, "frac": achieved / peak,
            "ex2_per_element": MUFU_EX2_PER_ELEMENT, "sm_mhz": mhz,
            "s_elements_per_clk_per_sm": elements / (attn_ms / 1e3) / (sms * mhz * 1e6)}


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise maximum of per-rank timings (the slowest rank counts); identity without a process group."""
    import torch

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def rank_seed(rank: int) -> int:
    """Each rank draws its own batch (weak scaling: one independent problem per GPU)."""
    return rank


def head_range(H: int, rank: int, world: int):
    """Heads [lo, hi) of one problem that rank `rank` computes when the heads are
    sharded over `world` ranks: contiguous, sizes differing by at most one."""
    base, extra = divmod(H, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def selected_workload(args):
    w = wl.WORKLOADS[args.workload]
    if args.heads:
        import dataclasses

        w = dataclasses.replace(w, H=args.heads)
    return w


QMAX_STUDY = (6.0, 6.5, 7.0, 7.25, 7.5, 7.75, 8.0)


def qmax_study(args):
    """Scale-boundary study: O error against exact attention (fp64, unquantized
    bf16 inputs) for boundaries Qmax in [6, 8] (8 = OCP), PNQ on and off, on
    four input distributions.  The error is the relative Frobenius norm over a
    seeded sample of query rows per head (all heads)."""
    import torch

    from mxfp4_microscaled_quantization_b200 import mxattn as mx

    torch.cuda.set_device(0)
    vid = wl.WORKLOADS["video_dit"]
    cases = [
        ("gaussian", wl.gaussian_qkv(1, 8, 4096, 128, seed=0)),
        ("student_t3", wl.student_t_qkv(1, 8, 4096, 128, seed=0)),
        ("outlier", wl.outlier_qkv(1, 8, 4096, 128, seed=0)),
        ("video_dit_4heads", wl.video_dit_qkv(1, 4, vid.frames, vid.rows, vid.cols, vid.d, seed=0)),
    ]
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)  # noqa: E731
    out_rows = []
    for name, (Q, K, V) in cases:
        q, k, v = to_dev(Q), to_dev(K), to_dev(V)
        B, H, N, d = q.shape
        rows = torch.from_numpy(np.sort(np.random.default_rng(7).choice(N, min(N, 512), replace=False))).cuda()
        qd, kd, vd = q.double(), k.double(), v.double()
        s = torch.einsum("bhrd,bhnd->bhrn", qd[:, :, rows], kd) / math.sqrt(d)
        exact = torch.einsum("bhrn,bhnd->bhrd", torch.softmax(s, dim=-1), vd)
        ws = mx.new_workspace(B, H, N, d)
        for qmax in QMAX_STUDY:
            for pnq in (True, False):
                o = mx.mxattn_forward(q, k, v, 128, pnq, qmax, workspace=ws)
                torch.cuda.synchronize()
                if mx.mxattn_workspace_status(ws) != 0:
                    raise RuntimeError("attention kernel reported a timeout")
                got = o[:, :, rows].double()
                rel = float((got - exact).norm() / exact.norm())
                out_rows.append({"inputs": name, "qmax": qmax, "pnq": pnq, "rel_err": rel})
        wsn = mx.new_nvfp4_workspace(B, H, N, d)
        for pnq in (True, False):
            o = mx.mxattn_nvfp4_forward(q, k, v, 128, pnq, workspace=wsn)
            torch.cuda.synchronize()
            if mx.mxattn_workspace_status(wsn) != 0:
                raise RuntimeError("NVFP4 attention kernel reported a timeout")
            rel = float((o[:, :, rows].double() - exact).norm() / exact.norm())
            out_rows.append({"inputs": name, "qmax": "nvfp4", "pnq": pnq, "rel_err": rel})
    line = {"study": "scale boundary Qmax (and the NVFP4 variant) vs O error against exact fp64 attention",
            "shapes": "gaussian / student_t3 / outlier: B=1 H=8 N=4096 d=128; video_dit_4heads: B=1 H=4 "
                      "N=32760 d=128; kv_tile 128; 512 seeded query rows per head",
            "rows": out_rows}
    print(json.dumps(line), flush=True)
    return 0


def run_gpu(args, rank, world, local_rank):
    import torch

    from mxfp4_microscaled_quantization_b200 import mxattn as mx

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    w_full = selected_workload(args)
    peaks, peak_kind = load_peaks()
    if args.shard == "heads":
        # One problem, its heads split over the ranks (no exchange: heads are independent).
        import dataclasses

        lo, hi = head_range(w_full.H, rank, world)
        if hi <= lo:
            raise ValueError(f"{w_full.H} heads cannot be sharded over {world} ranks")
        Q, K, V = (np.ascontiguousarray(a[:, lo:hi]) for a in wl.make_qkv(w_full, seed=0))
        w = dataclasses.replace(w_full, H=hi - lo)
    elif args.shard == "sequence":
        # One problem, its tokens split over the ranks (sequence parallelism): an
        # all-to-all regroups Q, K, V by head before the attention and O by token after.
        import dataclasses

        if w_full.H % world or w_full.N % world:
            raise ValueError(f"H={w_full.H} and N={w_full.N} must divide by the {world} ranks")
        n = w_full.N // world
        Q, K, V = (np.ascontiguousarray(a[:, :, rank * n:(rank + 1) * n]) for a in wl.make_qkv(w_full, seed=0))
        w = dataclasses.replace(w_full, H=w_full.H // world)  # what the kernels see after the exchange
    else:
        w = w_full
        Q, K, V = wl.make_qkv(w, seed=rank_seed(rank))
    seq = args.shard == "sequence"
    B, H, N, d = w.B, w.H, w.N, w.d
    # whole-job work per step: every rank's problem (replicas) or the one sharded problem
    job_flops = w_full.flops if args.shard in ("heads", "sequence") else world * w.flops
    base = None
    if rank == 0 and not args.quick and not seq:
        base = cpu_baseline(Q, K, V, w, budget_s=args.cpu_budget)
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)  # noqa: E731
    q, k, v = to_dev(Q), to_dev(K), to_dev(V)
    out = torch.empty((B, H, N, d), dtype=torch.float32, device="cuda")
    nv_step = args.format == "nvfp4"
    ws = mx.new_nvfp4_workspace(B, H, N, d) if nv_step else mx.new_workspace(B, H, N, d)
    stream = torch.cuda.current_stream()

    if seq:
        from mxfp4_microscaled_quantization_b200 import ulysses

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        qs, ks, vs = (ulysses.seq_to_head(t) for t in (q, k, v)) if seq else (q, k, v)
        if nv_step:
            mx.mxattn_nvfp4_prepare(qs, ks, vs, ws)
        else:
            mx.mxattn_prepare(qs, ks, vs, "uos", ws)
        if ev is not None:
            ev[1].record(stream)
        if nv_step:
            mx.mxattn_nvfp4_attend(ws, B, H, N, d, w.kv_tile, True, 0.0, out)
        else:
            mx.mxattn_attend(ws, B, H, N, d, w.kv_tile, True, "uos", 0.0, out)
        if ev is not None:
            ev[2].record(stream)
        if seq:
            ulysses.head_to_seq(out)  # this rank's tokens of O
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if mx.mxattn_workspace_status(ws) != 0:
        raise RuntimeError("attention kernel reported a timeout during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        for i in range(args.steps):
            step(evs[i])
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    total_ms = evs[0][0].elapsed_time(evs[-1][3])
    attn_ms = [e[1].elapsed_time(e[2]) for e in evs]
    prep_ms = [e[0].elapsed_time(e[1]) for e in evs]
    if mx.mxattn_workspace_status(ws) != 0:
        raise RuntimeError("attention kernel reported a timeout")
    total_ms, attn_avg_ms = max_over_ranks([total_ms, sum(attn_ms) / len(attn_ms)], dist, "cuda")
    ms_per_step = total_ms / args.steps
    value = job_flops / (ms_per_step / 1e3) / 1e12

    e2e_ms = None
    if not args.quick and not seq:
        e2e_ms = measure_e2e(torch, mx, Q, K, V, w, (q, k, v, out, ws), stream, args, dist)

    quant = None
    if rank == 0 and not args.quick and not args.no_quantize_sweep and not seq:
        quant = quantize_sweep(torch, mx, peaks, peak_kind)
    long_leg = None
    if rank == 0 and not args.quick and not seq and args.workload == "video_dit" and not args.heads:
        long_leg = long_video_leg(torch, mx)

    # The same attention step under every scale rule x PNQ combination: OCP
    # without PNQ is the comparator the method is measured against; the two mixed
    # ones separate the cost of UOS from that of PNQ.
    overhead = None
    if not args.quick and not seq:
        def attend_ms(rule, pnq):
            mx.mxattn_prepare(q, k, v, rule, ws)
            for _ in range(2):
                mx.mxattn_attend(ws, B, H, N, d, w.kv_tile, pnq, rule, 0.0, out)
            torch.cuda.synchronize()
            o0, o1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            o0.record(stream)
            for _ in range(5):
                mx.mxattn_attend(ws, B, H, N, d, w.kv_tile, pnq, rule, 0.0, out)
            o1.record(stream)
            torch.cuda.synchronize()
            return max_over_ranks([o0.elapsed_time(o1) / 5], dist, "cuda")[0]

        t = {(rule, pnq): attend_ms(rule, pnq) for rule in ("ocp", "uos") for pnq in (False, True)}
        ocp_ms = t[("ocp", False)]
        overhead = {"ocp_no_pnq_attn_ms": ocp_ms, "ocp_pnq_attn_ms": t[("ocp", True)],
                    "uos_no_pnq_attn_ms": t[("uos", False)], "uos_pnq_attn_ms": attn_avg_ms,
                    "uos_pnq_attn_ms_same_leg": t[("uos", True)],
                    "uos_pnq_over_ocp": attn_avg_ms / ocp_ms - 1.0,
                    "uos_over_ocp_with_pnq": t[("uos", True)] / t[("ocp", True)] - 1.0,
                    "uos_over_ocp_without_pnq": t[("uos", False)] / ocp_ms - 1.0,
                    "pnq_over_no_pnq_with_uos": t[("uos", True)] / t[("uos", False)] - 1.0}

    # The NVFP4 comparison variant (16-element blocks, E4M3 scales, per-head fp32
    # scales) on the same workload and kernel structure, PNQ on.
    nvfp4 = None
    if not args.quick and not seq:
        wsn = mx.new_nvfp4_workspace(B, H, N, d)
        mx.mxattn_nvfp4_prepare(q, k, v, wsn)
        mx.mxattn_nvfp4_attend(wsn, B, H, N, d, w.kv_tile, True, 0.0, out)
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(5)]
        for e in ev:
            e[0].record(stream)
            mx.mxattn_nvfp4_prepare(q, k, v, wsn)
            e[1].record(stream)
            mx.mxattn_nvfp4_attend(wsn, B, H, N, d, w.kv_tile, True, 0.0, out)
            e[2].record(stream)
        torch.cuda.synchronize()
        if mx.mxattn_workspace_status(wsn) != 0:
            raise RuntimeError("NVFP4 attention kernel reported a timeout")
        nv_prep, nv_attn = max_over_ranks([sum(e[0].elapsed_time(e[1]) for e in ev) / len(ev),
                                           sum(e[1].elapsed_time(e[2]) for e in ev) / len(ev)], dist, "cuda")
        nvfp4 = {"prepare_ms": nv_prep, "attn_ms": nv_attn, "attn_tflops": w.flops / (nv_attn / 1e3) / 1e12,
                 "step_tflops": w.flops / ((nv_prep + nv_attn) / 1e3) / 1e12,
                 "uos_pnq_attn_speedup": nv_attn / attn_avg_ms, "kernel": f"mxattn_fwd_kernel<{w.d},{w.kv_tile},1,nvfp4>"}
        del wsn

    # The ceiling of the attention kernel's own tensor-core instruction on this GPU:
    # its M = N = 128, K = 64 block-scaled FP4 MMA issued back to back from shared
    # memory, one CTA per SM (not part of the timed step).  Its wall-clock rate
    # depends on the clock the power cap allows during the burst; the SM cycle
    # count of each CTA gives the rate per clock, which is then taken at the clock
    # sampled while the attention kernel ran.
    mma_loop = None
    if rank == 0:
        sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
        iters = 20000
        cycles = torch.zeros(sms, dtype=torch.int64, device="cuda")
        mx.mxattn_mxf4_mma_loop(sms, iters, cycles=cycles, stream=stream)
        torch.cuda.synchronize()
        l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        l0.record(stream)
        st = mx.mxattn_mxf4_mma_loop(sms, iters, cycles=cycles, stream=stream)
        l1.record(stream)
        torch.cuda.synchronize()
        if int(st.item()) != 0:
            raise RuntimeError("tensor-core loop reported a timeout")
        loop_ms = l0.elapsed_time(l1)
        per_clk = float(np.median(iters * mx.MXF4_LOOP_FLOP_PER_ITER / cycles.cpu().numpy().astype(np.float64)))
        mma_loop = {"tflops_wall": sms * iters * mx.MXF4_LOOP_FLOP_PER_ITER / (loop_ms / 1e3) / 1e12, "ms": loop_ms,
                    "flop_per_clk_per_sm": per_clk, "ctas": sms, "iters": iters,
                    "what": "tcgen05.mma kind::mxf4 block32, M=N=128, K=64, back to back from shared memory"}

    if rank == 0:
        attn_tflops = w.flops / (attn_avg_ms / 1e3) / 1e12
        # Each launch is timed on its own, inside a sub-second region, and holds the maximum
        # SM clock (see `clocks`): the burst bf16 figure is the matching denominator.
        peak = peaks["bf16_tflops"] * FP4_PER_BF16
        clocks = clk.summary()
        mxf4_frac = None
        if mma_loop is not None:
            mhz = (clocks or {}).get("sm_mhz") or 1965.0
            mma_loop["sm_mhz"] = mhz
            mma_loop["tflops_at_sm_mhz"] = mma_loop["ctas"] * mma_loop["flop_per_clk_per_sm"] * mhz * 1e6 / 1e12
            mxf4_frac = attn_tflops / mma_loop["tflops_at_sm_mhz"]
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "strong" if args.shard in ("heads", "sequence") else "weak",
            "vs_baseline": None, "data": "synthetic",
            "dtype": ("nvfp4 (e2m1 x e4m3, fp32 accumulate)" if nv_step else "mxfp4 (e2m1 x e8m0, fp32 accumulate)"),
            "config": config_dict(w_full, world, args.shard),
            "pct_of_fp4_peak": 100.0 * value / world / peak,
            "roofline": {"bound": "tensor", "achieved": attn_tflops,
                         "kernel": f"mxattn_fwd_kernel<{w.d},{w.kv_tile}{',nvfp4' if nv_step else ''}>",
                         "peak": peak, "unit": "TFLOP/s", "frac": attn_tflops / peak,
                         "traffic": profiled_traffic() if (w == WORKLOAD and not nv_step) else None,
                         "peak_source": f"{peak_kind} bf16 burst {peaks['bf16_tflops']} TFLOP/s x "
                                        f"{FP4_PER_BF16:g} (nominal dense fp4:bf16)",
                         "attn_ms": attn_avg_ms, "prepare_ms": sum(prep_ms) / len(prep_ms),
                         "frac_of_9pf_spec": attn_tflops / 9000.0,
                         "mxf4_mma_loop": mma_loop,
                         "frac_of_mxf4_mma_loop": mxf4_frac},
            "cpu_baseline": base,
            "e2e": None if e2e_ms is None else {
                "value": job_flops / (e2e_ms / 1e3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": 3 * B * H * N * d * 2, "d2h_bytes_per_step": B * H * N * d * 4,
                "ms_per_step": e2e_ms, "steps": args.steps,
                "api": "mxattn_forward_host (C ABI, pinned host buffers)",
                "pipeline": "16 groups of (batch, head) slices; H2D, attention and D2H overlap on three streams"},
            "mufu_roofline": mufu_roofline(w, attn_avg_ms, clocks),
            "uos_pnq_overhead": overhead,
            "nvfp4": nvfp4,
            # per step: MXFP4 prepare (one fused quantize launch) + attention; NVFP4 prepare is
            # the amax pass and two quantizers, then attention
            "gpu_launches": (4 if nv_step else 2) * args.steps,
            "clocks": clocks,
            "quantize_sweep": quant,
            "long_video_dit": long_leg,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def measure_e2e(torch, mx, Q, K, V, w, bufs, stream, args, dist):
    """Same metric end to end through the public API with pinned host buffers:
    H2D of Q/K/V and D2H of O inside the timed region."""
    B, H, N, d = w.B, w.H, w.N, w.d
    q_h = torch.from_numpy(Q.view(np.int16)).view(torch.bfloat16).pin_memory()
    k_h = torch.from_numpy(K.view(np.int16)).view(torch.bfloat16).pin_memory()
    v_h = torch.from_numpy(V.view(np.int16)).view(torch.bfloat16).pin_memory()
    o_h = torch.empty((B, H, N, d), dtype=torch.float32).pin_memory()
    for _ in range(2):
        mx.attention_from_host(q_h, k_h, v_h, w.kv_tile, True, "uos", 0.0, bufs, o_h)
    torch.cuda.synchronize()
    e2e_steps = args.steps
    if dist is not None:
        dist.barrier()
    ee0, ee1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ee0.record(stream)
    for _ in range(e2e_steps):
        mx.attention_from_host(q_h, k_h, v_h, w.kv_tile, True, "uos", 0.0, bufs, o_h)
    ee1.record(stream)
    torch.cuda.synchronize()
    return max_over_ranks([ee0.elapsed_time(ee1) / e2e_steps], dist, "cuda")[0]


def launch_ranks(n: int) -> int:
    """`--gpus N` outside torchrun: start N ranks of this same command on this node
    (torch.distributed.run, rendezvous on 127.0.0.1); rank 0 prints the line."""
    import socket

    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-quantize-sweep", action="store_true")
    ap.add_argument("--workload", choices=sorted(wl.WORKLOADS), default="video_dit",
                    help="workload to time (default: the video-DiT configuration the metric is quoted on)")
    ap.add_argument("--heads", type=int, default=0, help="override H (smaller cases for profiling)")
    ap.add_argument("--shard", choices=["replicas", "heads", "sequence"], default="replicas",
                    help="N > 1: one independent batch per rank (weak scaling, default); the heads of one problem "
                         "split over the ranks; or its tokens split over the ranks with an all-to-all before and "
                         "after the attention (strong scaling)")
    ap.add_argument("--format", choices=["mxfp4", "nvfp4"], default="mxfp4",
                    help="operand format of the timed step (nvfp4: the comparison variant; only with --quick)")
    ap.add_argument("--qmax-study", action="store_true",
                    help="instead of the timed step: O error against exact attention over scale boundaries in [6, 8]")
    ap.add_argument("--quick", action="store_true",
                    help="timed steps only: no CPU baseline, no end-to-end leg, no quantize sweep")
    ap.add_argument("--ref-step-budget", type=float, default=0.0,
                    help="--impl reference: seconds of oracle work per step (default: about 2 minutes in all)")
    args = ap.parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return launch_ranks(args.gpus)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus if args.gpus == 1 else 1)))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    args.warmup = max(args.warmup, 3)  # timing rule: at least 3 warm-up steps
    if args.format == "nvfp4" and not args.quick:
        ap.error("--format nvfp4 times the comparison variant alone and needs --quick")
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.qmax_study:
        return qmax_study(args) if rank == 0 else 0
    return run_gpu(args, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
