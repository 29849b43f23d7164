#!/usr/bin/env python
"""Benchmark of the selective diagonal scan on B200: HybridMamba forward+backward.

One step = the whole hot path over one synthetic batch of the HybridMamba
workload (batch 8, L = 8192, 32 heads, P = 64, N = 128 = 64 real + 32
rotation pairs, two-endpoint writes, bf16 I/O, fp32 state): the forward scan
and the backward scan through the C ABI.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank scans its own batch (weak scaling); per-head
parameter gradients are summed over ranks with one NCCL all-reduce, the only
data-parallel exchange the path has.  HybridMamba's inputs (1.6 GB) exceed
the 126 MB L2, so steps run back to back; for a workload whose inputs fit in
twice the L2 (--workload mamba2_siso) every step is timed on its own and L2 is
flushed between steps.  --workload picks one of the other configured
workloads (their lines name it in config.workload).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from selective_diagonal_state_b200 import synthetic as S  # noqa: E402

METRIC = "HybridMamba scan tokens/s (fwd, fwd+bwd) at L=8192; % of HBM/TC roofline"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="hybridmamba", choices=list(S.WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target wall time of the bounded oracle sample")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the batch size (small cases for profiling only)")
    ap.add_argument("--variant", default="none", choices=sorted(VARIANTS),
                    help="a variant of the workload's scan (per-token angles, ZOH write, ...)")
    ap.add_argument("--op", default="scan", choices=["scan", "preact", "step", "gate", "cp"],
                    help="scan: forward + backward (the headline); preact: the dt / lambda "
                         "pre-activations, forward + backward; step: one decoding step; "
                         "gate: the forward with the mixer's output gate against the plain "
                         "forward; cp: the sequence-sharded training step with every "
                         "segment on this GPU, against the whole-sequence step")
    ap.add_argument("--segments", type=int, default=4,
                    help="--op cp: segments the sequence is cut into")
    return ap.parse_args()


# Variants of a workload's scan (rows beyond the hot path): the descriptor fields
# they change.
VARIANTS = {
    "none": {},
    "per_token_angles": dict(angle_mode=S.ANGLE_PER_TOKEN),
    "zoh": dict(two_endpoint=0, discretization=S.DISC_ZOH),
    "static_rows": dict(n_static=16),
    "rank_out_1": dict(rank_out=1),
    "rank_out_2": dict(rank_out=2),
}


# ---------------------------------------------------------------------------
# algorithmic bytes (read every input once, write every output once)
# ---------------------------------------------------------------------------
def tensor_bytes(shape: S.ScanShape) -> dict:
    s = shape
    e = 2 if s.dtype_io == S.DTYPE_BF16 else 4
    BL = s.batch * s.seqlen
    per_token = s.angle_mode == S.ANGLE_PER_TOKEN and s.n_pairs
    return {
        "x": BL * s.nheads * s.rank_in * s.headdim * e,
        "y": BL * s.nheads * s.rank_out * s.headdim * e,
        "B": BL * s.ngroups * s.rank_in * s.nstate * e,
        "C": BL * s.ngroups * s.rank_out * s.nstate * e,
        "dt": BL * s.nheads * e,
        "lam": BL * s.nheads * e if s.two_endpoint else 0,
        # per-token rotation angles (fp32), read by both directions, their gradient written
        "theta": BL * s.nheads * s.n_pairs * 4 if per_token else 0,
    }


def fwd_bytes(shape):
    t = tensor_bytes(shape)
    return t["x"] + t["B"] + t["C"] + t["dt"] + t["lam"] + t["theta"] + t["y"]


def bwd_bytes(shape):
    t = tensor_bytes(shape)
    reads = t["x"] + t["B"] + t["C"] + t["dt"] + t["lam"] + t["theta"] + t["y"]  # y-sized dy
    writes = t["x"] + t["B"] + t["C"] + t["dt"] + t["lam"] + t["theta"]
    return reads + writes


def kernel_bytes(shape, name: str) -> int:
    """Algorithmic bytes of one launch of each kernel: the path's inputs that the
    kernel has to read and the path's outputs it writes, each counted once.
    Workspace traffic between kernels is overhead of the design and is not
    counted, so a kernel that only touches workspace has 0 here."""
    s = shape
    t = tensor_bytes(shape)
    BLH = s.batch * s.seqlen * s.nheads
    ins = t["x"] + t["B"] + t["C"] + t["dt"] + t["lam"] + t["theta"]
    dy = t["y"]
    if name in ("k_fwd", "k_chunk_fwd"):
        return ins + t["y"]
    if name == "k_bwd_sweep1":   # inputs + dy -> per-head dC (fp32)
        return ins + dy + BLH * s.rank_out * s.nstate * 4
    if name == "k_bwd_sweep2":   # inputs + dy -> dx, sum_p G u^T (fp32), per-token scalars
        return (ins + dy + t["x"] + BLH * s.rank_in * s.nstate * 4
                + BLH * (2 + s.rank_in * s.rank_out) * 4)
    if name == "k_bwd_units_local":
        return (BLH * (s.rank_in + s.rank_out) * s.nstate * 4 + t["B"] + t["C"]
                + 2 * t["dt"] + 2 * t["lam"] + BLH * (2 + s.rank_in * s.rank_out) * 4)
    if name == "k_bwd_groups":
        return (BLH * (s.rank_in + s.rank_out) * s.nstate * 4 + t["C"] + t["B"] + t["C"]
                + t["dt"] + t["lam"])
    # tensor-core chain: path inputs read, path outputs written
    if name == "k_chunk_state_local":  # x, B, dt, lambda (chunk states go to workspace)
        return t["x"] + t["B"] + t["dt"] + t["lam"]
    if name == "k_chunk_bwd_dx":      # B, C, dt, lambda, dy -> dx
        return t["B"] + t["C"] + t["dt"] + t["lam"] + dy + t["x"]
    if name == "k_chunk_bwd_dx_saved":  # dy -> dx (the rest comes from the forward's workspace)
        return dy + t["x"]
    if name == "k_chunk_bwd_fused":   # x, B, C, dt, lambda, dy -> dB, dC (one head per group)
        out = t["B"] + t["C"] if s.nheads == s.ngroups else 0
        return ins + dy + out + t["theta"]   # and the per-token angle gradient
    if name == "k_bwd_units_final":   # dt, lambda -> ddt, dlambda
        return 2 * (t["dt"] + t["lam"])
    # scalar-decay chain
    if name == "k_ssd_fwd":           # x, B, C, dt, lambda -> y
        return ins + t["y"]
    if name == "k_ssd_bwd":           # x, B, C, dt, lambda, dy -> dx (+ dB, dC, one head per group)
        out = t["B"] + t["C"] if s.nheads == s.ngroups else 0
        return ins + dy + t["x"] + out
    if name == "k_ssd_tokens":        # dt, lambda -> ddt, dlambda
        return 2 * (t["dt"] + t["lam"])
    if name == "k_ssd_group_sum":     # -> dB, dC (groups of several heads)
        return t["B"] + t["C"]
    # channel scan
    if name == "k_m1_fwd":
        return ins + t["y"]
    if name == "k_m1_bwd":            # inputs + dy -> dx, ddt, dlambda
        return ins + dy + t["x"] + t["dt"] + t["lam"]
    if name == "k_m1_bc_sum":         # -> dB, dC
        return t["B"] + t["C"]
    return 0


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per batch row of
# the workload for the largest kernels, from one ncu capture of a smaller
# batch (the traffic is per 64-token chunk, so a launch moves batch x this),
# keyed by the kernel's source file and the first 16 hex digits of its SHA-256
# at capture time: an entry whose source has changed since is not reported
# (traffic null) instead of going stale.
NCU_TRAFFIC_PER_ROW = {
    # (workload, kernel): (dram read + write bytes per batch row of one launch, source hash)
    # ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum captures at batch 2
    # (HybridMamba, Mamba-1), 1 (SSD-MIMO) and the full Mamba-2 size; the traffic of
    # these kernels grows with the batch rows
    ("hybridmamba", "k_chunk_fwd"): (421.30e6, "45bd0acc068dc92e"),
    ("hybridmamba", "k_chunk_bwd_fused"): (603.87e6, "7a7cb7c7d5e041ac"),
    ("ssd_mimo_r4", "k_ssd_fwd"): (1182.60e6, "b0388a47d161e1c7"),
    ("ssd_mimo_r4", "k_ssd_bwd"): (1739.96e6, "b0388a47d161e1c7"),
    ("mamba2_siso", "k_ssd_fwd"): (31.07e6, "b0388a47d161e1c7"),
    ("mamba2_siso", "k_ssd_bwd"): (75.35e6, "b0388a47d161e1c7"),
    ("mamba1_siso", "k_m1_fwd"): (60.85e6, "21950b673a9f6706"),
    ("mamba1_siso", "k_m1_bwd"): (118.78e6, "21950b673a9f6706"),
}

# sources each kernel is compiled from: a traffic entry holds only while they
# are byte-identical to the build the counters were taken on
KERNEL_SOURCES = {
    "k_chunk_fwd": ("scan_chunk.cu", "chunk_common.cuh", "umma.cuh", "common.cuh"),
    "k_chunk_bwd_fused": ("scan_chunk_rev.cu", "chunk_common.cuh", "umma.cuh", "common.cuh"),
    "k_ssd_fwd": ("scan_ssd.cu", "chunk_common.cuh", "umma.cuh", "common.cuh"),
    "k_ssd_bwd": ("scan_ssd.cu", "chunk_common.cuh", "umma.cuh", "common.cuh"),
    "k_m1_fwd": ("scan_m1.cu", "common.cuh"),
    "k_m1_bwd": ("scan_m1.cu", "common.cuh"),
}


def source_sha16(kernel):
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES.get(kernel, ()):
        try:
            h.update(open(os.path.join(ROOT, "selective_diagonal_state_b200", "csrc", rel), "rb").read())
        except OSError:
            return None
    return h.hexdigest()[:16] if kernel in KERNEL_SOURCES else None


def ncu_traffic(shape, kernel):
    """Measured DRAM bytes of one launch of `kernel`, or None when there is no
    capture of the kernel's current sources."""
    ent = NCU_TRAFFIC_PER_ROW.get((shape.name, kernel))
    if ent is None:
        return None
    per_row, sha = ent
    if source_sha16(kernel) != sha:
        return None
    return per_row * shape.batch

# upper bound on library launches per fwd + bwd step (sizes the profiling session)
LAUNCHES_PER_STEP = 32


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.rows = []
        self.proc = None
        self.gpu = gpu_index
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [c.strip() for c in line.split(",")]))

    def mark(self, begin: bool):
        if begin:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = [r for (ts, r) in self.rows if self.t0 - 0.15 <= ts <= self.t1 + 0.15 and len(r) >= 10]
        if not rows:
            rows = [r for (_, r) in self.rows if len(r) >= 10][-3:]
        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[2]) for r in rows if num(r[2]) is not None]
        mx = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[6 + k].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU oracle sample (the reported baseline and the reference arm)
# ---------------------------------------------------------------------------
def oracle_sample_plan(shape, target_s):
    """(units, seqlen) of a sample taking about target_s of wall time."""
    import oracle
    cores = os.cpu_count() or 1
    cal = shape.replace(batch=1, nheads=1, ngroups=1, seqlen=256)
    inp = S.make_inputs(cal, seed=99)
    t = time.perf_counter()
    oracle.scan_fwd(cal, inp)
    oracle.scan_bwd(cal, inp, inp["dy"])
    per_unit_token = (time.perf_counter() - t) / 256.0
    # units run in parallel over the cores; keep the full sequence length
    units = max(1, min(shape.nheads * shape.batch, cores))
    L = shape.seqlen
    est = per_unit_token * L * -(-units // cores)
    if est > target_s:
        L = max(256, int(L * target_s / est))
    return units, L, cores


def oracle_sample_run(shape, units, L, seed=5):
    """Time one oracle fwd+bwd over `units` (batch row 0, heads 0..units-1) of length L."""
    import oracle
    h = min(units, shape.nheads)
    b = -(-units // shape.nheads)
    g = shape.ngroups if shape.ngroups == shape.nheads else max(1, shape.ngroups * h // shape.nheads)
    if shape.ngroups == shape.nheads:
        g = h
    sub = shape.replace(batch=b, nheads=h, ngroups=g if h % g == 0 else 1, seqlen=L)
    inp = S.make_inputs(sub, seed=seed)
    t = time.perf_counter()
    oracle.scan_fwd(sub, inp)
    oracle.scan_bwd(sub, inp, inp["dy"])
    dt = time.perf_counter() - t
    unit_tokens = sub.batch * sub.nheads * L
    return dt, unit_tokens / shape.nheads, sub


def cpu_threads():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def run_reference(args):
    """Reference arm: the fp64 oracle as it stands, on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    shape = S.WORKLOADS[args.workload].replace(**VARIANTS[args.variant])
    per_step_target = max(1.0, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    units, L, cores = oracle_sample_plan(shape, per_step_target)
    for _ in range(args.warmup):
        oracle_sample_run(shape, units, L)
    total_t, total_tok = 0.0, 0.0
    for _ in range(args.steps):
        dt, tok, sub = oracle_sample_run(shape, units, L)
        total_t += dt
        total_tok += tok
    value = total_tok / total_t
    sample = (f"{sub.batch}x{sub.nheads} (batch rows x heads) of {shape.name} at L={L}, fwd+bwd "
              f"per step; tokens counted as head-tokens / {shape.nheads}")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_t / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": shape.name, "batch": shape.batch, "seqlen": shape.seqlen,
                   "nheads": shape.nheads, "headdim": shape.headdim,
                   "state": f"{shape.n_real} real + {shape.n_pairs} pairs",
                   "sample": sample},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
L2_BYTES = 126 * 2 ** 20


def roofline_of(shape, dom, ms_launch, peaks):
    """Roofline entry of the dominant kernel: HBM bytes for every workload but
    the Mamba-1 recovery, whose per-(token, channel, state) exponentials make it
    bound by the special-function unit (MUFU)."""
    hbm = peaks.get("hbm_gbs")
    src = "measured" if hbm else "fallback"
    hbm = hbm or 6650.0
    if shape.name == "mamba1_siso" and dom in ("k_fwd", "k_bwd_sweep1", "k_bwd_sweep2",
                                                "k_m1_fwd", "k_m1_bwd"):
        # one ex2 per (token, channel, state row): the minimum of a pass over the
        # sequence (the channel-scan backward recomputes the states and does two, which
        # is overhead of the design and not counted); 16 ex2 per SM and clock, 148 SMs,
        # at the clock sampled under load
        ex2 = shape.batch * shape.seqlen * shape.nheads * shape.nstate
        clk = peaks.get("sm_mhz_under_load") or 1965.0
        peak = 16 * 148 * clk * 1e6 / 1e9   # G ex2 / s
        ach = ex2 / (ms_launch * 1e-3) / 1e9
        return {"bound": "alu", "achieved": ach, "peak": peak, "unit": "G ex2/s",
                "frac": ach / peak, "traffic": ncu_traffic(shape, dom), "kernel": dom,
                "algorithmic_ex2": ex2, "ms_per_launch": ms_launch,
                "peak_source": "MUFU ex2 16/clk/SM x 148 SMs x SM clock"}
    b = kernel_bytes(shape, dom)
    ach = b / (ms_launch * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
            "traffic": ncu_traffic(shape, dom), "kernel": dom, "algorithmic_bytes": b,
            "ms_per_launch": ms_launch, "peak_source": src}


def _clock_index(local):
    if "CUDA_VISIBLE_DEVICES" not in os.environ:
        return local
    return int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local])


def _peaks():
    pk = os.path.join(ROOT, "MEASURED_PEAKS.json")
    return json.load(open(pk)) if os.path.exists(pk) else {}


def run_op(args, shape):
    """--op preact | step | gate | cp: a row beyond the hot path on one GPU, timed like the
    scan (CUDA events on the launching stream around K calls after W warm-up
    calls, clocks sampled meanwhile, L2 flushed between calls when the data fit
    in it) against the HBM roofline of its algorithmic bytes.

    preact: ssm_preact_fwd + ssm_preact_bwd over the workload's (batch, L, heads):
      reads z (and the lambda logits), writes dt (and lambda); then reads z,
      ddt (and the logits, dlambda), writes dz (and dlambda_logit).
    step:   one ssm_scan_step for a decoding batch (--batch, default 128 rows) of
      the workload's heads: the fp32 state (and the previous write) read and
      written once, one token's x, dt, lambda, B, C read and y written.
    gate:   the forward with the output gate, beside the plain forward.
    cp:     the sequence cut into --segments segments, each scanned by its own
      buffers (state-only forward, exact forward, two backwards and the boundary
      combines) one after another on this GPU, beside the whole-sequence step;
      the roofline counts the whole sequence's scan bytes once."""
    import torch

    from selective_diagonal_state_b200 import abi, scan
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--op preact / step / gate / cp run on one GPU")
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (the library has no CPU path)")
    abi.load_library()
    e = 2 if shape.dtype_io == S.DTYPE_BF16 else 4
    two = bool(shape.two_endpoint)
    dtype = scan.io_dtype(shape)
    gen = torch.Generator(device="cuda").manual_seed(11)
    stream = torch.cuda.current_stream()
    if args.op == "preact":
        inp = S.make_inputs(shape, seed=S.WORKLOAD_ORDER.index(shape.name) + 1, with_dy=False,
                            with_raw=True)
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dtype).cuda()  # noqa: E731
        z, lg = dev(inp["z"]), dev(inp["lam_logit"])
        bias = torch.from_numpy(inp["dt_bias"]).cuda()
        dt, lam = torch.empty_like(z), torch.empty_like(lg)
        ddt = torch.randn(z.shape, generator=gen, device="cuda").to(dtype)
        dlam = torch.randn(z.shape, generator=gen, device="cuda").to(dtype)
        dz, dlg = torch.empty_like(z), torch.empty_like(lg)
        dbias = torch.empty(shape.nheads, dtype=torch.float32, device="cuda")
        desc = abi.make_desc(shape)

        def call():
            abi.ssm_preact_fwd(desc, z, bias, lg if two else None, dt, lam if two else None)
            abi.ssm_preact_bwd(desc, z, bias, lg if two else None, ddt, dlam if two else None,
                               dz, dbias, dlg if two else None)

        BLH = shape.batch * shape.seqlen * shape.nheads
        nbytes = BLH * e * (5 + 5 * two)
        tokens = shape.batch * shape.seqlen
        launches = 2
        cfg = {"batch": shape.batch, "seqlen": shape.seqlen, "nheads": shape.nheads}
        metric = "pre-activation (softplus dt, sigmoid lambda) fwd+bwd tokens/s"
    elif args.op == "gate":
        inp = S.make_inputs(shape, seed=S.WORKLOAD_ORDER.index(shape.name) + 1,
                            with_dy=False)
        d = scan.to_device(shape, inp)
        desc = abi.make_desc(shape)
        y, hT, wT = scan.alloc_fwd(shape)
        z = torch.randn(y.shape, generator=gen, device="cuda").to(dtype)
        ws, nb = scan.alloc_workspace(shape, abi.PASS_FWD_INFER, desc=desc)

        def plain():
            abi.ssm_scan_fwd(desc, d.x, d.dt, d.A_log, d.theta, d.Bm, d.Cm, d.D, d.lam, None, None,
                             y, hT, wT, ws, nb)

        def call():
            abi.ssm_scan_fwd_gated(desc, d.x, d.dt, d.A_log, d.theta, d.Bm, d.Cm, d.D, d.lam,
                                   None, None, z, y, None, hT, wT, ws, nb)

        tb = tensor_bytes(shape)
        nbytes = fwd_bytes(shape) + tb["y"]   # the scan's bytes and z
        tokens = shape.batch * shape.seqlen
        launches = 0   # counted by the profile session below
        cfg = {"batch": shape.batch, "seqlen": shape.seqlen, "nheads": shape.nheads}
        metric = "forward with the mixer's output gate, tokens/s"
        for _ in range(3):
            plain()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            plain()
        e1.record(stream)
        torch.cuda.synchronize()
        plain_ms = e0.elapsed_time(e1) / args.steps
    elif args.op == "cp":
        from selective_diagonal_state_b200 import cp
        nseg = args.segments
        if nseg < 1 or nseg > shape.seqlen:
            raise SystemExit("--segments must be in [1, seqlen]")
        inp = S.make_inputs(shape, seed=S.WORKLOAD_ORDER.index(shape.name) + 1)
        segs = []
        for k in range(nseg):
            a, b_ = cp.segment_bounds(shape.seqlen, nseg, k)
            sg = cp.SegmentScan(shape.replace(seqlen=b_ - a))
            sg.load(inp, a, b_)
            segs.append(sg)

        def call():
            cp.run_sharded(segs)

        # the whole-sequence training step on the same inputs, for the overhead
        d = scan.to_device(shape, inp)
        desc = abi.make_desc(shape)
        out, grads = scan.alloc_fwd(shape), scan.alloc_bwd(shape)
        wsf = scan.alloc_workspace(shape, abi.PASS_FWD, desc=desc)
        wsb = scan.alloc_workspace(shape, abi.PASS_BWD, desc=desc)

        def plain():
            scan.scan_forward(shape, d, out=out, desc=desc, workspace=wsf)
            scan.scan_backward(shape, d, grads=grads, workspace=wsb, desc=desc, saved=wsf)

        nbytes = fwd_bytes(shape) + bwd_bytes(shape)   # the whole sequence's scan bytes
        tokens = shape.batch * shape.seqlen
        launches = 0   # counted by the profile session below
        cfg = {"batch": shape.batch, "seqlen": shape.seqlen, "nheads": shape.nheads,
               "segments": nseg,
               "emulation": "every segment's kernels on this GPU one after another; the "
                            "all-gathers are stacks of the segments' boundary values"}
        metric = "sequence-sharded training step (all segments on one GPU) tokens/s"
        for _ in range(3):
            plain()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            plain()
        e1.record(stream)
        torch.cuda.synchronize()
        plain_ms = e0.elapsed_time(e1) / args.steps
    else:
        B = args.batch or 128
        sh = shape.replace(batch=B, seqlen=1)
        inp = S.make_inputs(sh, seed=S.WORKLOAD_ORDER.index(shape.name) + 1, with_dy=False,
                            with_state=True)
        d = scan.to_device(sh, inp)
        desc = abi.make_desc(sh)
        h = d.h0.clone()
        w = d.w0.clone() if two else None
        y = torch.empty((B, 1, sh.nheads, sh.rank_out, sh.headdim), dtype=dtype, device="cuda")
        per_token = sh.angle_mode == S.ANGLE_PER_TOKEN and sh.n_pairs
        th = d.theta[:, 0].contiguous() if per_token else d.theta

        def call():
            abi.ssm_scan_step(desc, d.x, d.dt, d.A_log, th, d.Bm, d.Cm, d.D,
                              d.lam if two else None, h, w, y)

        st = B * sh.nheads * sh.nstate * sh.headdim * 4
        tb = tensor_bytes(sh)
        nbytes = 2 * st * (2 if two else 1) + sum(tb.values())
        tokens = B
        launches = 1
        cfg = {"batch": B, "nheads": sh.nheads, "state_bytes": st * (2 if two else 1)}
        metric = "decode step tokens/s (one token per batch row and call)"
    flush = nbytes < 2 * L2_BYTES
    scratch = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda") if flush else None
    for _ in range(max(3, args.warmup)):
        call()
    torch.cuda.synchronize()
    abi.ssm_scan_poll_device_error()
    # per-kernel device times (events around each launch, in a separate pass)
    abi.ssm_scan_profile_start(max(launches, 16) * args.steps)
    for _ in range(args.steps):
        call()
    prof = abi.ssm_scan_profile_stop()
    kernel_ms = {n: tot / max(1, c) for n, (c, tot) in prof.items()}
    if not launches:
        launches = int(round(sum(c for c, _ in prof.values()) / args.steps))
    # the timed calls replay a CUDA graph of one call: these ops take microseconds,
    # so launching them from Python would time the host instead of the device
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    torch.cuda.synchronize()
    call = graph.replay
    clocks = ClockSampler(_clock_index(int(os.environ.get("LOCAL_RANK", "0"))))
    clocks.start()
    time.sleep(0.3)
    clocks.mark(True)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps if flush else 1)]
    if flush:
        for a, b in evs:
            scratch.fill_(1.0)
            a.record(stream)
            call()
            b.record(stream)
    else:
        evs[0][0].record(stream)
        for _ in range(args.steps):
            call()
        evs[0][1].record(stream)
    torch.cuda.synchronize()
    clocks.mark(False)
    clk = clocks.stop()
    ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    abi.ssm_scan_poll_device_error()
    peaks = _peaks()
    hbm = peaks.get("hbm_gbs") or 6650.0
    ach = nbytes / (ms * 1e-3) / 1e9
    line = {
        "metric": metric, "value": tokens / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if shape.dtype_io == S.DTYPE_BF16 else "f32", "data": "synthetic",
        "op": args.op,
        "config": dict(cfg, workload=shape.name, variant=args.variant,
                       l2=("data below twice L2: each call timed alone, L2 flushed between "
                           "calls" if flush else "data larger than twice L2; no flush")),
        "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s",
                     "frac": ach / hbm, "traffic": None, "algorithmic_bytes": nbytes,
                     "peak_source": "measured" if peaks.get("hbm_gbs") else "fallback"},
        "kernel_ms": kernel_ms,
        "timing": "CUDA graph replays of one call, CUDA events on the stream",
        "plain_forward_ms": plain_ms if args.op == "gate" else None,
        "plain_step_ms": plain_ms if args.op == "cp" else None,
        "gpu_launches": launches * args.steps,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.op != "scan":
        shape = S.WORKLOADS[args.workload].replace(**VARIANTS[args.variant])
        if args.batch and args.op != "step":
            shape = shape.replace(batch=args.batch)
        run_op(args, shape)
        return
    import torch
    import torch.distributed as dist

    from selective_diagonal_state_b200 import abi, scan
    from selective_diagonal_state_b200 import dist as sdist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (the scan has no CPU path)")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    abi.load_library()
    shape = S.WORKLOADS[args.workload].replace(**VARIANTS[args.variant])
    if args.batch:
        shape = shape.replace(batch=args.batch)
    inp = S.make_inputs(shape, seed=S.WORKLOAD_ORDER.index(shape.name) + 1000 * rank)
    dev = scan.to_device(shape, inp)
    desc = abi.make_desc(shape)
    fwd_out = scan.alloc_fwd(shape)
    grads = scan.alloc_bwd(shape)
    ws = scan.alloc_workspace(shape, abi.PASS_BWD, desc=desc)
    wsf = scan.alloc_workspace(shape, abi.PASS_FWD, desc=desc)
    stream = torch.cuda.current_stream()
    in_bytes = fwd_bytes(shape)   # x, B, C, dt, lambda and the y-sized dy
    flush = in_bytes < 2 * L2_BYTES
    scratch = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda") if flush else None

    def barrier():
        if world > 1:
            dist.barrier()

    def allreduce_params():
        if world > 1:
            sdist.allreduce_param_grads((grads.dA_log, grads.dtheta, grads.dD))

    def step():
        scan.scan_forward(shape, dev, out=fwd_out, desc=desc, workspace=wsf)
        scan.scan_backward(shape, dev, grads=grads, workspace=ws, desc=desc, saved=wsf)
        allreduce_params()

    def fwd_only():
        scan.scan_forward(shape, dev, out=fwd_out, desc=desc, workspace=wsf)

    def timed(fn, n):
        """Device ms per call of fn over n calls (CUDA events on our stream).  With
        inputs that fit in L2, every call is timed on its own and L2 is flushed by
        writing a buffer of twice its size between calls, outside the events."""
        if not flush:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n):
                fn()
            e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / n
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for a, b in evs:
            scratch.fill_(1.0)
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs) / n

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    abi.ssm_scan_poll_device_error()
    names = {abi.ROUTE_CHUNKED: "per-coordinate tensor-core chain",
             abi.ROUTE_RANGE_FALLBACK: "recurrent (range fallback)",
             abi.ROUTE_RECURRENT: "recurrent", abi.ROUTE_SSD: "scalar-decay tensor-core chain",
             abi.ROUTE_CHANNEL: "channel scan"}
    route_bwd = names[abi.ssm_scan_last_route()]
    fwd_only()
    route = {"fwd": names[abi.ssm_scan_last_route()], "bwd": route_bwd}

    # ---- the headline: K steps, nothing else on the stream -----------------------
    clocks = ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ else
                          int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local]))
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    clocks.mark(True)
    ms_step = timed(step, args.steps)
    barrier()
    clocks.mark(False)
    ms_fwd = timed(fwd_only, args.steps)
    clk = clocks.stop()

    # ---- per-kernel device times: a separate pass of K steps bracketed per launch
    abi.ssm_scan_profile_start(LAUNCHES_PER_STEP * args.steps)
    timed(step, args.steps)
    prof = abi.ssm_scan_profile_stop()
    launches_per_step = sum(c for c, _ in prof.values()) / args.steps
    avg = {n: tot / max(1, c) for n, (c, tot) in prof.items()}
    share = {n: tot / max(1e-9, sum(t for _, t in prof.values())) for n, (c, tot) in prof.items()}

    # ---- memory: what the training forward keeps for the backward, and the peak
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    base_alloc = torch.cuda.memory_allocated()
    step()
    torch.cuda.synchronize()
    peak_alloc = torch.cuda.max_memory_allocated()
    saved_bytes = int(wsf[1]) if wsf[0] is not None else 0
    memory = {"saved_for_backward_bytes": saved_bytes,
              "backward_workspace_bytes": int(ws[1]) if ws[0] is not None else 0,
              "peak_alloc_bytes": int(peak_alloc), "resident_alloc_bytes": int(base_alloc)}

    # max over ranks
    t = torch.tensor([ms_step, ms_fwd], dtype=torch.float64, device="cuda")
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_step, ms_fwd = float(t[0]), float(t[1])

    tokens = shape.batch * shape.seqlen * world
    value = tokens / (ms_step * 1e-3)
    fwd_value = tokens / (ms_fwd * 1e-3)

    peaks = {}
    pk = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pk):
        peaks = json.load(open(pk))
    if clk.get("sm_mhz"):
        peaks = dict(peaks, sm_mhz_under_load=clk["sm_mhz"])
    hbm = peaks.get("hbm_gbs") or 6650.0
    dom = max(avg, key=avg.get)
    roof = roofline_of(shape, dom, avg[dom], peaks)
    step_bytes = fwd_bytes(shape) + bwd_bytes(shape)

    # end to end through the public API with host buffers
    e2e = None
    if args.e2e_steps > 0:
        host = {k: torch.from_numpy(np.ascontiguousarray(v)).to(scan.io_dtype(shape)
                if k in ("x", "dt", "lam", "Bm", "Cm", "dy") else torch.float32).pin_memory()
                for k, v in inp.items() if v is not None}
        outs = [fwd_out[0], grads.dx, grads.ddt, grads.dBm, grads.dCm, grads.dA_log, grads.dD]
        outs += [t_ for t_ in (grads.dtheta, grads.dlam) if t_ is not None]
        host_out = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
        dev_map = {"x": dev.x, "dt": dev.dt, "lam": dev.lam, "Bm": dev.Bm, "Cm": dev.Cm,
                   "dy": dev.dy, "A_log": dev.A_log, "theta": dev.theta, "D": dev.D}
        h2d = sum(host[k].numel() * host[k].element_size() for k in dev_map
                  if k in host and dev_map[k] is not None)
        d2h = sum(o.numel() * o.element_size() for o in outs)

        def e2e_step():
            for k, d in dev_map.items():
                if d is not None and k in host:
                    d.copy_(host[k], non_blocking=True)
            step()
            for o, ho in zip(outs, host_out):
                ho.copy_(o, non_blocking=True)

        # Pipelined: two device input / output sets alternate, so a step's host copies
        # overlap its neighbours' compute (a loader's prefetch): step i's inputs go up on
        # one copy stream while step i - 1 computes, its outputs come down on another
        # while step i + 1 computes.  Every step still moves all of its bytes both ways.
        dev2 = scan.to_device(shape, inp)
        sets = [(dev, fwd_out, grads), (dev2, scan.alloc_fwd(shape), scan.alloc_bwd(shape))]
        up, down = torch.cuda.Stream(), torch.cuda.Stream()

        def in_map(d):
            return {"x": d.x, "dt": d.dt, "lam": d.lam, "Bm": d.Bm, "Cm": d.Cm, "dy": d.dy,
                    "A_log": d.A_log, "theta": d.theta, "D": d.D}

        def outs_of(fo, g):
            o = [fo[0], g.dx, g.ddt, g.dBm, g.dCm, g.dA_log, g.dD]
            return o + [t_ for t_ in (g.dtheta, g.dlam) if t_ is not None]

        def e2e_pipelined(n):
            ev_in = [torch.cuda.Event() for _ in range(n)]
            ev_comp = [torch.cuda.Event() for _ in range(n)]
            ev_out = [torch.cuda.Event() for _ in range(n)]
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(up)
            for i in range(n):
                d, fo, g = sets[i % 2]
                if i >= 2:
                    up.wait_event(ev_comp[i - 2])    # this set's inputs are consumed
                with torch.cuda.stream(up):
                    for k, t_ in in_map(d).items():
                        if t_ is not None and k in host:
                            t_.copy_(host[k], non_blocking=True)
                ev_in[i].record(up)
                stream.wait_event(ev_in[i])
                if i >= 2:
                    stream.wait_event(ev_out[i - 2])  # this set's outputs have come down
                scan.scan_forward(shape, d, out=fo, desc=desc, workspace=wsf)
                scan.scan_backward(shape, d, grads=g, workspace=ws, desc=desc, saved=wsf)
                if world > 1:
                    sdist.allreduce_param_grads((g.dA_log, g.dtheta, g.dD))
                ev_comp[i].record(stream)
                down.wait_event(ev_comp[i])
                with torch.cuda.stream(down):
                    for o, ho in zip(outs_of(fo, g), host_out):
                        ho.copy_(o, non_blocking=True)
                ev_out[i].record(down)
            t1.record(down)
            torch.cuda.synchronize()
            return t0.elapsed_time(t1) / n

        barrier()
        torch.cuda.synchronize()
        ms_serial = timed(e2e_step, args.e2e_steps)
        barrier()
        e2e_pipelined(2)   # warm the second set and the streams
        barrier()
        ms_e2e = e2e_pipelined(args.e2e_steps)
        te = torch.tensor([ms_e2e, ms_serial], dtype=torch.float64, device="cuda")
        if world > 1:
            dist.all_reduce(te, op=dist.ReduceOp.MAX)
        ms_e2e, ms_serial = float(te[0]), float(te[1])
        e2e = {"value": tokens / (ms_e2e * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": ms_e2e, "copies": "pipelined over two buffer sets",
               "ms_per_step_serial": ms_serial}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        units, L, cores = oracle_sample_plan(shape, args.cpu_seconds)
        dt_s, tok, sub = oracle_sample_run(shape, units, L)
        cpu = {"value": tok / dt_s, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": f"{sub.batch}x{sub.nheads} (batch rows x heads) of {shape.name} at "
                         f"L={L}, fwd+bwd, {dt_s:.1f} s; tokens = head-tokens / {shape.nheads}"}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    io = "bf16, fp32 state" if shape.dtype_io == S.DTYPE_BF16 else "fp32"
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if shape.dtype_io == S.DTYPE_BF16 else "f32",
        "data": "synthetic",
        "config": {"workload": shape.name, "variant": args.variant,
                   "batch_per_gpu": shape.batch, "seqlen": shape.seqlen,
                   "nheads": shape.nheads, "headdim": shape.headdim, "ngroups": shape.ngroups,
                   "state": f"{shape.n_real} real + {shape.n_pairs} rotation pairs",
                   "rank_in": shape.rank_in, "rank_out": shape.rank_out,
                   "two_endpoint": bool(shape.two_endpoint), "io": io,
                   "parallelism": f"dp{world}" if world > 1 else "single",
                   "l2": (f"inputs ({in_bytes / 1e9:.2f} GB) fit in L2: each step timed alone, "
                          f"L2 flushed between steps" if flush else
                          f"inputs ({in_bytes / 1e9:.2f} GB) larger than L2; no flush"),
                   "route": route},
        "fwd_tokens_per_s": fwd_value, "ms_fwd": ms_fwd,
        "roofline": roof,
        "step_roofline": {"algorithmic_bytes": step_bytes,
                          "achieved_gbs": step_bytes / (ms_step * 1e-3) / 1e9,
                          "frac": step_bytes / (ms_step * 1e-3) / 1e9 / hbm},
        "kernel_ms": avg, "kernel_share": share,
        "gpu_launches": int(round(launches_per_step * args.steps)),
        "memory": memory,
        "clocks": clk,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
