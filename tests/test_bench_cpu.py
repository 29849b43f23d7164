"""Host-side pieces of the benchmark, on the CPU: the algorithmic bytes the
roofline divides by (the path's tensors counted once per (token, head)), the
traffic table's source keys, and the command line of the side measurements."""
import sys

import pytest

import bench
from selective_diagonal_state_b200 import synthetic as S


def test_hybridmamba_algorithmic_bytes():
    """bf16 per (token, head): forward x 128 + B 256 + C 256 + dt 2 + lambda 2 +
    y 128 = 772 B; backward reads the same inputs and dy 128, writes dx, dB, dC,
    ddt, dlambda (1416 B)."""
    sh = S.WORKLOADS["hybridmamba"]
    th = sh.batch * sh.seqlen * sh.nheads
    assert bench.fwd_bytes(sh) == 772 * th
    assert bench.bwd_bytes(sh) == 1416 * th
    assert bench.fwd_bytes(sh) + bench.bwd_bytes(sh) == 4_588_568_576
    # the forward kernel is charged the whole forward; the fused backward reads the
    # inputs and dy (772 B) and writes dB and dC (512 B): 1284 B per (token, head)
    assert bench.kernel_bytes(sh, "k_chunk_fwd") == bench.fwd_bytes(sh)
    assert bench.kernel_bytes(sh, "k_chunk_bwd_fused") == 1284 * th == 2_692_743_168


def test_per_token_angles_charge_theta():
    """A per-token angle is an fp32 input of B L H n_pairs read by the forward and the
    backward and written back as its gradient."""
    sh = S.WORKLOADS["hybridmamba"]
    tok = sh.replace(angle_mode=S.ANGLE_PER_TOKEN)
    th = 4 * sh.batch * sh.seqlen * sh.nheads * sh.n_pairs
    assert bench.fwd_bytes(tok) - bench.fwd_bytes(sh) == th
    assert bench.bwd_bytes(tok) - bench.bwd_bytes(sh) == 2 * th


def test_traffic_entries_name_known_kernels():
    """Every measured-traffic entry is keyed by a workload and a kernel whose source
    files exist, so a stale entry is detected by its hash instead of a missing file."""
    for (wl, kern), (per_row, sha) in bench.NCU_TRAFFIC_PER_ROW.items():
        assert wl in S.WORKLOADS
        assert kern in bench.KERNEL_SOURCES
        assert per_row > 0 and len(sha) == 16
        assert bench.source_sha16(kern) is not None


@pytest.mark.parametrize("argv,op,segments", [
    ([], "scan", 4),
    (["--op", "cp", "--segments", "8"], "cp", 8),
    (["--op", "gate", "--workload", "ssd_mimo_r4"], "gate", 4),
])
def test_command_line(monkeypatch, argv, op, segments):
    monkeypatch.setattr(sys, "argv", ["bench.py"] + argv)
    args = bench.parse()
    assert args.op == op and args.segments == segments
    assert args.gpus == 1 and args.warmup >= 3
