"""Seeded synthetic inputs for the selective diagonal scan.

This module only draws random numbers and rounds them to the storage
precision; it contains none of the scan's arithmetic.  Both the CUDA path
(tests, bench) and the fp64 oracle consume the arrays it returns, so the two
always see bit-identical inputs.

Recipe (same for every workload; the pages publish no shapes or data, so
these synthetic draws stand in for their five H100 workloads):

* ``A_log ~ U(0, ln 16)`` so ``A = -exp(A_log)`` lies in ``[-16, -1]``
  (Mamba-1 recovery instead fixes ``A_n = -(n+1)``).
* ``dt = softplus(z + dt_bias)`` with ``z ~ N(0, variance 0.5)`` and
  ``dt_bias = log(expm1(dt0))``, ``dt0`` log-uniform in ``[1e-3, 1e-1]`` per
  head (per channel for the Mamba-1 workload) - the log-uniform step
  initialisation the robocikowo.com state-space-model glossary recommends.
* ``lambda = sigmoid(N(0, 1))`` (two-endpoint weight).
* ``theta ~ U(0, pi)`` per (head, rotation pair).
* ``B, C ~ N(0, 1/N)`` (``1/(N R)`` for rank-R routing), ``D ~ N(0, 1)``,
  ``x, dy ~ N(0, 1)``.
* per-token angles (``angle_mode = 1``): ``theta_t = dt_t theta_j (1 + 0.5 xi)``
  with ``xi ~ N(0, 1)``, drawn after every other tensor, fp32;
  ``inp["theta"]`` then holds them, ``[B, L, H, n_pairs]``.

Draw order, from one ``numpy.random.Generator(PCG64(seed))``:
``A_log, theta, D, dt0, z, lambda_logit, B, C, x, dy``.
Tensors stored as bf16 are rounded to nearest-even once, on the host.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

DTYPE_F32 = 0
DTYPE_BF16 = 1
DECAY_PER_HEAD = 0
DECAY_PER_COORD = 1
ANGLE_STATIC = 0
ANGLE_PER_TOKEN = 1
DISC_EULER = 0
DISC_ZOH = 1


@dataclasses.dataclass(frozen=True)
class ScanShape:
    """Problem sizes of one scan call (mirrors ``ssm_desc_t``)."""

    batch: int
    seqlen: int
    nheads: int
    headdim: int
    ngroups: int
    n_real: int
    n_pairs: int
    rank_in: int = 1
    rank_out: int = 1
    chunk: int = 0
    decay_mode: int = DECAY_PER_COORD
    two_endpoint: int = 1
    dtype_io: int = DTYPE_BF16
    # Mamba-1 recovery: A_n = -(n+1) instead of the random draw
    fixed_mamba1_A: bool = False
    name: str = ""
    # 0: rotation angle dt_t theta[h][j]; 1: per-token angles theta[b][t][h][j]
    # (the data-dependent angles of Mamba-3's complex state)
    angle_mode: int = 0
    # the first n_static real rows are static: transition exp(a_n) per step,
    # independent of dt_t (HybridMamba's real static rows)
    n_static: int = 0
    # 0: Euler / two-endpoint write (dt-scaled); 1: exact zero-order hold
    # (write scaled by (e^{dt lam} - 1) / lam per mode; needs two_endpoint = 0)
    discretization: int = 0

    @property
    def nstate(self) -> int:
        return self.n_real + 2 * self.n_pairs

    @property
    def n_decay(self) -> int:
        return 1 if self.decay_mode == DECAY_PER_HEAD else self.n_real + self.n_pairs

    def replace(self, **kw) -> "ScanShape":
        return dataclasses.replace(self, **kw)


# The five workloads of the selective diagonal scan (tiny hybrid parity case,
# Mamba-2 / Mamba-1 recoveries, HybridMamba, SSD-MIMO).
WORKLOADS = {
    "tiny_hybrid_fp32": ScanShape(
        batch=1, seqlen=256, nheads=2, headdim=16, ngroups=2, n_real=8, n_pairs=4,
        chunk=32, decay_mode=DECAY_PER_COORD, two_endpoint=1, dtype_io=DTYPE_F32,
        name="tiny_hybrid_fp32"),
    "mamba2_siso": ScanShape(
        batch=4, seqlen=2048, nheads=24, headdim=64, ngroups=3, n_real=128, n_pairs=0,
        chunk=64, decay_mode=DECAY_PER_HEAD, two_endpoint=0, dtype_io=DTYPE_BF16,
        name="mamba2_siso"),
    "mamba1_siso": ScanShape(
        batch=8, seqlen=4096, nheads=2048, headdim=1, ngroups=1, n_real=16, n_pairs=0,
        chunk=0, decay_mode=DECAY_PER_COORD, two_endpoint=0, dtype_io=DTYPE_BF16,
        fixed_mamba1_A=True, name="mamba1_siso"),
    "hybridmamba": ScanShape(
        batch=8, seqlen=8192, nheads=32, headdim=64, ngroups=32, n_real=64, n_pairs=32,
        chunk=64, decay_mode=DECAY_PER_COORD, two_endpoint=1, dtype_io=DTYPE_BF16,
        name="hybridmamba"),
    "ssd_mimo_r4": ScanShape(
        batch=4, seqlen=16384, nheads=16, headdim=64, ngroups=16, n_real=128, n_pairs=0,
        rank_in=4, rank_out=4, chunk=64, decay_mode=DECAY_PER_HEAD, two_endpoint=0,
        dtype_io=DTYPE_BF16, name="ssd_mimo_r4"),
}
WORKLOAD_ORDER = ["tiny_hybrid_fp32", "mamba2_siso", "mamba1_siso", "hybridmamba", "ssd_mimo_r4"]


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    bias = ((u >> 16) & 1) + 0x7FFF
    r = ((u + bias) & 0xFFFF0000).astype(np.uint32)
    out = r.view(np.float32).reshape(a.shape)
    nan = np.isnan(a)
    if nan.any():
        out = out.copy()
        out[nan] = np.nan
    return out


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Bit pattern (uint16) of values that are already bf16-representable."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def _softplus(v):
    return np.where(v > 20.0, v, np.log1p(np.exp(np.minimum(v, 20.0))))


def _sigmoid(v):
    return 1.0 / (1.0 + np.exp(-v))


def make_inputs(shape: ScanShape, seed: int, with_dy: bool = True,
                with_state: bool = False, with_raw: bool = False) -> dict:
    """Draw every input of one scan (and the upstream gradient ``dy``).

    Returns float32 numpy arrays holding values exactly representable in the
    storage dtype (bf16-rounded where ``dtype_io`` is bf16).  Layouts:
    ``x [B,L,H,R,P]``, ``dt/lam [B,L,H]``, ``A_log [H,n_decay]``,
    ``theta [H,n_pairs]``, ``D [H]``, ``Bm [B,L,G,R,N]``, ``Cm [B,L,G,O,N]``,
    ``dy [B,L,H,O,P]``; optional ``h0``/``w0`` ``[B,H,N,P]``; with ``with_raw``
    also the pre-activation inputs ``z``, ``lam_logit`` ``[B,L,H]`` and
    ``dt_bias [H]`` that ``dt`` and ``lam`` were made from (the draws are the
    same either way).
    """
    s = shape
    g = np.random.Generator(np.random.PCG64(seed))
    Bt, L, H, P, G = s.batch, s.seqlen, s.nheads, s.headdim, s.ngroups
    N, R, O = s.nstate, s.rank_in, s.rank_out
    f32 = np.float32

    A_log = g.uniform(0.0, math.log(16.0), size=(H, s.n_decay)).astype(f32)
    if s.fixed_mamba1_A:
        A_log = np.broadcast_to(np.log(np.arange(1, s.n_decay + 1, dtype=np.float64)),
                                (H, s.n_decay)).astype(f32)
    theta = g.uniform(0.0, math.pi, size=(H, s.n_pairs)).astype(f32)
    D = g.standard_normal(H, dtype=f32)
    dt0 = np.exp(g.uniform(math.log(1e-3), math.log(1e-1), size=H))
    dt_bias = np.log(np.expm1(dt0))
    z = g.standard_normal((Bt, L, H), dtype=f32) * f32(math.sqrt(0.5))
    dt = _softplus(z.astype(np.float64) + dt_bias[None, None, :]).astype(f32)
    lam_logit = g.standard_normal((Bt, L, H), dtype=f32)
    lam = _sigmoid(lam_logit.astype(np.float64)).astype(f32)
    bc_scale = f32(1.0 / math.sqrt(N * R))
    Bm = g.standard_normal((Bt, L, G, R, N), dtype=f32) * bc_scale
    Cm = g.standard_normal((Bt, L, G, O, N), dtype=f32) * f32(1.0 / math.sqrt(N * O))
    x = g.standard_normal((Bt, L, H, R, P), dtype=f32)
    out = dict(A_log=A_log, theta=theta, D=D, dt=dt, lam=lam, Bm=Bm, Cm=Cm, x=x)
    if with_dy:
        out["dy"] = g.standard_normal((Bt, L, H, O, P), dtype=f32)
    if with_state:
        out["h0"] = g.standard_normal((Bt, H, N, P), dtype=f32) * f32(0.5)
        out["w0"] = g.standard_normal((Bt, H, N, P), dtype=f32) * f32(0.5)
    if with_raw:
        out["z"], out["lam_logit"] = z, lam_logit
        out["dt_bias"] = dt_bias.astype(f32)
    if s.dtype_io == DTYPE_BF16:
        for k in ("dt", "lam", "Bm", "Cm", "x", "dy", "z", "lam_logit"):
            if k in out:
                out[k] = round_bf16(out[k])
    if s.angle_mode == ANGLE_PER_TOKEN:
        xi = g.standard_normal((Bt, L, H, s.n_pairs), dtype=f32)
        out["theta"] = (out["dt"][..., None] * theta[None, None] * (1.0 + 0.5 * xi)).astype(f32)
    return out
