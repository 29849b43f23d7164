"""GPU parity: the CUDA scan (through the C ABI) against the fp64 oracle, element
by element, on the same seeded inputs."""
import re

import numpy as np
import pytest

import oracle
from selective_diagonal_state_b200 import abi, scan
from selective_diagonal_state_b200 import synthetic as S
from tests.parity_util import compare, to_np

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from selective_diagonal_state_b200 import build
    build.build()
    abi.load_library()
    assert torch.cuda.is_available()


def chunk_eligible(shape):
    """Shapes the per-coordinate tensor-core kernels take."""
    return (shape.dtype_io == S.DTYPE_BF16 and shape.headdim == 64 and shape.rank_in == 1
            and shape.rank_out == 1 and shape.nstate in (64, 128) and shape.n_real % 8 == 0
            and shape.seqlen > 0 and shape.chunk != 1 and shape.n_static == 0)


def ssd_eligible(shape):
    """Shapes the scalar-decay (per-head) tensor-core kernels take."""
    return (shape.dtype_io == S.DTYPE_BF16 and shape.decay_mode == S.DECAY_PER_HEAD
            and shape.n_pairs == 0 and shape.headdim == 64 and shape.nstate in (64, 128)
            and shape.rank_in in (1, 2, 4) and shape.rank_out in (1, 2, 4)
            and shape.seqlen > 0 and shape.chunk != 1
            and shape.n_static == 0 and shape.discretization == S.DISC_EULER)


def channel_eligible(shape):
    """Shapes the channel scan (Mamba-1 channels) takes."""
    return (shape.dtype_io == S.DTYPE_BF16 and shape.headdim == 1 and shape.rank_in == 1
            and shape.rank_out == 1 and shape.n_pairs == 0 and shape.nstate in (8, 16)
            and (shape.nheads // shape.ngroups) % 64 == 0 and shape.seqlen > 0
            and shape.chunk != 1)


def expected_route(shape, backward=False):
    """Kernels expected to run the forward (backward) of `shape`."""
    if channel_eligible(shape):
        return abi.ROUTE_CHANNEL
    if ssd_eligible(shape):
        return abi.ROUTE_SSD
    return abi.ROUTE_CHUNKED if chunk_eligible(shape) else abi.ROUTE_RECURRENT


def run_gpu(shape, inp, backward=True, route=None):
    """Forward (and backward) through the C ABI; checks which kernels ran.  `route`
    overrides the expected route of both directions (a pair: each its own)."""
    if route is None:
        route = (expected_route(shape), expected_route(shape, backward=True))
    elif not isinstance(route, tuple):
        route = (route, route)
    dev = scan.to_device(shape, inp)
    y, hT, wT = scan.scan_forward(shape, dev)
    assert abi.ssm_scan_last_route() == route[0]
    g = None
    if backward:
        g = scan.scan_backward(shape, dev)
        assert abi.ssm_scan_last_route() == route[1]
    torch.cuda.synchronize()
    abi.ssm_scan_poll_device_error()
    return y, hT, wT, g


def check_all(shape, inp, backward=True, report=None, route=None, bounds=None):
    """Every output against the oracle; `bounds` maps an output name to a
    per-element max-abs bound derived for an input outside the workloads'
    ranges (parity_util.compare's `bound`)."""
    bounds = bounds or {}
    y, hT, wT, g = run_gpu(shape, inp, backward, route)
    ref = oracle.scan_fwd(shape, inp)
    dt = shape.dtype_io
    compare("y", to_np(y), ref["y"], dt, report)
    compare("hT", to_np(hT), ref["hT"], dt, report)
    compare("last_write", to_np(wT), ref["wT"], dt, report)
    if not backward:
        return
    gr = oracle.scan_bwd(shape, inp, inp["dy"])
    compare("dx", to_np(g.dx), gr["dx"], dt, report)
    compare("ddt", to_np(g.ddt), gr["ddt"], dt, report)
    compare("dB", to_np(g.dBm), gr["dBm"], dt, report,
            bound=bounds["dB"](gr["dBm"]) if "dB" in bounds else None)
    compare("dC", to_np(g.dCm), gr["dCm"], dt, report,
            bound=bounds["dC"](gr["dCm"]) if "dC" in bounds else None)
    compare("dA_log", to_np(g.dA_log), gr["dA_log"], dt, report)
    if shape.rank_in == shape.rank_out:
        compare("dD", to_np(g.dD), gr["dD"], dt, report)
    if shape.n_pairs:
        compare("dtheta", to_np(g.dtheta), gr["dtheta"], dt, report)
    if shape.two_endpoint:
        compare("dlambda", to_np(g.dlam), gr["dlam"], dt, report)
    compare("dh0", to_np(g.dh0), gr["dh0"], dt, report)
    compare("dprev_write", to_np(g.dw0), gr["dw0"], dt, report)


# Reduced copies of the five workloads: same heads/state/rank/group structure,
# fewer tokens (not a multiple of the 16/32-token staging tile) so the oracle
# finishes in seconds.
REDUCED = {
    "tiny_hybrid_fp32": dict(),
    "mamba2_siso": dict(batch=2, seqlen=203),
    "mamba1_siso": dict(batch=2, seqlen=157),
    "hybridmamba": dict(batch=2, seqlen=181),
    "ssd_mimo_r4": dict(batch=1, seqlen=133),
}


@pytest.mark.parametrize("name", S.WORKLOAD_ORDER)
def test_workload_parity(name):
    shape = S.WORKLOADS[name].replace(**REDUCED[name])
    inp = S.make_inputs(shape, seed=S.WORKLOAD_ORDER.index(name))
    check_all(shape, inp)


@pytest.mark.parametrize("name", ["mamba2_siso", "hybridmamba"])
def test_workload_parity_recurrent_path(name):
    """The same workloads through the token-by-token kernels (chunk = 1)."""
    shape = S.WORKLOADS[name].replace(**REDUCED[name]).replace(chunk=1)
    inp = S.make_inputs(shape, seed=S.WORKLOAD_ORDER.index(name))
    check_all(shape, inp)


@pytest.mark.parametrize("kw", [
    dict(seqlen=1), dict(seqlen=63), dict(seqlen=64), dict(seqlen=65), dict(seqlen=200),
    dict(seqlen=130, n_real=128, n_pairs=0),
    dict(seqlen=130, n_real=0, n_pairs=64),
    dict(seqlen=100, n_real=32, n_pairs=16),
    dict(seqlen=100, decay_mode=S.DECAY_PER_HEAD, two_endpoint=0, n_real=128, n_pairs=0,
         ngroups=2),
])
def test_chunked_shapes(kw):
    """Chunked tensor-core kernels: ragged tails around the 64-token chunk,
    64/128 state rows, real-only, pairs-only, grouped B/C, initial state."""
    base = S.WORKLOADS["hybridmamba"].replace(batch=2, nheads=4, ngroups=4, chunk=64)
    shape = base.replace(**kw)
    inp = S.make_inputs(shape, seed=31, with_state=True)
    check_all(shape, inp)


@pytest.mark.parametrize("kw", [
    dict(),                                  # Mamba-1: 16 state rows, B / C shared by all channels
    dict(n_real=8),                          # 8 state rows: one thread per channel
    dict(two_endpoint=1),                    # two-endpoint writes
    dict(decay_mode=S.DECAY_PER_HEAD),       # one decay per channel
    dict(nheads=256, ngroups=4),             # groups of 64 channels
    dict(seqlen=1), dict(seqlen=16), dict(seqlen=17),
])
def test_channel_scan_shapes(kw):
    """The channel scan (head dim 1) around its 16-token tiles and 64-channel
    blocks, with an initial state and a left endpoint."""
    base = S.WORKLOADS["mamba1_siso"].replace(batch=2, seqlen=70, nheads=128)
    shape = base.replace(**kw)
    inp = S.make_inputs(shape, seed=71, with_state=True)
    check_all(shape, inp)


@pytest.mark.parametrize("kw", [
    dict(),                                   # HybridMamba heads, bf16
    dict(dtype_io=S.DTYPE_F32),
    dict(n_real=0, n_pairs=5, headdim=16, seqlen=33),
    dict(decay_mode=S.DECAY_PER_HEAD, two_endpoint=0),
    dict(seqlen=1),
])
def test_per_token_angles(kw):
    """Per-token rotation angles theta[b][t][h][j] (the complex state of
    Mamba-3): forward, and the per-token angle gradient across several 64-token
    chunks -- on the tensor-core chain for the bf16 HybridMamba heads, on the
    recurrent kernels for the others."""
    base = S.WORKLOADS["hybridmamba"].replace(batch=2, nheads=4, ngroups=4, seqlen=150,
                                              angle_mode=S.ANGLE_PER_TOKEN)
    shape = base.replace(**kw)
    inp = S.make_inputs(shape, seed=91, with_state=True)
    assert inp["theta"].shape == (shape.batch, shape.seqlen, shape.nheads, shape.n_pairs)
    check_all(shape, inp)   # the tensor-core chain for bf16 HybridMamba heads


@pytest.mark.parametrize("kw", [
    dict(n_static=16),                        # HybridMamba heads: 16 static of 64 real rows
    dict(n_real=32, n_pairs=16, n_static=24),  # another mixture (N = 64)
    dict(n_static=64, dtype_io=S.DTYPE_F32),  # every real row static
    dict(n_static=8, decay_mode=S.DECAY_PER_HEAD, two_endpoint=0),
    dict(n_static=16, angle_mode=S.ANGLE_PER_TOKEN, seqlen=70),
])
def test_static_rows(kw):
    """Real static rows (transition e^{a} whatever dt) mixed with real and
    complex dynamic rows, as HybridMamba mixes its three row types."""
    base = S.WORKLOADS["hybridmamba"].replace(batch=2, nheads=4, ngroups=4, seqlen=150)
    shape = base.replace(**kw)
    inp = S.make_inputs(shape, seed=93, with_state=True)
    check_all(shape, inp, route=abi.ROUTE_RECURRENT)


@pytest.mark.parametrize("kw", [
    dict(),                                   # HybridMamba heads (Euler write off), bf16
    dict(dtype_io=S.DTYPE_F32),
    dict(angle_mode=S.ANGLE_PER_TOKEN),
    dict(decay_mode=S.DECAY_PER_HEAD, n_real=128, n_pairs=0, ngroups=2),
    dict(rank_in=2, rank_out=2, n_real=16, n_pairs=8, seqlen=70),
])
def test_zoh_write(kw):
    """Exact zero-order-hold write ((e^{dt lam} - 1) / lam per mode, complex on a
    rotation pair) against the oracle, forward and backward: on the per-coordinate
    tensor-core chain for bf16 heads of 64 channels, on the recurrent kernels
    otherwise."""
    base = S.WORKLOADS["hybridmamba"].replace(batch=2, nheads=4, ngroups=4, seqlen=150,
                                              two_endpoint=0, discretization=S.DISC_ZOH)
    shape = base.replace(**kw)
    inp = S.make_inputs(shape, seed=95, with_state=True)
    check_all(shape, inp)


@pytest.mark.parametrize("kw", [
    dict(rank_in=1, rank_out=2),
    dict(rank_in=2, rank_out=1, ngroups=2),                   # two heads per group
    dict(rank_in=1, rank_out=4),
    dict(rank_in=4, rank_out=1, ngroups=2),
    dict(rank_in=2, rank_out=4, two_endpoint=1, ngroups=2),
    dict(rank_in=4, rank_out=2, n_real=64, seqlen=97),         # 64 state rows
])
def test_scalar_decay_unequal_ranks(kw):
    """SSD-MIMO with R source and O != R target rows per token on the scalar-decay
    tensor-core chain (chunks of 128 / max(R, O) tokens; the narrower side's rank
    rows are zero-filled on load and dropped on store): every output against the
    oracle, with groups of one head and of two."""
    base = S.WORKLOADS["ssd_mimo_r4"].replace(batch=2, seqlen=150, nheads=4, ngroups=4)
    shape = base.replace(**kw)
    inp = S.make_inputs(shape, seed=97, with_state=True)
    check_all(shape, inp, route=abi.ROUTE_SSD)


@pytest.mark.parametrize("name", S.WORKLOAD_ORDER)
def test_workload_parity_with_state(name):
    shape = S.WORKLOADS[name].replace(**REDUCED[name]).replace(seqlen=37)
    inp = S.make_inputs(shape, seed=100 + S.WORKLOAD_ORDER.index(name), with_state=True)
    check_all(shape, inp)


@pytest.mark.parametrize("kw", [
    dict(seqlen=1),
    dict(seqlen=2),
    dict(seqlen=33, n_real=0, n_pairs=5),
    dict(seqlen=47, n_real=7, n_pairs=0),
    dict(seqlen=20, decay_mode=S.DECAY_PER_HEAD),
    dict(seqlen=29, rank_in=3, rank_out=3, ngroups=1),
    dict(seqlen=29, rank_in=2, rank_out=1),
    dict(seqlen=25, headdim=5, nheads=4, ngroups=2),
    dict(seqlen=25, headdim=48, nheads=3, ngroups=1),
    dict(seqlen=64, headdim=128, n_real=32, n_pairs=16, nheads=2),
])
@pytest.mark.parametrize("dtype", [S.DTYPE_F32, S.DTYPE_BF16])
def test_edge_shapes(kw, dtype):
    base = dict(batch=2, seqlen=16, nheads=2, headdim=16, ngroups=2, n_real=8, n_pairs=4,
                decay_mode=S.DECAY_PER_COORD, two_endpoint=1, dtype_io=dtype)
    base.update(kw)
    shape = S.ScanShape(**base)
    inp = S.make_inputs(shape, seed=7, with_state=True)
    check_all(shape, inp)


def test_empty_sequence():
    shape = S.WORKLOADS["tiny_hybrid_fp32"].replace(seqlen=0)
    inp = S.make_inputs(shape, seed=1, with_state=True)
    dev = scan.to_device(shape, inp)
    y, hT, wT = scan.scan_forward(shape, dev)
    torch.cuda.synchronize()
    assert y.numel() == 0
    np.testing.assert_array_equal(to_np(hT), inp["h0"])
    np.testing.assert_array_equal(to_np(wT), inp["w0"])
    g = scan.scan_backward(shape, dev)
    torch.cuda.synchronize()
    assert float(g.dA_log.abs().max()) == 0.0 and float(g.dh0.abs().max()) == 0.0


def test_carry_continuation_on_gpu():
    shape = S.WORKLOADS["hybridmamba"].replace(batch=1, seqlen=90, dtype_io=S.DTYPE_F32)
    inp = S.make_inputs(shape, seed=3)
    full = scan.scan_forward(shape, scan.to_device(shape, inp))
    L1 = 41
    cut = lambda a, sl: a[:, sl] if a is not None else None  # noqa: E731
    part = {k: (cut(v, slice(0, L1)) if k in ("x", "dt", "lam", "Bm", "Cm", "dy") else v)
            for k, v in inp.items()}
    s1 = shape.replace(seqlen=L1)
    y1, h1, w1 = scan.scan_forward(s1, scan.to_device(s1, part))
    rest = {k: (cut(v, slice(L1, None)) if k in ("x", "dt", "lam", "Bm", "Cm", "dy") else v)
            for k, v in inp.items()}
    s2 = shape.replace(seqlen=shape.seqlen - L1)
    dev2 = scan.to_device(s2, rest)
    dev2.h0, dev2.w0 = h1, w1
    y2, h2, _ = scan.scan_forward(s2, dev2)
    torch.cuda.synchronize()
    yc = torch.cat([y1, y2], 1)
    assert float((yc - full[0]).abs().max()) <= 1e-5 * float(full[0].abs().max())
    assert float((h2 - full[1]).abs().max()) <= 1e-5 * float(full[1].abs().max())


def test_strided_views():
    """x / y / B / C as head-strided views of wider buffers give the dense result."""
    shape = S.WORKLOADS["hybridmamba"].replace(batch=2, seqlen=40, nheads=4, ngroups=2,
                                                dtype_io=S.DTYPE_F32)
    inp = S.make_inputs(shape, seed=11)
    dev = scan.to_device(shape, inp)
    y_ref, _, _ = scan.scan_forward(shape, dev)
    d = abi.make_desc(shape)

    def widen(t, extra):
        big = torch.zeros(*t.shape[:3], t.shape[3] * t.shape[4] + extra, dtype=t.dtype,
                          device=t.device)
        big[..., : t.shape[3] * t.shape[4]] = t.reshape(*t.shape[:3], -1)
        return big

    xb, Bb, Cb = widen(dev.x, 24), widen(dev.Bm, 8), widen(dev.Cm, 40)
    yb = torch.zeros(*y_ref.shape[:3], y_ref.shape[3] * y_ref.shape[4] + 16, device="cuda")
    for arr, big in (("stride_x", xb), ("stride_B", Bb), ("stride_C", Cb), ("stride_y", yb)):
        st = getattr(d, arr)
        st[0], st[1], st[2] = big.stride(0), big.stride(1), big.stride(2)
    y = torch.zeros_like(y_ref)
    abi.ssm_scan_fwd(d, xb, dev.dt, dev.A_log, dev.theta, Bb, Cb, dev.D, dev.lam, None, None, yb)
    torch.cuda.synchronize()
    got = yb[..., : y_ref.shape[3] * y_ref.shape[4]].reshape(y_ref.shape)
    assert float((got - y_ref).abs().max()) == 0.0


@pytest.mark.parametrize("name", ["mamba2_siso", "mamba1_siso"])
def test_unaligned_tensors_take_recurrent_route(name):
    """dy 2 bytes past a 16-byte boundary: the backward cannot take the chain
    whose workspace ssm_scan_workspace_size reports; when the recurrent kernels
    need more it says so (with the size), and with their workspace it gives the
    oracle's gradients."""
    shape = S.WORKLOADS[name].replace(**REDUCED[name])
    inp = S.make_inputs(shape, seed=17)
    dev = scan.to_device(shape, inp)
    buf = torch.empty(dev.dy.numel() + 1, dtype=dev.dy.dtype, device="cuda")
    dy_off = buf[1:].view(dev.dy.shape)
    dy_off.copy_(dev.dy)
    dev.dy = dy_off
    ws = scan.alloc_workspace(shape, abi.PASS_BWD)
    try:
        g = scan.scan_backward(shape, dev, workspace=ws)
    except abi.SsmError as e:
        # the recurrent kernels need more than the chain the size was taken for
        assert e.code == -6
        need = int(re.search(r"needs (\d+) bytes", str(e)).group(1))
        assert need > ws[1]
        ws = (torch.empty(need, dtype=torch.uint8, device="cuda"), need)
        g = scan.scan_backward(shape, dev, workspace=ws)
    assert abi.ssm_scan_last_route() == abi.ROUTE_RECURRENT
    torch.cuda.synchronize()
    gr = oracle.scan_bwd(shape, inp, inp["dy"])
    for k, a, b in (("dx", g.dx, gr["dx"]), ("ddt", g.ddt, gr["ddt"]), ("dB", g.dBm, gr["dBm"]),
                    ("dC", g.dCm, gr["dCm"]), ("dA_log", g.dA_log, gr["dA_log"])):
        compare(k, to_np(a), b, shape.dtype_io)


def test_backward_deterministic():
    shape = S.WORKLOADS["mamba2_siso"].replace(batch=2, seqlen=64)
    inp = S.make_inputs(shape, seed=5)
    dev = scan.to_device(shape, inp)
    g1 = scan.scan_backward(shape, dev)
    a = [t.clone() for t in (g1.dx, g1.ddt, g1.dBm, g1.dCm, g1.dA_log, g1.dD)]
    g2 = scan.scan_backward(shape, dev)
    torch.cuda.synchronize()
    for x1, x2 in zip(a, (g2.dx, g2.ddt, g2.dBm, g2.dCm, g2.dA_log, g2.dD)):
        assert torch.equal(x1, x2)


def _scaled_dt(shape, inp, factor, rows=None):
    """Copy of the inputs with dt scaled (bf16-rounded again); `rows` limits it to
    some batch rows and a token range."""
    out = dict(inp)
    dt = inp["dt"].copy()
    if rows is None:
        dt = dt * factor
    else:
        b, t0, t1 = rows
        dt[b, t0:t1] = dt[b, t0:t1] * factor
    out["dt"] = S.round_bf16(dt) if shape.dtype_io == S.DTYPE_BF16 else dt
    return out


@pytest.mark.parametrize("kw", [dict(), dict(decay_mode=S.DECAY_PER_HEAD, two_endpoint=0,
                                             n_real=128, n_pairs=0, ngroups=2)])
def test_large_decay_takes_recurrent_route(kw):
    """Inputs whose per-sub-block decay leaves the folding range (|A| log2(e)
    sum of 16 dt > 100) give the oracle's result through the recurrent kernels
    in the per-coordinate chain; the scalar-decay chain has no range condition
    and keeps them."""
    shape = S.WORKLOADS["hybridmamba"].replace(batch=2, seqlen=150, nheads=4, ngroups=4).replace(**kw)
    inp = _scaled_dt(shape, S.make_inputs(shape, seed=41, with_state=True), 60.0)
    a_max = np.exp(inp["A_log"].max(axis=1))
    span = np.array([[inp["dt"][b, 16 * k:16 * k + 16, h].sum() for k in range(150 // 16 + 1)]
                     for b in range(2) for h in range(4)])
    assert (span.max() * a_max.max() * np.log2(np.e)) > 100.0
    bounds = None
    if ssd_eligible(shape):
        # dt scaled 60-fold makes sigma up to ~6, so the bf16 operand (dS (.) W) of the
        # dB / dC contractions reaches magnitudes where its own rounding (2^-9
        # relative, summed over the chunk's 128 rows) adds about one bf16 step of the
        # result on top of the output's own rounding: 5e-2 + 2^-7 |ref| instead of
        # 5e-2 + 2^-8 |ref| (measured: 0.122 at |ref| 17.5, bound 0.187)
        rel2 = lambda ref: 5e-2 + 2.0 ** -7 * np.abs(ref)  # noqa: E731
        bounds = {"dB": rel2, "dC": rel2}
    check_all(shape, inp, route=abi.ROUTE_SSD if ssd_eligible(shape) else abi.ROUTE_RANGE_FALLBACK,
              bounds=bounds)


def test_one_hot_sub_block_takes_recurrent_route():
    """A single out-of-range stretch in one batch row moves the whole call."""
    shape = S.WORKLOADS["hybridmamba"].replace(batch=2, seqlen=130, nheads=4, ngroups=4)
    inp = _scaled_dt(shape, S.make_inputs(shape, seed=43), 200.0, rows=(1, 70, 90))
    check_all(shape, inp, route=abi.ROUTE_RANGE_FALLBACK)


def test_moderate_decay_stays_chunked():
    """Large but in-range sub-block decays keep the tensor-core kernels and
    their parity."""
    shape = S.WORKLOADS["hybridmamba"].replace(batch=2, seqlen=140, nheads=4, ngroups=4)
    inp = S.make_inputs(shape, seed=45)
    # scale dt so that the largest sub-block exponent is about 60 (of the 100 allowed)
    a_max = np.exp(inp["A_log"].max())
    span = max(inp["dt"][b, 16 * k:16 * k + 16, h].sum()
               for b in range(2) for h in range(4) for k in range(140 // 16 + 1))
    f = 60.0 / (a_max * np.log2(np.e) * span)
    inp = _scaled_dt(shape, inp, f)
    check_all(shape, inp, route=abi.ROUTE_CHUNKED)


@pytest.mark.parametrize("kw", [dict(), dict(seqlen=64), dict(seqlen=1),
                                dict(decay_mode=S.DECAY_PER_HEAD, two_endpoint=0, n_real=128,
                                     n_pairs=0, ngroups=2),
                                dict(angle_mode=S.ANGLE_PER_TOKEN),
                                dict(two_endpoint=0, discretization=S.DISC_ZOH),
                                dict(two_endpoint=0, discretization=S.DISC_ZOH,
                                     angle_mode=S.ANGLE_PER_TOKEN, ngroups=2)])
def test_backward_from_saved_states(kw):
    """The backward that reads the forward's chunk states gives the same
    gradients as the one that recomputes them, and the oracle's.  Everything but
    dx is bit for bit; dx takes the forward's saved score and chunk-end tiles
    (summed in another order), so it agrees to bf16 rounding."""
    shape = S.WORKLOADS["hybridmamba"].replace(batch=2, seqlen=150, nheads=4, ngroups=4).replace(**kw)
    inp = S.make_inputs(shape, seed=47, with_state=True)
    dev = scan.to_device(shape, inp)
    y_inf = scan.scan_forward(shape, dev, workspace=scan.alloc_workspace(shape, abi.PASS_FWD_INFER))[0].clone()
    wsf = scan.alloc_workspace(shape, abi.PASS_FWD)
    y_tr = scan.scan_forward(shape, dev, workspace=wsf)[0]
    torch.cuda.synchronize()
    assert torch.equal(y_inf, y_tr)   # saving the backward's products changes nothing
    g_saved = scan.scan_backward(shape, dev, saved=wsf)
    assert abi.ssm_scan_last_route() == expected_route(shape, backward=True)
    g_plain = scan.scan_backward(shape, dev)
    torch.cuda.synchronize()
    abi.ssm_scan_poll_device_error()
    for name in ("ddt", "dBm", "dCm", "dA_log", "dD", "dh0", "dw0", "dtheta", "dlam"):
        a, b = getattr(g_saved, name), getattr(g_plain, name)
        if a is not None:
            assert torch.equal(a, b), name
    a, b = g_saved.dx.float(), g_plain.dx.float()
    assert float((a - b).norm() / b.norm()) < 2e-3
    gr = oracle.scan_bwd(shape, inp, inp["dy"])
    dt = shape.dtype_io
    compare("dx", to_np(g_saved.dx), gr["dx"], dt)
    compare("dA_log", to_np(g_saved.dA_log), gr["dA_log"], dt)
    compare("ddt", to_np(g_saved.ddt), gr["ddt"], dt)


@pytest.mark.parametrize("name", S.WORKLOAD_ORDER)
def test_state_only_forward(name):
    """y = NULL: only the final state and last write, equal to the full forward's."""
    shape = S.WORKLOADS[name].replace(**REDUCED[name])
    inp = S.make_inputs(shape, seed=120, with_state=True)
    dev = scan.to_device(shape, inp)
    desc = abi.make_desc(shape)
    y_ref, hT_ref, wT_ref = scan.scan_forward(shape, dev)
    route = abi.ssm_scan_last_route()
    hT, wT = torch.empty_like(hT_ref), torch.empty_like(wT_ref)
    ws, nb = scan.alloc_workspace(shape, abi.PASS_FWD, desc=desc)
    abi.ssm_scan_fwd(desc, dev.x, dev.dt, dev.A_log, dev.theta, dev.Bm, dev.Cm, dev.D, dev.lam,
                     dev.h0, dev.w0, None, hT, wT, ws, nb)
    assert abi.ssm_scan_last_route() == route
    torch.cuda.synchronize()
    abi.ssm_scan_poll_device_error()
    ref = oracle.scan_fwd(shape, inp)
    compare("hT", to_np(hT), ref["hT"], shape.dtype_io)
    compare("last_write", to_np(wT), ref["wT"], shape.dtype_io)
    assert float((hT - hT_ref).abs().max()) <= 1e-3 * max(1.0, float(hT_ref.abs().max()))
