"""GPU parity of the recurrent step (decoding): calling ssm_scan_step once per
token, from h0 / prev_write, reproduces the oracle's sequence forward -- every
token's output, the final state and the last write."""
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


def step_through(shape, inp, with_w=True):
    """Run ssm_scan_step token by token on device slices of the full tensors."""
    dev = scan.to_device(shape, inp)
    desc = abi.make_desc(shape)          # strides of the whole sequence ...
    desc.seqlen = 1                      # ... one token per call
    h = dev.h0.clone()
    w = dev.w0.clone() if with_w else None
    y = torch.zeros((shape.batch, shape.seqlen, shape.nheads, shape.rank_out, shape.headdim),
                    dtype=scan.io_dtype(shape), device="cuda")
    per_token = shape.angle_mode == S.ANGLE_PER_TOKEN and shape.n_pairs
    for t in range(shape.seqlen):
        lam_t = dev.lam[:, t] if shape.two_endpoint else None
        th = dev.theta[:, t].contiguous() if per_token else dev.theta   # dense [B][H][np]
        abi.ssm_scan_step(desc, dev.x[:, t], dev.dt[:, t], dev.A_log, th, dev.Bm[:, t],
                          dev.Cm[:, t], dev.D, lam_t, h, w, y[:, t])
    torch.cuda.synchronize()
    abi.ssm_scan_poll_device_error()
    return y, h, w


CASES = {
    "tiny_hybrid_fp32": dict(seqlen=9),
    "hybridmamba": dict(batch=2, nheads=4, ngroups=4, seqlen=7),
    "mamba2_siso": dict(batch=2, nheads=6, ngroups=3, seqlen=6),
    "mamba1_siso": dict(batch=2, nheads=64, seqlen=6),
    "ssd_mimo_r4": dict(batch=1, nheads=2, ngroups=2, seqlen=5),
}


@pytest.mark.parametrize("name", list(CASES))
def test_steps_match_sequence(name):
    shape = S.WORKLOADS[name].replace(**CASES[name])
    inp = S.make_inputs(shape, seed=11, with_dy=False, with_state=True)
    y, h, w = step_through(shape, inp)
    ref = oracle.scan_fwd(shape, inp)
    compare("y", to_np(y), ref["y"], shape.dtype_io)
    compare("hT", to_np(h), ref["hT"], shape.dtype_io)
    compare("last_write", to_np(w), ref["wT"], shape.dtype_io)


def test_steps_with_per_token_angles():
    shape = S.WORKLOADS["hybridmamba"].replace(batch=2, nheads=4, ngroups=4, seqlen=7,
                                               angle_mode=S.ANGLE_PER_TOKEN)
    inp = S.make_inputs(shape, seed=14, with_dy=False, with_state=True)
    y, h, w = step_through(shape, inp)
    ref = oracle.scan_fwd(shape, inp)
    compare("y", to_np(y), ref["y"], shape.dtype_io)
    compare("hT", to_np(h), ref["hT"], shape.dtype_io)
    compare("last_write", to_np(w), ref["wT"], shape.dtype_io)


def test_steps_with_static_rows():
    shape = S.WORKLOADS["hybridmamba"].replace(batch=2, nheads=4, ngroups=4, seqlen=7,
                                               n_static=24)
    inp = S.make_inputs(shape, seed=15, with_dy=False, with_state=True)
    y, h, w = step_through(shape, inp)
    ref = oracle.scan_fwd(shape, inp)
    compare("y", to_np(y), ref["y"], shape.dtype_io)
    compare("hT", to_np(h), ref["hT"], shape.dtype_io)
    compare("last_write", to_np(w), ref["wT"], shape.dtype_io)


@pytest.mark.parametrize("kw", [dict(), dict(angle_mode=S.ANGLE_PER_TOKEN)])
def test_steps_with_zoh_write(kw):
    shape = S.WORKLOADS["hybridmamba"].replace(batch=2, nheads=4, ngroups=4, seqlen=7,
                                               two_endpoint=0, discretization=S.DISC_ZOH, **kw)
    inp = S.make_inputs(shape, seed=16, with_dy=False, with_state=True)
    y, h, w = step_through(shape, inp)
    ref = oracle.scan_fwd(shape, inp)
    compare("y", to_np(y), ref["y"], shape.dtype_io)
    compare("hT", to_np(h), ref["hT"], shape.dtype_io)
    compare("last_write", to_np(w), ref["wT"], shape.dtype_io)


@pytest.mark.parametrize("kw", [
    # sixteen channels per head, up to nine heads per CTA, ranks 8: the staged kernel
    # with 83 KB of coefficients (above the default shared-memory limit)
    dict(headdim=16, nheads=18, ngroups=9, n_real=96, n_pairs=16, rank_in=8, rank_out=8),
    # 256 state rows at ranks 8: 166 KB of coefficients, too large for shared memory,
    # the per-channel kernel
    dict(headdim=16, nheads=9, ngroups=9, n_real=128, n_pairs=64, rank_in=8, rank_out=8),
    # one channel per head: the per-channel kernel
    dict(headdim=1, nheads=256, ngroups=2, n_real=12, n_pairs=2, rank_in=2, rank_out=3),
    # a head width that does not divide the CTA (its heads straddle CTAs)
    dict(headdim=48, nheads=5, ngroups=5, n_real=9, n_pairs=3),
])
def test_steps_kernel_layouts(kw):
    """The step's CTA layouts: several heads per CTA, heads straddling CTAs, and the
    per-channel kernel taken for one-channel heads or coefficients too large for
    shared memory."""
    shape = S.WORKLOADS["tiny_hybrid_fp32"].replace(batch=2, seqlen=5, **kw)
    inp = S.make_inputs(shape, seed=17, with_dy=False, with_state=True)
    y, h, w = step_through(shape, inp)
    ref = oracle.scan_fwd(shape, inp)
    compare("y", to_np(y), ref["y"], shape.dtype_io)
    compare("hT", to_np(h), ref["hT"], shape.dtype_io)
    compare("last_write", to_np(w), ref["wT"], shape.dtype_io)


def test_euler_write_needs_no_w():
    shape = S.WORKLOADS["tiny_hybrid_fp32"].replace(seqlen=6, two_endpoint=0)
    inp = S.make_inputs(shape, seed=12, with_dy=False, with_state=True)
    inp["w0"] = np.zeros_like(inp["w0"])   # the Euler write never reads a previous write
    y, h, _ = step_through(shape, inp, with_w=False)
    ref = oracle.scan_fwd(shape, inp)
    compare("y", to_np(y), ref["y"], shape.dtype_io)
    compare("hT", to_np(h), ref["hT"], shape.dtype_io)


def test_step_continues_a_forward_call():
    """A prompt through ssm_scan_fwd, then decoding steps from its (hT, last_write)."""
    shape = S.WORKLOADS["hybridmamba"].replace(batch=1, nheads=2, ngroups=2, seqlen=70)
    inp = S.make_inputs(shape, seed=13, with_dy=False, with_state=True)
    L0 = 66
    pre = {k: (v[:, :L0] if k in ("x", "dt", "lam", "Bm", "Cm") else v) for k, v in inp.items()}
    dev_pre = scan.to_device(shape.replace(seqlen=L0), pre)
    _, hT, wT = scan.scan_forward(shape.replace(seqlen=L0), dev_pre)
    post_shape = shape.replace(seqlen=shape.seqlen - L0)
    post = {k: (v[:, L0:] if k in ("x", "dt", "lam", "Bm", "Cm") else v) for k, v in inp.items()}
    post["h0"], post["w0"] = to_np(hT).astype(np.float32), to_np(wT).astype(np.float32)
    y, h, w = step_through(post_shape, post)
    ref = oracle.scan_fwd(shape, inp)
    compare("y", to_np(y), ref["y"][:, L0:], shape.dtype_io)
    compare("hT", to_np(h), ref["hT"], shape.dtype_io)
    compare("last_write", to_np(w), ref["wT"], shape.dtype_io)
