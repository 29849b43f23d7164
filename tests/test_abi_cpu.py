"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/ssm_scan.h declares, and rejects bad arguments before
any launch."""
import ctypes
import os
import re

import pytest

from selective_diagonal_state_b200 import abi, build
from selective_diagonal_state_b200 import synthetic as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssm_scan.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return abi.load_library()


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"SSM_API\s+[\w\s\*]+?\b(ssm_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    syms = set(declared_symbols())
    assert {"ssm_scan_fwd", "ssm_scan_bwd", "ssm_scan_workspace_size",
            "ssm_scan_last_error"} <= syms


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert set(abi.EXPORTED) >= set(declared_symbols())


def test_abi_version(lib):
    assert abi.ssm_scan_abi_version() == 3


def test_desc_layout_matches_header(lib):
    """ssm_desc_t: five int64 sizes, eight int32 fields, six int64[3] stride
    arrays, angle_mode, n_static, discretization and a reserved word: 208
    bytes, no padding."""
    assert ctypes.sizeof(abi.Desc) == 5 * 8 + 8 * 4 + 6 * 3 * 8 + 4 * 4
    assert abi.Desc.angle_mode.offset == 5 * 8 + 8 * 4 + 6 * 3 * 8


def test_angle_mode_validation(lib):
    sh = S.WORKLOADS["hybridmamba"].replace(batch=2, seqlen=100)
    d = abi.make_desc(sh)
    d.angle_mode = 2
    assert abi.ssm_scan_workspace_size(d, abi.PASS_FWD) == 0
    assert b"angle_mode" in lib.ssm_scan_last_error()
    d.angle_mode = 0
    for bad in (-1, sh.n_real + 1):
        d.n_static = bad
        assert abi.ssm_scan_workspace_size(d, abi.PASS_FWD) == 0
        assert b"n_static" in lib.ssm_scan_last_error()
    d.n_static = 0
    d.discretization = 2
    assert abi.ssm_scan_workspace_size(d, abi.PASS_FWD) == 0
    assert b"discretization" in lib.ssm_scan_last_error()
    d.discretization = S.DISC_ZOH          # ZOH needs the Euler form (two_endpoint == 0)
    assert abi.ssm_scan_workspace_size(d, abi.PASS_FWD) == 0
    assert b"ZOH" in lib.ssm_scan_last_error()
    d.two_endpoint = 0
    # the ZOH write takes the tensor-core chain: the same workspace as the Euler form
    zoh_ws = abi.ssm_scan_workspace_size(d, abi.PASS_FWD)
    d.discretization = 0
    assert zoh_ws == abi.ssm_scan_workspace_size(d, abi.PASS_FWD) > 0
    d.discretization = 0
    d.reserved_ = 1
    assert abi.ssm_scan_workspace_size(d, abi.PASS_FWD) == 0
    # static rows run on the recurrent kernels too
    st = abi.make_desc(sh.replace(n_static=16))
    assert st.n_static == 16
    assert abi.ssm_scan_workspace_size(st, abi.PASS_FWD) == 0
    # per-token angles take the tensor-core chain as static ones do: the same
    # chunk workspace
    pt = abi.make_desc(sh.replace(angle_mode=S.ANGLE_PER_TOKEN))
    assert abi.ssm_scan_workspace_size(pt, abi.PASS_FWD) == \
        abi.ssm_scan_workspace_size(abi.make_desc(sh), abi.PASS_FWD) > 0


def test_wait_limit_setter(lib):
    old = abi.ssm_scan_set_wait_limit(123)
    assert old == 1 << 22
    assert abi.ssm_scan_set_wait_limit(old) == 123
    with pytest.raises(abi.SsmError) as ei:
        abi.ssm_scan_set_wait_limit(-1)
    assert ei.value.code == -1
    assert abi.ssm_scan_set_wait_limit(old) == old


def test_contiguous_strides(lib):
    sh = S.WORKLOADS["ssd_mimo_r4"]
    d = abi.make_desc(sh)
    N, P, R, O, H, G, L = sh.nstate, sh.headdim, sh.rank_in, sh.rank_out, sh.nheads, sh.ngroups, sh.seqlen
    assert list(d.stride_x) == [L * H * R * P, H * R * P, R * P]
    assert list(d.stride_y) == [L * H * O * P, H * O * P, O * P]
    assert list(d.stride_B) == [L * G * R * N, G * R * N, R * N]
    assert list(d.stride_C) == [L * G * O * N, G * O * N, O * N]
    assert list(d.stride_dt) == [L * H, H, 1]


def test_workspace_size(lib):
    sh = S.WORKLOADS["hybridmamba"].replace(batch=2, seqlen=100)
    d = abi.make_desc(sh)
    # tensor-core chain: a forward alone needs the two fp32 carry slots and the
    # counter of every (b, h); a training forward also keeps, per chunk, the
    # entering state (32 KB), the chunk decays and the products the backward
    # reuses (8 + 16 KB + 64 floats)
    nc = (100 + 63) // 64
    ni = abi.ssm_scan_workspace_size(d, abi.PASS_FWD_INFER)
    assert ni >= 2 * 32 * 2 * 128 * 64 * 4 + (2 * 32 + 2) * 4 and ni % 256 == 0
    nf = abi.ssm_scan_workspace_size(d, abi.PASS_FWD)
    assert nf % 256 == 0
    assert nf - ni >= 2 * 32 * nc * (128 * 64 * 4 + 128 * 2 * 4 + 8192 + 16384 + 256)
    # the recurrent chain needs none
    for kw in (dict(chunk=1), dict(dtype_io=S.DTYPE_F32), dict(headdim=32)):
        assert abi.ssm_scan_workspace_size(abi.make_desc(sh.replace(**kw)), abi.PASS_FWD) == 0
    n = abi.ssm_scan_workspace_size(d, abi.PASS_BWD)
    BLH = 2 * 100 * 32
    assert n >= BLH * (2 * 128 + 2 + 1) * 4
    assert n % 256 == 0
    bad = abi.make_desc(sh)
    bad.ngroups = 5
    assert abi.ssm_scan_workspace_size(bad, abi.PASS_BWD) == 0


def _fwd_status(lib, d, **ptrs):
    names = ["x", "dt", "A_log", "theta", "B", "C", "D", "lam", "h0", "w0", "y", "hT", "wT", "ws"]
    args = [ptrs.get(n) for n in names]
    return lib.ssm_scan_fwd(ctypes.byref(d) if d is not None else None, *args, 0, None)


FAKE = 1 << 40  # never dereferenced: validation fails first


@pytest.mark.parametrize("mutate,code", [
    (lambda d: setattr(d, "ngroups", 5), -1),
    (lambda d: setattr(d, "nheads", 0), -1),
    (lambda d: setattr(d, "decay_mode", 7), -1),
    (lambda d: setattr(d, "dtype_io", 3), -1),
    (lambda d: setattr(d, "two_endpoint", 2), -1),
    (lambda d: (setattr(d, "n_real", 0), setattr(d, "n_pairs", 0)), -1),
    (lambda d: d.stride_x.__setitem__(1, -4), -1),
    (lambda d: setattr(d, "batch", 70000), -2),
])
def test_bad_descriptor_rejected(lib, mutate, code):
    d = abi.make_desc(S.WORKLOADS["tiny_hybrid_fp32"])
    mutate(d)
    full = dict(x=FAKE, dt=FAKE, A_log=FAKE, theta=FAKE, B=FAKE, C=FAKE, D=FAKE, lam=FAKE, y=FAKE)
    assert _fwd_status(lib, d, **full) == code
    assert lib.ssm_scan_last_error().decode()


def test_null_descriptor(lib):
    assert _fwd_status(lib, None) == -1


@pytest.mark.parametrize("missing", ["x", "dt", "A_log", "theta", "B", "C", "D", "lam", "y"])
def test_missing_pointer_rejected(lib, missing):
    d = abi.make_desc(S.WORKLOADS["tiny_hybrid_fp32"])
    full = dict(x=FAKE, dt=FAKE, A_log=FAKE, theta=FAKE, B=FAKE, C=FAKE, D=FAKE, lam=FAKE, y=FAKE)
    full[missing] = None
    assert _fwd_status(lib, d, **full) == -1
    assert missing in lib.ssm_scan_last_error().decode()


def test_misaligned_pointer_rejected(lib):
    d = abi.make_desc(S.WORKLOADS["mamba2_siso"])
    full = dict(x=FAKE + 1, dt=FAKE, A_log=FAKE, B=FAKE, C=FAKE, D=FAKE, y=FAKE)
    assert _fwd_status(lib, d, **full) == -3


def test_backward_needs_workspace(lib):
    d = abi.make_desc(S.WORKLOADS["hybridmamba"].replace(batch=1, seqlen=8))
    p = [FAKE] * 22
    rc = lib.ssm_scan_bwd(ctypes.byref(d), *p, 0, None)
    assert rc == -6
    assert "workspace" in lib.ssm_scan_last_error().decode()


def test_unsupported_rank_reported(lib):
    d = abi.make_desc(S.WORKLOADS["tiny_hybrid_fp32"].replace(rank_in=8, rank_out=8))
    full = dict(x=FAKE, dt=FAKE, A_log=FAKE, theta=FAKE, B=FAKE, C=FAKE, D=FAKE, lam=FAKE, y=FAKE)
    assert _fwd_status(lib, d, **full) == -2


def test_host_tensor_refused():
    torch = pytest.importorskip("torch")
    with pytest.raises(ValueError):
        abi._ptr(torch.zeros(3))


def _step_status(lib, d, **ptrs):
    names = ["x", "dt", "A_log", "theta", "B", "C", "D", "lam", "h", "w", "y"]
    return lib.ssm_scan_step(ctypes.byref(d), *[ptrs.get(n) for n in names], None)


def test_step_argument_checks(lib):
    full = dict(x=FAKE, dt=FAKE, A_log=FAKE, theta=FAKE, B=FAKE, C=FAKE, D=FAKE, lam=FAKE,
                h=FAKE, w=FAKE, y=FAKE)
    d = abi.make_desc(S.WORKLOADS["tiny_hybrid_fp32"].replace(seqlen=3))
    assert _step_status(lib, d, **full) == -1          # one token per call
    assert "one token" in lib.ssm_scan_last_error().decode()
    d = abi.make_desc(S.WORKLOADS["tiny_hybrid_fp32"].replace(seqlen=1))
    assert _step_status(lib, d, **dict(full, w=None)) == -1     # two-endpoint needs w
    assert "w" in lib.ssm_scan_last_error().decode()
    assert _step_status(lib, d, **dict(full, h=None)) == -1
    d = abi.make_desc(S.WORKLOADS["tiny_hybrid_fp32"].replace(seqlen=1, rank_in=9, rank_out=9))
    assert _step_status(lib, d, **full) == -2


def test_preact_argument_checks(lib):
    d = abi.make_desc(S.WORKLOADS["hybridmamba"].replace(batch=1, seqlen=8))
    ok = dict(z=FAKE, bias=FAKE, logit=FAKE, dt=FAKE, lam=FAKE)
    def fwd(**kw):
        a = dict(ok, **kw)
        return lib.ssm_preact_fwd(ctypes.byref(d), a["z"], a["bias"], a["logit"], a["dt"], a["lam"], None)
    assert fwd(z=None) == -1 and "z" in lib.ssm_scan_last_error().decode()
    assert fwd(bias=None) == -1
    assert fwd(lam=None) == -1          # two-endpoint shapes need lambda
    assert fwd(z=FAKE + 1) == -3        # bf16 tensors need 2-byte alignment
    assert lib.ssm_preact_bwd(ctypes.byref(d), FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE,
                              None) == -1


def test_sequence_sharding_calls_validate_before_launch(lib):
    """The ssm_cp_* calls check their arguments on the host (nothing is launched)."""
    sh = S.WORKLOADS["hybridmamba"].replace(batch=2, seqlen=100)
    d = abi.make_desc(sh)
    assert lib.ssm_cp_tail_rows(ctypes.byref(d)) == 2 * sh.nstate        # bf16: value + remainder
    d32 = abi.make_desc(S.WORKLOADS["tiny_hybrid_fp32"])
    assert lib.ssm_cp_tail_rows(ctypes.byref(d32)) == S.WORKLOADS["tiny_hybrid_fp32"].nstate
    bad = abi.make_desc(sh)
    bad.ngroups = 5
    assert lib.ssm_cp_tail_rows(ctypes.byref(bad)) == -1
    p = [FAKE] * 8
    # segment index out of range
    assert lib.ssm_cp_state_combine(ctypes.byref(d), 2, 2, *p, None) == -1
    assert "segment" in lib.ssm_scan_last_error().decode()
    assert lib.ssm_cp_adjoint_combine(ctypes.byref(d), 0, 0, *p[:6], None) == -1
    # missing outputs
    assert lib.ssm_cp_state_combine(ctypes.byref(d), 2, 1, FAKE, FAKE, FAKE, FAKE, None, None,
                                    None, FAKE, None) == -1
    assert "h_in" in lib.ssm_scan_last_error().decode()
    # the end-adjoint rows cannot carry per-token angles or static rows through
    for kw in (dict(angle_mode=S.ANGLE_PER_TOKEN), dict(n_static=8)):
        dd = abi.make_desc(sh.replace(**kw))
        assert lib.ssm_cp_fill_tail(ctypes.byref(dd), *([FAKE] * 7), None) == -2
    # the fill takes every input row buffer or none of them (dy only), and always dy
    assert lib.ssm_cp_fill_tail(ctypes.byref(d), None, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                                None) == -1
    assert "x" in lib.ssm_scan_last_error().decode()
    assert lib.ssm_cp_fill_tail(ctypes.byref(d), *([None] * 5), None, None, None) == -1
    assert "dy" in lib.ssm_scan_last_error().decode()
    # transition: n_pairs above 64
    wide = abi.make_desc(S.WORKLOADS["tiny_hybrid_fp32"].replace(n_real=0, n_pairs=65))
    assert lib.ssm_cp_segment_transition(ctypes.byref(wide), *([FAKE] * 6), None) == -2


def test_gated_forward_and_state_only_forward_validate(lib):
    """The gated forward needs z and y; a plain forward may drop y (state only)
    but not every output."""
    d = abi.make_desc(S.WORKLOADS["tiny_hybrid_fp32"])
    ins = [FAKE] * 10   # x, dt, A_log, theta, B, C, D, lambda, h0, prev_write
    # z missing
    rc = lib.ssm_scan_fwd_gated(ctypes.byref(d), *ins, None, FAKE, None, FAKE, None, None, 0, None)
    assert rc == -1 and "z" in lib.ssm_scan_last_error().decode()
    # y_gated missing
    rc = lib.ssm_scan_fwd_gated(ctypes.byref(d), *ins, FAKE, None, None, FAKE, None, None, 0, None)
    assert rc == -1 and "y" in lib.ssm_scan_last_error().decode()
    # state-only forward with nothing to write
    rc = lib.ssm_scan_fwd(ctypes.byref(d), *ins, None, None, None, None, 0, None)
    assert rc == -1 and "NULL" in lib.ssm_scan_last_error().decode()
    # the gate's backward checks every pointer
    rc = lib.ssm_gate_bwd(ctypes.byref(d), FAKE, None, FAKE, FAKE, FAKE, None)
    assert rc == -1 and "y_pre" in lib.ssm_scan_last_error().decode()
