"""tcgen05 operand and accumulator layouts (the descriptors the chunked scan
builds), checked one MMA sequence at a time against numpy."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gpu_probes", "umma_probe.cu")
OUT = os.path.join(HERE, "_build", "umma_probe.cubin")


@pytest.fixture(scope="module")
def probe():
    os.makedirs(os.path.dirname(OUT), exist_ok=True)
    subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2",
                           "-cubin", SRC, "-o", OUT])
    from cuda.bindings import driver as cu  # cuda-python
    torch.cuda.init()
    torch.zeros(1, device="cuda")
    err, mod = cu.cuModuleLoad(OUT.encode())
    assert err == cu.CUresult.CUDA_SUCCESS, err
    err, fn = cu.cuModuleGetFunction(mod, b"umma_probe")
    assert err == cu.CUresult.CUDA_SUCCESS, err
    return cu, fn


def bf16(a):
    return torch.from_numpy(a).to(torch.bfloat16).float().numpy()


@pytest.mark.parametrize("M,N,K,a_code,b_code,d_lane", [
    (128, 64, 32, 0, 0, 0),   # K-major A and B
    (128, 64, 64, 1, 2, 0),   # MN-major A, 128B-swizzled MN-major B (state MMA shape)
    (64, 64, 64, 2, 1, 0),    # swizzled MN-major A (X^T), MN-major B (P^T)
    (64, 16, 64, 0, 0, 16),   # M=64 accumulator in the upper half-lanes
    (64, 64, 32, 1, 0, 0),    # MN-major A (state^T), K-major B
    (64, 64, 64, 3, 3, 0),    # 128B-swizzled K-major A and B (dY . X^T)
    (128, 64, 64, 0, 3, 0),   # K-major A (state rows), swizzled K-major B (K_prev . dY^T)
    (128, 16, 32, 1, 0, 0),   # MN-major A read from a K-major tile, K-major B (B_i^T . Gm^T)
])
def test_umma_layout(probe, M, N, K, a_code, b_code, d_lane):
    cu, fn = probe
    rng = np.random.default_rng(M + N + K + a_code + b_code)
    A = rng.standard_normal((M, K)).astype(np.float32)
    B = rng.standard_normal((N, K)).astype(np.float32)
    dA = torch.from_numpy(A).cuda()
    dB = torch.from_numpy(B).cuda()
    dD = torch.full((M, N), float("nan"), device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    args = [ctypes.c_int(M), ctypes.c_int(N), ctypes.c_int(K), ctypes.c_int(a_code),
            ctypes.c_int(b_code), ctypes.c_int(d_lane), ctypes.c_void_p(dA.data_ptr()),
            ctypes.c_void_p(dB.data_ptr()), ctypes.c_void_p(dD.data_ptr()),
            ctypes.c_void_p(st.data_ptr())]
    ptrs = (ctypes.c_void_p * len(args))(*[ctypes.addressof(a) for a in args])
    err, = cu.cuLaunchKernel(fn, 1, 1, 1, 128, 1, 1, 0, 0, ctypes.addressof(ptrs), 0)
    assert err == cu.CUresult.CUDA_SUCCESS, err
    torch.cuda.synchronize()
    assert int(st.item()) == 0, "mbarrier wait timed out"
    ref = bf16(A) @ bf16(B).T
    got = dD.cpu().numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-4, atol=1e-3)
