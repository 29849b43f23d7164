"""Data-parallel path on CPU with world size 2 (gloo): every rank scans its own
batch rows and the per-head parameter gradients are all-reduced.  The compute
here is the fp64 oracle (no GPU on this host); what is tested is the sharding
and the exchange, which the benchmark uses unchanged over NCCL."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from selective_diagonal_state_b200 import dist as sdist
from selective_diagonal_state_b200 import synthetic as S

SHAPE = S.WORKLOADS["hybridmamba"].replace(batch=5, seqlen=24, nheads=2, ngroups=2,
                                            dtype_io=S.DTYPE_F32)
BATCHED = ("x", "dt", "lam", "Bm", "Cm", "dy", "h0", "w0")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = S.make_inputs(SHAPE, seed=4, with_state=True)
        lo, hi = sdist.shard_batch(SHAPE.batch, world, rank)
        part = {k: (v[lo:hi] if k in BATCHED else v) for k, v in inp.items()}
        sh = SHAPE.replace(batch=hi - lo)
        g = oracle.scan_bwd(sh, part, part["dy"])
        params = [torch.from_numpy(g[k].copy()) for k in ("dA_log", "dtheta", "dD")]
        sdist.allreduce_param_grads(params)
        out[rank] = {"lo": lo, "hi": hi, "dx": g["dx"], "dBm": g["dBm"],
                     "params": [p.numpy() for p in params]}
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_data_parallel_param_grads_match_full_batch(world):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    inp = S.make_inputs(SHAPE, seed=4, with_state=True)
    full = oracle.scan_bwd(SHAPE, inp, inp["dy"])
    for r in range(world):
        res = out[r]
        np.testing.assert_allclose(res["dx"], full["dx"][res["lo"]:res["hi"]], rtol=1e-12,
                                   atol=1e-12)
        np.testing.assert_allclose(res["dBm"], full["dBm"][res["lo"]:res["hi"]], rtol=1e-12,
                                   atol=1e-12)
        for got, key in zip(res["params"], ("dA_log", "dtheta", "dD")):
            np.testing.assert_allclose(got, full[key], rtol=1e-10, atol=1e-12)


def test_shard_batch_covers_every_row_once():
    for batch in (1, 5, 8, 13):
        for world in (1, 2, 3, 8):
            rows = []
            for r in range(world):
                lo, hi = sdist.shard_batch(batch, world, r)
                rows += list(range(lo, hi))
            assert rows == list(range(batch))
