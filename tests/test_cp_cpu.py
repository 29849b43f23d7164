"""Host side of sequence sharding (no GPU): segment bounds, the shapes that are
refused, and the all-gather of boundary values over world-size-2 gloo ranks."""
import os

import pytest

from selective_diagonal_state_b200 import cp
from selective_diagonal_state_b200 import synthetic as S

torch = pytest.importorskip("torch")


@pytest.mark.parametrize("L,n", [(300, 3), (257, 2), (7, 4), (64, 1)])
def test_segment_bounds_tile_the_sequence(L, n):
    b = [cp.segment_bounds(L, n, k) for k in range(n)]
    assert b[0][0] == 0 and b[-1][1] == L
    assert all(b[k][1] == b[k + 1][0] for k in range(n - 1))
    lens = [hi - lo for lo, hi in b]
    assert max(lens) - min(lens) <= 1


def test_segment_bounds_reject_bad_index():
    with pytest.raises(ValueError):
        cp.segment_bounds(10, 2, 2)


@pytest.mark.parametrize("kw", [dict(angle_mode=S.ANGLE_PER_TOKEN), dict(n_static=8)])
def test_unsupported_shapes_are_refused(kw):
    shape = S.WORKLOADS["hybridmamba"].replace(batch=1, seqlen=64, **kw)
    with pytest.raises(ValueError):
        cp.SegmentScan(shape, device="cpu")


def _gather_worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = torch.full((2, 3), float(rank + 1))
        g = cp.all_gather_stacked(t, world)
        q.put((rank, g.tolist()))
    finally:
        dist.destroy_process_group()


def test_all_gather_stacks_in_rank_order():
    import socket

    import torch.multiprocessing as mp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_gather_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(2):
        g = res[r]
        assert [row[0][0] for row in g] == [1.0, 2.0]   # segment k at index k
