"""Multi-rank plumbing of bench.py on CPU: two gloo ranks.

bench.py runs one independent replica per GPU (the step does not shard), so
the only cross-rank work is the barrier around the timed region and the MAX
of the per-rank times.  These checks run that plumbing with the gloo backend.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    r, w, lr = bench.rank_env()
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        got = bench.max_over_ranks(10.0 + 5.0 * r, w)
        again = bench.max_over_ranks(100.0 - r, w)
        dist.barrier()
        # the reference arm runs on rank 0 only; other ranks return at once
        other = None
        if r != 0:
            other = bench.run_reference(None, r, w)
        q.put((r, w, lr, got, again, other))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert [x[0] for x in res] == [0, 1]
    for r, w, lr, got, again, other in res:
        assert w == world and lr == r
        assert got == pytest.approx(15.0)
        assert again == pytest.approx(100.0)
        assert other is None


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25


class _FakeDecoder:
    def __init__(self, code, masked):
        import torch
        self.code = code
        self.masked = torch.tensor(masked, dtype=torch.uint8)

    def device_status(self):
        return self.code


def test_clean_run_check():
    sys.path.insert(0, ROOT)
    import bench
    bench.check_clean(_FakeDecoder(0, [0, 0]), finished=True)
    bench.check_clean(_FakeDecoder(0, [1, 0]))            # mid-run: masked rows are fine
    with pytest.raises(RuntimeError, match="status word"):
        bench.check_clean(_FakeDecoder(4, [0, 0]))
    with pytest.raises(RuntimeError, match="masked"):
        bench.check_clean(_FakeDecoder(0, [0, 1]), finished=True)
