"""The benchmark's multi-process plumbing on CPU with the gloo backend
(world size 2): process-group set-up from the launcher's environment, the
barrier, and the max / sum reductions the timing uses.  With N GPUs every
rank runs an independent replica of the same workload (the path does not
shard), so these reductions are the only cross-rank steps."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "S12_BENCH_BACKEND": "gloo"})
    import bench
    import torch.distributed as dist
    w, r, local = bench.dist_init()
    assert (w, r, local) == (world, rank, rank)
    bench.barrier(w)
    mx = bench.max_over_ranks(1.5 + rank, w)
    sm = bench.sum_over_ranks(10.0 * (rank + 1), w)
    bench.barrier(w)
    q.put((rank, mx, sm))
    dist.destroy_process_group()


def test_two_rank_reductions_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, mx, sm in got:
        assert mx == pytest.approx(2.5)   # the slowest rank's time
        assert sm == pytest.approx(30.0)  # units summed over ranks


def test_single_process_needs_no_group():
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.sum_over_ranks(3.0, 1) == 3.0
    bench.barrier(1)
