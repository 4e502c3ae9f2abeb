"""The bench's multi-process plumbing on CPU (gloo, world size 2): process
group set-up from the torchrun environment, the max-over-ranks timing rule,
and the weak-scaling whole-job value (units of all ranks / slowest rank)."""
import os
import socket

import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist

    import bench

    w, r, _ = bench.setup_dist(None, backend="gloo")
    # rank r "took" 10 + 5r ms for the same per-rank work
    ms = bench.max_over_ranks(10.0 + 5.0 * r, w)
    bench.barrier(w)
    flops_per_rank = 8.0e12
    value = w * flops_per_rank / (ms * 1e-3) / 1e12
    q.put((r, w, ms, value))
    dist.destroy_process_group()


def test_two_rank_max_and_weak_scaling_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [2, 2]
    assert all(o[2] == 15.0 for o in out)  # every rank reports the slowest rank's time
    assert abs(out[0][3] - 2 * 8.0 / 0.015) < 1e-6
