"""The multi-process plumbing of bench.py (one process per GPU under torchrun) on
the CPU: two gloo ranks rendezvous on 127.0.0.1 from the torchrun environment
variables, the timing reduction takes the maximum over ranks, the barrier
returns on every rank, and the process group shuts down cleanly.  The mixer
itself has no exchange step (rows are independent): several GPUs run replicas."""
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(None)
    t = bench.max_over_ranks(10.0 + 5.0 * r, w)  # per-rank times: the job's time is the slowest rank's
    bench.barrier(w)
    q.put((r, w, t, dist.get_backend()))
    dist.destroy_process_group()


def test_two_gloo_ranks_reduce_the_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res == [(0, 2, 15.0, "gloo"), (1, 2, 15.0, "gloo")]
