"""The multi-GPU plumbing of bench.py with world_size 2 on the gloo backend (CPU).

One process per GPU, each rank processing its own batch: the only collective
steps are the barrier and the max over ranks of the timed region.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    import workloads
    w, r, _ = bench.dist_setup()
    try:
        bench.barrier(w)
        # each rank draws its own batch (weak scaling): different seeds give different data
        wl = workloads.generate("prefill", B=1, S=8, Nk=2, Nv=4, D=16, seed=2 + 1000 * r)
        slow = bench.all_max(10.0 + r, w)
        rate = bench.weak_scaling_rate(int(wl.lengths.sum()), 5, slow, w)
        q.put((r, slow, rate, float(wl.q[0, 0, 0, 0])))
        bench.barrier(w)
    finally:
        import torch.distributed as dist
        dist.destroy_process_group()


def test_two_rank_gloo_max_and_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0, p.exitcode
    res = sorted(q.get(timeout=10) for _ in range(2))
    # both ranks agree on the slowest rank's time and on the job rate
    assert res[0][1] == res[1][1] == 11.0
    assert res[0][2] == res[1][2] == pytest.approx(2 * 8 * 5 / 0.011)
    # and their batches differ
    assert res[0][3] != res[1][3]


def test_single_rank_rate():
    import bench
    assert bench.weak_scaling_rate(16384, 10, 100.0, 1) == pytest.approx(1638400.0)
