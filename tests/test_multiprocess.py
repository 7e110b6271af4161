"""The N > 1 path of bench.py on CPU: two gloo ranks (replicas, no data-path
collective) agree on the slowest rank's time and the whole-job throughput,
and the reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import bench
    w, r, _ = bench.dist_setup(None)
    ms_local = 100.0 + 50.0 * rank                  # rank 1 is the slow one
    ms_max, value = bench.aggregate(w, 4096, 8, ms_local)
    bench.dist_barrier(w)
    from qi21_synth import configs as C

    class A:
        warmup, steps, gpus = 0, 1, world
    rc = bench.run_reference(A, C.make_workload("toy"), w, r) if r == 1 else 0
    bench.dist_done(w)
    q.put((rank, w, ms_max, value, rc))


@pytest.mark.timeout(180)
def test_two_gloo_ranks_report_max_time_and_total_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(150)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, world, ms_max, value, rc in res:
        assert world == 2
        assert ms_max == 150.0                       # the slowest rank's time on every rank
        assert abs(value - 2 * 4096 * 8 / 0.150) < 1e-6
        assert rc == 0                               # non-zero ranks of the reference arm exit cleanly
