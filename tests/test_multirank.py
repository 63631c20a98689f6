"""The benchmark's N > 1 path on CPU: two gloo ranks run the cross-rank pieces bench.py
uses under torchrun (rank environment, barriers, the maximum of the per-rank step times,
the whole-job throughput, the reference arm's rank-0-only rule).  Requests are
independent, so nothing else crosses ranks."""
import multiprocessing as mp
import os
import socket
import sys
from datetime import timedelta

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        w, r, local = bench.rank_env()
        bench.barrier(w)
        step_ms = [0.8, 1.3][rank]                      # per-rank device times of one step
        m = bench.max_over_ranks(step_ms, w, "cpu")
        value = bench.job_value(w, 32, m)
        ref = "not run"
        if rank == 1:
            class Args:
                workload, steps, warmup = "csa_decode_bf16_128k", 1, 0
            ref = bench.run_reference(Args())          # ranks other than 0 do no work
        bench.barrier(w)
        q.put((rank, w, r, local, m, value, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, w, r, local, m, value, ref in res:
        assert (w, r, local) == (2, rank, rank)
        assert m == 1.3                                 # the slowest rank's step time
        assert abs(value - 2 * 32 / 1.3e-3) < 1e-6      # both ranks' requests over that time
    assert res[1][6] is None
