"""The N > 1 paths on CPU, as two gloo ranks.

* bench.py under torchrun: the rank environment, barriers, the maximum of the per-rank step
  times, the whole-job throughput, the reference arm's rank-0-only rule (requests are
  independent, so nothing else crosses ranks);
* context parallelism for one long request (long_context_sparse_06_b200.cp): the exchange of
  top-k candidates and attention partials between ranks that each hold a shard of the
  entries, with the per-rank compute done by the oracle.
"""
import multiprocessing as mp
import os
import socket
import sys
from datetime import timedelta

import numpy as np

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


# ------------------------------------------------- context parallelism over two gloo ranks
class _OracleOps:
    """The per-rank compute of the CP step done by the oracle on CPU tensors, so that the
    exchange itself (shards, offsets, rank order, the merge) runs over two real ranks."""

    def __init__(self, orc):
        self.orc = orc

    def index_topk(self, qI, w, kI, k, N_c):
        import torch
        sc = [self.orc.index_scores_f32(qI[b].numpy(), w[b].numpy(), kI[b].numpy()) for b in range(qI.shape[0])]
        idx = [self.orc.topk(s, k) for s in sc]
        return torch.from_numpy(np.stack(idx)), torch.from_numpy(np.stack(sc))

    def candidates(self, scores, idx, offset):
        import torch
        valid = idx >= 0
        cs = torch.where(valid, torch.gather(scores, 1, idx.clamp(min=0).long()), torch.tensor(-np.inf))
        ci = torch.where(valid, idx + offset, torch.tensor(-1, dtype=torch.int32))
        return cs.float(), ci.int()

    def select(self, cs, ci, offset, S):
        import torch
        G, B, k = cs.shape
        rows = cs.permute(1, 0, 2).reshape(B, G * k).numpy()
        cidx = ci.permute(1, 0, 2).reshape(B, G * k).numpy()
        ig = np.full((B, k), -1, np.int32)
        il = np.full((B, k), -1, np.int32)
        for b in range(B):
            pos = self.orc.topk(rows[b], k)
            g = [int(cidx[b, p]) for p in pos if p >= 0 and cidx[b, p] >= 0]
            ig[b, :len(g)] = g
            loc = [x - offset for x in g if offset <= x < offset + S]
            il[b, :len(loc)] = loc
        return torch.from_numpy(ig), torch.from_numpy(il)

    def attend(self, q, comp, win, idx_local, d_v, scale):
        import torch
        B, H, D = q.shape
        o, lse = np.zeros((B, H, d_v)), np.zeros((B, H))
        for b in range(B):
            wv = win[b].double().numpy() if win is not None else np.zeros((0, D))
            o[b], lse[b] = self.orc.csa_attend(q[b].double().numpy(), comp[b].double().numpy(), idx_local[b].numpy(),
                                               wv, 0, -1, 128, d_v, scale)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def merge(self, o, lse, out_dtype):
        import torch
        lse = lse.numpy()
        M = lse.max(axis=0)
        wgt = np.where(np.isfinite(lse), np.exp(lse - M), 0.0)
        out = (wgt[..., None] * o.numpy()).sum(axis=0) / wgt.sum(axis=0)[..., None]
        return torch.from_numpy(out)


def _cp_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from helpers import randn
    from long_context_sparse_06_b200 import cp
    from oracle import oracle as orc
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        B, H, D, dv, HI, DI, Nc, k = 2, 8, 64, 48, 4, 32, 1500, 64
        qq = randn("mr.cp.q", (B, H, D))
        comp = randn("mr.cp.c", (B, Nc, D))
        win = randn("mr.cp.w", (B, 128, D))
        qI = randn("mr.cp.qi", (B, HI, DI))
        w = randn("mr.cp.wi", (B, HI), std=0.5)
        kI = randn("mr.cp.k", (B, Nc, DI))
        shards = [(0, 700), (700, 800)]
        off, S = shards[rank]
        out, idx = cp.cp_decode_step(qq, comp[:, off:off + S].contiguous(), win if rank == world - 1 else None, qI, w,
                                     kI[:, off:off + S].contiguous(), k, off, dv, 1 / 8, ops=_OracleOps(orc),
                                     out_dtype=torch.float64)
        q.put((rank, out.numpy(), idx.numpy()))
    finally:
        dist.destroy_process_group()


def test_cp_exchange_two_gloo_ranks():
    """Two ranks, each with its shard of the entries (the window on the last): the exchanged
    selection equals the unsplit top-k and the merged attention the unsplit attention."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from helpers import randn
    from oracle import oracle as orc
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    B, H, D, dv, HI, DI, Nc, k = 2, 8, 64, 48, 4, 32, 1500, 64
    qq = randn("mr.cp.q", (B, H, D))
    comp = randn("mr.cp.c", (B, Nc, D))
    win = randn("mr.cp.w", (B, 128, D))
    qI = randn("mr.cp.qi", (B, HI, DI))
    w = randn("mr.cp.wi", (B, HI), std=0.5)
    kI = randn("mr.cp.k", (B, Nc, DI))
    for b in range(B):
        ref_idx = orc.topk(orc.index_scores_f32(qI[b].numpy(), w[b].numpy(), kI[b].numpy()), k)
        ref_o, _ = orc.csa_attend(qq[b].double().numpy(), comp[b].double().numpy(), ref_idx,
                                  win[b].double().numpy(), 0, -1, 128, dv, 1 / 8)
        for rank, out, idx in res:
            np.testing.assert_array_equal(idx[b], ref_idx)
            np.testing.assert_allclose(out[b], ref_o, rtol=0, atol=1e-12)
