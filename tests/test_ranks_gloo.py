"""The multi-rank bench path on CPU: two gloo ranks, no GPU.

Every rank processes its own batch (weak scaling); the step time is the
slowest rank's, the throughput counts every rank's tokens, and ranks draw
different sequences.  These are the only cross-rank operations of the path.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_delta_rule_138_b200 import inputs as gen
from gated_delta_rule_138_b200 import ranks


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [3.0, 5.0][rank]                      # the slower rank decides
        tokens = [100, 300][rank]
        t_max = ranks.reduce_max(ms, world)
        n_all = ranks.reduce_sum(tokens, world)
        value = ranks.weak_scaling_throughput(n_all, t_max)
        w = gen.WORKLOADS["bf16_B8_T4096_H32_d128"]
        x = gen.draw_forward(1, 4, 2, 8, 8, "bf16", w.seed + ranks.rank_seed_offset(rank))["q"]
        xs = [torch.zeros_like(x, dtype=torch.float32) for _ in range(world)]
        dist.all_gather(xs, x.float())
        ranks.barrier(world)
        q.put((rank, t_max, n_all, value, bool(torch.equal(xs[0], xs[1]))))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, t_max, n_all, value, same in res:
        assert t_max == 5.0 and n_all == 400
        assert value == pytest.approx(400 / 5e-3)
        assert not same          # ranks draw independent batches


def test_single_rank_is_identity():
    assert ranks.reduce_max(2.5, 1) == 2.5
    assert ranks.reduce_sum(7, 1) == 7
    assert ranks.rank_seed_offset(0) == 0
