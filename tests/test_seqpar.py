"""Sequence-parallel forward (time segments on different ranks) against the
oracle.  The segment maps are pinned to their definition through the oracle
itself: with v = 0 and S0 = I the final state is M, with S0 = 0 it is N."""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_138_b200 as kda
from gated_delta_rule_138_b200 import inputs as gen
from gated_delta_rule_138_b200.seqpar import split_time

from _parity import check_o, check_S, np32, oracle_forward

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_segment_maps_match_their_definition():
    B, T, H, d = 2, 300, 2, 128
    inp = gen.draw_forward(B, T, H, d, d, "bf16", 1300, device=DEV, s0=False)
    # slow gates and weak writes, so that M stays of order one over 300 tokens
    # (with the workload's gates it decays below the fp32 range and both sides are ~0)
    g = torch.Generator(device="cpu").manual_seed(1302)
    inp["alpha"] = (1.0 - 0.005 * torch.rand(inp["alpha"].shape, generator=g)).to(DEV, torch.bfloat16)
    inp["beta"] = torch.full(inp["beta"].shape, 0.125, dtype=torch.bfloat16, device=DEV)
    maps = kda.kda_segment_maps(inp["k"], inp["v"], inp["alpha"], inp["beta"])
    torch.cuda.synchronize()
    f = lambda t: np32(t)
    eye = np.broadcast_to(np.eye(d, dtype=np.float32), (B, H, d, d)).copy()
    zero_v = np.zeros_like(f(inp["k"]))
    _, M = oracle.forward(f(inp["q"]), f(inp["k"]), zero_v, f(inp["alpha"]), f(inp["beta"]), eye)
    _, N = oracle.forward(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["alpha"]), f(inp["beta"]),
                          None)
    got = f(maps)
    assert np.abs(M).max() > 0.1          # a non-trivial map
    check_S(got[..., :d], M, 2e-2)
    check_S(got[..., d:], N, 2e-2)


def test_segment_scan_composes_in_order():
    G, N, H, d = 3, 2, 2, 128
    g = torch.Generator(device="cpu").manual_seed(1301)
    maps = (0.05 * torch.randn(G, N, H, d, 2 * d, generator=g)).to(DEV)
    S0 = torch.randn(N, H, d, d, generator=g).to(DEV)
    out = kda.kda_segment_scan(maps, S0)
    torch.cuda.synchronize()
    ref = S0.double().cpu().numpy()
    m = maps.double().cpu().numpy()
    for i in range(G):
        ref = m[i, ..., :d] @ ref + m[i, ..., d:]
    check_S(np32(out), ref, 1e-5)
    # no maps: a copy of S0; in place allowed
    same = kda.kda_segment_scan(maps[:0], S0.clone())
    torch.cuda.synchronize()
    assert torch.equal(same, S0)


@pytest.mark.parametrize("world,T", [(2, 64 * 12), (4, 64 * 12 + 0), (3, 64 * 9)])
def test_ranks_emulated_in_one_process(world, T):
    """Every rank's steps in turn on one GPU: maps of the earlier segments, scan,
    forward from the scanned start state; outputs and final state against the
    oracle over the whole sequence."""
    B, H, d = 1, 2, 128
    inp = gen.draw_forward(B, T, H, d, d, "bf16", 1310 + world, device=DEV, s0=True)
    sl = {n: [split_time(inp[n], world, r) for r in range(world)]
          for n in ("q", "k", "v", "alpha", "beta")}
    maps = torch.stack([kda.kda_segment_maps(sl["k"][r], sl["v"][r], sl["alpha"][r], sl["beta"][r])
                        for r in range(world)])
    outs = []
    for r in range(world):
        start = kda.kda_segment_scan(maps[:r].contiguous(), inp["S0"]) if r else inp["S0"]
        o, S_end = kda.kda_forward(sl["q"][r], sl["k"][r], sl["v"][r], sl["alpha"][r],
                                   sl["beta"][r], start)
        outs.append(o)
    torch.cuda.synchronize()
    ro, rS = oracle_forward(inp)
    check_o(np32(torch.cat(outs, dim=1)), ro, 2e-2)
    check_S(np32(S_end), rS, 2e-2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, T, q):
    import torch.distributed as dist
    from gated_delta_rule_138_b200.seqpar import kda_forward_sequence_parallel
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        torch.cuda.set_device(0)
        inp = gen.draw_forward(1, T, 2, 128, 128, "bf16", 1320, device="cpu", s0=True)
        part = {n: split_time(inp[n], world, rank).to(DEV) for n in ("q", "k", "v", "alpha", "beta")}
        out, S_end = kda_forward_sequence_parallel(part["q"], part["k"], part["v"], part["alpha"],
                                                   part["beta"], inp["S0"].to(DEV))
        torch.cuda.synchronize()
        q.put((rank, out.float().cpu().numpy(), S_end.cpu().numpy()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_through_torch_distributed():
    """Two processes on this GPU (each launches only its own kernels; the maps
    travel through a gloo all-gather), against the oracle."""
    import torch.multiprocessing as mp
    world, T, port = 2, 64 * 10, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, T, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict((r, (o, s)) for r, o, s in (q.get(timeout=300) for _ in range(world)))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = gen.draw_forward(1, T, 2, 128, 128, "bf16", 1320, device="cpu", s0=True)
    ro, rS = oracle_forward(inp)
    out = np.concatenate([res[r][0] for r in range(world)], axis=1)
    check_o(out, ro, 2e-2)
    check_S(res[world - 1][1], rS, 2e-2)
