"""Pooled state slots (serving): decode and multi-token forward steps that read
and update S_pool[slots[n]] in place, against the oracle on the gathered states.
Slots not named stay bit-identical; a slot outside the pool is padding."""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_138_b200 as kda
from gated_delta_rule_138_b200 import inputs as gen

from _parity import check_o, check_S, np32, tolerance

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _pool(P, H, dk, dv, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (0.1 * torch.randn(P, H, dk, dv, generator=g)).to(DEV)


@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 64, 64), ("f32", 128, 64)])
def test_decode_step_indexed(dtype, dk, dv):
    N, H, P = 4, 3, 7
    slots_l = [5, 0, -1, 3]                       # sequence 2 is padding
    d = gen.draw_decode(N, H, dk, dv, 1, dtype, 1400 + dk + dv, device=DEV)
    pool = _pool(P, H, dk, dv, 1401)
    before = pool.clone()
    slots = torch.tensor(slots_l, dtype=torch.int32, device=DEV)
    out = kda.kda_decode_step_indexed(d["q"][0], d["k"][0], d["v"][0], d["alpha"][0], d["beta"][0],
                                      pool, slots)
    torch.cuda.synchronize()
    S_in = torch.stack([before[s] if s >= 0 else torch.zeros_like(before[0]) for s in slots_l])
    ro, rS = oracle.decode_steps(np32(d["q"]), np32(d["k"]), np32(d["v"]), np32(d["alpha"]),
                                 np32(d["beta"]), np32(S_in))
    tol = tolerance(d["q"].dtype)
    check_o(np32(out)[None], ro, tol, time_axis=0)
    for n, s in enumerate(slots_l):
        if s >= 0:
            check_S(np32(pool[s]), rS[n], tol)
    for s in set(range(P)) - {x for x in slots_l if x >= 0}:
        assert torch.equal(pool[s], before[s])


@pytest.mark.parametrize("dtype,dk,dv,T", [("bf16", 128, 128, 4), ("bf16", 128, 128, 16),
                                           ("bf16", 128, 128, 1), ("f32", 64, 64, 4),
                                           ("bf16", 128, 128, 70)])
def test_forward_indexed_multi_token(dtype, dk, dv, T):
    """A multi-token step (T tokens per sequence) from pooled states."""
    N, H, P = 5, 2, 9
    slots_l = [8, 2, 40, 0, 5]                     # 40 is outside the pool: padding
    inp = gen.draw_forward(N, T, H, dk, dv, dtype, 1410 + T + dk, device=DEV, s0=False)
    pool = _pool(P, H, dk, dv, 1411)
    before = pool.clone()
    slots = torch.tensor(slots_l, dtype=torch.int32, device=DEV)
    out = kda.kda_forward_indexed(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], pool,
                                  slots)
    torch.cuda.synchronize()
    S_in = torch.stack([before[s] if 0 <= s < P else torch.zeros_like(before[0]) for s in slots_l])
    ro, rS = oracle.forward(np32(inp["q"]), np32(inp["k"]), np32(inp["v"]), np32(inp["alpha"]),
                            np32(inp["beta"]), np32(S_in))
    tol = tolerance(inp["q"].dtype)
    check_o(np32(out), ro, tol)
    for n, s in enumerate(slots_l):
        if 0 <= s < P:
            check_S(np32(pool[s]), rS[n], tol)
    for s in set(range(P)) - set(slots_l):
        assert torch.equal(pool[s], before[s])


def test_forward_indexed_equals_decode_steps():
    """Four tokens through one multi-token step equal four decode steps."""
    N, H, P, T = 6, 2, 6, 4
    slots = torch.tensor([3, 1, 0, 5, 2, 4], dtype=torch.int32, device=DEV)
    inp = gen.draw_forward(N, T, H, 128, 128, "bf16", 1420, device=DEV, s0=False)
    pool_a = _pool(P, H, 128, 128, 1421)
    pool_b = pool_a.clone()
    out_a = kda.kda_forward_indexed(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                                    pool_a, slots)
    outs = [kda.kda_decode_step_indexed(inp["q"][:, t].contiguous(), inp["k"][:, t].contiguous(),
                                        inp["v"][:, t].contiguous(), inp["alpha"][:, t].contiguous(),
                                        inp["beta"][:, t].contiguous(), pool_b, slots)
            for t in range(T)]
    torch.cuda.synchronize()
    check_o(np32(out_a), np32(torch.stack(outs, dim=1)), 2e-2)
    check_S(np32(pool_a), np32(pool_b), 2e-2)


def test_forward_indexed_packed():
    lengths = [3, 0, 17, 64]
    H, P = 2, 6
    slots_l = [4, 1, 0, 3]
    inp = gen.draw_varlen(lengths, H, 128, 128, "bf16", 1430, device=DEV, s0=False)
    pool = _pool(P, H, 128, 128, 1431)
    before = pool.clone()
    slots = torch.tensor(slots_l, dtype=torch.int32, device=DEV)
    out = kda.kda_forward_indexed(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], pool,
                                  slots, cu_seqlens=inp["cu_seqlens"])
    torch.cuda.synchronize()
    S_in = torch.stack([before[s] for s in slots_l])
    ro, rS = oracle.forward(np32(inp["q"]), np32(inp["k"]), np32(inp["v"]), np32(inp["alpha"]),
                            np32(inp["beta"]), np32(S_in),
                            np32(inp["cu_seqlens"]).astype(np.int32))
    check_o(np32(out), ro, 2e-2)
    for n, s in enumerate(slots_l):
        check_S(np32(pool[s]), rS[n], 2e-2)
    assert torch.equal(pool[1], before[1])        # zero-length sequence: state unchanged
    assert torch.equal(pool[2], before[2]) and torch.equal(pool[5], before[5])


def test_forward_indexed_zero_tokens_keeps_pool():
    inp = gen.draw_forward(3, 0, 2, 128, 128, "bf16", 1440, device=DEV, s0=False)
    pool = _pool(4, 2, 128, 128, 1441)
    before = pool.clone()
    out = kda.kda_forward_indexed(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], pool,
                                  torch.tensor([0, 2, 3], dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert out.numel() == 0 and torch.equal(pool, before)
