"""Fused input-side transforms (gates from logits, q and k normalised inside
the kernels) against the oracle on the transformed inputs."""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_138_b200 as kda

from _parity import check_o, check_S, np32

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _raw(B, T, H, dk, dv, dtype, seed, device=DEV):
    """Unnormalised q, k and gate logits (the generators' draws before their transforms)."""
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    g = torch.Generator(device="cpu").manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=g)
    out = dict(q=r(B, T, H, dk), k=r(B, T, H, dk), v=r(B, T, H, dv), alpha=r(B, T, H, dk),
               beta=r(B, T, H))
    out = {n: x.to(td).to(device) for n, x in out.items()}
    out["S0"] = (0.1 * r(B, H, dk, dv)).to(device)
    return out


def _oracle(inp, cu=None):
    qh, kh, a, b = oracle.fused_inputs(np32(inp["q"]), np32(inp["k"]), np32(inp["alpha"]),
                                       np32(inp["beta"]))
    return oracle.forward(qh, kh, np32(inp["v"]), a, b, np32(inp["S0"]), cu)


@pytest.mark.parametrize("B,T,H", [(2, 300, 3), (1, 64, 2), (1, 64 * 65 + 37, 2)])
def test_forward_fused(B, T, H):
    """Tensor-core kernel with fused transforms; the last case is split along time."""
    inp = _raw(B, T, H, 128, 128, "bf16", 1500 + T)
    out, Sf = kda.kda_forward_fused(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                                    inp["S0"])
    torch.cuda.synchronize()
    ro, rS = _oracle(inp)
    check_o(np32(out), ro, 2e-2)
    check_S(np32(Sf), rS, 2e-2)


def test_forward_fused_equals_forward_on_transformed_inputs():
    inp = _raw(2, 200, 2, 128, 128, "bf16", 1510)
    out_f, S_f = kda.kda_forward_fused(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                                       inp["S0"])
    qf, kf = inp["q"].float(), inp["k"].float()
    qn = (qf / qf.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    kn = (kf / kf.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    al = torch.sigmoid(-inp["alpha"].float()).to(torch.bfloat16)
    be = torch.sigmoid(inp["beta"].float()).to(torch.bfloat16)
    out_p, S_p = kda.kda_forward(qn, kn, inp["v"], al, be, inp["S0"])
    torch.cuda.synchronize()
    check_o(np32(out_f), np32(out_p), 2e-2)
    check_S(np32(S_f), np32(S_p), 2e-2)


def test_forward_fused_packed():
    lengths = [5, 0, 130, 64]
    H = 2
    g = torch.Generator(device="cpu").manual_seed(1520)
    parts = [_raw(1, L, H, 128, 128, "bf16", 1520 + i) for i, L in enumerate(lengths)]
    inp = {n: torch.cat([p[n] for p in parts], dim=1) for n in ("q", "k", "v", "alpha", "beta")}
    inp["S0"] = torch.cat([p["S0"] for p in parts], dim=0)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device=DEV)
    out, Sf = kda.kda_forward_fused(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                                    inp["S0"], cu_seqlens=cu)
    torch.cuda.synchronize()
    ro, rS = _oracle(inp, np32(cu).astype(np.int32))
    check_o(np32(out), ro, 2e-2)
    check_S(np32(Sf), rS, 2e-2)
    del g


@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 64, 64), ("f32", 128, 64)])
def test_decode_step_fused(dtype, dk, dv):
    N, H = 5, 3
    inp = _raw(N, 1, H, dk, dv, dtype, 1530 + dk + dv)
    S = inp["S0"].clone()
    sq = lambda x: x[:, 0].contiguous()
    out = kda.kda_decode_step_fused(sq(inp["q"]), sq(inp["k"]), sq(inp["v"]), sq(inp["alpha"]),
                                    sq(inp["beta"]), S)
    torch.cuda.synchronize()
    ro, rS = _oracle(inp)
    tol = 1e-5 if dtype == "f32" else 2e-2
    check_o(np32(out)[:, None], ro, tol)
    check_S(np32(S), rS, tol)


def test_forward_fused_rejects_other_configurations():
    inp = _raw(1, 64, 1, 64, 64, "f32", 1540)
    with pytest.raises(kda.KdaError):
        kda.kda_forward_fused(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S0"])
