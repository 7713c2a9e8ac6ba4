"""GPU parity of kda_backward (through the C ABI) against the oracle's backward.

The oracle is the fp64 reverse mode of the token recurrence, pinned in
test_backward_oracle.py.  Two kernels sit behind the entry point:

- bf16 inputs with d_k = d_v = 128 take the tensor-core chunk form (bf16 MMA
  operands, fp32 accumulation): every gradient is held to the bf16 bar, 2e-2,
  over the whole tensor, per (sequence, head) and per token (tests/_parity.py);
- every other case takes the token-sequential kernel, which computes in fp32
  from the same input values (bf16 inputs widen exactly): the fp32 bar, 1e-5.

Cases span several 8-token checkpoints and 64-token chunks with ragged last
chunks, both input dtypes, the head-dimension pairs, packed sequences (empty,
one-token and ragged ones), absent S0 / dS_final, the clamp's blocked gradients
and a caller-owned workspace.
"""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_138_b200 as kda
from gated_delta_rule_138_b200 import inputs as gen

from _parity import check, np32

pytestmark = pytest.mark.gpu
TOL = 1e-5       # token-sequential fp32 kernel
TOL_TC = 2e-2    # tensor-core kernel (bf16 operands)
NAMES = ("dq", "dk", "dv", "dalpha", "dbeta", "dS0")


def _tc(dtype, dk, dv):
    return dtype == "bf16" and dk == 128 and dv == 128


def _case(B, T, H, dk, dv, dtype, seed, s0=True, dsf=True):
    inp = gen.draw_forward(B, T, H, dk, dv, dtype, seed, device="cpu", s0=s0)
    g = torch.Generator().manual_seed(seed + 77)
    dout = torch.randn(B, T, H, dv, generator=g).to(inp["q"].dtype)
    dSf = torch.randn(B, H, dk, dv, generator=g) if dsf else None
    return inp, dout, dSf


def _gpu(inp, dout, dSf, cu=None, **kw):
    d = lambda t: None if t is None else t.cuda()
    return kda.kda_backward(d(inp["q"]), d(inp["k"]), d(inp["v"]), d(inp["alpha"]), d(inp["beta"]),
                            d(dout), d(inp["S0"]), d(dSf), cu_seqlens=d(cu), **kw)


def _oracle(inp, dout, dSf, cu=None):
    return oracle.backward(np32(inp["q"]), np32(inp["k"]), np32(inp["v"]), np32(inp["alpha"]),
                           np32(inp["beta"]), np32(dout), np32(inp["S0"]), np32(dSf),
                           cu_seqlens=None if cu is None else np.asarray(cu, np.int32))


def _check(got, ref, skip_dS0=False, tol=TOL):
    """Every gradient against the oracle's: the three bars of tests/_parity.py
    (token gradients per (sequence, head) and per token, dS0 per (sequence, head)
    and per key row)."""
    torch.cuda.synchronize()
    for name, x, r in zip(NAMES, got, ref):
        if name == "dS0" and skip_dS0:
            assert x is None
            continue
        x = np32(x)
        if name == "dS0":
            check(x, r, tol, None, name)
        elif name == "dbeta":
            check(x[..., None], np.asarray(r)[..., None], tol, 1, name)
        else:
            check(x, r, tol, 1, name)


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_matches_oracle(dk, dv, dtype):
    inp, dout, dSf = _case(2, 150, 2, dk, dv, dtype, seed=11)
    _check(_gpu(inp, dout, dSf), _oracle(inp, dout, dSf), tol=TOL_TC if _tc(dtype, dk, dv) else TOL)


@pytest.mark.parametrize("T", [1, 7, 8, 9, 15, 16, 17, 31, 32, 33, 63, 64, 65, 128, 200])
def test_backward_chunk_boundaries(T):
    """Tensor-core path: 64-token chunks, 32-token sub-chunks and ragged last chunks."""
    inp, dout, dSf = _case(1, T, 3, 128, 128, "bf16", seed=12)
    _check(_gpu(inp, dout, dSf), _oracle(inp, dout, dSf), tol=TOL_TC)


@pytest.mark.parametrize("T", [1, 9, 17, 65])
def test_backward_chunk_boundaries_fp32_kernel(T):
    inp, dout, dSf = _case(1, T, 3, 128, 128, "f32", seed=12)
    _check(_gpu(inp, dout, dSf), _oracle(inp, dout, dSf))


def test_backward_without_state_inputs():
    inp, dout, _ = _case(2, 96, 2, 64, 64, "f32", seed=13, s0=False, dsf=False)
    _check(_gpu(inp, dout, None), _oracle(inp, dout, None))
    got = _gpu(inp, dout, None, want_dS0=False)
    _check(got, _oracle(inp, dout, None), skip_dS0=True)


def test_backward_packed_sequences():
    lens = [1, 63, 64, 65, 130, 0, 7]
    T = sum(lens)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    inp = gen.draw_forward(1, T, 2, 64, 128, "bf16", 14, device="cpu")
    g = torch.Generator().manual_seed(91)
    inp["S0"] = 0.1 * torch.randn(len(lens), 2, 64, 128, generator=g)
    dout = torch.randn(1, T, 2, 128, generator=g).to(torch.bfloat16)
    dSf = torch.randn(len(lens), 2, 64, 128, generator=g)
    _check(_gpu(inp, dout, dSf, cu=cu), _oracle(inp, dout, dSf, cu=cu.numpy()))


def test_backward_packed_sequences_tensor_cores():
    lens = [1, 63, 64, 65, 130, 0, 7, 200]
    T = sum(lens)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    inp = gen.draw_forward(1, T, 2, 128, 128, "bf16", 24, device="cpu")
    g = torch.Generator().manual_seed(92)
    inp["S0"] = 0.1 * torch.randn(len(lens), 2, 128, 128, generator=g)
    dout = torch.randn(1, T, 2, 128, generator=g).to(torch.bfloat16)
    dSf = torch.randn(len(lens), 2, 128, 128, generator=g)
    _check(_gpu(inp, dout, dSf, cu=cu), _oracle(inp, dout, dSf, cu=cu.numpy()), tol=TOL_TC)


def test_backward_tensor_cores_without_state_inputs():
    inp, dout, _ = _case(2, 100, 2, 128, 128, "bf16", seed=23, s0=False, dsf=False)
    _check(_gpu(inp, dout, None), _oracle(inp, dout, None), tol=TOL_TC)
    got = _gpu(inp, dout, None, want_dS0=False)
    _check(got, _oracle(inp, dout, None), skip_dS0=True, tol=TOL_TC)


def test_backward_tensor_cores_clamp_blocks_gradient():
    inp, dout, dSf = _case(1, 70, 2, 128, 128, "bf16", seed=25)
    al = inp["alpha"]
    al[0, 3, 0, :8] = 1e-4          # below e^-5
    al[0, 40, 1, 8:16] = 1.0        # on the bound: passes
    got = _gpu(inp, dout, dSf)
    _check(got, _oracle(inp, dout, dSf), tol=TOL_TC)
    dal = np32(got[3])
    assert np.all(dal[0, 3, 0, :8] == 0)
    assert np.any(dal[0, 40, 1, 8:16] != 0)


def test_backward_clamp_blocks_gradient():
    inp, dout, dSf = _case(1, 70, 2, 64, 64, "f32", seed=15)
    al = inp["alpha"]
    al[0, 3, 0, :8] = 1e-4          # below e^-5
    al[0, 40, 1, 8:16] = 1.5        # above 1
    al[0, 41, 1, 16:24] = 1.0       # on the bound: passes
    got = _gpu(inp, dout, dSf)
    _check(got, _oracle(inp, dout, dSf))
    dal = np32(got[3])
    assert np.all(dal[0, 3, 0, :8] == 0) and np.all(dal[0, 40, 1, 8:16] == 0)
    assert np.any(dal[0, 41, 1, 16:24] != 0)


def test_backward_caller_workspace_gives_the_same_bits():
    inp, dout, dSf = _case(2, 130, 2, 128, 128, "bf16", seed=16)
    a = _gpu(inp, dout, dSf)
    nbytes = kda.kda_backward_workspace_bytes(2, 130, 2, 128, 128)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    ws.fill_(0xFF)   # contents are not an input
    b = _gpu(inp, dout, dSf, workspace=ws)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.slow
def test_backward_full_size_sampled():
    """The bench workload's shape (B=8, T=4096, H=32, d=128, bf16): the whole
    backward on the GPU, one (sequence, head) against the oracle."""
    B, T, H = 8, 4096, 32
    inp = gen.draw_forward(B, T, H, 128, 128, "bf16", 1001, device="cuda", s0=True)
    g = torch.Generator(device="cuda").manual_seed(5)
    dout = torch.randn(B, T, H, 128, generator=g, device="cuda").to(torch.bfloat16)
    dSf = torch.randn(B, H, 128, 128, generator=g, device="cuda")
    got = kda.kda_backward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], dout,
                           inp["S0"], dSf)
    torch.cuda.synchronize()
    b, h = 5, 17
    sl = lambda x: np32(x[b:b + 1, :, h:h + 1])
    ref = oracle.backward(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["alpha"]),
                          sl(inp["beta"]), sl(dout), np32(inp["S0"][b:b + 1, h:h + 1]),
                          np32(dSf[b:b + 1, h:h + 1]))
    for name, x, r in zip(NAMES, got, ref):
        part = np32(x[b:b + 1, h:h + 1] if name == "dS0" else x[b:b + 1, :, h:h + 1])
        if name == "dS0":
            check(part, r, TOL_TC, None, name)
        elif name == "dbeta":
            check(part[..., None], np.asarray(r)[..., None], TOL_TC, 1, name)
        else:
            check(part, r, TOL_TC, 1, name)
