"""Helpers for the GPU-vs-oracle parity tests (no method arithmetic here)."""
import numpy as np
import torch

import oracle

TOL_F32 = 1e-5   # relative L2 bar for fp32 inputs
TOL_BF16 = 2e-2  # relative L2 bar for bf16 inputs (oracle on the same bf16 values)


def rel_l2(x, ref) -> float:
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    assert np.all(np.isfinite(x)), "non-finite values in the kernel output"
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    return float(num / den) if den > 0 else float(num)


def np32(t):
    return None if t is None else t.detach().float().cpu().numpy()


def oracle_forward(inp, b=None, h=None, t1=None, cu=None):
    """Oracle on (optionally) one batch row b, one head h and the first t1 tokens."""
    sl = lambda x: x
    q, k, v, al, be, S0 = (inp[n] for n in ("q", "k", "v", "alpha", "beta", "S0"))
    if b is not None:
        q, k, v, al, be = (x[b:b + 1] for x in (q, k, v, al, be))
        S0 = None if S0 is None else S0[b:b + 1]
    if h is not None:
        q, k, v, al, be = (x[:, :, h:h + 1] for x in (q, k, v, al, be))
        S0 = None if S0 is None else S0[:, h:h + 1]
    if t1 is not None:
        q, k, v, al, be = (x[:, :t1] for x in (q, k, v, al, be))
    del sl
    return oracle.forward(np32(q), np32(k), np32(v), np32(al), np32(be), np32(S0),
                          None if cu is None else np.asarray(cu, np.int32))


def tolerance(dtype: torch.dtype) -> float:
    return TOL_F32 if dtype == torch.float32 else TOL_BF16
