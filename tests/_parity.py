"""Helpers for the GPU-vs-oracle parity tests (no method arithmetic here).

Every comparison is made three ways (the tolerance metric of the survey's
oracle section: relative L2 in fp64, reported for the whole tensor and for the
worst (sequence, head)):

- the whole tensor: ||x - ref|| / ||ref|| <= tol;
- every (sequence, head) slab on its own (o over its tokens and value channels,
  S over its d_k x d_v entries): the same bar, so one bad head cannot hide in
  the average of the others;
- every row (one token's output vector, one key row of a state) on its own:
  ||x_row - ref_row|| <= ROW_FACTOR * tol * max(||ref_row||, rms row norm of its
  slab).  A token that is wrong outright (an error of the size of its head's
  outputs) fails it even in a 4096-token head, where it moves the slab's relative
  L2 by only ~1.6 %.  The rms floor keeps rows whose output nearly cancels (a
  query almost orthogonal to the state) from being judged against their own tiny
  norm: their absolute error is set by the state's rounding, not by the row.

With the environment variable KDA_PARITY_LOG set to a file path, every check
appends one line (test id, tensor, global / worst-slab / worst-row error) there.
"""
import json
import os

import numpy as np
import torch

import oracle

TOL_F32 = 1e-5   # relative L2 bar for fp32 inputs
TOL_BF16 = 2e-2  # relative L2 bar for bf16 inputs (oracle on the same bf16 values)
ROW_FACTOR = 5   # per-row bar = ROW_FACTOR * tol, against max(row norm, rms row norm of its slab)


def rel_l2(x, ref) -> float:
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    assert np.all(np.isfinite(x)), "non-finite values in the kernel output"
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    return float(num / den) if den > 0 else float(num)


def _ratio(num, den):
    """num / den elementwise, with an absolute error where the reference is 0."""
    den = np.asarray(den, np.float64)
    return np.where(den > 0, num / np.where(den > 0, den, 1.0), num)


def parity_stats(x, ref, time_axis):
    """Global, worst-slab and worst-row relative errors.

    x, ref: arrays whose last axis is the feature axis (d_v, or the value
    columns of a state).  time_axis: the token axis of an output ([B, T, H, d]:
    1; decode steps [steps, N, H, d]: 0), or None for states [N, H, d_k, d_v]
    (a slab is then one (sequence, head) matrix, a row one key channel).
    """
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    assert np.all(np.isfinite(x)), "non-finite values in the kernel output"
    if x.size == 0:
        return {"rel_l2": 0.0, "worst_slab": 0.0, "worst_row": 0.0}
    err = x - ref
    glob = rel_l2(x, ref)
    red = (x.ndim - 2, x.ndim - 1) if time_axis is None else (time_axis, x.ndim - 1)
    s_num = np.sqrt(np.sum(err * err, axis=red, keepdims=True))
    s_den = np.sqrt(np.sum(ref * ref, axis=red, keepdims=True))
    worst_slab = float(np.max(_ratio(s_num, s_den)))
    r_num = np.sqrt(np.sum(err * err, axis=-1, keepdims=True))
    r_den = np.sqrt(np.sum(ref * ref, axis=-1, keepdims=True))
    rows_per_slab = x.shape[red[0]]
    floor = s_den / np.sqrt(rows_per_slab)           # rms row norm of the slab
    worst_row = float(np.max(_ratio(r_num, np.maximum(r_den, floor))))
    return {"rel_l2": glob, "worst_slab": worst_slab, "worst_row": worst_row}


def _log(name, stats, tol):
    path = os.environ.get("KDA_PARITY_LOG")
    if not path:
        return
    rec = {"test": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0], "tensor": name,
           "tol": tol}
    rec.update({k: float(f"{v:.4g}") for k, v in stats.items()})
    with open(path, "a") as f:
        f.write(json.dumps(rec) + "\n")


def check(x, ref, tol, time_axis, name):
    st = parity_stats(x, ref, time_axis)
    _log(name, st, tol)
    assert st["rel_l2"] <= tol, (name, st)
    assert st["worst_slab"] <= tol, (name, st)
    assert st["worst_row"] <= ROW_FACTOR * tol, (name, st)
    return st


def check_o(x, ref, tol, time_axis=1):
    """An output o: [B, T, H, d_v] (time_axis 1) or [steps, N, H, d_v] (0)."""
    return check(x, ref, tol, time_axis, "o")


def check_S(x, ref, tol):
    """A state: [N, H, d_k, d_v]."""
    return check(x, ref, tol, None, "S")


def np32(t):
    return None if t is None else t.detach().float().cpu().numpy()


def oracle_forward(inp, b=None, h=None, t1=None, cu=None):
    """Oracle on (optionally) one batch row b, one head h and the first t1 tokens."""
    q, k, v, al, be, S0 = (inp[n] for n in ("q", "k", "v", "alpha", "beta", "S0"))
    if b is not None:
        q, k, v, al, be = (x[b:b + 1] for x in (q, k, v, al, be))
        S0 = None if S0 is None else S0[b:b + 1]
    if h is not None:
        q, k, v, al, be = (x[:, :, h:h + 1] for x in (q, k, v, al, be))
        S0 = None if S0 is None else S0[:, h:h + 1]
    if t1 is not None:
        q, k, v, al, be = (x[:, :t1] for x in (q, k, v, al, be))
    return oracle.forward(np32(q), np32(k), np32(v), np32(al), np32(be), np32(S0),
                          None if cu is None else np.asarray(cu, np.int32))


def tolerance(dtype: torch.dtype) -> float:
    return TOL_F32 if dtype == torch.float32 else TOL_BF16
