"""KDA oracle -- TEST INFRASTRUCTURE ONLY.

A plain fp64 CPU implementation of the KDA forward pass (token-by-token gated
delta rule) and of its reverse mode (the backward pass), used to check the CUDA
path.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import
this package.  It shares no code with ``gated_delta_rule_138_b200`` and the
product never imports it.

Source of the method: the worldcybernews article "Kimi K3 Open Model Surpasses
Closed GPT and Anthropic Systems on Independent Benchmarks", paragraph 2
(state matrix S, delta-rule update, beta write strength, alpha forgetting,
alpha clamped to [e^-5, 1]).  The equation it computes, per sequence and head:

    a_t = clamp(alpha_t, e^-5, 1);  S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T;
    o_t = S_t^T q_t

All pins that tie it to the page and to mathematics live in
tests/test_oracle_pins.py.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_libs = {}


def _load(path=None):
    """Load the oracle library (built on demand).  `path` selects another build
    of the same source; the pin tests use it to load deliberately broken copies
    and check that the pins catch them."""
    key = path or "default"
    if key not in _libs:
        lib = ctypes.CDLL(path or _build.build())
        lib.kda_oracle_forward.restype = ctypes.c_int
        lib.kda_oracle_forward.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
            ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
            ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32]
        lib.kda_oracle_backward.restype = ctypes.c_int
        lib.kda_oracle_backward.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int64,
            ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_int32]
        lib.kda_oracle_alpha_min.restype = ctypes.c_double
        lib.kda_oracle_alpha_min.argtypes = []
        _libs[key] = lib
    return _libs[key]


def alpha_min(lib_path=None) -> float:
    """The clamp's lower bound: e^-5 rounded to fp32, widened to fp64."""
    return float(_load(lib_path).kda_oracle_alpha_min())


def _f32(x):
    if x is None:
        return None
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data


def forward(q, k, v, alpha, beta, S0=None, cu_seqlens=None, nthreads=0, lib_path=None):
    """Token-by-token KDA forward in fp64.

    q, k, alpha: [B, T, H, dk]; v: [B, T, H, dv]; beta: [B, T, H]; all are
    taken as fp32 values (bf16 values widen to fp32 exactly).  S0: None or
    [N, H, dk, dv] with N = B (dense) or len(cu_seqlens) - 1 (packed, B == 1).
    Returns (out fp64 [B, T, H, dv], S_final fp64 [N, H, dk, dv]).
    """
    q, k, v, alpha, beta, S0 = (_f32(x) for x in (q, k, v, alpha, beta, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and alpha.shape == q.shape
    assert v.shape == (B, T, H, dv) and beta.shape == (B, T, H)
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        nseq = cu.shape[0] - 1
        assert B == 1
    else:
        cu = None
        nseq = B
    if S0 is not None:
        assert S0.shape == (nseq, H, dk, dv)
    out = np.zeros((B, T, H, dv), dtype=np.float64)
    S_final = np.zeros((nseq, H, dk, dv), dtype=np.float64)
    rc = _load(lib_path).kda_oracle_forward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S0), _ptr(cu),
        nseq, B, T, H, dk, dv, _ptr(out), _ptr(S_final), int(nthreads))
    if rc != 0:
        raise ValueError("kda_oracle_forward rejected its arguments (rc=%d)" % rc)
    return out, S_final


def backward(q, k, v, alpha, beta, dout, S0=None, dS_final=None, cu_seqlens=None,
             nthreads=0, lib_path=None):
    """Reverse mode of the token recurrence in fp64 (the backward pass).

    Inputs as `forward`, plus dout (dL/d out, like v) and dS_final (dL/d S_final,
    like S0, or None for zero).  The clamp passes the gradient where alpha lies
    in [e^-5, 1] (bounds included) and blocks it outside.  Returns fp64
    (dq, dk, dv, dalpha, dbeta, dS0), each shaped like its input (dS0 like S0,
    [N, H, dk, dv], also when S0 is None).
    """
    q, k, v, alpha, beta, S0, dout, dS_final = (
        _f32(x) for x in (q, k, v, alpha, beta, S0, dout, dS_final))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and alpha.shape == q.shape
    assert v.shape == (B, T, H, dv) and beta.shape == (B, T, H) and dout.shape == v.shape
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        nseq = cu.shape[0] - 1
        assert B == 1
    else:
        cu = None
        nseq = B
    for x in (S0, dS_final):
        if x is not None:
            assert x.shape == (nseq, H, dk, dv)
    dq = np.zeros((B, T, H, dk)); dk_ = np.zeros((B, T, H, dk)); dal = np.zeros((B, T, H, dk))
    dv_ = np.zeros((B, T, H, dv)); dbe = np.zeros((B, T, H)); dS0 = np.zeros((nseq, H, dk, dv))
    rc = _load(lib_path).kda_oracle_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S0), _ptr(dout),
        _ptr(dS_final), _ptr(cu), nseq, B, T, H, dk, dv, _ptr(dq), _ptr(dk_), _ptr(dv_),
        _ptr(dal), _ptr(dbe), _ptr(dS0), int(nthreads))
    if rc != 0:
        raise ValueError("kda_oracle_backward rejected its arguments (rc=%d)" % rc)
    return dq, dk_, dv_, dal, dbe, dS0


def decode_steps(q, k, v, alpha, beta, S, nthreads=0):
    """Consecutive single-token steps: inputs [steps, N, H, d], S [N, H, dk, dv].

    One decode step per sequence is the same recurrence with one token, so a run
    of steps is the forward over T = steps tokens of each sequence.  Returns
    (out fp64 [steps, N, H, dv], S after the last step, fp64).
    """
    sw = lambda x: np.ascontiguousarray(np.swapaxes(np.asarray(x, np.float32), 0, 1))
    out, S_final = forward(sw(q), sw(k), sw(v), sw(alpha), sw(beta), S,
                           nthreads=nthreads)
    return np.ascontiguousarray(np.swapaxes(out, 0, 1)), S_final


def available_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def fused_inputs(q, k, alpha_logits, beta_logits):
    """Input-side transforms of the fused entry points, written from their plain
    definitions in fp64 (the pages name none of them; the workload generators draw
    the gates this way):
        alpha = exp(-softplus(x)) = exp(-log(1 + e^x)),   beta = 1 / (1 + e^-y),
        q_hat = q / sqrt(max(||q||^2, 1e-12)) over the last axis (per token and head),
        k_hat likewise.
    Returns (q_hat, k_hat, alpha, beta) as fp64 arrays."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    x = np.asarray(alpha_logits, dtype=np.float64)
    y = np.asarray(beta_logits, dtype=np.float64)
    with np.errstate(over="ignore"):
        alpha = np.exp(-np.log1p(np.exp(x)))
        beta = 1.0 / (1.0 + np.exp(-y))
    nq = np.sqrt(np.maximum((q * q).sum(-1, keepdims=True), 1e-12))
    nk = np.sqrt(np.maximum((k * k).sum(-1, keepdims=True), 1e-12))
    return q / nq, k / nk, alpha, beta
