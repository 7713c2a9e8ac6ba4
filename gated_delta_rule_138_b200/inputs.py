"""Seeded synthetic inputs for the KDA forward pass and decode step.

This module is shared by the tests, the benchmark and the CPU oracle's
callers.  It holds none of the method's arithmetic: it only draws the random
inputs (q, k, v, beta, alpha, initial state) in the shapes and distributions
of the workloads below.  The forget gate is NOT clamped here; clamping alpha
to [e^-5, 1] is the method's job and both the kernels and the oracle do it.

Distributions (every workload):
  q, k  ~ N(0, 1) per element, then L2-normalised per (token, head) in fp32;
  v     ~ N(0, 1);
  beta  = sigmoid(N(0, 1));
  alpha = exp(-softplus(N(0, 1))) per key channel (in (0, 1); values below
          e^-5 occur with probability ~3e-7 and are left for the clamp);
  S0    ~ N(0, 0.1^2) fp32 (read as standard deviation 0.1), where used.
Values are drawn in fp32 and rounded to nearest-even when the input dtype is
bf16.  Draw order per tensor group: q, k, v, beta, alpha, S0.

The long-context workload additionally pins, per head, a seeded choice of
10% of key channels (13 of 128) to alpha = 1 and another 10% to the bf16
value just below e^-5 (0.0067138671875), which the clamp raises to exactly
fp32(e^-5): "channels at exactly e^-5" after the clamp, stressing it.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

BF16_BELOW_EXP_M5 = 0.0067138671875  # largest bf16 value below e^-5


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "forward" | "decode" | "varlen" | "pooled"
    dtype: str                # input dtype: "f32" | "bf16"
    H: int
    dk: int
    dv: int
    B: int = 1
    T: int = 0
    chunk: int = 64
    s0: bool = False
    special_alpha: bool = False
    steps: int = 0            # decode only
    nseq: int = 0             # varlen only; pooled: slots in the state pool
    min_len: int = 0
    max_len: int = 0
    seed: int = 0
    out_dtype: str = "bf16"

    def tokens(self) -> int:
        if self.kind == "decode":
            return self.B * self.steps
        return self.B * self.T


WORKLOADS = {
    # fp32 inputs, one head, small: the oracle finishes in milliseconds
    "fp32_T256_d64": Workload("fp32_T256_d64", "forward", "f32", H=1, dk=64, dv=64,
                              B=1, T=256, s0=False, seed=1000, out_dtype="f32"),
    # bf16 inputs, fp32 state: the headline batch
    "bf16_B8_T4096_H32_d128": Workload("bf16_B8_T4096_H32_d128", "forward", "bf16", H=32,
                                       dk=128, dv=128, B=8, T=4096, s0=True, seed=1001),
    # bf16, one 1M-token sequence per head, clamp-stressing alpha channels
    "bf16_B1_T1M_H32_d128": Workload("bf16_B1_T1M_H32_d128", "forward", "bf16", H=32,
                                     dk=128, dv=128, B=1, T=1 << 20, s0=False,
                                     special_alpha=True, seed=1002),
    # the same recipe on 65,536 tokens: a small case of the same time-split kernels (for
    # profiling captures that must stay a few GB on the device)
    "bf16_B1_T64K_H32_d128": Workload("bf16_B1_T64K_H32_d128", "forward", "bf16", H=32,
                                      dk=128, dv=128, B=1, T=1 << 16, s0=False,
                                      special_alpha=True, seed=1002),
    # single-token decode: 256 sequences x 32 heads, 128 consecutive steps
    "decode_N256_H32_d128": Workload("decode_N256_H32_d128", "decode", "bf16", H=32,
                                     dk=128, dv=128, B=256, steps=128, s0=True, seed=1003),
    # packed variable-length batch: 64 sequences, log-uniform lengths
    # serving step: 4 tokens for each of 256 sequences whose states live in a pool of
    # 512 slots (a seeded choice of slots)
    "pooled_N256_T4_H32_d128": Workload("pooled_N256_T4_H32_d128", "pooled", "bf16", H=32,
                                        dk=128, dv=128, B=256, T=4, nseq=512, seed=5000),
    "varlen_64seq_H16_d128": Workload("varlen_64seq_H16_d128", "varlen", "bf16", H=16,
                                      dk=128, dv=128, nseq=64, min_len=128, max_len=32768,
                                      s0=True, seed=4000),
}


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _l2norm_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def draw_forward(B: int, T: int, H: int, dk: int, dv: int, dtype: str, seed: int,
                 device="cpu", s0: bool = False, special_alpha: bool = False,
                 slice_tokens: int = 1 << 16) -> dict:
    """Draw q, k, v, beta, alpha [B, T, H, *] in `dtype` and S0 [B, H, dk, dv] fp32.

    Large T is drawn in slices of `slice_tokens` tokens so that the fp32
    temporaries stay small; every slice draws q, k, v, beta, alpha in that
    order from the same generator, so the values are fixed by (shape, seed).
    """
    td = torch_dtype(dtype)
    g = _gen(seed, device)
    q = torch.empty(B, T, H, dk, dtype=td, device=device)
    k = torch.empty_like(q)
    al = torch.empty_like(q)
    v = torch.empty(B, T, H, dv, dtype=td, device=device)
    be = torch.empty(B, T, H, dtype=td, device=device)
    for t0 in range(0, T, slice_tokens):
        t1 = min(T, t0 + slice_tokens)
        n = t1 - t0
        f = dict(device=device, dtype=torch.float32, generator=g)
        q[:, t0:t1] = _l2norm_rows(torch.randn(B, n, H, dk, **f)).to(td)
        k[:, t0:t1] = _l2norm_rows(torch.randn(B, n, H, dk, **f)).to(td)
        v[:, t0:t1] = torch.randn(B, n, H, dv, **f).to(td)
        be[:, t0:t1] = torch.sigmoid(torch.randn(B, n, H, **f)).to(td)
        al[:, t0:t1] = torch.exp(-torch.nn.functional.softplus(
            torch.randn(B, n, H, dk, **f))).to(td)
    S0 = None
    if s0:
        S0 = 0.1 * torch.randn(B, H, dk, dv, device=device, dtype=torch.float32, generator=g)
    if special_alpha:
        n_special = int(round(0.1 * dk))
        gp = _gen(seed + 7919, "cpu")
        for h in range(H):
            perm = torch.randperm(dk, generator=gp)
            ones, lows = perm[:n_special].to(device), perm[n_special:2 * n_special].to(device)
            al[:, :, h, ones] = 1.0
            al[:, :, h, lows] = BF16_BELOW_EXP_M5
    return dict(q=q, k=k, v=v, alpha=al, beta=be, S0=S0)


def varlen_lengths(nseq: int, min_len: int, max_len: int, seed: int) -> list:
    """Log-uniform lengths in [min_len, max_len]: round(exp(U(ln min, ln max)))."""
    g = _gen(seed, "cpu")
    u = torch.rand(nseq, generator=g, dtype=torch.float64)
    lo, hi = math.log(min_len), math.log(max_len)
    lens = torch.exp(lo + (hi - lo) * u).round().clamp(min_len, max_len).to(torch.int64)
    return [int(x) for x in lens]


def draw_varlen(lengths: list, H: int, dk: int, dv: int, dtype: str, seed: int,
                device="cpu", s0: bool = True) -> dict:
    """Packed batch: sequence i drawn from seed + i, concatenated along tokens.

    Returns q, k, v, alpha, beta [1, total, H, *], S0 [nseq, H, dk, dv] fp32 (or
    None) and cu_seqlens int32 [nseq + 1].
    """
    parts = [draw_forward(1, L, H, dk, dv, dtype, seed + i, device=device, s0=s0)
             for i, L in enumerate(lengths)]
    out = {name: torch.cat([p[name] for p in parts], dim=1)
           for name in ("q", "k", "v", "alpha", "beta")}
    out["S0"] = torch.cat([p["S0"] for p in parts], dim=0) if s0 else None
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + L)
    out["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32, device=device)
    return out


def draw_decode(N: int, H: int, dk: int, dv: int, steps: int, dtype: str, seed: int,
                device="cpu") -> dict:
    """Decode run: S [N, H, dk, dv] fp32 first, then per step q, k, v, beta, alpha.

    Returns S and per-step stacks q, k, alpha [steps, N, H, dk], v [steps, N, H, dv],
    beta [steps, N, H].
    """
    td = torch_dtype(dtype)
    g = _gen(seed, device)
    f = dict(device=device, dtype=torch.float32, generator=g)
    S = 0.1 * torch.randn(N, H, dk, dv, **f)
    qs, ks, vs, bs, als = [], [], [], [], []
    for _ in range(steps):
        qs.append(_l2norm_rows(torch.randn(N, H, dk, **f)).to(td))
        ks.append(_l2norm_rows(torch.randn(N, H, dk, **f)).to(td))
        vs.append(torch.randn(N, H, dv, **f).to(td))
        bs.append(torch.sigmoid(torch.randn(N, H, **f)).to(td))
        als.append(torch.exp(-torch.nn.functional.softplus(torch.randn(N, H, dk, **f))).to(td))
    return dict(S=S, q=torch.stack(qs), k=torch.stack(ks), v=torch.stack(vs),
                beta=torch.stack(bs), alpha=torch.stack(als))


def draw_workload(w: Workload, device="cpu", **over) -> dict:
    """Inputs of a named workload (sizes may be overridden, e.g. T=... for a slice)."""
    if w.kind == "forward":
        kw = dict(B=w.B, T=w.T, H=w.H, dk=w.dk, dv=w.dv)
        kw.update({k_: v_ for k_, v_ in over.items() if k_ in kw})
        return draw_forward(kw["B"], kw["T"], kw["H"], kw["dk"], kw["dv"], w.dtype, w.seed,
                            device=device, s0=w.s0, special_alpha=w.special_alpha)
    if w.kind == "varlen":
        nseq = over.get("nseq", w.nseq)
        lengths = over.get("lengths") or varlen_lengths(nseq, w.min_len, w.max_len, w.seed + 999)
        return draw_varlen(lengths, w.H, w.dk, w.dv, w.dtype, w.seed, device=device, s0=w.s0)
    if w.kind == "decode":
        return draw_decode(over.get("B", w.B), w.H, w.dk, w.dv, over.get("steps", w.steps),
                           w.dtype, w.seed, device=device)
    if w.kind == "pooled":
        out = draw_forward(w.B, w.T, w.H, w.dk, w.dv, w.dtype, w.seed, device=device, s0=False)
        g = _gen(w.seed + 1, "cpu")
        out["S_pool"] = (0.1 * torch.randn(w.nseq, w.H, w.dk, w.dv, generator=g)).to(device)
        out["slots"] = torch.randperm(w.nseq, generator=g)[:w.B].to(torch.int32).to(device)
        return out
    raise ValueError(w.kind)
