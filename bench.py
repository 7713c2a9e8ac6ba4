#!/usr/bin/env python
"""KDA forward benchmark on B200: tokens/s and TFLOP/s against the HBM roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one kda_forward call (the whole chunk-parallel forward) over one
batch of seeded synthetic inputs already resident in HBM.  The default workload
is the long-context one (B=1, H=32, T=2^20, d=128): few (sequence, head) pairs,
so the forward splits every sequence into time segments (one pass over every
segment giving its state map, its zero-start outputs and map rows; the scan of
the start states; the start states' share of the outputs: three launches per
step, timed together).
For N > 1 (launched with torch.distributed.run, one process per GPU) every
rank runs its own batch (independent sequences, no data-path collective:
weak scaling); the time is the max over ranks and `value` counts all ranks'
tokens.  Rank 0 prints ONE JSON line.

--seqpar (forward workloads with one sequence per batch row) instead splits
time across the ranks: rank r runs the r-th contiguous segment of every
sequence; segment state maps are all-gathered (NCCL) and scanned to each rank's
start state (strong scaling, the same total tokens at every N).

--impl reference times the CPU oracle (fp64, token by token) as it stands on
the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "KDA fwd tokens/s and TFLOP/s (% roofline) at H=32, d=128, 1 B200"
DEFAULT_WORKLOAD = "bf16_B1_T1M_H32_d128"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------- work model

def esize(dtype: str) -> int:
    return 4 if dtype == "f32" else 2


def forward_bytes(w, n_token_heads: int, n_seq_heads: int, has_s0: bool) -> int:
    """Algorithmic HBM bytes of one forward: q, k, alpha, v, beta read and o
    written once per (token, head); S0 read and S_final written once per
    (sequence, head)."""
    ei, eo = esize(w.dtype), esize(w.out_dtype)
    per_th = ei * (3 * w.dk + w.dv + 1) + eo * w.dv
    per_sh = 4 * w.dk * w.dv * ((1 if has_s0 else 0) + 1)
    return per_th * n_token_heads + per_sh * n_seq_heads


def forward_flops(w, n_token_heads: int) -> int:
    """Chunk-form flops per (token, head): 6 dk dv + 2 C (3 dk + 2 dv)."""
    return (6 * w.dk * w.dv + 2 * w.chunk * (3 * w.dk + 2 * w.dv)) * n_token_heads


def backward_bytes(w, n_token_heads: int, n_seq_heads: int, has_s0: bool) -> int:
    """Algorithmic HBM bytes of one backward: q, k, alpha, v, beta and dout read,
    fp32 dq, dk, dalpha, dv, dbeta written once per (token, head); S0 (if any)
    and dS_final read and dS0 written once per (sequence, head)."""
    ei = esize(w.dtype)
    per_th = ei * (3 * w.dk + 2 * w.dv + 1) + 4 * (3 * w.dk + w.dv + 1)
    per_sh = 4 * w.dk * w.dv * ((1 if has_s0 else 0) + 2)
    return per_th * n_token_heads + per_sh * n_seq_heads


def backward_flops(w, n_token_heads: int) -> int:
    """Flops per (token, head) as the backward kernel executes them: two forward
    recomputations (5 dk dv each) and the reverse step (21 dk dv)."""
    return 31 * w.dk * w.dv * n_token_heads


def backward_tc_flops(w, n_token_heads: int) -> int:
    """Tensor-core backward (d_k = d_v = 128, C = 64): the MMA flops per chunk, per
    (token, head).  Record pass: [A/beta ; P] (128 x 96 x 128), (k*gamma) S0
    (64 x 128 x 128), U (64 x 128 x 64), the state update (128 x 128 x 64) and the
    32 -> 64 solve step (2 x 64 x 32 x 32); state-gradient pass: dU (64 x 128 x 192),
    dY (64 x 128 x 64), dS (128 x 128 x 128); chunk pass: [dY ; dO] U^T (128 x 64 x 128),
    [A/beta ; P] (128 x 96 x 128), dS U^T (128 x 64 x 128), S0 [dR ; dO]^T, R^T G^T,
    L^T G (128 x 128 x 128, 128 x 128 x 96, 128 x 128 x 128)."""
    C = w.chunk
    mnk = [(128, 96, 128), (64, 128, 128), (64, 128, 64), (128, 128, 64), (64, 32, 32), (64, 32, 32),
           (64, 128, 192), (64, 128, 64), (128, 128, 128),
           (128, 64, 128), (128, 96, 128), (128, 64, 128), (128, 128, 128), (128, 128, 96),
           (128, 128, 128)]
    per_chunk = sum(2 * m * n * k for m, n, k in mnk)
    return per_chunk * n_token_heads // C


def decode_bytes(w, n_seq_heads: int) -> int:
    ei, eo = esize(w.dtype), esize(w.out_dtype)
    return n_seq_heads * (8 * w.dk * w.dv + ei * (3 * w.dk + w.dv + 1) + eo * w.dv)


def decode_flops(w, n_seq_heads: int) -> int:
    return n_seq_heads * 6 * w.dk * w.dv


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def code_only(src: str) -> str:
    """C/C++/CUDA source without its comments, whitespace runs collapsed to one
    space: what the compiler sees, so that a record survives edits to comments only."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":   # a string or character literal, kept whole
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_digest(names: str) -> str:
    """sha256 (16 hex digits) of the code (comments and whitespace runs aside, see
    code_only) of the comma-separated csrc files, in order."""
    h = hashlib.sha256()
    for name in names.split(","):
        with open(os.path.join(ROOT, "gated_delta_rule_138_b200", "csrc", name),
                  encoding="utf-8") as fh:
            h.update(code_only(fh.read()).encode("utf-8"))
        h.update(b"\0")
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """dram read+write bytes per launch from the committed ncu summary, if it
    was taken on the kernel source as it is now (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    for ln in lines:
        if ln.startswith("#") or not ln.strip():
            continue
        f = ln.split()
        # kernel workload source_file source_sha bytes_per_launch
        if len(f) >= 5 and f[0] == kernel and f[1] == workload:
            try:
                if kernel_source_digest(f[2]) == f[3]:
                    return float(f[4])
            except OSError:
                return None
    return None


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self._h = pynvml.nvmlDeviceGetHandleByUUID(
                    uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as exc:  # pragma: no cover - depends on the machine
            self.error = repr(exc)
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except AttributeError:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                self.samples.append((time.monotonic(), mhz, rs))
            except Exception:
                pass
            time.sleep(self._period)

    def start(self):
        if self._h is not None:
            self._t.start()
        return self

    def stop(self):
        self._stop.set()
        if self._t.is_alive():
            self._t.join(timeout=2)

    def summary(self, t0: float, t1: float):
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        if not win and self.samples:   # region shorter than the period: nearest
            mid = 0.5 * (t0 + t1)
            win = [min(self.samples, key=lambda s: abs(s[0] - mid))]
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "note": getattr(self, "error", "no samples")}
        reasons = set()
        for _, _, rs in win:
            for bit, name in self.REASONS.items():
                if rs & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[1] for s in win), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(win)}


# ---------------------------------------------------------------- helpers

def dist_setup(n_gpus: int):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d (launch N>1 with torch.distributed.run)"
                         % (n_gpus, world))
    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def barrier(world):
    from gated_delta_rule_138_b200 import ranks
    ranks.barrier(world)


def max_over_ranks(x: float, world: int) -> float:
    from gated_delta_rule_138_b200 import ranks
    return ranks.reduce_max(x, world, device="cuda")


def sum_over_ranks(x: float, world: int) -> float:
    from gated_delta_rule_138_b200 import ranks
    return ranks.reduce_sum(x, world, device="cuda")


def make_inputs(w, device, seed_offset: int):
    from gated_delta_rule_138_b200 import inputs as gen
    import dataclasses
    w2 = dataclasses.replace(w, seed=w.seed + seed_offset)
    return gen.draw_workload(w2, device=device)


def counts(w, inp):
    """(tokens, token-heads, sequence-heads) of one forward step."""
    if w.kind == "varlen":
        tokens = int(inp["q"].shape[1])
        nseq = int(inp["cu_seqlens"].numel() - 1)
    elif w.kind == "decode":
        tokens = w.B
        nseq = w.B
    else:
        tokens = w.B * w.T
        nseq = w.B
    return tokens, tokens * w.H, nseq * w.H


# ---------------------------------------------------------------- CPU oracle timing

def time_oracle(w, inp, budget_s: float, cores: int):
    """Time the fp64 oracle on a bounded sample of this workload's inputs.

    The sample is the first P (sequence, head) pairs over their first Ts tokens,
    grown until one timed run takes about `budget_s` or covers the workload.
    Returns (tokens_per_s, seconds, description).
    """
    import numpy as np
    import oracle
    f = lambda t: t.detach().float().cpu().numpy()
    if w.kind == "decode":
        # one decode step of P (sequence, head) pairs is T = 1 of the forward
        q, k, v, al, be = (inp[n][0] for n in ("q", "k", "v", "alpha", "beta"))
        S = inp["S"]
        total_pairs = S.shape[0] * S.shape[1]
        P = min(total_pairs, 64)
        while True:
            n_seq = max(1, P // w.H)
            t0 = time.perf_counter()
            oracle.decode_steps(f(q[None, :n_seq]), f(k[None, :n_seq]), f(v[None, :n_seq]),
                                f(al[None, :n_seq]), f(be[None, :n_seq]), f(S[:n_seq]),
                                nthreads=cores)
            dt = time.perf_counter() - t0
            if dt >= 0.5 * budget_s or n_seq >= S.shape[0]:
                return n_seq / dt, dt, "%d sequences x %d heads, one decode step" % (n_seq, w.H)
            P = min(total_pairs, int(P * max(2.0, budget_s / max(dt, 1e-3))))

    if w.kind == "varlen":
        cu = inp["cu_seqlens"].cpu().numpy()
        starts, lens = cu[:-1], np.diff(cu)
    else:
        starts = np.arange(w.B) * w.T
        lens = np.full(w.B, w.T)
    Tmax = int(lens.max()) if len(lens) else 0
    flat = {n: inp[n].reshape(-1, *inp[n].shape[2:]) for n in ("q", "k", "v", "alpha", "beta")}
    S0 = inp["S_pool"][inp["slots"].long()] if w.kind == "pooled" else inp.get("S0")
    pairs = [(s, h) for s in range(len(lens)) for h in range(w.H)]
    P, Ts = min(len(pairs), 2 * cores), min(Tmax, 1024)
    while True:
        sel = pairs[:P]
        qs, ks, vs, als, bes, s0s = [], [], [], [], [], []
        for s, h in sel:
            a = int(starts[s])
            L = min(int(lens[s]), Ts)
            pad = Ts - L
            sl = lambda x: np.pad(f(x[a:a + L, h]), [(0, pad)] + [(0, 0)] * (x.dim() - 2))
            qs.append(sl(flat["q"])); ks.append(sl(flat["k"])); vs.append(sl(flat["v"]))
            als.append(sl(flat["alpha"])); bes.append(sl(flat["beta"]))
            s0s.append(f(S0[s, h]) if S0 is not None else np.zeros((w.dk, w.dv), np.float32))
        st = lambda xs: np.stack(xs)[:, :, None]
        t0 = time.perf_counter()
        oracle.forward(st(qs), st(ks), st(vs), st(als), np.stack(bes)[:, :, None],
                       np.stack(s0s)[:, None], nthreads=cores)
        dt = time.perf_counter() - t0
        covered = P == len(pairs) and Ts == Tmax
        if dt >= 0.5 * budget_s or covered:
            tok_heads = P * Ts
            desc = "%d (sequence, head) pairs x first %d tokens (%d token-heads of %d)" % (
                P, Ts, tok_heads, int(lens.sum()) * w.H)
            return (tok_heads / w.H) / dt, dt, desc
        grow = max(2.0, min(8.0, budget_s / max(dt, 1e-3)))
        if Ts < Tmax:
            Ts = min(Tmax, int(Ts * grow))
        else:
            P = min(len(pairs), int(P * grow))


def time_oracle_backward(w, inp, dout, dSf, budget_s: float, cores: int):
    """Time the oracle's fp64 backward on a bounded sample of a dense forward workload:
    the first P (sequence, head) pairs over their first Ts tokens (the oracle keeps
    every state, so Ts stays at most 1024), grown until a run takes about `budget_s`.
    Returns (tokens_per_s, seconds, description)."""
    import numpy as np
    import oracle
    f = lambda t: t.detach().float().cpu().numpy()
    B, T, H = inp["q"].shape[0], inp["q"].shape[1], w.H
    pairs = [(b, h) for b in range(B) for h in range(H)]
    P, Ts = min(len(pairs), max(1, cores)), min(T, 256)
    while True:
        sel = pairs[:P]
        pick = lambda x: np.stack([f(x[b, :Ts, h]) for b, h in sel])[:, :, None]
        s0 = (np.stack([f(inp["S0"][b, h]) for b, h in sel])[:, None]
              if inp.get("S0") is not None else None)
        dsf = np.stack([f(dSf[b, h]) for b, h in sel])[:, None]
        t0 = time.perf_counter()
        oracle.backward(pick(inp["q"]), pick(inp["k"]), pick(inp["v"]), pick(inp["alpha"]),
                        np.stack([f(inp["beta"][b, :Ts, h]) for b, h in sel])[:, :, None],
                        pick(dout), s0, dsf, nthreads=cores)
        dt = time.perf_counter() - t0
        if dt >= 0.5 * budget_s or (P == len(pairs) and Ts == min(T, 1024)):
            desc = "%d (sequence, head) pairs x first %d tokens, backward" % (P, Ts)
            return (P * Ts / H) / dt, dt, desc
        grow = max(2.0, min(8.0, budget_s / max(dt, 1e-3)))
        if Ts < min(T, 1024):
            Ts = min(T, 1024, int(Ts * grow))
        else:
            P = min(len(pairs), int(P * grow))


# ---------------------------------------------------------------- parity on a sample

def _parity_stats(x, ref, time_axis):
    """Relative L2 of the whole sample, of its worst (sequence, head) slab and of
    its worst row (token output, or key row of a state), in fp64."""
    import numpy as np
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    err = x - ref
    nrm = lambda a, ax: np.sqrt(np.sum(a * a, axis=ax, keepdims=True))
    glob = float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300))
    red = (x.ndim - 2, x.ndim - 1) if time_axis is None else (time_axis, x.ndim - 1)
    s_num, s_den = nrm(err, red), nrm(ref, red)
    worst_slab = float(np.max(s_num / np.maximum(s_den, 1e-300)))
    floor = s_den / np.sqrt(x.shape[red[0]])          # rms row norm of the slab
    worst_row = float(np.max(nrm(err, -1) / np.maximum(np.maximum(nrm(ref, -1), floor), 1e-300)))
    return {"rel_l2": glob, "worst_head": worst_slab, "worst_row": worst_row}


def parity_ok(par, bar):
    """False if a sampled comparison is not finite or exceeds its bar (global and
    worst-slab errors within `bar`, worst row within 5 x `bar`, as in the tests)."""
    import math
    for key in ("o", "S_final"):
        st = (par or {}).get(key)
        if not st:
            continue
        vals = (st["rel_l2"], st["worst_head"], st["worst_row"])
        if not all(math.isfinite(v) for v in vals):
            return False
        if vals[0] > bar or vals[1] > bar or vals[2] > 5 * bar:
            return False
    return True


def bench_parity(w, inp, out, Sf, max_tokens=8192):
    """The bench's own outputs against the oracle on sampled (sequence, head) pairs:
    o over the first `max_tokens` tokens of each pair, S_final where the pair's
    whole sequence fits in that budget.  Seconds of host time, not the tests."""
    import numpy as np
    import oracle
    f = lambda t: t.detach().float().cpu().numpy()
    if w.kind not in ("forward", "varlen"):
        return None
    if w.kind == "forward":
        B, T = inp["q"].shape[0], inp["q"].shape[1]
        # (batch row, first token, head, length, sequence index)
        picks = [(0, 0, 0, T, 0), (B - 1, 0, w.H - 1, T, B - 1)]
    else:
        cu = f(inp["cu_seqlens"]).astype(np.int64)
        lens = np.diff(cu)
        picks = [(0, int(cu[n]), h, int(lens[n]), n)
                 for n, h in ((int(np.argmin(lens)), 0), (int(np.argmax(lens)), w.H - 1))]
    res = {"o": [], "S": []}
    for bb, a, h, L, n in picks:
        t1 = min(L, max_tokens)
        sl = lambda x: f(x[bb:bb + 1, a:a + t1, h:h + 1])
        S0 = inp.get("S0")
        s0 = None if S0 is None else f(S0[n:n + 1, h:h + 1])
        ro, rS = oracle.forward(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["alpha"]),
                                sl(inp["beta"]), s0)
        res["o"].append((f(out[bb:bb + 1, a:a + t1, h:h + 1]), ro))
        if t1 == L:
            res["S"].append((f(Sf[n:n + 1, h:h + 1]), rS))
    pack = lambda pairs: (np.concatenate([p[0] for p in pairs], axis=2),
                          np.concatenate([p[1] for p in pairs], axis=2))
    line = {"sample": "%d (sequence, head) pairs, o over the first <= %d tokens%s"
            % (len(picks), max_tokens, ", S_final" if res["S"] else "")}
    # slabs are the sampled heads (axis 2 after concatenation)
    xo, ro = pack(res["o"]) if w.kind == "forward" else (None, None)
    if w.kind == "forward":
        line["o"] = _parity_stats(xo, ro, 1)
    else:
        st = [_parity_stats(x, r, 1) for x, r in res["o"]]
        line["o"] = {k: max(d[k] for d in st) for k in st[0]}
    if res["S"]:
        st = [_parity_stats(x, r, None) for x, r in res["S"]]
        line["S_final"] = {k: max(d[k] for d in st) for k in st[0]}
    return line


# ---------------------------------------------------------------- arms

def run_reference(args, w):
    """The CPU oracle as the reference arm: rank 0 only, host cores."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    import oracle
    import torch
    cores = oracle.available_cores()
    inp = make_inputs(w, "cpu", 0) if w.kind != "forward" or w.T <= 8192 else None
    if inp is None:   # long sequences: draw only the first slice of tokens
        from gated_delta_rule_138_b200 import inputs as gen
        inp = gen.draw_forward(w.B, 8192, w.H, w.dk, w.dv, w.dtype, w.seed, device="cpu",
                               s0=w.s0, special_alpha=w.special_alpha)
    per_step = max(1.0, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        time_oracle(w, inp, per_step * 0.25, cores)
    rates, secs, desc = [], 0.0, ""
    for _ in range(args.steps):
        r, dt, desc = time_oracle(w, inp, per_step, cores)
        rates.append(r)
        secs += dt
    value = statistics.median(rates) if rates else 0.0
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(config_of(w, args.gpus), l2=l2_note(workload_bytes(w))),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    del torch


def workload_bytes(w) -> int:
    """Algorithmic bytes of one step of a named workload, from its definition alone."""
    if w.kind == "decode":
        return decode_bytes(w, w.B * w.H)
    if w.kind == "varlen":
        from gated_delta_rule_138_b200 import inputs as gen
        total = int(sum(gen.varlen_lengths(w.nseq, w.min_len, w.max_len, w.seed + 999)))
        return forward_bytes(w, total * w.H, w.nseq * w.H, w.s0)
    if w.kind == "pooled":
        return forward_bytes(w, w.B * w.T * w.H, w.B * w.H, True)
    return forward_bytes(w, w.B * w.T * w.H, w.B * w.H, w.s0)


def l2_note(algo_bytes) -> str:
    return "no flush: inputs %.2f GB per step > 126 MB L2" % (algo_bytes / 1e9)


def config_of(w, n_gpus):
    c = {"workload": w.name, "H": w.H, "d_k": w.dk, "d_v": w.dv, "chunk": w.chunk,
         "in_dtype": w.dtype, "out_dtype": w.out_dtype, "state": "fp32",
         "parallelism": "replicas x%d (independent sequences per GPU)" % n_gpus}
    if w.kind == "forward":
        c.update({"B": w.B, "T": w.T, "global_batch": w.B * n_gpus, "seq_len": w.T})
    elif w.kind == "varlen":
        c.update({"num_seqs": w.nseq, "len_range": [w.min_len, w.max_len]})
    elif w.kind == "pooled":
        c.update({"N": w.B, "tokens_per_seq": w.T, "pool_slots": w.nseq})
    else:
        c.update({"N": w.B, "steps_per_run": w.steps})
    return c


def run_ours(args, w):
    import torch
    import gated_delta_rule_138_b200 as kda

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    parity_failed = False
    from gated_delta_rule_138_b200 import ranks
    inp = make_inputs(w, dev, ranks.rank_seed_offset(rank))
    tokens, n_th, n_sh = counts(w, inp)
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream()

    if w.kind == "decode":
        S = inp["S"].clone()
        out = torch.empty(w.B, w.H, w.dv, dtype=torch.bfloat16, device=dev)
        n_steps_avail = inp["q"].shape[0]
        state = {"i": 0}

        def step():
            i = state["i"] % n_steps_avail
            state["i"] += 1
            kda.kda_decode_step(inp["q"][i], inp["k"][i], inp["v"][i], inp["alpha"][i],
                                inp["beta"][i], S, out=out)
        kname = "decode_f32state"
        segments = None
        algo_bytes = decode_bytes(w, n_sh)
        algo_flops = decode_flops(w, n_sh)
    elif w.kind == "pooled":
        # a serving step: T tokens per sequence from and into pooled state slots
        out = torch.empty(w.B, w.T, w.H, w.dv, dtype=torch.bfloat16, device=dev)
        pool = inp["S_pool"]

        def step():
            kda.kda_forward_indexed(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], pool,
                                    inp["slots"], out=out, chunk=w.chunk)
        # steps of at most 16 tokens run on the token-sequential kernel (state on chip)
        kname = ("decode_f32state_steps" if w.T <= 16 else
                 kda.kda_forward_kernel_name(w.dk, w.dv, w.chunk, inp["q"].dtype, out.dtype))
        segments = 1
        algo_bytes = forward_bytes(w, n_th, n_sh, True)   # state read and written once
        algo_flops = forward_flops(w, n_th)
    else:
        cu = inp.get("cu_seqlens")
        B, T = inp["q"].shape[0], inp["q"].shape[1]
        out = torch.empty(B, T, w.H, w.dv, dtype=torch.bfloat16 if w.out_dtype == "bf16"
                          else torch.float32, device=dev)
        nseq = B if cu is None else cu.numel() - 1
        Sf = torch.empty(nseq, w.H, w.dk, w.dv, dtype=torch.float32, device=dev)

        def step():
            kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S0"],
                            cu_seqlens=cu, out=out, S_final=Sf, chunk=w.chunk)
        if args.fused:
            # the same tensors read as raw inputs: alpha and beta as logits, q and k unnormalised
            def step():
                kda.kda_forward_fused(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                                      inp["S0"], cu_seqlens=cu, out=out, S_final=Sf, chunk=w.chunk)
        if args.backward:
            # gradients of the same forward: dout like out, dS_final like S_final
            gb = torch.Generator(device=dev).manual_seed(int(w.seed) + 5)
            dout = torch.randn(out.shape, generator=gb, device=dev).to(inp["q"].dtype)
            dSf = torch.randn(Sf.shape, generator=gb, device=dev)
            ws = torch.empty(kda.kda_backward_workspace_bytes(
                B, T, w.H, w.dk, w.dv, None if cu is None else nseq), dtype=torch.uint8,
                device=dev)

            def step():
                kda.kda_backward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], dout,
                                 inp["S0"], dSf, cu_seqlens=cu, workspace=ws)
        if args.seqpar and w.kind == "forward":
            # this rank's time segment; maps exchanged through the process group
            from gated_delta_rule_138_b200.seqpar import kda_forward_sequence_parallel, split_time
            part = {n: split_time(inp[n], world, rank) for n in ("q", "k", "v", "alpha", "beta")}
            S0 = inp["S0"]
            del inp
            inp = dict(part, S0=S0)

            def step():
                kda_forward_sequence_parallel(part["q"], part["k"], part["v"], part["alpha"],
                                              part["beta"], S0)
        kname = kda.kda_forward_kernel_name(w.dk, w.dv, w.chunk, inp["q"].dtype, out.dtype)
        if args.fused:
            kname += "_fused"   # its own compile-time variant (no DRAM-traffic record)
        if args.backward:
            kname = ("backward_tc_bf16" if (w.dtype == "bf16" and w.dk == 128 and w.dv == 128)
                     else "backward_f32")
        # time segments per sequence of the tensor-core path (1: unsplit); with g > 1 a
        # step is three launches (dual pass, scan, o += Qg S_g) timed together
        segments = (kda.kda_forward_segments(nseq, -(-B * T // nseq), w.H)
                    if kname.startswith("chunk_tc_bf16") else 1)
        algo_bytes = forward_bytes(w, n_th, n_sh, inp["S0"] is not None)
        algo_flops = forward_flops(w, n_th)
        if args.backward:
            algo_bytes = backward_bytes(w, n_th, n_sh, inp["S0"] is not None)
            algo_flops = (backward_tc_flops(w, n_th) if kname == "backward_tc_bf16"
                          else backward_flops(w, n_th))

    warm = max(3, args.warmup)
    for _ in range(warm):
        step()
    torch.cuda.synchronize()

    sampler = ClockSampler(local).start()
    time.sleep(0.05)
    barrier(world)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = kda.kda_launch_count()
    h0 = time.monotonic()
    e0.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    h1 = time.monotonic()
    barrier(world)
    launches = kda.kda_launch_count() - n0
    sampler.stop()
    clocks = sampler.summary(h0, h1)
    elapsed_ms = max_over_ranks(e0.elapsed_time(e1), world)
    kern_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    kern_ms = max_over_ranks(kern_ms, world)
    seqpar = bool(args.seqpar and w.kind == "forward")
    # replicas: every rank's own tokens; sequence-parallel: one job split over the ranks
    total_tokens = tokens * args.steps if seqpar else sum_over_ranks(tokens * args.steps, world)
    value = ranks.weak_scaling_throughput(total_tokens, elapsed_ms)
    ms_per_step = elapsed_ms / args.steps

    # end to end: pinned host inputs -> device -> kda_forward -> host results
    e2e = run_e2e(args, w, inp, dev, stream, world) \
        if w.kind in ("forward", "varlen") and args.e2e_steps > 0 and not seqpar \
        and not args.backward \
        else None

    if rank == 0:
        # per GPU: a sequence-parallel step moves 1/world of the job's bytes on each GPU
        share = world if seqpar else 1
        achieved = algo_bytes / share / (kern_ms * 1e-3) / 1e9
        tflops = algo_flops / share / (kern_ms * 1e-3) / 1e12
        cfg = config_of(w, world)
        if args.fused:
            cfg["inputs"] = "raw: gate logits, unnormalised q and k (kda_forward_fused)"
        if args.backward:
            cfg["pass"] = "backward (kda_backward: dq, dk, dv, dalpha, dbeta, dS0 in fp32)"
        if seqpar:
            cfg["parallelism"] = "sequence x%d (time segments per rank, maps all-gathered)" % world
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": warm, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "strong" if seqpar else "weak",
            "vs_baseline": None,
            "dtype": "bf16" if kname.startswith("chunk_tc_bf16") else "f32",
            "data": "synthetic (seeded generators, the workload's shapes and distributions)",
            "config": dict(cfg, l2=l2_note(algo_bytes)),
            "tflops": tflops,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "traffic": recorded_traffic(kname, w.name),
                         "kernel": kname, "time_segments": segments,
                         "algorithmic_bytes": algo_bytes,
                         "kernel_ms": kern_ms, "peak_source": peak_src},
            "tensor": {"achieved_tflops": tflops, "peak": peaks["bf16_tflops"],
                       "frac": tflops / peaks["bf16_tflops"], "flops_per_step": algo_flops},
            "clocks": clocks,
            "gpu_launches": int(launches),
            "e2e": e2e,
        }
        if w.kind in ("forward", "varlen") and not args.backward and not seqpar \
                and not args.fused and not args.no_parity:
            par = bench_parity(w, inp, out, Sf)
            if par is not None:
                par["bar"] = 2e-2 if w.dtype == "bf16" else 1e-5
                par["ok"] = parity_ok(par, par["bar"])
                parity_failed = not par["ok"]
            line["parity"] = par
        # (the backward's sample is taken over dense sequences only)
        if world == 1 and not args.no_cpu_baseline and not (args.backward and w.kind != "forward"):
            import oracle
            cores = oracle.available_cores()
            if args.backward:
                r, dt, desc = time_oracle_backward(w, inp, dout, dSf, args.cpu_budget, cores)
            else:
                r, dt, desc = time_oracle(w, inp, args.cpu_budget, cores)
            line["cpu_baseline"] = {"value": r, "unit": "tokens/s", "cores": cores,
                                    "kind": "oracle", "sample": desc, "seconds": dt}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if parity_failed:   # the line stands as printed; the run does not pass
        print("bench: the sampled outputs fail the oracle check (parity.ok false)", file=sys.stderr)
        sys.exit(3)


def e2e_pieces(w, B, T):
    """How one step's batch is cut for the copy / compute / copy pipeline of the
    end-to-end leg: (axis, piece length).  Independent sequences are cut along
    the batch; a single long sequence along time, each piece starting from the
    previous piece's S_final (kda_forward's S0 / S_final chaining)."""
    if w.kind != "forward":
        return None, 0
    if B >= 2:
        return 0, max(1, B // 4)
    return 1, max(64, min(T, 1 << 17))


def run_e2e(args, w, inp, dev, stream, world):
    """Same metric through the public API with host buffers: every step copies
    its inputs from pinned host memory and reads its outputs (out and S_final)
    back.  Host -> device copies, kda_forward calls and device -> host copies run
    on three streams ordered by events over pieces of the batch (e2e_pieces):
    piece j+1 is copied in and piece j-1 copied out while piece j computes, and
    consecutive steps overlap the same way.  One cudaMemcpyAsync per tensor and
    piece."""
    import torch
    import gated_delta_rule_138_b200 as kda
    names = [n for n in ("q", "k", "v", "alpha", "beta") if inp.get(n) is not None]
    cu_d = inp.get("cu_seqlens")
    B, T = inp["q"].shape[0], inp["q"].shape[1]
    nseq = B if cu_d is None else cu_d.numel() - 1
    odt = torch.bfloat16 if w.out_dtype == "bf16" else torch.float32
    try:
        host = {n: torch.empty(inp[n].shape, dtype=inp[n].dtype, pin_memory=True).copy_(inp[n])
                for n in names}
        S0_h = (torch.empty(inp["S0"].shape, dtype=torch.float32, pin_memory=True).copy_(inp["S0"])
                if inp.get("S0") is not None else None)
        out_h = torch.empty(B, T, w.H, w.dv, dtype=odt, pin_memory=True)
        Sf_h = torch.empty(nseq, w.H, w.dk, w.dv, dtype=torch.float32, pin_memory=True)
    except RuntimeError as exc:
        return {"value": None, "unit": "tokens/s", "note": "pinned host alloc failed: %s" % exc}
    axis, plen = e2e_pieces(w, B, T)
    extent = B if axis == 0 else T
    bounds = ([(0, extent)] if axis is None else
              [(a, min(extent, a + plen)) for a in range(0, extent, plen)])
    sl = lambda t, a, b: t if axis is None else (t[a:b] if axis == 0 else t[:, a:b])
    nslot = 2
    pb = bounds[0][1] - bounds[0][0]
    shape_of = lambda t: ((pb,) + tuple(t.shape[1:]) if axis == 0 else
                          (t.shape[0], pb) + tuple(t.shape[2:]) if axis == 1 else tuple(t.shape))
    dslot = [{n: torch.empty(shape_of(inp[n]), dtype=inp[n].dtype, device=dev) for n in names}
             for _ in range(nslot)]
    oslot = [torch.empty(shape_of(out_h), dtype=odt, device=dev) for _ in range(nslot)]
    cu = cu_d.clone() if cu_d is not None else None
    # state chaining: batch pieces own their rows of S0 / S_final; time pieces pass S along
    S0_d = torch.empty(nseq, w.H, w.dk, w.dv, dtype=torch.float32, device=dev) \
        if S0_h is not None else None
    Sbuf = [torch.empty(nseq, w.H, w.dk, w.dv, dtype=torch.float32, device=dev) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    s_cmp = stream
    ev = lambda: torch.cuda.Event()
    h2d = sum(host[n].numel() * host[n].element_size() for n in names) + (
        S0_h.numel() * 4 if S0_h is not None else 0)
    d2h = out_h.numel() * out_h.element_size() + Sf_h.numel() * 4
    slot_free = [None] * nslot      # compute of the slot's last piece has read its inputs
    out_free = [None] * nslot       # its output copy has left the device buffer
    sf_read = [None]                # the previous step's S_final copy has left Sbuf
    cu_h = cu_d.cpu().pin_memory() if cu_d is not None else None
    if cu_h is not None:
        h2d += cu_h.numel() * 4

    def step():
        if sf_read[0] is not None:
            s_cmp.wait_event(sf_read[0])
        if cu_h is not None:
            with torch.cuda.stream(s_in):
                cu.copy_(cu_h, non_blocking=True)
        if S0_d is not None or cu_h is not None:
            if S0_d is not None:
                with torch.cuda.stream(s_in):
                    S0_d.copy_(S0_h, non_blocking=True)
            e = ev(); e.record(s_in); s_cmp.wait_event(e)
        S_prev = S0_d
        last_sf = None
        for j, (a, b) in enumerate(bounds):
            k = j % nslot
            d, o = dslot[k], oslot[k]
            n_rows = b - a
            with torch.cuda.stream(s_in):
                if slot_free[k] is not None:
                    s_in.wait_event(slot_free[k])
                for n in names:
                    sl(d[n], 0, n_rows).copy_(sl(host[n], a, b), non_blocking=True)
                e_in = ev(); e_in.record(s_in)
            s_cmp.wait_event(e_in)
            if out_free[k] is not None:
                s_cmp.wait_event(out_free[k])
            with torch.cuda.stream(s_cmp):
                dd = {n: sl(d[n], 0, n_rows) for n in names}
                oo = sl(o, 0, n_rows)
                if axis == 0:
                    s0 = None if S0_d is None else S0_d[a:b]
                    sf = Sbuf[0][a:b]
                else:
                    s0 = S_prev
                    sf = Sbuf[j % 2]
                kda.kda_forward(dd["q"], dd["k"], dd["v"], dd["alpha"], dd["beta"], s0,
                                cu_seqlens=cu, out=oo, S_final=sf, chunk=w.chunk)
                S_prev, last_sf = sf, sf
                slot_free[k] = ev(); slot_free[k].record(s_cmp)
            s_out.wait_event(slot_free[k])
            with torch.cuda.stream(s_out):
                sl(out_h, a, b).copy_(oo, non_blocking=True)
                out_free[k] = ev(); out_free[k].record(s_out)
        with torch.cuda.stream(s_out):
            Sf_h.copy_(Sbuf[0] if axis == 0 else last_sf, non_blocking=True)
            sf_read[0] = ev(); sf_read[0].record(s_out)

    n = max(1, min(args.steps, args.e2e_steps))
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_cmp)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for _ in range(n):
        step()
    for s_ in (s_in, s_out):
        e = ev(); e.record(s_); s_cmp.wait_event(e)
    e1.record(s_cmp)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    tokens, _, _ = counts(w, inp)
    total = sum_over_ranks(tokens * n, world)
    return {"value": total / (ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": n, "pieces": len(bounds),
            "overlap": "h2d / compute / d2h streams, %d device slots" % nslot}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle time for the cpu_baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-parity", action="store_true",
                    help="skip the oracle check of the bench's own outputs on sampled heads")
    ap.add_argument("--fused", action="store_true",
                    help="forward workloads through kda_forward_fused (gates as logits, q and k "
                         "normalised inside the kernel)")
    ap.add_argument("--backward", action="store_true",
                    help="time kda_backward (all input gradients) on a forward workload")
    ap.add_argument("--seqpar", action="store_true",
                    help="split every sequence's time axis across the ranks (strong scaling)")
    ap.add_argument("--e2e-steps", type=int, default=10,
                    help="steps of the end-to-end (host buffers) measurement; 0 skips it")
    ap.add_argument("--batch", type=int, default=0,
                    help="a dense workload with this many sequences instead of its own B "
                         "(smaller cases of the same kernels, for profiler captures)")
    args = ap.parse_args()
    if args.backward and (args.fused or args.seqpar):
        ap.error("--backward times kda_backward alone (not with --fused or --seqpar)")
    from gated_delta_rule_138_b200 import inputs as gen
    w = gen.WORKLOADS[args.workload]
    if args.batch > 0:
        if w.kind != "forward":
            ap.error("--batch applies to the dense forward workloads")
        import dataclasses
        w = dataclasses.replace(w, B=args.batch, name="%s_batch%d" % (w.name, args.batch))
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
