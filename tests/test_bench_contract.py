"""CPU checks of bench.py: the work model behind `roofline` and `tensor`, the
DRAM-traffic record lookup, and the JSON line of the reference (oracle) arm.

The byte and flop counts are the ones the measurement section states: per (token, head)
q, k, alpha, v, beta read and o written once; per (sequence, head) S0 read and S_final
written once; chunk-form flops 6 d_k d_v + 2 C (3 d_k + 2 d_v).
"""
import importlib.util
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _workload(name):
    sys.path.insert(0, ROOT)
    from gated_delta_rule_138_b200 import inputs
    return inputs.WORKLOADS[name]


def test_default_workload_is_the_long_context_one():
    b = _bench()
    w = _workload(b.DEFAULT_WORKLOAD)
    assert (w.kind, w.B, w.T, w.H, w.dk, w.dv, w.chunk) == ("forward", 1, 1 << 20, 32, 128, 128, 64)
    # 1282 B per (token, head) over 2^20 x 32 token-heads, S_final written (no S0)
    assert b.forward_bytes(w, w.T * w.H, w.H, w.s0) == 1282 * (1 << 25) + 65536 * 32


def test_e2e_pieces():
    b = _bench()
    w = _workload("bf16_B8_T4096_H32_d128")
    assert b.e2e_pieces(w, 8, 4096) == (0, 2)           # batch rows, four pieces
    w2 = _workload(b.DEFAULT_WORKLOAD)
    assert b.e2e_pieces(w2, 1, 1 << 20) == (1, 1 << 17)  # time slices, S chained
    assert b.e2e_pieces(_workload("varlen_64seq_H16_d128"), 1, 1000) == (None, 0)


def test_forward_bytes_and_flops_of_the_batch_workload():
    b = _bench()
    w = _workload("bf16_B8_T4096_H32_d128")
    n_th, n_sh = w.B * w.T * w.H, w.B * w.H
    # bf16 d_k = d_v = 128: 2 (3*128 + 128 + 1) + 2*128 = 1282 B per (token, head)
    assert b.forward_bytes(w, 1, 0, True) == 1282
    # fp32 S0 and S_final: 2 * 4 * 128 * 128 B per (sequence, head); without S0 only S_final
    assert b.forward_bytes(w, 0, 1, True) == 131072
    assert b.forward_bytes(w, 0, 1, False) == 65536
    assert b.forward_bytes(w, n_th, n_sh, True) == 1377828864
    assert b.forward_flops(w, 1) == 6 * 128 * 128 + 2 * 64 * (3 * 128 + 2 * 128) == 180224


def test_backward_bytes_and_flops():
    b = _bench()
    w = _workload("bf16_B8_T4096_H32_d128")
    # per (token, head): bf16 q, k, alpha, v, dout, beta read; fp32 dq, dk, dalpha, dv, dbeta written
    assert b.backward_bytes(w, 1, 0, True) == 2 * (3 * 128 + 2 * 128 + 1) + 4 * (3 * 128 + 128 + 1)
    # per (sequence, head): S0 and dS_final read, dS0 written (fp32)
    assert b.backward_bytes(w, 0, 1, True) == 3 * 4 * 128 * 128
    assert b.backward_bytes(w, 0, 1, False) == 2 * 4 * 128 * 128
    assert b.backward_flops(w, 1) == 31 * 128 * 128


def test_oracle_backward_baseline_sample():
    """The backward line's cpu_baseline times the oracle's backward (not its forward)
    on a bounded sample of the workload."""
    import torch
    b = _bench()
    w = _workload("fp32_T256_d64")
    sys.path.insert(0, ROOT)
    from gated_delta_rule_138_b200 import inputs
    inp = inputs.draw_forward(2, 64, 3, 64, 64, "f32", 5, device="cpu", s0=True)
    w = type(w)(**dict(w.__dict__, B=2, T=64, H=3))
    g = torch.Generator().manual_seed(1)
    dout = torch.randn(2, 64, 3, 64, generator=g)
    dSf = torch.randn(2, 3, 64, 64, generator=g)
    rate, secs, desc = b.time_oracle_backward(w, inp, dout, dSf, 0.01, 2)
    assert rate > 0 and secs > 0 and "backward" in desc


def test_decode_bytes():
    b = _bench()
    w = _workload("decode_N256_H32_d128")
    # the fp32 state read and written once, the token's inputs and output once
    assert b.decode_bytes(w, 1) == 8 * 128 * 128 + 2 * (3 * 128 + 128 + 1) + 2 * 128
    assert b.decode_flops(w, 1) == 6 * 128 * 128


def test_recorded_traffic_lookup():
    b = _bench()
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    rows = [ln.split() for ln in open(path).read().splitlines()
            if ln.strip() and not ln.startswith("#")]
    assert rows, "no DRAM-traffic records"
    for kernel, workload, files, digest, nbytes in rows:
        got = b.recorded_traffic(kernel, workload)
        # a record counts only while the kernel sources still hash to the recorded digest
        if b.kernel_source_digest(files) == digest:
            assert got == float(nbytes)
        else:
            assert got is None
    # no record for a workload or kernel variant that was never captured
    assert b.recorded_traffic("chunk_tc_bf16", "no_such_workload") is None
    assert b.recorded_traffic("chunk_tc_bf16_fused", "bf16_B8_T4096_H32_d128") is None


def _run_reference(extra_env=None):
    env = dict(os.environ)
    env.update(extra_env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--workload", "fp32_T256_d64", "--steps", "1", "--warmup", "3"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_json_line():
    r = _run_reference()
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "fp32_T256_d64"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_do_no_work():
    r = _run_reference({"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_batch_override_is_for_dense_forward_workloads_only():
    """--batch (a smaller batch of the same kernels, for profiler captures) is refused
    before any GPU work on workloads that are not dense forwards."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--workload",
                        "decode_N256_H32_d128", "--batch", "2"], capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 2
    assert "--batch applies to the dense forward workloads" in r.stderr


def test_traffic_records_are_keyed_to_code_not_comments():
    """A DRAM-traffic record stays valid across edits to comments and whitespace only,
    and goes stale on any change to the code itself (string and character literals
    included)."""
    a = "int f(int x) { return x + 1; }  // one\n/* two */ const char* s = \"a // b\";\n"
    b = "int f(int x) {\n  return x + 1;   /* edited */ }\nconst char* s = \"a // b\";  // new\n"
    code_only = _bench().code_only
    assert code_only(a) == code_only(b)
    assert code_only(a) != code_only(a.replace("x + 1", "x + 2"))
    assert code_only(a) != code_only(a.replace("a // b", "a // c"))
    assert code_only("char c = '/'; // x\n") == "char c = '/';"


def test_parity_verdict_fails_on_nan_and_on_the_bars():
    """The bench's own oracle check fails the run (after printing its line) when a
    sampled comparison is not finite or over the bars the tests use."""
    ok = _bench().parity_ok
    good = {"o": {"rel_l2": 3e-3, "worst_head": 3e-3, "worst_row": 5e-3}}
    assert ok(good, 2e-2) and ok(None, 2e-2) and ok({"sample": "x"}, 2e-2)
    nan = float("nan")
    assert not ok({"o": {"rel_l2": nan, "worst_head": nan, "worst_row": nan}}, 2e-2)
    assert not ok({"o": {"rel_l2": 3e-2, "worst_head": 3e-3, "worst_row": 5e-3}}, 2e-2)
    assert not ok({"o": {"rel_l2": 3e-3, "worst_head": 3e-3, "worst_row": 0.11}}, 2e-2)
    assert ok({"o": {"rel_l2": 3e-3, "worst_head": 3e-3, "worst_row": 0.09}}, 2e-2)
    assert not ok(dict(good, S_final={"rel_l2": 1e-4, "worst_head": 1e-4, "worst_row": nan}), 2e-2)
