"""GPU parity: the CUDA path, called through the C ABI, against the fp64 oracle
on the same seeded inputs.  Bars: relative L2 <= 1e-5 for fp32 inputs and
<= 2e-2 for bf16 inputs (the oracle then runs on the same bf16 values)."""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_138_b200 as kda
from gated_delta_rule_138_b200 import inputs as gen

from _parity import check_o, check_S, np32, oracle_forward, tolerance

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _forward_case(B, T, H, dk, dv, dtype, chunk, s0, seed, out_dtype=None):
    inp = gen.draw_forward(B, T, H, dk, dv, dtype, seed, device=DEV, s0=s0)
    out, Sf = kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                              inp["S0"], chunk=chunk, out_dtype=out_dtype)
    torch.cuda.synchronize()
    ref_o, ref_S = oracle_forward(inp)
    return inp, out, Sf, ref_o, ref_S


def test_fp32_small_workload():
    """fp32, B=1, H=1, T=256, d=64, chunk 64, S0 = 0: the oracle-sized workload."""
    w = gen.WORKLOADS["fp32_T256_d64"]
    _, out, Sf, ro, rS = _forward_case(w.B, w.T, w.H, w.dk, w.dv, w.dtype, w.chunk, w.s0, w.seed)
    assert out.dtype == torch.float32
    check_o(np32(out), ro, 1e-5)
    check_S(np32(Sf), rS, 1e-5)


@pytest.mark.parametrize("B,T,H,dk,dv,chunk,s0", [
    (1, 1, 1, 64, 64, 64, False),      # one token
    (2, 37, 3, 64, 128, 16, True),     # ragged tail, chunk 16
    (1, 130, 2, 128, 64, 32, True),    # ragged, chunk 32
    (1, 200, 2, 128, 128, 64, True),   # several chunks + tail
    (3, 64, 1, 64, 64, 64, True),      # exactly one chunk
])
def test_fp32_shapes(B, T, H, dk, dv, chunk, s0):
    _, out, Sf, ro, rS = _forward_case(B, T, H, dk, dv, "f32", chunk, s0, 11 + T)
    check_o(np32(out), ro, 1e-5)
    check_S(np32(Sf), rS, 1e-5)


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("B,T,H,dk,dv", [(2, 300, 4, 128, 128), (1, 65, 2, 64, 128)])
def test_bf16_small(B, T, H, dk, dv, out_dtype):
    _, out, Sf, ro, rS = _forward_case(B, T, H, dk, dv, "bf16", 64, True, 21 + T,
                                       out_dtype=out_dtype)
    assert out.dtype == out_dtype
    check_o(np32(out), ro, 2e-2)
    check_S(np32(Sf), rS, 2e-2)


def test_zero_length_keeps_state():
    inp = gen.draw_forward(2, 0, 3, 64, 64, "f32", 5, device=DEV, s0=True)
    out, Sf = kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S0"])
    torch.cuda.synchronize()
    assert out.numel() == 0
    assert torch.equal(Sf, inp["S0"])


def test_state_in_place_alias():
    inp = gen.draw_forward(1, 100, 2, 128, 128, "f32", 6, device=DEV, s0=True)
    S = inp["S0"].clone()
    ro, rS = oracle_forward(inp)
    out, Sf = kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], S,
                              S_final=S)
    torch.cuda.synchronize()
    assert Sf.data_ptr() == S.data_ptr()
    check_S(np32(S), rS, 1e-5)
    check_o(np32(out), ro, 1e-5)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_varlen_small(dtype):
    lengths = [1, 15, 0, 64, 65, 130, 7]
    inp = gen.draw_varlen(lengths, 2, 128, 128, dtype, 300, device=DEV, s0=True)
    out, Sf = kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                              inp["S0"], cu_seqlens=inp["cu_seqlens"])
    torch.cuda.synchronize()
    ro, rS = oracle_forward(inp, cu=np32(inp["cu_seqlens"]).astype(np.int32))
    tol = tolerance(inp["q"].dtype)
    check_o(np32(out), ro, tol)
    check_S(np32(Sf), rS, tol)


def test_output_canaries_untouched():
    """Poisoned guard regions around out and S_final stay as they were."""
    B, T, H, dk, dv = 1, 77, 2, 128, 128
    inp = gen.draw_forward(B, T, H, dk, dv, "bf16", 8, device=DEV, s0=True)
    n_out, n_S = B * T * H * dv, B * H * dk * dv
    pad = 4096
    ob = torch.full((n_out + 2 * pad,), 1536.0, device=DEV).to(torch.bfloat16)
    sb = torch.full((n_S + 2 * pad,), -777.0, device=DEV)
    out = ob[pad:pad + n_out].view(B, T, H, dv)
    Sf = sb[pad:pad + n_S].view(B, H, dk, dv)
    kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S0"],
                    out=out, S_final=Sf)
    torch.cuda.synchronize()
    assert torch.all(ob[:pad] == 1536.0) and torch.all(ob[pad + n_out:] == 1536.0)
    assert torch.all(sb[:pad] == -777.0) and torch.all(sb[pad + n_S:] == -777.0)
    ro, rS = oracle_forward(inp)
    check_o(np32(out), ro, 2e-2)
    check_S(np32(Sf), rS, 2e-2)


# ------------------------------------------------------------------ decode

def _decode_run(N, H, dk, dv, steps, dtype, seed):
    d = gen.draw_decode(N, H, dk, dv, steps, dtype, seed, device=DEV)
    S = d["S"].clone()
    outs = []
    for t in range(steps):
        outs.append(kda.kda_decode_step(d["q"][t], d["k"][t], d["v"][t], d["alpha"][t],
                                        d["beta"][t], S))
    torch.cuda.synchronize()
    return d, torch.stack(outs), S


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_decode_small(dtype, dk, dv):
    N, H, steps = 5, 3, 6
    d, out, S = _decode_run(N, H, dk, dv, steps, dtype, 40 + dk + dv)
    ro, rS = oracle.decode_steps(np32(d["q"]), np32(d["k"]), np32(d["v"]), np32(d["alpha"]),
                                 np32(d["beta"]), np32(d["S"]))
    tol = tolerance(d["q"].dtype)
    check_o(np32(out), ro, tol, time_axis=0)
    check_S(np32(S), rS, tol)


def test_decode_canaries_untouched():
    N, H, dk, dv = 3, 2, 128, 128
    d = gen.draw_decode(N, H, dk, dv, 1, "bf16", 9, device=DEV)
    pad = 1024
    sb = torch.full((N * H * dk * dv + 2 * pad,), 55.0, device=DEV)
    S = sb[pad:pad + N * H * dk * dv].view(N, H, dk, dv)
    S.copy_(d["S"])
    ob = torch.full((N * H * dv + 2 * pad,), 3.0, device=DEV).to(torch.bfloat16)
    out = ob[pad:pad + N * H * dv].view(N, H, dv)
    kda.kda_decode_step(d["q"][0], d["k"][0], d["v"][0], d["alpha"][0], d["beta"][0], S, out=out)
    torch.cuda.synchronize()
    assert torch.all(sb[:pad] == 55.0) and torch.all(sb[-pad:] == 55.0)
    assert torch.all(ob[:pad] == 3.0) and torch.all(ob[-pad:] == 3.0)


# ------------------------------------------------ full-size workloads, sampled

def test_full_bf16_batch_sampled():
    """B=8, H=32, T=4096, d=128: whole run on the GPU, oracle on sampled (b, h)."""
    w = gen.WORKLOADS["bf16_B8_T4096_H32_d128"]
    inp = gen.draw_workload(w, device=DEV)
    out, Sf = kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                              inp["S0"], chunk=w.chunk)
    torch.cuda.synchronize()
    for b, h in [(0, 0), (3, 17), (7, 31)]:
        ro, rS = oracle_forward(inp, b=b, h=h)
        check_o(np32(out[b:b + 1, :, h:h + 1]), ro, 2e-2)
        check_S(np32(Sf[b:b + 1, h:h + 1]), rS, 2e-2)


def test_full_decode_sampled():
    """N=256, H=32, d=128, 128 consecutive steps; oracle on sampled (n, h)."""
    w = gen.WORKLOADS["decode_N256_H32_d128"]
    d, out, S = _decode_run(w.B, w.H, w.dk, w.dv, w.steps, w.dtype, w.seed)
    for n, h in [(0, 0), (100, 5), (255, 31)]:
        sl = lambda x: np32(x[:, n:n + 1, h:h + 1])
        ro, rS = oracle.decode_steps(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["alpha"]),
                                     sl(d["beta"]), np32(d["S"][n:n + 1, h:h + 1]))
        check_o(np32(out[:, n:n + 1, h:h + 1]), ro, 2e-2, time_axis=0)
        check_S(np32(S[n:n + 1, h:h + 1]), rS, 2e-2)


def test_full_varlen_sampled():
    """64 packed sequences, log-uniform lengths in [128, 32768], H=16, d=128."""
    w = gen.WORKLOADS["varlen_64seq_H16_d128"]
    inp = gen.draw_workload(w, device=DEV)
    cu = np32(inp["cu_seqlens"]).astype(np.int64)
    out, Sf = kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                              inp["S0"], cu_seqlens=inp["cu_seqlens"], chunk=w.chunk)
    torch.cuda.synchronize()
    lens = np.diff(cu)
    picks = [int(np.argmin(lens)), int(np.argmax(lens)), 17]
    for n in picks:
        a, b = int(cu[n]), int(cu[n + 1])
        for h in (0, 15):
            sub = {key: inp[key][:, a:b] for key in ("q", "k", "v", "alpha", "beta")}
            sub["S0"] = inp["S0"][n:n + 1]
            ro, rS = oracle_forward(sub, h=h)
            check_o(np32(out[:, a:b, h:h + 1]), ro, 2e-2)
            check_S(np32(Sf[n:n + 1, h:h + 1]), rS, 2e-2)


def test_full_long_context_sampled():
    """B=1, H=32, T=2^20, d=128 with clamp-stressing gates: o on the first 65,536
    tokens of two heads and S_final after all 2^20 tokens of one head."""
    w = gen.WORKLOADS["bf16_B1_T1M_H32_d128"]
    inp = gen.draw_workload(w, device=DEV)
    out, Sf = kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                              None, chunk=w.chunk)
    torch.cuda.synchronize()
    for h in (0, 31):
        ro, _ = oracle_forward(inp, h=h, t1=65536)
        check_o(np32(out[:, :65536, h:h + 1]), ro, 2e-2)
    _, rS = oracle_forward(inp, h=7)
    check_S(np32(Sf[:, 7:8]), rS, 2e-2)


# ------------------------------------------------ tensor-core path specifics

def test_tc_kernel_selected_for_bf16_d128():
    assert kda.kda_forward_kernel_name(128, 128, 64, torch.bfloat16) == "chunk_tc_bf16"
    assert kda.kda_forward_kernel_name(128, 128, 64, torch.bfloat16, torch.float32) == "chunk_simt_f32"
    assert kda.kda_forward_kernel_name(64, 64, 64, torch.float32) == "chunk_simt_f32"


@pytest.mark.parametrize("T", [1, 63, 64, 65, 64 * 5 + 17])
def test_tc_ragged_lengths(T):
    inp = gen.draw_forward(2, T, 3, 128, 128, "bf16", 500 + T, device=DEV, s0=True)
    out, Sf = kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S0"])
    torch.cuda.synchronize()
    kda.kda_device_status()
    ro, rS = oracle_forward(inp)
    check_o(np32(out), ro, 2e-2)
    check_S(np32(Sf), rS, 2e-2)


def test_tc_extreme_gates():
    """Whole channels at alpha = 1, below the clamp floor, and at the floor: the
    sub-chunk factors reach e^-80 and 1/pi reaches e^80."""
    inp = gen.draw_forward(1, 300, 2, 128, 128, "bf16", 600, device=DEV, s0=True)
    al = inp["alpha"]
    al[..., :40] = 1.0
    al[..., 40:80] = 1e-4
    al[..., 80:90] = gen.BF16_BELOW_EXP_M5
    out, Sf = kda.kda_forward(inp["q"], inp["k"], inp["v"], al, inp["beta"], inp["S0"])
    torch.cuda.synchronize()
    ro, rS = oracle_forward(inp)
    check_o(np32(out), ro, 2e-2)
    check_S(np32(Sf), rS, 2e-2)


def test_tc_matches_fp32_path():
    """The tensor-core kernel and the fp32 CUDA-core kernel agree on the same
    bf16 inputs (the latter selected by asking for an fp32 output)."""
    inp = gen.draw_forward(2, 333, 4, 128, 128, "bf16", 700, device=DEV, s0=True)
    o_tc, S_tc = kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S0"])
    o_f, S_f = kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S0"],
                               out_dtype=torch.float32)
    torch.cuda.synchronize()
    check_o(np32(o_tc), np32(o_f), 2e-2)
    check_S(np32(S_tc), np32(S_f), 2e-2)


# ------------------------------------------------ time segments (sequence split + scan)

@pytest.mark.parametrize("B,T,H", [(1, 64 * 65 + 37, 2), (2, 64 * 40, 1)])
def test_tc_time_segments(B, T, H):
    """Few (sequence, head) pairs and long sequences: the forward is split along
    time (segment maps, fp32 scan of start states, forward of every segment).
    Parity with the oracle, and with the unsplit kernel on the same inputs."""
    nseg = kda.kda_forward_segments(B, T, H)
    assert nseg > 1
    inp = gen.draw_forward(B, T, H, 128, 128, "bf16", 900 + T, device=DEV, s0=True)
    out, Sf = kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S0"])
    o1 = torch.empty_like(out)
    S1 = torch.empty_like(Sf)
    kda.kda_forward_noalloc(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], o1, S1,
                            inp["S0"])
    torch.cuda.synchronize()
    kda.kda_device_status()
    ro, rS = oracle_forward(inp)
    check_o(np32(out), ro, 2e-2)
    check_S(np32(Sf), rS, 2e-2)
    check_o(np32(out), np32(o1), 1e-2)
    check_S(np32(Sf), np32(S1), 1e-2)


def test_tc_time_segments_varlen_with_empty_segments():
    """A packed batch whose short sequences leave some segments empty (one
    chunk, zero tokens) next to a long one that is cut into several."""
    lengths = [20000, 40, 0, 3000]
    total = sum(lengths)
    assert kda.kda_forward_segments(len(lengths), -(-total // len(lengths)), 1) >= 4
    inp = gen.draw_varlen(lengths, 1, 128, 128, "bf16", 910, device=DEV, s0=True)
    out, Sf = kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                              inp["S0"], cu_seqlens=inp["cu_seqlens"])
    torch.cuda.synchronize()
    kda.kda_device_status()
    ro, rS = oracle_forward(inp, cu=np32(inp["cu_seqlens"]).astype(np.int32))
    check_o(np32(out), ro, 2e-2)
    for n in range(len(lengths)):
        check_S(np32(Sf[n:n + 1]), rS[n:n + 1], 2e-2)
    # the empty sequence keeps its start state exactly
    assert torch.equal(Sf[2], inp["S0"][2])


def test_tc_time_segments_state_in_place():
    """S_final aliasing S0 under the split: the start states are taken by the
    scan before any segment writes S_final."""
    B, T, H = 1, 64 * 48 + 5, 2
    assert kda.kda_forward_segments(B, T, H) > 1
    inp = gen.draw_forward(B, T, H, 128, 128, "bf16", 920, device=DEV, s0=True)
    ro, rS = oracle_forward(inp)
    S = inp["S0"].clone()
    out, _ = kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], S, S_final=S)
    torch.cuda.synchronize()
    check_o(np32(out), ro, 2e-2)
    check_S(np32(S), rS, 2e-2)


# ------------------------------------------------ failure detection (no fault, no hang)

def test_bounded_wait_reports_timeout_and_context_survives():
    """A wait on a barrier that nothing arrives on gives up after its limit and
    reports KDA_ERR_DEVICE_TIMEOUT through the status word; the context stays
    usable and a later forward is still correct."""
    kda.kda_device_status()                       # clean slate
    kda.kda_selftest_timeout(2_000_000)           # 2 ms limit
    with pytest.raises(kda.KdaError) as ei:
        kda.kda_device_status()
    assert ei.value.status == 4                   # KDA_ERR_DEVICE_TIMEOUT
    kda.kda_device_status()                       # cleared by the read
    _, out, Sf, ro, rS = _forward_case(1, 100, 2, 128, 128, "bf16", 64, True, 808)
    check_o(np32(out), ro, 2e-2)
    check_S(np32(Sf), rS, 2e-2)
