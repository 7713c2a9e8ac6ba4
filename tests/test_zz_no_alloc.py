"""kda_forward_noalloc: the tensor-core forward for callers that cannot call
cudaMalloc (a process that has handed its device memory to its own pool, or a
latency-critical loop in which an allocation may synchronise the device).  It
keeps its scratch in a fixed array compiled into the library instead of
allocating.  Its results must equal kda_forward's, call after call.

This file is collected last on purpose; it must pass alone in a fresh process
and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import gated_delta_rule_138_b200 as kda
from gated_delta_rule_138_b200 import inputs as gen

from _parity import np32, rel_l2

pytestmark = pytest.mark.gpu

MAX_SEQ_HEADS = 16384  # KDA_NOALLOC_MAX_SEQ_HEADS in include/kda.h


def _pair(inp, cu=None):
    ref_o, ref_S = kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                                   inp["S0"], cu_seqlens=cu)
    out = torch.full_like(ref_o, float("nan"))
    Sf = torch.full_like(ref_S, float("nan"))
    kda.kda_forward_noalloc(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], out, Sf,
                            S0=inp["S0"], cu_seqlens=cu)
    torch.cuda.synchronize()
    return (out, Sf), (ref_o, ref_S)


def test_noalloc_matches_kda_forward_on_consecutive_calls():
    # first call: dense batch with ragged tail; second call: a packed varlen batch
    inp1 = gen.draw_forward(2, 200, 3, 128, 128, "bf16", 901, device="cuda", s0=True)
    (o1, s1), (r1, rs1) = _pair(inp1)
    inp2 = gen.draw_varlen([1, 70, 0, 129], 2, 128, 128, "bf16", 902, device="cuda", s0=True)
    (o2, s2), (r2, rs2) = _pair(inp2, inp2["cu_seqlens"])
    for got, ref in ((o1, r1), (s1, rs1), (o2, r2), (s2, rs2)):
        assert rel_l2(np32(got), np32(ref)) <= 2e-2


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = kda.load_library()
    p = ctypes.c_void_p(0x10000)
    H = 32
    B = MAX_SEQ_HEADS // H + 1          # one (sequence, head) pair too many
    st = lib.kda_forward_noalloc(p, p, p, p, p, None, None, 0, p, None, B, 64, H, 128, 128, 64,
                                 1, 1, None)
    assert st == 2  # KDA_ERR_UNSUPPORTED, before anything is launched
    assert "exceed" in lib.kda_last_error().decode()
    st = lib.kda_forward_noalloc(p, p, p, p, p, None, None, 0, p, None, 1, 64, 2, 64, 64, 64,
                                 1, 1, None)
    assert st == 2  # not the tensor-core configuration
