"""kda_forward_noalloc: the tensor-core forward for callers that cannot call
cudaMalloc (a process that has handed its device memory to its own pool, or a
latency-critical loop in which an allocation may synchronise the device).  It
keeps its scratch -- one status word per (sequence, head) -- in a fixed array
compiled into the library instead of allocating.

Checked here, through the C ABI, on two calls in a row:
- its results equal kda_forward's bit for bit (same kernel, unsplit shapes),
  and match the oracle within the bf16 bar;
- its status words read back as 0, and a bounded wait that gives up is
  reported through them (kda_noalloc_status), after which a call is correct;
- it allocates no device memory.

This file is collected last on purpose; it must pass alone in a fresh process
and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import gated_delta_rule_138_b200 as kda
from gated_delta_rule_138_b200 import inputs as gen

from _parity import check_o, check_S, np32, oracle_forward

pytestmark = pytest.mark.gpu

MAX_SEQ_HEADS = 16384  # KDA_NOALLOC_MAX_SEQ_HEADS in include/kda.h


def _run(inp, cu=None):
    ref_o, ref_S = kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                                   inp["S0"], cu_seqlens=cu)
    out = torch.full_like(ref_o, float("nan"))
    Sf = torch.full_like(ref_S, float("nan"))
    torch.cuda.synchronize()
    before = (torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0])
    kda.kda_forward_noalloc(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], out, Sf,
                            S0=inp["S0"], cu_seqlens=cu)
    torch.cuda.synchronize()
    after = (torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0])
    return (out, Sf), (ref_o, ref_S), before, after


def _check_call(inp, cu, nseq, H):
    (o, s), (ro, rs), before, after = _run(inp, cu)
    # the same tensor-core kernel on the same inputs: identical bits
    assert torch.equal(o, ro) and torch.equal(s, rs)
    # and the oracle on the same bf16 values
    oo, oS = oracle_forward(inp, cu=None if cu is None else np32(cu).astype(np.int32))
    check_o(np32(o), oo, 2e-2)
    check_S(np32(s), oS, 2e-2)
    # every (sequence, head) CTA reported a completed run
    words = kda.kda_noalloc_status(nseq * H)
    assert words == [0] * (nseq * H)
    return before, after


def test_noalloc_matches_kda_forward_and_oracle_on_consecutive_calls():
    # first call: dense batch with a ragged tail; second: a packed batch with an empty sequence
    inp1 = gen.draw_forward(2, 200, 3, 128, 128, "bf16", 901, device="cuda", s0=True)
    _check_call(inp1, None, 2, 3)
    inp2 = gen.draw_varlen([1, 70, 0, 129], 2, 128, 128, "bf16", 902, device="cuda", s0=True)
    before, after = _check_call(inp2, inp2["cu_seqlens"], 4, 2)
    # the second call (its kernel already loaded) allocates nothing, through torch or not
    assert after == before


def test_noalloc_reports_a_timeout_through_its_status_words():
    """A bounded wait that gives up (nothing arrives on its barrier) is written
    into the fixed array as a forward CTA writes it; kda_noalloc_status reports
    it, and the next call is correct and reports clean words."""
    kda.kda_noalloc_selftest_timeout(2_000_000, 5)        # 2 ms limit, word 5
    words = kda.kda_noalloc_status(8, check=False)
    assert words[5] == 1
    with pytest.raises(kda.KdaError) as ei:
        kda.kda_noalloc_status(8)
    assert ei.value.status == 4                           # KDA_ERR_DEVICE_TIMEOUT
    inp = gen.draw_forward(2, 130, 3, 128, 128, "bf16", 903, device="cuda", s0=True)
    _check_call(inp, None, 2, 3)                          # rewrites words 0..5


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
