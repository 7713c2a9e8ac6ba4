"""The C-ABI library loads without a GPU, exports every entry point the header
declares, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_138_b200 as kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(kda_\w+)\s*\(", src))
    return names


def test_header_declares_the_entry_points():
    names = _declared_symbols()
    for want in ("kda_forward", "kda_decode_step", "kda_status_string",
                 "kda_forward_workspace_bytes", "kda_last_error"):
        assert want in names


def test_library_exports_every_declared_symbol():
    lib = kda.load_library()
    missing = [n for n in sorted(_declared_symbols()) if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings():
    assert kda.kda_status_string(0) == "KDA_OK"
    assert kda.kda_status_string(1) == "KDA_ERR_INVALID_ARG"
    assert kda.kda_status_string(2) == "KDA_ERR_UNSUPPORTED"
    assert kda.kda_status_string(3) == "KDA_ERR_CUDA"
    assert kda.kda_status_string(4) == "KDA_ERR_DEVICE_TIMEOUT"
    assert kda.kda_status_string(99) == "KDA_ERR_UNKNOWN"


def _fwd_raw(**over):
    """Call kda_forward with fake (never dereferenced) aligned pointers."""
    lib = kda.load_library()
    p = ctypes.c_void_p(0x10000)
    args = dict(q=p, k=p, v=p, alpha=p, beta=p, S0=None, cu=None, nseq=0, out=p, Sf=None,
                B=1, T=64, H=1, dk=64, dv=64, chunk=64, idt=0, odt=0)
    args.update(over)
    return lib.kda_forward(args["q"], args["k"], args["v"], args["alpha"], args["beta"],
                           args["S0"], args["cu"], args["nseq"], args["out"], args["Sf"],
                           args["B"], args["T"], args["H"], args["dk"], args["dv"],
                           args["chunk"], args["idt"], args["odt"], None)


@pytest.mark.parametrize("over,status", [
    (dict(H=0), 1),                                  # no heads
    (dict(B=-1), 1),
    (dict(T=-5), 1),
    (dict(idt=7), 1),                                # unknown dtype
    (dict(q=None), 1),                               # missing input with tokens
    (dict(q=ctypes.c_void_p(0x10002)), 1),           # q misaligned (needs 16 bytes)
    (dict(beta=ctypes.c_void_p(0x10001)), 1),        # beta not element-aligned
    (dict(cu=ctypes.c_void_p(0x20000), B=2, nseq=1), 1),  # packed needs B == 1
    (dict(dk=96), 2),                                # head dim without a kernel
    (dict(dv=256), 2),
    (dict(chunk=48), 2),
    (dict(B=0), 0),                                  # nothing to do: OK, no launch
])
def test_forward_rejects_before_launch(over, status):
    assert _fwd_raw(**over) == status


def test_decode_rejects_before_launch():
    lib = kda.load_library()
    p = ctypes.c_void_p(0x10000)
    call = lambda N=1, H=1, dk=128, dv=128, q=p, S=p: lib.kda_decode_step(
        q, p, p, p, p, S, p, N, H, dk, dv, 1, 1, None)
    assert call(H=0) == 1
    assert call(q=None) == 1
    assert call(S=ctypes.c_void_p(0x10008)) == 1       # S needs 16 bytes
    assert call(dk=32) == 2
    assert call(N=0) == 0


def test_workspace_query_is_host_only():
    assert kda.kda_forward_workspace_bytes(8, 4096, 32, 128, 128, 64) >= 0


def test_forward_workspace_covers_the_split():
    """The split forward's workspace: per segment a map [M | N] and a start state
    (fp32, d_k (d_k + 2 d_v) values per head and sequence) and, for every token, its
    map row Qg (bf16, as large as the output); unsplit calls need only the status word."""
    assert kda.kda_forward_segments(8, 4096, 32) == 1
    assert kda.kda_forward_workspace_bytes(8, 4096, 32, 128, 128, 64) == 4
    T = 1 << 20
    g = kda.kda_forward_segments(1, T, 32)
    assert g > 1
    assert kda.kda_forward_workspace_bytes(1, T, 32, 128, 128, 64) == \
        4 + 4 * g * 32 * 128 * (128 + 2 * 128) + 2 * T * 32 * 128
    # the fp32 CUDA-core path never splits
    assert kda.kda_forward_workspace_bytes(1, T, 32, 64, 64, 64) == 4


def test_release_workspace_answers_without_a_pool():
    """Trimming the split forward's workspace pool launches nothing: OK when no pool
    exists yet (or CUDA's error code when no device is visible), never a crash."""
    assert kda.load_library().kda_release_workspace() in (0, 3)


def test_selftest_rejects_bad_limit():
    lib = kda.load_library()
    assert lib.kda_selftest_timeout(0, None) == 1
    assert lib.kda_selftest_timeout(20_000_000_000, None) == 1


def test_time_segment_choice():
    """Host logic of the sequence split: only when few (sequence, head) pairs
    would leave SMs idle and the sequences are long enough."""
    seg = kda.kda_forward_segments
    assert seg(8, 4096, 32, 148) == 1            # 256 CTAs already fill 148 SMs
    assert seg(64, 5000, 16, 148) == 1           # packed batch of 1024 CTAs
    assert seg(1, 64 * 31, 1, 148) == 1          # too short for two 16-chunk segments
    assert seg(1, 64 * 32, 1, 148) == 2
    g = seg(1, 1 << 20, 32, 148)                 # 32 CTAs on 148 SMs, 16384 chunks each
    assert 4 <= g <= 64
    last = (32 * g) % 148
    assert last == 0 or last > 100 or (32 * g) <= 148  # the last wave is mostly full
    assert seg(0, 100, 4, 148) == 1 and seg(1, 0, 4, 148) == 1
    for units_h in (1, 2, 4, 8, 16, 32, 64):
        assert 1 <= seg(1, 1 << 22, units_h, 148) <= 64


def test_segment_calls_reject_before_launch():
    lib = kda.load_library()
    # unsupported shape or dtype: no launch, no device touched
    assert lib.kda_segment_maps(None, None, None, None, None, 0, None, 0, 0, 1, 128, 128, 64,
                                0, None) == 2          # fp32 inputs
    assert lib.kda_segment_maps(None, None, None, None, None, 0, None, 0, 0, 1, 64, 64, 64,
                                1, None) == 2          # d = 64
    assert lib.kda_segment_maps(None, None, None, None, None, 0, None, 1, 64, 1, 128, 128, 64,
                                1, None) == 1          # tokens but no pointers
    assert lib.kda_segment_scan(None, None, -1, None, 1, 1, 128, 128, None) == 1
    assert lib.kda_segment_scan(None, None, 0, None, 1, 1, 64, 128, None) == 2
    assert lib.kda_segment_scan(None, None, 1, None, 1, 1, 128, 128, None) == 1   # no out / maps
    assert lib.kda_segment_scan(None, None, 0, None, 0, 1, 128, 128, None) == 0   # nothing to do


def test_split_time_slices():
    import torch
    from gated_delta_rule_138_b200.seqpar import split_time
    x = torch.arange(2 * 12 * 3).reshape(2, 12, 3)
    parts = [split_time(x, 4, r) for r in range(4)]
    assert all(p.shape == (2, 3, 3) for p in parts)
    assert torch.equal(torch.cat(parts, dim=1), x)
    with pytest.raises(ValueError):
        split_time(x, 5, 0)


def test_sequence_parallel_without_process_group_is_one_rank(monkeypatch):
    """No process group: one rank, no maps, no exchange -- just the forward."""
    from gated_delta_rule_138_b200 import seqpar
    calls = []
    monkeypatch.setattr(seqpar.kda, "kda_forward", lambda *a, **k: calls.append("fwd") or ("o", "s"))
    monkeypatch.setattr(seqpar.kda, "kda_segment_maps", lambda *a, **k: calls.append("maps"))
    import torch
    x = torch.zeros(1, 4, 1, 8)
    assert seqpar.kda_forward_sequence_parallel(x, x, x, x, x[..., 0]) == ("o", "s")
    assert calls == ["fwd"]


def test_indexed_calls_reject_before_launch():
    lib = kda.load_library()
    # negative pool size, missing slots, unsupported head dim: no launch
    assert lib.kda_decode_step_indexed(None, None, None, None, None, None, -1, None, None, 0, 1,
                                       128, 128, 1, 1, None) == 1
    assert lib.kda_decode_step_indexed(None, None, None, None, None, None, 4, None, None, 2, 1,
                                       128, 128, 1, 1, None) == 1
    assert lib.kda_forward_indexed(None, None, None, None, None, None, 4, None, None, 0, None,
                                   1, 4, 1, 96, 128, 64, 1, 1, None) == 1   # no pool / slots
    assert lib.kda_forward_indexed(None, None, None, None, None, None, 4, None, None, 0, None,
                                   0, 4, 1, 96, 128, 64, 1, 1, None) == 2   # d_k = 96


def test_backward_rejects_before_launch():
    lib = kda.load_library()
    p = ctypes.c_void_p(0x10000)
    need = kda.kda_backward_workspace_bytes(2, 128, 4, 128, 128)

    def call(B=2, T=128, H=4, dk=128, dv=128, q=p, S0=None, ws=p, ws_bytes=need, dt=1, cu=None,
             nseq=0):
        return lib.kda_backward(q, p, p, p, p, S0, p, None, cu, nseq, p, p, p, p, p, None,
                                B, T, H, dk, dv, dt, ws, ws_bytes, None)
    assert call(H=0) == 1
    assert call(q=None) == 1
    assert call(dt=7) == 1
    assert call(S0=ctypes.c_void_p(0x10008)) == 1        # S0 read with 16-byte accesses
    assert call(ws=ctypes.c_void_p(0x10004)) == 1        # workspace likewise
    assert call(ws_bytes=need - 1) == 1                  # workspace too small
    assert call(dk=32) == 2
    assert call(B=0) == 0                                # nothing to do, nothing launched
    assert call(B=2, cu=p, nseq=1) == 1                  # packed batches have B == 1


def test_backward_workspace_sizes():
    mat = 128 * 128 * 4
    # dense: ceil(T / 8) checkpoints per (sequence, head) plus an 8-state slab
    assert kda.kda_backward_workspace_bytes(8, 4096, 32, 128, 128) == (8 * 512 + 8 * 8) * 32 * mat
    assert kda.kda_backward_workspace_bytes(1, 9, 1, 128, 128) == (2 + 8) * mat
    # packed: floor(T / 8) + num_seqs checkpoints per head
    assert kda.kda_backward_workspace_bytes(1, 1000, 2, 128, 128, num_seqs=3) == \
        ((1000 // 8 + 3) * 2 + 3 * 2 * 8) * mat


def test_noalloc_status_rejects_bad_counts_before_any_copy():
    lib = kda.load_library()
    assert lib.kda_noalloc_status(-1, None, None) == 1
    assert lib.kda_noalloc_status(16384 + 1, None, None) == 1
    assert lib.kda_noalloc_selftest_timeout(0, 0, None) == 1          # zero limit
    assert lib.kda_noalloc_selftest_timeout(1000, -1, None) == 1      # word out of range
    assert lib.kda_noalloc_selftest_timeout(1000, 16384, None) == 1
