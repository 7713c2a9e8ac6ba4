"""Host-side checks of the tensor-core backward's per-(chunk, head) record layout
(gated_delta_rule_138_b200/csrc/kda_bwd_record.cuh), which three kernels share: the
forward in record mode writes it, the state-gradient and chunk-gradient kernels read
it back as raw 128-byte-swizzled operand tiles.  Every region must hold its tile,
regions must not overlap, and every tile must start on a 1024-byte boundary (a raw
copy into a 1024-aligned shared buffer keeps the swizzle phase).  Also: the workspace
query covers the records and their headers."""
import os
import re

import gated_delta_rule_138_b200 as kda

HERE = os.path.dirname(os.path.abspath(__file__))
HDR = os.path.join(HERE, "..", "gated_delta_rule_138_b200", "csrc", "kda_bwd_record.cuh")

# bytes of each tile (bf16 unless noted): what the kernels copy into and out of the record
SIZES = {
    "S": 128 * 128 * 2,          # S at the chunk start
    "L": 128 * 128 * 2,          # [k*lam ; q*lam]
    "R": 96 * 128 * 2,           # [k*rho^0 ; k*rho^1]
    "QT": 64 * 128 * 2, "KT": 64 * 128 * 2, "KH": 64 * 128 * 2,
    "P": 64 * 64 * 2, "T": 64 * 64 * 2,
    "RV": 64 * 128 * 2, "U": 64 * 128 * 2,
    "GC": 128 * 4,               # gamma_C, fp32
    "DS": 128 * 128 * 2, "DY": 64 * 128 * 2,
}


def _offsets():
    text = open(HDR).read()
    vals = dict(re.findall(r"constexpr uint32_t (\w+) = (\d+);", text))
    return {k: int(v) for k, v in vals.items()}


def test_regions_fit_align_and_do_not_overlap():
    off = _offsets()
    assert set(SIZES) <= set(off), set(SIZES) - set(off)
    spans = sorted((off[n], off[n] + SIZES[n], n) for n in SIZES)
    for (a0, a1, an), (b0, b1, bn) in zip(spans, spans[1:]):
        assert a1 <= b0, (an, bn)
    for a0, _, n in spans:
        assert a0 % 1024 == 0, n
    assert spans[-1][1] <= off["BYTES"]
    assert off["BYTES"] % 1024 == 0


def test_workspace_query_covers_the_records():
    rec = _offsets()["BYTES"]
    # one chunk of one head: a record and a 1024-byte-rounded header block
    assert kda.kda_backward_workspace_bytes(1, 64, 1, 128, 128) >= rec + 1024
    # B=8, T=4096, H=32: 16384 records (the query is the larger of the two kernels' needs)
    assert kda.kda_backward_workspace_bytes(8, 4096, 32, 128, 128) >= 16384 * rec
    # packed: ceil(T / 64) + num_seqs chunks per head at most
    assert kda.kda_backward_workspace_bytes(1, 1000, 2, 128, 128, num_seqs=3) >= (16 + 3) * 2 * rec
