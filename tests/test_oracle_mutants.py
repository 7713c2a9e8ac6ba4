"""The pins must catch plausible mistakes in the oracle.

Each mutant is a copy of oracle/kda_oracle.c with one deliberate error planted
(on the CPU, in a temporary build); every pin of test_oracle_pins.py is run
against it and at least one must fail.  The real oracle is never modified.
"""
import os
import subprocess

import pytest

import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "kda_oracle.c")

MUTANTS = {
    # the delta projection added instead of subtracted
    "projection_sign": ("S[(size_t)c * w + j] -= bt * kd[c] * proj[j];",
                        "S[(size_t)c * w + j] += bt * kd[c] * proj[j];"),
    # beta dropped from the write term
    "write_without_beta": ("S[(size_t)c * w + j] += bt * kd[c] * (double)vt[j0 + j];",
                           "S[(size_t)c * w + j] += kd[c] * (double)vt[j0 + j];"),
    # the query read with the key (o_t = S_t^T k_t)
    "output_uses_key": ("s += S[(size_t)c * w + j] * (double)qt[c];",
                        "s += S[(size_t)c * w + j] * (double)kt[c];"),
    # the clamp's lower bound set to e^-4
    "clamp_bound": ("0x1.b993fep-8f", "0x1.2c2a4cp-6f"),
    # the clamp's upper bound dropped
    "no_upper_clamp": ("if (y > 1.0f) y = 1.0f;", ""),
    # decay applied after the projection instead of before it
    "decay_after_projection": (
        "        /* S <- Diag(a) S   (row c is key channel c) */\n"
        "        for (int c = 0; c < dk; ++c)\n"
        "            for (int j = 0; j < w; ++j) S[(size_t)c * w + j] *= a[c];\n",
        ""),
    # the gate of token t read from token t-1's slot
    "alpha_off_by_one": ("const float* at = alpha + t * tok_stride_k;",
                         "const float* at = alpha + (t > 0 ? t - 1 : 0) * tok_stride_k;"),
    # the value read from the wrong head (head stride ignored)
    "value_head_offset": ("v + t0 * sv + (int64_t)h * dv", "v + t0 * sv"),
    # the initial state not loaded
    "S0_ignored": ("S[(size_t)c * w + j] = S0 ? (double)S0[(size_t)c * dv + j0 + j] : 0.0;",
                   "S[(size_t)c * w + j] = 0.0;"),
    # the initial state read transposed
    "S0_transposed": ("(double)S0[(size_t)c * dv + j0 + j]", "(double)S0[(size_t)(j0 + j) * dk + c]"),
}

# the after-projection decay mutant needs the decay re-inserted after the write
_DECAY_AFTER = ("        /* o_t = S_t^T q_t */\n",
                "        for (int c = 0; c < dk; ++c)\n"
                "            for (int j = 0; j < w; ++j) S[(size_t)c * w + j] *= a[c];\n"
                "        /* o_t = S_t^T q_t */\n")

PIN_TESTS = [name for name in dir(pins) if name.startswith("test_")]


def _build_mutant(tmp_path, name):
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    src = src.replace(old, new)
    if name == "decay_after_projection":
        src = src.replace(*_DECAY_AFTER)
    c = tmp_path / ("m_%s.c" % name)
    so = tmp_path / ("libm_%s.so" % name)
    c.write_text(src)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(so),
                    str(c), "-lm"], check=True)
    return str(so)


def _run_pin(fn):
    import inspect
    params = inspect.signature(fn).parameters
    if "T" in params:           # parametrized brute force: try all its sizes
        for T in (1, 2, 4, 6):
            fn(T)
    else:
        fn()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(tmp_path, name):
    path = _build_mutant(tmp_path, name)
    caught = []
    pins._LIB = path
    try:
        for t in PIN_TESTS:
            try:
                _run_pin(getattr(pins, t))
            except AssertionError:
                caught.append(t)
    finally:
        pins._LIB = None
    assert caught, "no pin caught mutant %r" % name
