"""Pins of the oracle's backward pass (reverse mode of the token recurrence).

The pages give no backward formulas; the gradients are defined by the forward
(the worldcybernews article "Kimi K3 Open Model Surpasses Closed GPT and
Anthropic Systems on Independent Benchmarks", paragraph 2, read as the oracle's
recurrence).  So the backward is pinned to the forward itself, not to a second
statement of the same formulas:

* central finite differences of the oracle's forward, L = sum(dout * out) +
  sum(dS_final * S_final), for every input element of small problems;
* closed forms with beta = 0, where the state only decays: S_t =
  Diag(prod_{s<=t} a_s) S0, so every gradient is a sum of explicit products;
* the clamp: no gradient reaches alpha outside [e^-5, 1], and the other
  gradients equal those of the pre-clamped gates;
* packed sequences: the packed result equals the per-sequence results;
* planted mistakes (a dropped term, a wrong sign, a transposed operand) in
  copies of the oracle source each fail at least one pin.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "kda_oracle.c")
GRID = 2.0 ** -16     # inputs on this grid: x +- H_FD stays exact in fp32
H_FD = 2.0 ** -10


def _grid(rng, shape, lo, hi):
    return (np.round(rng.uniform(lo, hi, shape) / GRID) * GRID).astype(np.float32)


def _problem(seed, B=2, T=6, H=1, dk=3, dv=2, beta_zero=False):
    rng = np.random.default_rng(seed)
    p = dict(q=_grid(rng, (B, T, H, dk), -1, 1), k=_grid(rng, (B, T, H, dk), -1, 1),
             v=_grid(rng, (B, T, H, dv), -1, 1), alpha=_grid(rng, (B, T, H, dk), 0.3, 0.95),
             beta=_grid(rng, (B, T, H), 0.1, 0.9), S0=_grid(rng, (B, H, dk, dv), -1, 1))
    if beta_zero:
        p["beta"][:] = 0.0
    up = dict(dout=_grid(rng, (B, T, H, dv), -1, 1), dS_final=_grid(rng, (B, H, dk, dv), -1, 1))
    return p, up


def _loss(p, up, lib_path=None):
    out, Sf = oracle.forward(p["q"], p["k"], p["v"], p["alpha"], p["beta"], p["S0"],
                             lib_path=lib_path)
    return float((out * up["dout"]).sum() + (Sf * up["dS_final"]).sum())


def _grads(p, up, lib_path=None):
    dq, dk, dv, dal, dbe, dS0 = oracle.backward(p["q"], p["k"], p["v"], p["alpha"], p["beta"],
                                                up["dout"], p["S0"], up["dS_final"],
                                                lib_path=lib_path)
    return dict(q=dq, k=dk, v=dv, alpha=dal, beta=dbe, S0=dS0)


def _rel(x, ref):
    den = np.linalg.norm(ref.ravel())
    return float(np.linalg.norm((x - ref).ravel()) / (den if den > 0 else 1.0))


def test_backward_matches_finite_differences(lib_path=None):
    p, up = _problem(1)
    g = _grads(p, up, lib_path)
    for name in ("q", "k", "v", "alpha", "beta", "S0"):
        fd = np.zeros(p[name].shape)
        for idx in np.ndindex(*p[name].shape):
            keep = p[name][idx]
            p[name][idx] = keep + np.float32(H_FD)
            lp = _loss(p, up)
            p[name][idx] = keep - np.float32(H_FD)
            lm = _loss(p, up)
            p[name][idx] = keep
            fd[idx] = (lp - lm) / (2 * H_FD)
        assert _rel(g[name], fd) < 1e-8, (name, _rel(g[name], fd))


def test_backward_pure_decay_closed_form(lib_path=None):
    # beta = 0: S_t = Diag(G_t) S0 with G_t = prod_{s<=t} a_s, o_t = S_t^T q_t
    p, up = _problem(2, B=1, T=5, H=1, dk=3, dv=2, beta_zero=True)
    g = _grads(p, up, lib_path)
    a = p["alpha"][0, :, 0].astype(np.float64)           # [T, dk]
    q = p["q"][0, :, 0].astype(np.float64)
    do = up["dout"][0, :, 0].astype(np.float64)           # [T, dv]
    S0 = p["S0"][0, 0].astype(np.float64)                 # [dk, dv]
    dSf = up["dS_final"][0, 0].astype(np.float64)
    Gt = np.cumprod(a, axis=0)                            # [T, dk]
    T = a.shape[0]
    dq = np.stack([(Gt[t][:, None] * S0) @ do[t] for t in range(T)])
    dS0 = sum(np.outer(Gt[t] * q[t], do[t]) for t in range(T)) + Gt[-1][:, None] * dSf
    # dL/da_s = sum_{t>=s} (G_t / a_s) q_t . (S0 do_t) + (G_T / a_s) sum_n S0 dSf
    w = np.stack([q[t] * (S0 @ do[t]) for t in range(T)])   # [T, dk]
    fin = (S0 * dSf).sum(1)
    dal = np.stack([(sum(Gt[t] * w[t] for t in range(s, T)) + Gt[-1] * fin) / a[s]
                    for s in range(T)])
    assert _rel(g["q"][0, :, 0], dq) < 1e-13
    assert _rel(g["S0"][0, 0], dS0) < 1e-13
    assert _rel(g["alpha"][0, :, 0], dal) < 1e-13
    assert np.abs(g["k"]).max() == 0.0 and np.abs(g["v"]).max() == 0.0
    # dbeta_t = du . (v_t - x_t) with du = G^T k_t: zero only by accident, so check it
    # by a one-sided perturbation of beta away from 0 instead
    eps = 2.0 ** -20
    for t in range(T):
        p["beta"][0, t, 0] = np.float32(eps)
        lp = _loss(p, up)
        p["beta"][0, t, 0] = 0.0
        l0 = _loss(p, up)
        assert abs((lp - l0) / eps - g["beta"][0, t, 0]) < 1e-4 * (1 + abs(g["beta"][0, t, 0]))


def test_backward_clamp(lib_path=None):
    p, up = _problem(3, B=1, T=6, H=2, dk=4, dv=3)
    amin = oracle.alpha_min()
    raw = p["alpha"].copy()
    raw[0, 1, 0, 0] = 0.001          # below e^-5
    raw[0, 3, 1, 2] = 1.25           # above 1
    raw[0, 4, 0, 1] = 1.0            # on the bound: passes
    p_raw = dict(p, alpha=raw)
    p_clamped = dict(p, alpha=np.clip(raw, np.float32(amin), np.float32(1.0)).astype(np.float32))
    g_raw, g_cl = _grads(p_raw, up, lib_path), _grads(p_clamped, up, lib_path)
    assert g_raw["alpha"][0, 1, 0, 0] == 0.0 and g_raw["alpha"][0, 3, 1, 2] == 0.0
    assert g_raw["alpha"][0, 4, 0, 1] != 0.0
    for name in ("q", "k", "v", "beta", "S0"):
        assert np.array_equal(g_raw[name], g_cl[name]), name
    mask = np.ones(raw.shape, bool)
    mask[0, 1, 0, 0] = mask[0, 3, 1, 2] = False
    assert np.array_equal(g_raw["alpha"][mask], g_cl["alpha"][mask])


def test_backward_packed_equals_per_sequence(lib_path=None):
    rng = np.random.default_rng(4)
    lens = [3, 7, 1, 5]
    H, dk, dv = 2, 4, 3
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    f = lambda *s: rng.standard_normal(s).astype(np.float32)
    q, k, v, do = f(1, T, H, dk), f(1, T, H, dk), f(1, T, H, dv), f(1, T, H, dv)
    al = rng.uniform(0.2, 1.0, (1, T, H, dk)).astype(np.float32)
    be = rng.uniform(0, 1, (1, T, H)).astype(np.float32)
    S0, dSf = f(len(lens), H, dk, dv), f(len(lens), H, dk, dv)
    packed = oracle.backward(q, k, v, al, be, do, S0, dSf, cu_seqlens=cu, lib_path=lib_path)
    for n, (a0, a1) in enumerate(zip(cu[:-1], cu[1:])):
        sl = lambda x: x[:, a0:a1]
        one = oracle.backward(sl(q), sl(k), sl(v), sl(al), sl(be), sl(do), S0[n:n + 1],
                              dSf[n:n + 1], lib_path=lib_path)
        for i in range(5):
            assert np.array_equal(packed[i][:, a0:a1], one[i])
        assert np.array_equal(packed[5][n:n + 1], one[5])


PINS = [test_backward_matches_finite_differences, test_backward_pure_decay_closed_form,
        test_backward_clamp, test_backward_packed_equals_per_sequence]

MUTANTS = {
    # the second contribution to dk (through x_t = S'^T k_t) dropped
    "dk_without_projection_term": ("            dkk[t * sk + c] += s;\n", ""),
    # dx taken with the wrong sign
    "dx_sign": ("dx[n] = -bt * s;", "dx[n] = bt * s;"),
    # the carried gradient not decayed (G = dS' instead of Diag(a) dS')
    "carry_without_decay": ("G[(size_t)c * dv + n] = a[c] * dSp[(size_t)c * dv + n];",
                            "G[(size_t)c * dv + n] = dSp[(size_t)c * dv + n];"),
    # the gate gradient taken against S'_t instead of S_{t-1}
    "dalpha_against_decayed": ("s += dSp[(size_t)c * dv + n] * Sprev[(size_t)c * dv + n];",
                               "s += dSp[(size_t)c * dv + n] * Sp[(size_t)c * dv + n];"),
    # dq read from the state before the update
    "dq_from_previous_state": ("s += Scur[(size_t)c * dv + n] * (double)dot[n];",
                               "s += Sprev[(size_t)c * dv + n] * (double)dot[n];"),
    # the output's contribution to G added with q and do swapped (transposed operand)
    "G_output_term_transposed": (
        "G[(size_t)c * dv + n] += (double)qt[c] * (double)dot[n];",
        "G[(size_t)c * dv + n] += (double)qt[n % dk] * (double)dot[c % dv];"),
    # dbeta without the value term
    "dbeta_without_v": ("db += s * ((double)vt[n] - x[n]);", "db += s * (-x[n]);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_backward_pins_catch_mutant(tmp_path, name):
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    c = tmp_path / ("bm_%s.c" % name)
    so = tmp_path / ("libbm_%s.so" % name)
    c.write_text(src.replace(old, new))
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(so),
                    str(c), "-lm"], check=True)
    caught = []
    for pin in PINS:
        try:
            pin(lib_path=str(so))
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, "no pin caught mutant %s" % name
