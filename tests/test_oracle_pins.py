"""Pins for the fp64 CPU oracle (oracle/), checked against what the page and
the mathematics fix -- never against the oracle itself.

Source page: "Kimi K3 Open Model Surpasses Closed GPT and Anthropic Systems on
Independent Benchmarks" (worldcybernews), paragraph 2: a fixed-size state S
updated by the delta rule, beta the write strength, alpha the forgetting,
alpha clamped between e^-5 and 1.  Reading (the page prints no equation):
S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T, o_t = S_t^T q_t,
a_t = clamp(alpha_t, e^-5, 1) per key channel.

Each pin is chosen to catch a class of plausible mistakes:
  hand-worked cases     -> order of decay and write, rows vs columns, sign of
                           the projection, output from the updated state
  identity / pure decay -> Diag(alpha) on key rows, cumulative gating
  write exactness       -> the delta rule's defining property (S^T k = v)
  orthonormal DeltaNet  -> textbook closed form of the ungated delta rule
  clamp                 -> bounds and where the clamp is taken
  linearity, stability, resume, varlen, brute-force matrix product
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng_seed = 20240607
# Which build of the oracle the pins check (None = the real one).  The mutant
# test points this at deliberately broken builds to show the pins catch them.
_LIB = None


def _fwd(*args, **kw):
    return oracle.forward(*args, lib_path=_LIB, **kw)


def _run(q, k, v, alpha, beta, S0=None, cu=None):
    return _fwd(np.asarray(q, np.float32), np.asarray(k, np.float32),
                          np.asarray(v, np.float32), np.asarray(alpha, np.float32),
                          np.asarray(beta, np.float32),
                          None if S0 is None else np.asarray(S0, np.float32), cu)


def _one(x):
    """[T, d] -> [1, T, 1, d] ; [T] -> [1, T, 1]"""
    x = np.asarray(x, np.float64)
    return x[None, :, None, ...] if x.ndim == 2 else x[None, :, None]


def _random_case(rng, T, dk, dv, unit_k=True):
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal(T)))
    alpha = np.exp(-np.log1p(np.exp(rng.standard_normal((T, dk)))))
    S0 = 0.3 * rng.standard_normal((dk, dv))
    f = lambda a: np.asarray(a, np.float32).astype(np.float64)
    return f(q), f(k), f(v), f(alpha), f(beta), f(S0)


def _read_page_constants():
    vals = {}
    with open(os.path.join(GOLDEN, "page_constants.txt")) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if line:
                name, expr = (s.strip() for s in line.split("=", 1))
                vals[name] = expr
    return vals


# ---------------------------------------------------------------- hand-worked

def test_hand_worked_two_steps():
    """d_k = d_v = 2, T = 2, exact arithmetic done by hand.

    S0 = [[1, 2], [3, 4]]  (row c = key channel c)
    t=1: a=(1/2, 1) b=1/2 k=(1,0) v=(2,6) q=(1,1)
         Diag(a)S0 = [[.5, 1], [3, 4]];  k^T S' = (.5, 1)
         S1 = S' - 1/2 k (.5, 1) + 1/2 k (2, 6) = [[1.25, 3.5], [3, 4]]
         o1 = S1^T q = (4.25, 7.5)
    t=2: a=(1, 1/4) b=1 k=(0,1) v=(-1,2) q=(2,-1)
         S' = [[1.25, 3.5], [.75, 1]];  k^T S' = (.75, 1)
         S2 = S' - k (.75, 1) + k (-1, 2) = [[1.25, 3.5], [-1, 2]]
         o2 = S2^T q = (3.5, 5)
    """
    q = [[1, 1], [2, -1]]
    k = [[1, 0], [0, 1]]
    v = [[2, 6], [-1, 2]]
    alpha = [[0.5, 1], [1, 0.25]]
    beta = [0.5, 1]
    S0 = [[[[1, 2], [3, 4]]]]
    out, Sf = _run(_one(q), _one(k), _one(v), _one(alpha), _one(beta), S0)
    assert np.array_equal(out[0, :, 0], [[4.25, 7.5], [3.5, 5.0]])
    assert np.array_equal(Sf[0, 0], [[1.25, 3.5], [-1.0, 2.0]])


def test_hand_worked_projection_sign():
    """Non-axis key, exercises -b k (k^T S) with both channels.

    S0 = [[2], [0]], a = (1, 1), b = 1/2, k = (1, 1), v = (4), q = (1, 0)
    k^T S0 = 2;  S1 = S0 - 1/2 (1,1)^T 2 + 1/2 (1,1)^T 4 = [[3], [1]];  o1 = 3
    (a '+' projection would give [[5], [3]]).
    """
    out, Sf = _run(_one([[1, 0]]), _one([[1, 1]]), _one([[4]]), _one([[1, 1]]),
                   _one([0.5]), [[[[2], [0]]]])
    assert out[0, 0, 0, 0] == 3.0
    assert np.array_equal(Sf[0, 0], [[3.0], [1.0]])


def test_hand_worked_clamp():
    """Inputs outside [e^-5, 1] are clamped (page: alpha between e^-5 and 1).

    S0 = [[1], [1]]
    t=1: alpha = (2, 0) -> a = (1, m) with m = fp32(e^-5); b = 0
         S1 = [[1], [m]];  q = (1, 1000) -> o1 = 1 + 1000 m
    t=2: alpha = (-1, 1.5) -> a = (m, 1); b = 1, k = (1, 0), v = (3)
         S' = [[m], [m]];  k^T S' = m;  S2 = [[3], [m]];  q = (1, 1) -> o2 = 3 + m
    """
    m = Fraction(float(np.float32(math.exp(-5.0))))
    out, Sf = _run(_one([[1, 1000], [1, 1]]), _one([[0, 0], [1, 0]]), _one([[0], [3]]),
                   _one([[2, 0], [-1, 1.5]]), _one([0, 1]), [[[[1], [1]]]])
    assert out[0, 0, 0, 0] == float(1 + 1000 * m)
    assert out[0, 1, 0, 0] == float(3 + m)
    assert np.array_equal(Sf[0, 0, :, 0], [3.0, float(m)])


# ---------------------------------------------------------------- page values

def test_clamp_bounds_are_the_pages():
    c = _read_page_constants()
    assert c["alpha_lower"] == "exp(-5)" and c["alpha_upper"] == "1"
    lo = float(np.float32(math.exp(-5.0)))
    assert oracle.alpha_min(_LIB) == lo
    # pure decay of a single channel over one token, alpha at/below/above the bounds
    for raw, eff in [(1e-9, lo), (lo, lo), (0.5, 0.5), (1.0, 1.0), (7.0, 1.0), (-3.0, lo)]:
        _, Sf = _run(_one([[0.0]]), _one([[0.0]]), _one([[0.0]]), _one([[raw]]),
                     _one([0.0]), [[[[1.0]]]])
        assert Sf[0, 0, 0, 0] == float(np.float32(eff))


def test_context_length_constant():
    assert int(_read_page_constants()["context_length"]) == 1 << 20


# ---------------------------------------------------------------- invariants

def test_identity_alpha1_beta0():
    rng = np.random.default_rng(rng_seed)
    T, dk, dv = 9, 5, 3
    q, k, v, _, _, S0 = _random_case(rng, T, dk, dv)
    out, Sf = _run(_one(q), _one(k), _one(v), _one(np.ones((T, dk))), _one(np.zeros(T)),
                   S0[None, None])
    assert np.array_equal(Sf[0, 0], S0)
    np.testing.assert_allclose(out[0, :, 0], q @ S0, rtol=0, atol=1e-14)


def test_write_exactness_unit_key():
    """a = 1, b = 1, ||k|| = 1 exactly  =>  S_t^T k_t = v_t, and S_t^T w = S_{t-1}^T w
    for every w orthogonal to k_t (the delta rule replaces the value stored
    along k_t and leaves the orthogonal complement alone)."""
    rng = np.random.default_rng(rng_seed + 1)
    T, dk, dv = 7, 8, 3
    # keys with four entries of +-1/2: exactly unit norm in binary
    k = np.zeros((T, dk))
    for t in range(T):
        idx = rng.choice(dk, 4, replace=False)
        k[t, idx] = 0.5 * rng.choice([-1.0, 1.0], 4)
    q, _, v, _, _, S0 = _random_case(rng, T, dk, dv)
    ones = np.ones((T, dk))
    prev = S0
    for t in range(1, T + 1):
        _, Sf = _run(_one(q[:t]), _one(k[:t]), _one(v[:t]), _one(ones[:t]), _one(np.ones(t)),
                     S0[None, None])
        St = Sf[0, 0]
        np.testing.assert_allclose(St.T @ k[t - 1], v[t - 1], rtol=0, atol=1e-14)
        w = rng.standard_normal(dk)
        w -= (w @ k[t - 1]) * k[t - 1]
        np.testing.assert_allclose(St.T @ w, prev.T @ w, rtol=0, atol=1e-13)
        prev = St


def test_pure_decay_closed_form():
    """b = 0: S_T = Diag(prod_t a_t) S0 and o_t = (Diag(prod_{s<=t} a_s) S0)^T q_t."""
    rng = np.random.default_rng(rng_seed + 2)
    T, dk, dv = 11, 6, 4          # dk != dv: a column-wise Diag would fail
    q, k, v, alpha, _, S0 = _random_case(rng, T, dk, dv)
    out, Sf = _run(_one(q), _one(k), _one(v), _one(alpha), _one(np.zeros(T)), S0[None, None])
    cum = np.cumprod(alpha, axis=0)
    for t in range(T):
        np.testing.assert_allclose(out[0, t, 0], (cum[t][:, None] * S0).T @ q[t],
                                   rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(Sf[0, 0], cum[-1][:, None] * S0, rtol=1e-13, atol=0)


def test_scalar_gate_reduces_to_power():
    """alpha equal on all channels (scalar gate), b = 0: S_T = g^T S0."""
    T, dk, dv = 6, 4, 3
    g = 0.75
    S0 = np.arange(dk * dv, dtype=np.float64).reshape(dk, dv) - 5
    _, Sf = _run(_one(np.zeros((T, dk))), _one(np.zeros((T, dk))), _one(np.zeros((T, dv))),
                 _one(np.full((T, dk), g)), _one(np.zeros(T)), S0[None, None])
    assert np.array_equal(Sf[0, 0], g ** T * S0)


def test_orthonormal_deltanet_closed_form():
    """a = 1, b = 1, k_1..k_T orthonormal (plain delta rule):
    S_T = (I - sum_t k_t k_t^T) S0 + sum_t k_t v_t^T."""
    dk, dv = 8, 3
    h4 = 0.5 * np.array([[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]], float)
    basis = np.zeros((dk, dk))
    basis[:4, :4] = h4
    basis[4:, 4:] = h4
    rng = np.random.default_rng(rng_seed + 3)
    order = rng.permutation(dk)[:6]
    k = basis[order]
    T = k.shape[0]
    q, _, v, _, _, S0 = _random_case(rng, T, dk, dv)
    _, Sf = _run(_one(q), _one(k), _one(v), _one(np.ones((T, dk))), _one(np.ones(T)),
                 S0[None, None])
    expect = (np.eye(dk) - k.T @ k) @ S0 + k.T @ v
    np.testing.assert_allclose(Sf[0, 0], expect, rtol=0, atol=1e-14)


def test_clamp_equivalence_random():
    """Raw alpha outside [e^-5, 1] == the same run on pre-clamped alpha."""
    rng = np.random.default_rng(rng_seed + 4)
    T, dk, dv = 13, 6, 5
    q, k, v, alpha, beta, S0 = _random_case(rng, T, dk, dv)
    raw = alpha.copy()
    raw[rng.random((T, dk)) < 0.3] = 1.5
    raw[rng.random((T, dk)) < 0.3] = 1e-4
    raw[0, 0] = -2.0
    lo = np.float32(math.exp(-5.0))
    pre = np.clip(raw.astype(np.float32), lo, np.float32(1.0))
    a = _run(_one(q), _one(k), _one(v), _one(raw), _one(beta), S0[None, None])
    b = _run(_one(q), _one(k), _one(v), _one(pre), _one(beta), S0[None, None])
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_linearity_in_v_and_S0():
    rng = np.random.default_rng(rng_seed + 5)
    T, dk, dv = 10, 5, 4
    q, k, v1, alpha, beta, S01 = _random_case(rng, T, dk, dv)
    v2 = np.asarray(rng.standard_normal((T, dv)), np.float32).astype(np.float64)
    S02 = np.asarray(rng.standard_normal((dk, dv)), np.float32).astype(np.float64)
    # sums of fp32 values are rounded back to fp32 by the call: compare to 1e-6
    o1, s1 = _run(_one(q), _one(k), _one(v1), _one(alpha), _one(beta), S01[None, None])
    o2, s2 = _run(_one(q), _one(k), _one(v2), _one(alpha), _one(beta), S02[None, None])
    o3, s3 = _run(_one(q), _one(k), _one(v1 + v2), _one(alpha), _one(beta),
                  (S01 + S02)[None, None])
    np.testing.assert_allclose(o3, o1 + o2, rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(s3, s1 + s2, rtol=1e-6, atol=1e-6)


def test_stability_bound():
    """b in [0,1], ||k|| = 1, a <= 1: ||S_t||_F <= ||S_{t-1}||_F + b_t ||v_t||."""
    rng = np.random.default_rng(rng_seed + 6)
    T, dk, dv = 12, 6, 4
    q, k, v, alpha, beta, S0 = _random_case(rng, T, dk, dv)
    k = k / np.linalg.norm(k, axis=1, keepdims=True)
    prev = np.linalg.norm(S0)
    for t in range(1, T + 1):
        _, Sf = _run(_one(q[:t]), _one(k[:t]), _one(v[:t]), _one(alpha[:t]), _one(beta[:t]),
                     S0[None, None])
        cur = np.linalg.norm(Sf[0, 0])
        assert cur <= prev + beta[t - 1] * np.linalg.norm(v[t - 1]) + 1e-6
        prev = cur


def test_resume_from_final_state():
    """forward(T) == forward(t0) -> S_final -> forward(T - t0)."""
    rng = np.random.default_rng(rng_seed + 7)
    T, t0, dk, dv = 20, 7, 6, 5
    q, k, v, alpha, beta, S0 = _random_case(rng, T, dk, dv)
    full_o, full_S = _run(_one(q), _one(k), _one(v), _one(alpha), _one(beta), S0[None, None])
    o1, S1 = _run(_one(q[:t0]), _one(k[:t0]), _one(v[:t0]), _one(alpha[:t0]), _one(beta[:t0]),
                  S0[None, None])
    o2, S2 = _run(_one(q[t0:]), _one(k[t0:]), _one(v[t0:]), _one(alpha[t0:]), _one(beta[t0:]),
                  S1.astype(np.float32))
    np.testing.assert_array_equal(o1[0, :, 0], full_o[0, :t0, 0])
    # the hand-off rounds S to fp32, so the tail agrees to fp32 precision
    np.testing.assert_allclose(o2[0, :, 0], full_o[0, t0:, 0], rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(S2, full_S, rtol=1e-5, atol=1e-6)


def test_varlen_equals_independent_sequences():
    rng = np.random.default_rng(rng_seed + 8)
    H, dk, dv = 2, 4, 3
    lens = [5, 1, 0, 9]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    tot = int(cu[-1])
    f = lambda *s: np.asarray(rng.standard_normal(s), np.float32)
    q, k, al, v = f(1, tot, H, dk), f(1, tot, H, dk), f(1, tot, H, dk), f(1, tot, H, dv)
    al = 1 / (1 + np.exp(-al))
    be = 1 / (1 + np.exp(-f(1, tot, H)))
    S0 = f(len(lens), H, dk, dv)
    out, Sf = _fwd(q, k, v, al, be, S0, cu)
    for n, L in enumerate(lens):
        a, b = cu[n], cu[n + 1]
        o_n, S_n = _fwd(q[:, a:b], k[:, a:b], v[:, a:b], al[:, a:b], be[:, a:b],
                                  S0[n:n + 1])
        assert np.array_equal(out[:, a:b], o_n)
        assert np.array_equal(Sf[n], S_n[0])
    # dense batch of equal lengths == packed
    o_d, S_d = _fwd(np.concatenate([q[:, :5], q[:, 6:11]]),
                              np.concatenate([k[:, :5], k[:, 6:11]]),
                              np.concatenate([v[:, :5], v[:, 6:11]]),
                              np.concatenate([al[:, :5], al[:, 6:11]]),
                              np.concatenate([be[:, :5], be[:, 6:11]]),
                              np.stack([S0[0], S0[3]]))
    o_p, S_p = _fwd(q[:, np.r_[0:5, 6:11]], k[:, np.r_[0:5, 6:11]],
                              v[:, np.r_[0:5, 6:11]], al[:, np.r_[0:5, 6:11]],
                              be[:, np.r_[0:5, 6:11]], np.stack([S0[0], S0[3]]),
                              np.array([0, 5, 10], np.int32))
    assert np.array_equal(o_d.reshape(1, 10, H, dv), o_p) and np.array_equal(S_d, S_p)


def test_heads_are_independent():
    rng = np.random.default_rng(rng_seed + 9)
    B, T, H, dk, dv = 2, 6, 3, 4, 5
    f = lambda *s: np.asarray(rng.standard_normal(s), np.float32)
    q, k, v = f(B, T, H, dk), f(B, T, H, dk), f(B, T, H, dv)
    al = 1 / (1 + np.exp(-f(B, T, H, dk)))
    be = 1 / (1 + np.exp(-f(B, T, H)))
    S0 = f(B, H, dk, dv)
    out, Sf = _fwd(q, k, v, al, be, S0)
    for b in range(B):
        for h in range(H):
            o1, s1 = _fwd(q[b:b + 1, :, h:h + 1], k[b:b + 1, :, h:h + 1],
                                    v[b:b + 1, :, h:h + 1], al[b:b + 1, :, h:h + 1],
                                    be[b:b + 1, :, h:h + 1], S0[b:b + 1, h:h + 1])
            assert np.array_equal(out[b, :, h], o1[0, :, 0])
            assert np.array_equal(Sf[b, h], s1[0, 0])


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("T", [1, 2, 4, 6])
def test_brute_force_matrix_product(T):
    """d_k = 3, d_v = 2: explicit update matrices M_t = (I - b_t k_t k_t^T) Diag(a_t),
    S_t = (prod_{s<=t} M_s) S0 + sum_{s<=t} (prod_{s<r<=t} M_r) b_s k_s v_s^T."""
    rng = np.random.default_rng(100 + T)
    dk, dv = 3, 2
    q, k, v, alpha, beta, S0 = _random_case(rng, T, dk, dv, unit_k=False)
    out, Sf = _run(_one(q), _one(k), _one(v), _one(alpha), _one(beta), S0[None, None])
    M = [(np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ np.diag(alpha[t]) for t in range(T)]
    for t in range(T):
        P = np.eye(dk)
        for s in range(t + 1):
            P = M[s] @ P
        St = P @ S0
        for s in range(t + 1):
            R = np.eye(dk)
            for r in range(s + 1, t + 1):
                R = M[r] @ R
            St = St + R @ (beta[s] * np.outer(k[s], v[s]))
        np.testing.assert_allclose(out[0, t, 0], St.T @ q[t], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(Sf[0, 0], St, rtol=1e-13, atol=1e-14)


def test_fused_input_transforms():
    """The fused entry points' transforms against closed forms and limits."""
    x = np.array([-30.0, -2.0, 0.0, 0.5, 3.0, 50.0, 800.0])
    q = np.array([[3.0, 4.0], [0.0, 0.0], [1e-9, 0.0]])
    qh, kh, a, b = oracle.fused_inputs(q, 2 * q, x, x)
    np.testing.assert_allclose(a[:-1], 1.0 / (1.0 + np.exp(x[:-1])), rtol=1e-12, atol=0)
    assert a[2] == 0.5 and b[2] == 0.5 and a[-1] == 0.0 and b[-1] == 1.0
    np.testing.assert_allclose(a + b, 1.0, rtol=0, atol=1e-15)      # sigma(-x) + sigma(x) = 1
    np.testing.assert_allclose(qh[0], [0.6, 0.8], rtol=1e-15)
    np.testing.assert_allclose(kh[0], [0.6, 0.8], rtol=1e-15)       # scale-free
    assert np.all(qh[1] == 0.0)                                      # zero stays zero
    np.testing.assert_allclose(qh[2], [1e-9 / 1e-6, 0.0], rtol=1e-12)   # floored norm
