"""The chunk-parallel form of the backward pass, restated in fp64 numpy and
checked against the oracle's token-by-token reverse mode.

The pages give neither the chunk form nor any backward; the forward chunk form
is the one of test_chunk_form.py (per chunk of C tokens with start state S0,
a = clamp(alpha), g_r = sum_{s<=r} log a_s per key channel, gamma = e^g):

    Kt = K * gamma,  Qt = Q * gamma,  Z = K / gamma,  Kh = K * gamma_C / gamma
    A  = strict_lower(diag(beta) Kt Z^T),   P = lower(Qt Z^T),   T = (I + A)^-1
    R  = V - Kt S0,  Y = diag(beta) R,  U = T Y
    O  = Qt S0 + P U,   S_C = diag(gamma_C) S0 + Kh^T U

Its reverse mode, chunk by chunk from the last, carrying only dS across chunk
boundaries (the order a chunk-parallel backward kernel would use):

    dU  = P^T dO + Kh dS_C;          dP = lower(dO U^T)
    dQt = dO S0^T + dP Z;            dZ = dP^T Qt
    dS0 = Qt^T dO + diag(gamma_C) dS_C;   dKh = U dS_C^T
    dY  = T^T dU;  dT = dU Y^T;  dR = diag(beta) dY;  dbeta = rowsum(R * dY)
    dA  = strict_lower(-T^T dT T^T)
    dV  = dR;  dKt = -dR S0^T;  dS0 -= Kt^T dR
    dM  = diag(beta) dA (M = Kt Z^T);  dbeta += rowsum(dA * M);  dKt += dM Z;  dZ += dM^T Kt
    dK  = dKt * gamma + dZ / gamma + dKh * gamma_C / gamma;   dQ = dQt * gamma
    dg  = dKt * Kt - dZ * Z + dQt * Qt - dKh * Kh;   dg[C-1] += sum_j dKh_j * Kh_j + gamma_C * rowsum(S0 * dS_C)
    dlog a_s = sum_{r >= s} dg_r;    dalpha = dlog a / a where e^-5 <= alpha <= 1, else 0

Plain gamma ratios are exact enough in fp64 (a 64-token product of gates >= e^-5
stays above e^-320).  In fp32 a kernel takes the decay gradients of A and P from
the tensor-core forward's bounded sub-chunk factors instead; the last test shows
that form gives the same gradients.
"""
import numpy as np
import pytest

import oracle


def _clamp(alpha):
    lo = np.float32(np.exp(-5.0))
    a32 = alpha.astype(np.float32)
    a = np.clip(a32, lo, np.float32(1.0)).astype(np.float64)
    mask = ((a32 >= lo) & (a32 <= np.float32(1.0))).astype(np.float64)
    return a, mask


def chunk_backward_one(q, k, v, alpha, beta, S0, dout, dSf, C, rnd=None, rnd_decay=None,
                       rnd_elem=None):
    """One (sequence, head): q, k, alpha [T, dk]; v, dout [T, dv]; beta [T];
    S0, dSf [dk, dv].  Returns dq, dk, dv, dalpha, dbeta, dS0 (fp64).

    rnd / rnd_decay (default: none) round the operands of every matrix product, as a
    tensor-core kernel would stage them; rnd_decay applies to the products that feed
    the decay gradient (dQt, dKt, dZ, dKh), rnd to all others.  rnd_elem (default:
    none) rounds the operands Kt, Z, Qt, Kh where the decay gradient multiplies them
    element-wise by their gradients."""
    r = rnd or (lambda x: x)
    r2 = rnd_decay or r
    re_ = rnd_elem or (lambda x: x)
    T, dk = q.shape
    dv = v.shape[1]
    a_all, mask = _clamp(alpha)
    q, k, v, beta, dout = (np.asarray(x, np.float64) for x in (q, k, v, beta, dout))
    nck = (T + C - 1) // C

    def chunk(ci):
        t0 = ci * C
        L = min(C, T - t0)
        Q = np.zeros((C, dk)); K = np.zeros((C, dk)); V = np.zeros((C, dv))
        a = np.ones((C, dk)); b = np.zeros(C); dO = np.zeros((C, dv))
        Q[:L], K[:L], V[:L], a[:L], b[:L], dO[:L] = (q[t0:t0 + L], k[t0:t0 + L], v[t0:t0 + L],
                                                     a_all[t0:t0 + L], beta[t0:t0 + L],
                                                     dout[t0:t0 + L])
        g = np.cumsum(np.log(a), axis=0)
        gam = np.exp(g)
        gC = gam[-1]
        Kt, Qt, Z, Kh = K * gam, Q * gam, K / gam, K * (gC / gam)
        lower = np.tril(np.ones((C, C)))
        strict = np.tril(np.ones((C, C)), -1)
        M = r(Kt) @ r(Z).T
        A = strict * (b[:, None] * M)
        P = lower * (r(Qt) @ r(Z).T)
        Tm = np.linalg.inv(np.eye(C) + A)
        return dict(L=L, t0=t0, Q=Q, K=K, V=V, a=a, b=b, dO=dO, gam=gam, gC=gC, Kt=Kt, Qt=Qt,
                    Z=Z, Kh=Kh, M=M, A=A, P=P, T=Tm, lower=lower, strict=strict)

    # forward over the chunks: the start state of each
    S = np.asarray(S0, np.float64).copy()
    starts = []
    for ci in range(nck):
        c = chunk(ci)
        starts.append(S.copy())
        R = c["V"] - r(c["Kt"]) @ r(S)
        U = r(c["T"]) @ r(c["b"][:, None] * R)
        S = c["gC"][:, None] * S + r(c["Kh"]).T @ r(U)

    dq = np.zeros((T, dk)); dkk = np.zeros((T, dk)); dvv = np.zeros((T, dv))
    dal = np.zeros((T, dk)); dbe = np.zeros(T)
    dS = np.asarray(dSf, np.float64).copy()
    for ci in range(nck - 1, -1, -1):
        c = chunk(ci)
        S0c = starts[ci]
        R = c["V"] - r(c["Kt"]) @ r(S0c)
        Y = c["b"][:, None] * R
        U = r(c["T"]) @ r(Y)
        dO, Tm = c["dO"], c["T"]
        dU = r(c["P"]).T @ r(dO) + r(c["Kh"]) @ r(dS)
        dP = c["lower"] * (r(dO) @ r(U).T)
        dQt = r2(dO) @ r2(S0c).T + r2(dP) @ r2(c["Z"])
        dZ = r2(dP).T @ r2(c["Qt"])
        dS0 = r(c["Qt"]).T @ r(dO) + c["gC"][:, None] * dS
        dKh = r2(U) @ r2(dS).T
        dgC = c["gC"] * (S0c * dS).sum(1)
        dY = r(Tm).T @ r(dU)
        dT = r(dU) @ r(Y).T
        dR = c["b"][:, None] * dY
        db = (R * dY).sum(1)
        dA = c["strict"] * (-(r(Tm).T @ r(dT) @ r(Tm).T))
        dV = dR
        dKt = -r2(dR) @ r2(S0c).T
        dS0 -= r(c["Kt"]).T @ r(dR)
        dM = c["b"][:, None] * dA
        db += (dA * c["M"]).sum(1)
        dKt += r2(dM) @ r2(c["Z"])
        dZ += r2(dM).T @ r2(c["Kt"])
        gam, gC = c["gam"], c["gC"]
        dK = dKt * gam + dZ / gam + dKh * (gC / gam)
        dQ = dQt * gam
        dg = dKt * re_(c["Kt"]) - dZ * re_(c["Z"]) + dQt * re_(c["Qt"]) - dKh * re_(c["Kh"])
        dg[-1] += (dKh * re_(c["Kh"])).sum(0) + dgC
        dloga = np.cumsum(dg[::-1], axis=0)[::-1]
        L, t0 = c["L"], c["t0"]
        dq[t0:t0 + L], dkk[t0:t0 + L], dvv[t0:t0 + L] = dQ[:L], dK[:L], dV[:L]
        dbe[t0:t0 + L] = db[:L]
        dal[t0:t0 + L] = (dloga[:L] / c["a"][:L]) * mask[t0:t0 + L]
        dS = dS0
    return dq, dkk, dvv, dal, dbe, dS


def _rel(x, ref):
    den = np.linalg.norm(ref.ravel())
    return float(np.linalg.norm((x - ref).ravel()) / (den if den > 0 else 1.0))


@pytest.mark.parametrize("C", [16, 32, 64])
@pytest.mark.parametrize("T", [1, 40, 64, 150])
def test_chunk_backward_equals_token_backward(C, T):
    rng = np.random.default_rng(1000 + 7 * C + T)
    dk, dv = 16, 12
    f = lambda *s: rng.standard_normal(s).astype(np.float32)
    q, k = f(T, dk), f(T, dk)
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v, do = f(T, dv), f(T, dv)
    al = np.exp(-np.log1p(np.exp(rng.standard_normal((T, dk))))).astype(np.float32)
    al[:, 0] = 1.0                 # a channel on the upper bound
    al[::7, 1] = 1e-4              # gates below the clamp floor (gradient blocked)
    be = (1 / (1 + np.exp(-rng.standard_normal(T)))).astype(np.float32)
    S0, dSf = f(dk, dv), f(dk, dv)
    got = chunk_backward_one(q, k, v, al, be, S0, do, dSf, C)
    x = lambda a: a[None, :, None]
    ref = oracle.backward(x(q), x(k), x(v), x(al), be[None, :, None], x(do), S0[None, None],
                          dSf[None, None])
    names = ("dq", "dk", "dv", "dalpha", "dbeta", "dS0")
    for name, g_, r in zip(names, got, ref):
        r = r[0, :, 0] if name != "dS0" else r[0, 0]
        assert _rel(g_, r) < 1e-9, (name, _rel(g_, r))


def _decay_grads_gamma_form(K, Q, b, g, dA, dP):
    """dg of A and P through plain gamma = e^g (the form above): X dX - Z dZ + Qt dQt."""
    gam = np.exp(g)
    X, Z, Qt = K * gam, K / gam, Q * gam
    dX = b[:, None] * (dA @ Z)                      # A = strict(diag(b) X Z^T)
    dZ = (b[:, None] * dA).T @ X + dP.T @ Qt        # and P = lower(Qt Z^T)
    dQt = dP @ Z
    return X * dX - Z * dZ + Qt * dQt


def _decay_grads_factored(K, Q, b, g, dA, dP, sub=32):
    """The same gradients from the tensor-core kernel's factors: sub-chunks I of `sub`
    tokens with reference token ref_I = sub I + sub/2 - 1, left factors
    lam_r = e^{g_r - g_ref(I(r))} and right factors rho^I_j = e^{g_ref(I) - g_j}
    (j < end of I), so that D(r, j) = lam_r rho^{I(r)}_j.  With L = K lam, Lq = Q lam,
    R^I = K rho^I:  dg_r = L_r dL_r + Lq_r dLq_r - sum_I R^I_r dR^I_r  (the reference's
    own derivative cancels between left and right)."""
    C = K.shape[0]
    nsub = C // sub
    ref = np.array([sub * (r // sub) + sub // 2 - 1 for r in range(C)])
    lam = np.exp(g - g[ref])
    L, Lq = K * lam, Q * lam
    dg = np.zeros_like(g)
    dL = np.zeros_like(K)
    dLq = np.zeros_like(K)
    for I in range(nsub):
        rows = slice(sub * I, sub * (I + 1))
        cols = slice(0, sub * (I + 1))                 # j < end of I
        rho = np.exp(g[sub * I + sub // 2 - 1] - g[cols])
        R = K[cols] * rho
        dAI, dPI = dA[rows, cols], dP[rows, cols]
        dL[rows] = b[rows, None] * (dAI @ R)
        dLq[rows] = dPI @ R
        dR = (b[rows, None] * dAI).T @ L[rows] + dPI.T @ Lq[rows]
        dg[cols] -= R * dR
        # every factor stays within the fp32 range (e^88): a row is at most sub/2 tokens
        # from its reference and each gate is >= e^-5, so |log lam| <= 5 sub/2 = 80, and
        # log rho <= 80 (tokens before the reference give rho <= 1)
        assert np.all(np.abs(np.log(lam[rows])) <= 5.0 * sub / 2 + 1e-9)
        assert np.all(np.log(rho) <= 5.0 * sub / 2 + 1e-9)
    dg += L * dL + Lq * dLq
    return dg


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_factored_decay_gradients_equal_gamma_form(seed):
    rng = np.random.default_rng(seed)
    C, dk = 64, 24
    K, Q = rng.standard_normal((C, dk)), rng.standard_normal((C, dk))
    a = np.clip(np.exp(-np.log1p(np.exp(rng.standard_normal((C, dk))))), np.exp(-5.0), 1.0)
    a[:, :3] = np.exp(-5.0)                         # channels decaying as fast as allowed
    g = np.cumsum(np.log(a), axis=0)
    b = rng.uniform(0, 1, C)
    dA = np.tril(rng.standard_normal((C, C)), -1)
    dP = np.tril(rng.standard_normal((C, C)))
    want = _decay_grads_gamma_form(K, Q, b, g, dA, dP)
    got = _decay_grads_factored(K, Q, b, g, dA, dP)
    assert np.allclose(got, want, rtol=1e-9, atol=1e-9 * np.abs(want).max())


def _bf16(x):
    """Round to bf16 (nearest even) and widen back, on the host."""
    import torch
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).double().numpy()


def _tf32(x):
    """Round to tf32 (10 mantissa bits, nearest, ties away) and widen back."""
    a = np.array(np.asarray(x, np.float32), copy=True)
    i = a.view(np.uint32)
    i += np.uint32(0x1000)
    i &= np.uint32(0xFFFFE000)
    return a.astype(np.float64)


def test_operand_precision_budget():
    """Which operand precision a tensor-core form of this backward needs.  With every
    product staged in bf16 and the element-wise decay terms taken against unrounded
    operands, dq, dk, dv, dbeta and dS0 stay near 3e-3 of the oracle but dalpha does
    not: the decay gradient sums operand * operand-gradient products that largely
    cancel.  Staging the products that feed it (dQt, dKt, dZ, dKh) in tf32 keeps every
    gradient inside the bf16 bar of 2e-2; so does rounding the element-wise operands
    the way the MMA operands are rounded, with every product in bf16."""
    rng = np.random.default_rng(0)
    T, dk, dv = 256, 128, 128
    n = lambda *s: rng.standard_normal(s)
    q = n(T, dk); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = n(T, dk); k /= np.linalg.norm(k, axis=1, keepdims=True)
    v, do = n(T, dv), n(T, dv)
    al = np.exp(-np.log1p(np.exp(n(T, dk))))
    be = 1 / (1 + np.exp(-n(T)))
    q, k, v, do, al, be = (_bf16(x).astype(np.float32) for x in (q, k, v, do, al, be))
    S0 = (0.1 * n(dk, dv)).astype(np.float32)
    dSf = n(dk, dv).astype(np.float32)
    x = lambda a: a[None, :, None]
    ref = oracle.backward(x(q), x(k), x(v), x(al), be[None, :, None], x(do), S0[None, None],
                          dSf[None, None])
    ref = [r[0, :, 0] for r in ref[:5]] + [ref[5][0, 0]]

    def errs(rnd, rnd_decay, rnd_elem=None):
        got = chunk_backward_one(q, k, v, al, be, S0, do, dSf, 64, rnd, rnd_decay, rnd_elem)
        return [_rel(g_, r) for g_, r in zip(got, ref)]
    all_bf16 = errs(_bf16, _bf16)
    mixed = errs(_bf16, _tf32)
    assert max(all_bf16[i] for i in (0, 1, 2, 4, 5)) < 1e-2
    assert max(mixed) < 2e-2, mixed
    assert all_bf16[3] > 3 * mixed[3], (all_bf16[3], mixed[3])   # dalpha: the sensitive one
    # ... unless the element-wise products take the same bf16 operand values the MMAs
    # read: each (r, j) pair's two ends then cancel exactly, and all-bf16 products keep
    # every gradient, dalpha included, inside the bar (the tensor-core backward's choice)
    consistent = errs(_bf16, _bf16, _bf16)
    assert max(consistent) < 1e-2, consistent
    assert consistent[3] < all_bf16[3] / 3, (consistent[3], all_bf16[3])
