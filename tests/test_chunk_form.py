"""The chunk-parallel algebra the CUDA kernels use, restated in fp64 numpy and
checked against the token-by-token oracle.

"FlashKDA parallelizes token processing inside each chunk ... and uses
prefix-scan operations ... to reconstruct correct sequential states" (the
worldcybernews article "Kimi K3 Open Model Surpasses Closed GPT and Anthropic
Systems on Independent Benchmarks", paragraph 3).  The page gives no algebra;
this file writes out the one the kernels implement, so that the algebra is
known to be exact (to fp64 rounding) before any kernel runs:

Per chunk of C tokens (positions r = 0..C-1) with start state S0, a = clamp(alpha):
  decay from token j (exclusive) to token r (inclusive), per key channel:
      D(r, j) = prod_{s=j+1..r} a_s
  A[r, j] = beta_r sum_c k_rc k_jc D(r, j)_c        (j < r, else 0)
  P[r, j] =        sum_c q_rc k_jc D(r, j)_c        (j <= r, else 0)
  T  = (I + A)^-1
  K~ = k * gamma, Q~ = q * gamma, gamma_r = prod_{s<=r} a_s
  K^ = k * eta,   eta_j = prod_{s>j} a_s
  W  = T diag(beta) K~,   U~ = T diag(beta) V
  U  = U~ - W S0
  O  = Q~ S0 + P U  =  (Q~ - P W) S0 + P U~
  S_C = Diag(gamma_{C-1}) S0 + K^^T U

D(r, j) is never formed as a ratio of long products (those leave the fp32
range: a >= e^-5 over 64 tokens reaches e^-320).  It is split at 16-token
sub-chunk boundaries, where a product stays >= e^-80 > the fp32 minimum:
  phi_r = prod_{s=start(I)..r} a_s,   psi_j = prod_{s=j+1..end(J)} a_s,
  pi_I  = prod over sub-chunk I,     Delta_IJ = prod_{J<M<I} pi_M
  I > J:  D(r, j) = (phi_r Delta_IJ) * psi_j
  I = J:  D(r, j) = (phi_r / pi_I) * psi_j      (j <= r)
so A and P are products of a left operand x_r phi_r Delta'_IJ and one right
operand k_j psi_j, with no factor above e^80.  (fp32 CUDA-core kernel.)

The tensor-core kernel uses 32-token sub-chunks with the reference at each
sub-chunk's 16th token instead (one left operand per row, two right operands):
  lam_r   = e^{g_r - g_ref(I(r))}  in [e^-80, e^75]
  rho^I_j = e^{g_ref(I) - g_j}     in (0, e^80], for j < end(I)
with D(r, j) = lam_r rho^{I(r)}_j; a right factor may underflow only where the
true product is negligible.  Both factorizations are checked below.
"""
import numpy as np
import pytest

import oracle

SUB = 16


def _clamp(alpha):
    lo = np.float64(np.float32(np.exp(-5.0)))
    return np.clip(alpha.astype(np.float32).astype(np.float64), lo, 1.0)


def chunk_forward_one(q, k, v, alpha, beta, S0, C):
    """One (sequence, head): q, k, alpha [T, dk]; v [T, dv]; beta [T]; S0 [dk, dv]."""
    T, dk = q.shape
    dv = v.shape[1]
    a_all = _clamp(alpha)
    S = S0.astype(np.float64).copy()
    out = np.zeros((T, dv))
    for t0 in range(0, T, C):
        L = min(C, T - t0)
        # masked tail rows: k = q = v = 0, beta = 0, a = 1
        Q = np.zeros((C, dk)); K = np.zeros((C, dk)); V = np.zeros((C, dv))
        a = np.ones((C, dk)); b = np.zeros(C)
        Q[:L], K[:L], V[:L], a[:L], b[:L] = (q[t0:t0 + L], k[t0:t0 + L], v[t0:t0 + L],
                                             a_all[t0:t0 + L], beta[t0:t0 + L])
        nsub = C // SUB
        phi = np.empty((C, dk)); psi = np.empty((C, dk)); pi = np.empty((nsub, dk))
        for I in range(nsub):
            s, e = I * SUB, (I + 1) * SUB
            phi[s:e] = np.cumprod(a[s:e], axis=0)
            rev = np.ones((SUB, dk))
            for r in range(SUB - 2, -1, -1):
                rev[r] = rev[r + 1] * a[s + r + 1]
            psi[s:e] = rev
            pi[I] = phi[e - 1]
        # left/right operands and A, P by sub-chunk blocks
        R = K * psi
        A = np.zeros((C, C)); P = np.zeros((C, C))
        for I in range(nsub):
            rs = slice(I * SUB, (I + 1) * SUB)
            for J in range(I + 1):
                js = slice(J * SUB, (J + 1) * SUB)
                if I == J:
                    dprime = 1.0 / pi[I]
                else:
                    dprime = np.prod(pi[J + 1:I], axis=0) if I > J + 1 else np.ones(dk)
                A[rs, js] = (K[rs] * phi[rs] * dprime) @ R[js].T
                P[rs, js] = (Q[rs] * phi[rs] * dprime) @ R[js].T
        A = np.tril(A, -1) * b[:, None]
        P = np.tril(P, 0)
        Tm = np.linalg.inv(np.eye(C) + A)
        # chunk-level decays from the sub-chunk products
        gamma = np.empty((C, dk)); eta = np.empty((C, dk))
        for I in range(nsub):
            rs = slice(I * SUB, (I + 1) * SUB)
            before = np.prod(pi[:I], axis=0) if I > 0 else np.ones(dk)
            after = np.prod(pi[I + 1:], axis=0) if I < nsub - 1 else np.ones(dk)
            gamma[rs] = before * phi[rs]
            eta[rs] = psi[rs] * after
        Kt, Qt, Kh = K * gamma, Q * gamma, K * eta
        W = Tm @ (b[:, None] * Kt)
        Ut = Tm @ (b[:, None] * V)
        U = Ut - W @ S
        O1 = Qt @ S + P @ U
        O2 = (Qt - P @ W) @ S + P @ Ut
        assert np.allclose(O1, O2, rtol=1e-10, atol=1e-12)
        out[t0:t0 + L] = O1[:L]
        S = gamma[C - 1][:, None] * S + Kh.T @ U
    return out, S


def mid_reference_factors(a):
    """lam [C, dk], rho0 [32, dk], rho1 [64, dk] for one 64-token chunk of gates a."""
    C, dk = a.shape
    assert C == 64
    phi = np.empty_like(a); psi = np.empty_like(a); pi = np.empty((4, dk))
    for Q in range(4):
        blk = a[16 * Q:16 * Q + 16]
        phi[16 * Q:16 * Q + 16] = np.cumprod(blk, axis=0)
        for i in range(16):
            psi[16 * Q + i] = np.prod(blk[i + 1:], axis=0)
        pi[Q] = phi[16 * Q + 15]
    dq = [1 / pi[0], np.ones(dk), 1 / pi[2], np.ones(dk)]
    c0 = [np.ones(dk), 1 / pi[1]]
    c1 = [pi[1] * pi[2], pi[2], np.ones(dk), 1 / pi[3]]
    lam = np.array([phi[r] * dq[r // 16] for r in range(64)])
    rho0 = np.array([psi[j] * c0[j // 16] for j in range(32)])
    rho1 = np.array([psi[j] * c1[j // 16] for j in range(64)])
    return lam, rho0, rho1


@pytest.mark.parametrize("extreme", [False, True])
def test_mid_reference_factorization(extreme):
    rng = np.random.default_rng(77 + extreme)
    a = np.exp(-np.log1p(np.exp(rng.standard_normal((64, 16)))))
    if extreme:
        a[:, :4] = np.exp(-5.0)
        a[:, 4:8] = 1.0
    lam, rho0, rho1 = mid_reference_factors(a)
    for r in range(64):
        for j in range(r + 1):
            D = np.prod(a[j + 1:r + 1], axis=0)
            rho = rho0[j] if r < 32 else rho1[j]
            np.testing.assert_allclose(lam[r] * rho, D, rtol=1e-12, atol=0)
    lo = np.log(np.float64(np.float32(np.exp(-5.0))))
    assert np.log(lam).min() >= 16 * lo - 1e-9 and np.log(lam).max() <= -15 * lo + 1e-9
    assert np.log(rho0).max() <= -16 * lo + 1e-9 and np.log(rho1).max() <= -16 * lo + 1e-9


def _case(seed, T, dk, dv, extreme=False):
    rng = np.random.default_rng(seed)
    f32 = lambda x: np.asarray(x, np.float32)
    q = rng.standard_normal((T, dk)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((T, dk)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal(T)))
    alpha = np.exp(-np.log1p(np.exp(rng.standard_normal((T, dk)))))
    if extreme:
        # whole channels pinned at the clamp's bounds and below it
        alpha[:, : dk // 4] = 1.0
        alpha[:, dk // 4: dk // 2] = 1e-4
    S0 = 0.1 * rng.standard_normal((dk, dv))
    return f32(q), f32(k), f32(v), f32(alpha), f32(beta), f32(S0)


@pytest.mark.parametrize("C", [16, 32, 64])
@pytest.mark.parametrize("T,extreme", [(1, False), (37, False), (130, False), (200, True)])
def test_chunk_form_equals_oracle(C, T, extreme):
    dk, dv = 32, 16
    q, k, v, al, be, S0 = _case(1000 + T + C, T, dk, dv, extreme)
    ref_o, ref_S = oracle.forward(q[None, :, None], k[None, :, None], v[None, :, None],
                                  al[None, :, None], be[None, :, None], S0[None, None])
    o, S = chunk_forward_one(*(x.astype(np.float64) for x in (q, k, v, al, be, S0)), C)
    np.testing.assert_allclose(o, ref_o[0, :, 0], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S, ref_S[0, 0], rtol=1e-11, atol=1e-12)


def test_subchunk_factors_stay_in_fp32_range():
    """With every gate at the clamp's floor the factors used for A and P stay
    inside the fp32 range: phi, psi >= e^-80 and 1/pi <= e^80."""
    lo = np.float64(np.float32(np.exp(-5.0)))
    phi_min = lo ** SUB
    assert phi_min > np.finfo(np.float32).tiny
    assert 1.0 / phi_min < np.finfo(np.float32).max
    # one token more per sub-chunk would still fit, two sub-chunks would not
    assert lo ** (2 * SUB) < np.finfo(np.float32).tiny


def chunk_maps_one(k, alpha, beta, v, C):
    """The affine state map of a run of tokens, S_end = M S_start + N, built the
    way the tensor-core kernel's summary mode builds it: per chunk
    M_c = Diag(gamma_C) - (k*eta)^T W and N_c = (k*eta)^T Tb V, composed in order."""
    T, dk = k.shape
    dv = v.shape[1]
    a_all = _clamp(alpha)
    M = np.eye(dk)
    N = np.zeros((dk, dv))
    for t0 in range(0, T, C):
        L = min(C, T - t0)
        K = np.zeros((C, dk)); V = np.zeros((C, dv)); a = np.ones((C, dk)); b = np.zeros(C)
        K[:L], V[:L], a[:L], b[:L] = k[t0:t0 + L], v[t0:t0 + L], a_all[t0:t0 + L], beta[t0:t0 + L]
        A = np.zeros((C, C))
        for r in range(C):
            for j in range(r):
                A[r, j] = b[r] * np.sum(K[r] * K[j] * np.prod(a[j + 1:r + 1], axis=0))
        Tb = np.linalg.inv(np.eye(C) + A) * b[None, :]
        gamma = np.cumprod(a, axis=0)
        eta = np.array([np.prod(a[j + 1:], axis=0) for j in range(C)])
        W = Tb @ (K * gamma)
        Mc = np.diag(gamma[C - 1]) - (K * eta).T @ W
        Nc = (K * eta).T @ (Tb @ V)
        M, N = Mc @ M, Mc @ N + Nc
    return M, N


@pytest.mark.parametrize("T,nseg,extreme", [(300, 3, False), (256, 4, True), (130, 5, False), (40, 5, False)])
def test_time_segments_scan_equals_oracle(T, nseg, extreme):
    """Cutting a sequence into runs of whole chunks, chaining the runs' affine
    maps S_{g+1} = M_g S_g + N_g and re-running every run from its own start
    state gives the token recurrence's outputs and final state (the prefix
    scan of the article's paragraph 3, here over segments of one sequence)."""
    C, dk, dv = 16, 16, 8
    q, k, v, al, be, S0 = (x.astype(np.float64) for x in _case(2000 + T, T, dk, dv, extreme))
    ref_o, ref_S = oracle.forward(*(x[None, :, None].astype(np.float32) for x in (q, k, v, al, be)),
                                  S0[None, None].astype(np.float32))
    nch = -(-T // C)
    cps = -(-nch // nseg)
    bounds = [(min(g * cps * C, T), min((g + 1) * cps * C, T)) for g in range(nseg)]
    assert bounds[-1][1] == T
    starts = [S0]
    for g in range(nseg - 1):
        t0, t1 = bounds[g]
        M, N = chunk_maps_one(k[t0:t1], al[t0:t1], be[t0:t1], v[t0:t1], C)
        # the map agrees with running the recurrence from two start states
        o_a, S_a = chunk_forward_one(q[t0:t1], k[t0:t1], v[t0:t1], al[t0:t1], be[t0:t1], starts[-1], C) \
            if t1 > t0 else (None, starts[-1])
        np.testing.assert_allclose(M @ starts[-1] + N, S_a, rtol=1e-10, atol=1e-12)
        starts.append(M @ starts[-1] + N)
    outs = []
    for g, (t0, t1) in enumerate(bounds):
        if t1 == t0:
            continue
        o, S_end = chunk_forward_one(q[t0:t1], k[t0:t1], v[t0:t1], al[t0:t1], be[t0:t1], starts[g], C)
        outs.append(o)
    np.testing.assert_allclose(np.concatenate(outs), ref_o[0, :, 0], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S_end, ref_S[0, 0], rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("T,nseg,extreme", [(300, 3, False), (256, 4, True), (130, 5, False), (40, 5, False)])
def test_split_forward_zero_start_outputs_and_map_rows(T, nseg, extreme):
    """The split forward's one pass per segment: the chunk recurrence on the
    widened state [M | N] from [I | 0], with values [0 | V], ends at the
    segment's map and outputs [Qg | O0], O0 the outputs from a zero start state.
    The output is affine in the start state like the state itself, so with the
    start states chained by the maps, o = O0 + Qg S_g is the token recurrence's
    output and the last map applied to the last start state its final state (the
    prefix scan of the article's paragraph 3)."""
    C, dk, dv = 16, 16, 8
    q, k, v, al, be, S0 = (x.astype(np.float64) for x in _case(2100 + T, T, dk, dv, extreme))
    ref_o, ref_S = oracle.forward(*(x[None, :, None].astype(np.float32) for x in (q, k, v, al, be)),
                                  S0[None, None].astype(np.float32))
    nch = -(-T // C)
    cps = -(-nch // nseg)
    bounds = [(min(g * cps * C, T), min((g + 1) * cps * C, T)) for g in range(nseg)]
    start = S0
    outs = []
    for t0, t1 in bounds:
        v_wide = np.concatenate([np.zeros((t1 - t0, dk)), v[t0:t1]], axis=1)
        if t1 > t0:
            o_wide, MN = chunk_forward_one(q[t0:t1], k[t0:t1], v_wide, al[t0:t1], be[t0:t1],
                                           np.concatenate([np.eye(dk), np.zeros((dk, dv))], axis=1), C)
            Qg, O0 = o_wide[:, :dk], o_wide[:, dk:]
            outs.append(O0 + Qg @ start)
        else:   # an empty segment: the identity map
            MN = np.concatenate([np.eye(dk), np.zeros((dk, dv))], axis=1)
        start = MN[:, :dk] @ start + MN[:, dk:]
    np.testing.assert_allclose(np.concatenate(outs), ref_o[0, :, 0], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(start, ref_S[0, 0], rtol=1e-10, atol=1e-12)
