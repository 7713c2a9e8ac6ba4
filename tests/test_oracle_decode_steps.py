"""Pins for oracle.decode_steps, the checker of every decode and serving-step GPU
test.  It re-lays [steps, N, H, d] inputs as [N, steps, H, d] for the token
recurrence; these tests tie that re-layout to things that do not go through it:

- a closed form (alpha = 1, beta = 0 leave S unchanged, so o[t, n, h] =
  S0[n, h]^T q[t, n, h]; worldcybernews article "Kimi K3 Open Model Surpasses
  Closed GPT and Anthropic Systems on Independent Benchmarks", paragraph 2:
  beta is the write strength, alpha the forgetting);
- single-token oracle calls chained by hand, one step at a time, with the state
  carried from each call's S_final into the next call's S0;
- a copy of the adaptor with the plausible mistake (steps taken as sequences)
  fails the same comparison.
"""
import numpy as np

import oracle


def _draw(steps, N, H, dk, dv, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((steps, N, H, dk)).astype(np.float32)
    k = rng.standard_normal((steps, N, H, dk)).astype(np.float32)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((steps, N, H, dv)).astype(np.float32)
    al = rng.uniform(0.3, 1.0, (steps, N, H, dk)).astype(np.float32)
    be = rng.uniform(0.1, 0.9, (steps, N, H)).astype(np.float32)
    S0 = (0.5 * rng.standard_normal((N, H, dk, dv))).astype(np.float32)
    return q, k, v, al, be, S0


def test_identity_gives_readout_of_start_state():
    steps, N, H, dk, dv = 4, 3, 2, 5, 3
    q, k, v, _, _, S0 = _draw(steps, N, H, dk, dv, 1)
    al = np.ones_like(q)
    be = np.zeros((steps, N, H), np.float32)
    out, S = oracle.decode_steps(q, k, v, al, be, S0)
    assert out.shape == (steps, N, H, dv) and S.shape == (N, H, dk, dv)
    want = np.einsum("nhcd,tnhc->tnhd", S0.astype(np.float64), q.astype(np.float64))
    np.testing.assert_allclose(out, want, rtol=0, atol=1e-13)
    np.testing.assert_array_equal(S, S0.astype(np.float64))


def _hand_chained(q, k, v, al, be, S0):
    """One oracle.forward call per step (T = 1 tokens, B = N sequences)."""
    S = S0
    outs = []
    for t in range(q.shape[0]):
        o, S = oracle.forward(q[t][:, None], k[t][:, None], v[t][:, None], al[t][:, None],
                              be[t][:, None], S)
        outs.append(o[:, 0])
    return np.stack(outs), S


def test_equals_single_steps_chained_by_hand():
    q, k, v, al, be, S0 = _draw(3, 2, 2, 6, 4, 2)
    out, S = oracle.decode_steps(q, k, v, al, be, S0)
    ho, hS = _hand_chained(q, k, v, al, be, S0)
    # the hand chain rounds the carried state to fp32 between calls (the oracle
    # takes S0 in fp32); nothing else differs
    np.testing.assert_allclose(out, ho, rtol=0, atol=1e-6)
    np.testing.assert_allclose(S, hS, rtol=0, atol=1e-6)
    # the first step is one call on identical inputs: bit for bit
    o1, S1 = oracle.decode_steps(q[:1], k[:1], v[:1], al[:1], be[:1], S0)
    np.testing.assert_array_equal(o1, ho[:1])


def test_a_misread_layout_is_caught():
    """Steps taken as sequences (no re-layout) does not pass the hand-chain check."""
    q, k, v, al, be, S0 = _draw(3, 3, 2, 6, 4, 3)

    def broken(q, k, v, al, be, S):
        out, S_final = oracle.forward(q, k, v, al, be, S)      # [steps, N] read as [B, T]
        return out, S_final

    ho, hS = _hand_chained(q, k, v, al, be, S0)
    bo, bS = broken(q, k, v, al, be, S0)
    assert np.abs(bo - ho).max() > 1e-2
    assert np.abs(bS - hS).max() > 1e-2
