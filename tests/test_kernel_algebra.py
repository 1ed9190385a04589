"""The tensor-core prefill's restatement of the chunk algebra, in fp64 on the CPU, against
the oracle's sequential recurrence.

The kernels keep raw K, Q, V as tensor-core operands and move normalisation and decay
into per-block matrices and row scales (the block record), then step the state 64 tokens
at a time over two 32-token solves.  This test writes that step out from its formulas --
nothing here is shared with the CUDA code -- and requires it to reproduce the oracle to
rounding, for the rule and for its erase=False form, with a ragged last block.  A slip
in the restated algebra (a sign, a missing decay factor, a misplaced row scale, the
coupling of the two solves) fails here without a GPU.
"""

import numpy as np
import pytest

from gated_delta_rule_145_b200 import synth

EPS = 1e-6


@pytest.mark.parametrize("erase", [True, False])
def test_decode_step_restatement_matches_the_recurrence(erase):
    """The decode kernel reads only k^T S and q^T S of the old state: with gamma = e^g,
    u = k^T S, p = q^T S: delta = beta (v - gamma u) (erase=False: beta v),
    o = gamma p + (q . k) delta, S' = gamma S + k delta^T (q, k normalised)."""
    from oracle import oracle

    inp = synth.make_inputs(3, 1, 2, 4, 8, 8, "f32", seed=77, s0_std=0.5)
    ro, rS = oracle.forward(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                            inp.init_state, erase=erase)
    qh, kh, g, beta = oracle.prepare(inp.q, inp.k, inp.a, inp.b, inp.A_log, inp.dt_bias)
    for bq in range(3):
        for h in range(4):
            kk, qq = kh[bq, 0, h // 2], qh[bq, 0, h // 2]
            S = inp.init_state[bq, h].astype(np.float64)
            gam, bt, v = np.exp(g[bq, 0, h]), beta[bq, 0, h], inp.v[bq, 0, h].astype(np.float64)
            u, p = kk @ S, qq @ S
            delta = bt * (v - gam * u) if erase else bt * v
            o = gam * p + (qq @ kk) * delta
            S1 = gam * S + np.outer(kk, delta)
            np.testing.assert_allclose(o, ro[bq, 0, h], rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(S1, rS[bq, h], rtol=1e-10, atol=1e-12)


def _forward_substitution(A):
    """(I + A)^-1 for strictly lower-triangular A, row by row."""
    n = A.shape[0]
    T = np.zeros((n, n))
    for i in range(n):
        T[i, i] = 1.0
        for j in range(i):
            T[i, j] = -sum(A[i, m] * T[m, j] for m in range(j, i))
    return T


def _blocked_inverse(A, leaf):
    """(I + A)^-1 as the intra-block kernel builds it: forward substitution on the leaf
    diagonal blocks, then at each level T = [[T_a, 0], [-T_b A_ba T_a, T_b]]."""
    n = A.shape[0]
    if n <= leaf:
        return _forward_substitution(A)
    h = n // 2
    Ta, Tb = _blocked_inverse(A[:h, :h], leaf), _blocked_inverse(A[h:, h:], leaf)
    T = np.zeros((n, n))
    T[:h, :h], T[h:, h:] = Ta, Tb
    T[h:, :h] = -Tb @ A[h:, :h] @ Ta
    return T


def _block_step_prefill(q, k, v, beta, g, S0, CB, leaf, erase):
    """The state kernel's step over a block of CB tokens (two solve blocks of CB / 2):
    B = diag(beta) V - diag(w) K S, Delta = T B, O = diag(E) Q S + P Delta,
    S' = gamma S + K^T diag(D) Delta, with T from the blocked inverse."""
    T_len, dk = k.shape
    n = -(-T_len // CB)
    pad = n * CB - T_len
    padz = lambda x: np.concatenate([x, np.zeros((pad,) + x.shape[1:])]) if pad else x
    q, k, v, beta, g = (padz(x) for x in (q, k, v, beta, g))
    o = np.zeros((n * CB, v.shape[1]))
    S = S0.copy()
    lower = np.tril(np.ones((CB, CB), dtype=bool))
    for c in range(n):
        s = slice(c * CB, (c + 1) * CB)
        Kc, Qc, Vc, bc, gc = k[s], q[s], v[s], beta[s], g[s]
        rk = 1.0 / np.sqrt((Kc * Kc).sum(1) + EPS)
        rq = 1.0 / np.sqrt((Qc * Qc).sum(1) + EPS) / np.sqrt(dk)
        G = np.cumsum(gc)
        dec = np.where(lower, np.exp(np.where(lower, G[:, None] - G[None, :], 0.0)), 0.0)
        A = np.where(np.tril(lower, -1), bc[:, None] * dec * rk[:, None] * rk[None, :] * (Kc @ Kc.T), 0.0)
        if not erase:
            A = np.zeros_like(A)
        Tm = _blocked_inverse(A, leaf)
        w = bc * np.exp(G) * rk if erase else np.zeros(CB)
        P = dec * rq[:, None] * rk[None, :] * (Qc @ Kc.T)
        B = bc[:, None] * Vc - w[:, None] * (Kc @ S)
        delta = Tm @ B
        o[s] = (np.exp(G) * rq)[:, None] * (Qc @ S) + P @ delta
        S = np.exp(G[-1]) * S + Kc.T @ ((np.exp(G[-1] - G) * rk)[:, None] * delta)
    return o[:T_len], S


@pytest.mark.parametrize("erase", [True, False])
@pytest.mark.parametrize("T,CB,leaf", [(23, 8, 2), (37, 16, 4), (5, 8, 2), (64, 16, 4)])
def test_block_step_algebra_matches_the_recurrence(erase, T, CB, leaf):
    """The 64-token state step (CB = 64, solves of 32, leaves of 16 in the kernels) at
    small sizes: equal to the oracle's recurrence to rounding, ragged last block included.
    A sign slip in the coupling T_ba = -T_b A_ba T_a, or T_a and T_b swapped, fails here."""
    from oracle import oracle

    inp = synth.make_inputs(1, T, 2, 4, 8, 8, "f32", seed=500 + T + CB, s0_std=0.3)
    ro, rS = oracle.forward(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                            inp.init_state, erase=erase)
    _, _, g, beta = oracle.prepare(inp.q, inp.k, inp.a, inp.b, inp.A_log, inp.dt_bias)
    for h in range(4):
        kh = h // 2
        o, S = _block_step_prefill(inp.q[0, :, kh].astype(np.float64),
                                   inp.k[0, :, kh].astype(np.float64),
                                   inp.v[0, :, h].astype(np.float64), beta[0, :, h], g[0, :, h],
                                   inp.init_state[0, h].astype(np.float64), CB, leaf, erase)
        np.testing.assert_allclose(o, ro[0, :, h], rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(S, rS[0, h], rtol=1e-9, atol=1e-11)


def test_blocked_inverse_is_the_inverse():
    """The leaf/coupling construction equals numpy's inverse of I + A (64 x 64, leaves of
    16: the intra-block kernel's sizes)."""
    rng = np.random.default_rng(11)
    A = np.tril(rng.standard_normal((64, 64)) * 0.2, -1)
    np.testing.assert_allclose(_blocked_inverse(A, 16), np.linalg.inv(np.eye(64) + A),
                               rtol=1e-10, atol=1e-12)
