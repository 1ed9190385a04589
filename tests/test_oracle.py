"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each ``check_*`` function raises AssertionError on a mismatch.  The tests run them
on the oracle as built, and ``test_planted_mistakes_are_caught`` runs them on copies
of the oracle with one plausible mistake compiled in (a flipped erase sign, a dropped
1/sqrt(dk), the output taken before the update, a flipped gate sign): each copy must
fail at least one pin, which shows the pins bite.

Sources: Mila "GatedDeltaRule.ixx File Reference", Detailed Description (the step,
the normalisation, the gates, the two forms); tessera PR #77 "Track L -- genuine
gated delta rule + Mamba2 SSM", summary (brute-force erase check, erase=False as
gated linear attention, chunk-size invariance, streaming decode equal to recompute,
the contraction / numeric-policy finding).
"""

import math
import os

import numpy as np
import pytest

from oracle import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_raw(rng, T, Hk, Hv, dk, dv, s0=0.3, nseq=1):
    q = rng.standard_normal((1, T, Hk, dk)).astype(np.float32)
    k = rng.standard_normal((1, T, Hk, dk)).astype(np.float32)
    v = rng.standard_normal((1, T, Hv, dv)).astype(np.float32)
    a = rng.standard_normal((1, T, Hv)).astype(np.float32)
    b = rng.standard_normal((1, T, Hv)).astype(np.float32)
    A_log = rng.uniform(0, math.log(16), Hv).astype(np.float32)
    dt = np.exp(rng.uniform(math.log(1e-3), math.log(1e-1), Hv))
    dt_bias = np.log(np.expm1(dt)).astype(np.float32)
    S0 = (s0 * rng.standard_normal((nseq, Hv, dk, dv))).astype(np.float64)
    return q, k, v, a, b, A_log, dt_bias, S0


def _close(x, y, rtol, what):
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    scale = max(1.0, float(np.max(np.abs(y))))
    err = float(np.max(np.abs(x - y))) if x.size else 0.0
    assert err <= rtol * scale, f"{what}: max abs err {err:.3e} > {rtol:.1e} * {scale:.3e}"


# ------------------------------------------------------------------------------ pins


def check_bruteforce(lib):
    """(i) O1 equals the explicit erase-matrix products (O2), tiny sizes, dk != dv too."""
    rng = np.random.default_rng(11)
    for dk, dv, T in ((4, 4, 9), (6, 3, 12), (3, 7, 8)):
        q, k, v, a, b, A_log, dtb, S0 = _rand_raw(rng, T, 1, 1, dk, dv)
        qh, kh, g, beta = oracle.prepare(q, k, a, b, A_log, dtb, lib=lib)
        o, S = oracle.core(qh, kh, v, g, beta, S0, lib=lib)
        o2, states = oracle.bruteforce_states(qh[0, :, 0], kh[0, :, 0], v[0, :, 0].astype(
            np.float64), g[0, :, 0], beta[0, :, 0], S0[0, 0])
        _close(o[0, :, 0], o2, 1e-12, f"o vs brute force dk={dk} dv={dv}")
        _close(S[0, 0], states[-1], 1e-12, f"S vs brute force dk={dk} dv={dv}")


def check_gla(lib):
    """(ii) erase=False is gated linear attention: equals the closed-form sum (O3)."""
    rng = np.random.default_rng(12)
    dk, dv, T = 5, 4, 20
    q, k, v, a, b, A_log, dtb, S0 = _rand_raw(rng, T, 1, 1, dk, dv)
    qh, kh, g, beta = oracle.prepare(q, k, a, b, A_log, dtb, lib=lib)
    o, S = oracle.core(qh, kh, v, g, beta, S0, erase=False, lib=lib)
    o3, S3 = oracle.gla_closed_form(qh[0, :, 0], kh[0, :, 0], v[0, :, 0].astype(np.float64),
                                    g[0, :, 0], beta[0, :, 0], S0[0, 0])
    _close(o[0, :, 0], o3, 1e-12, "o vs GLA closed form")
    _close(S[0, 0], S3, 1e-12, "S vs GLA closed form")


def check_chunk_invariance(lib):
    """(iii) the chunked UT algebra (O4) equals O1 for every chunk size, ragged tail."""
    rng = np.random.default_rng(13)
    dk, dv, T = 8, 6, 70
    q, k, v, a, b, A_log, dtb, S0 = _rand_raw(rng, T, 1, 1, dk, dv)
    qh, kh, g, beta = oracle.prepare(q, k, a, b, A_log, dtb, lib=lib)
    o, S = oracle.core(qh, kh, v, g, beta, S0, lib=lib)
    args = (qh[0, :, 0], kh[0, :, 0], v[0, :, 0].astype(np.float64), g[0, :, 0],
            beta[0, :, 0], S0[0, 0])
    for C in (1, 2, 4, 8, 16, 32, 64, T):
        o4, S4 = oracle.chunked_ut(*args, C)
        _close(o[0, :, 0], o4, 1e-11, f"o vs chunked C={C}")
        _close(S[0, 0], S4, 1e-11, f"S vs chunked C={C}")


def check_beta_one_retrieval(lib):
    """(iv) beta = 1 and q = k: the output reads back the value just written, v / sqrt(dk)."""
    rng = np.random.default_rng(14)
    dk, dv, T = 16, 8, 10
    q, k, v, a, b, A_log, dtb, S0 = _rand_raw(rng, T, 1, 1, dk, dv)
    b[:] = 40.0  # sigmoid(40) == 1 in double
    o, _ = oracle.forward(k, k, v, a, b, A_log, dtb, S0, lib=lib)
    _close(o[0, :, 0], v[0, :, 0] / math.sqrt(dk), 1e-6, "beta=1 retrieval")


def check_beta_zero_decay(lib):
    """(v) beta ~ 0 (b = -40): pure decay, S_t = exp(G_t) S0 and o_t = exp(G_t) q_t^T S0."""
    rng = np.random.default_rng(15)
    dk, dv, T = 8, 5, 12
    q, k, v, a, b, A_log, dtb, S0 = _rand_raw(rng, T, 1, 1, dk, dv, s0=1.0)
    b[:] = -40.0
    o, S = oracle.forward(q, k, v, a, b, A_log, dtb, S0, lib=lib)
    # gates and normalised q from the definition, independently of the oracle
    x = a[0, :, 0].astype(np.float64) + float(dtb[0])
    sp = np.maximum(x, 0) + np.log1p(np.exp(-np.abs(x)))
    G = np.cumsum(-np.exp(float(A_log[0])) * sp)
    qq = q[0, :, 0].astype(np.float64)
    qh = qq / np.sqrt((qq * qq).sum(-1, keepdims=True) + 1e-6) / math.sqrt(dk)
    _close(S[0, 0], math.exp(G[-1]) * S0[0, 0], 1e-12, "beta=0 final state")
    _close(o[0, :, 0], np.exp(G)[:, None] * (qh @ S0[0, 0]), 1e-12, "beta=0 outputs")


def check_full_decay_keeps_only_the_last_write(lib):
    """Saturated decay (a = +40, so each token's gamma is below e^-30): the state carries
    only the current token's write, S_t = beta_t k_t v_t^T, so o_t = beta_t (q_t . k_t) v_t
    and the final state is the last write, whatever S0 held."""
    rng = np.random.default_rng(16)
    dk, dv, T = 8, 6, 12
    q, k, v, a, b, A_log, dtb, S0 = _rand_raw(rng, T, 1, 1, dk, dv, s0=1.0)
    a[:] = 40.0
    o, S = oracle.forward(q, k, v, a, b, A_log, dtb, S0, lib=lib)
    qq, kk = q[0, :, 0].astype(np.float64), k[0, :, 0].astype(np.float64)
    qh = qq / np.sqrt((qq * qq).sum(-1, keepdims=True) + 1e-6) / math.sqrt(dk)
    kh = kk / np.sqrt((kk * kk).sum(-1, keepdims=True) + 1e-6)
    beta = 1.0 / (1.0 + np.exp(-b[0, :, 0].astype(np.float64)))
    vv = v[0, :, 0].astype(np.float64)
    _close(o[0, :, 0], (beta * (qh * kh).sum(-1))[:, None] * vv, 1e-12, "full-decay outputs")
    _close(S[0, 0], beta[-1] * np.outer(kh[-1], vv[-1]), 1e-12, "full-decay final state")


def check_first_step(lib):
    """(vi) T = 1 from zero state with beta = 1/2, gamma = 1/2: S = k v^T / 2, o = (q.k) v / 2."""
    dk, dv = 4, 3
    q = np.array([[[[2.0, 0.0, 0.0, 0.0]]]], dtype=np.float32)
    k = np.array([[[[1.0, 1.0, 1.0, 1.0]]]], dtype=np.float32)
    v = np.array([[[[2.0, -4.0, 6.0]]]], dtype=np.float32)
    a = np.array([[[-0.5]]], dtype=np.float32)
    b = np.zeros((1, 1, 1), dtype=np.float32)
    o, S = oracle.forward(q, k, v, a, b, np.zeros(1, np.float32), np.full(1, 0.5, np.float32),
                          lib=lib)
    kh = np.full(dk, 0.5)
    qh = np.array([0.5, 0, 0, 0])
    _close(S[0, 0], 0.5 * np.outer(kh, v[0, 0, 0]), 1e-6, "first-step state")
    _close(o[0, 0, 0], 0.5 * (qh @ kh) * v[0, 0, 0], 1e-6, "first-step output")


def check_orthogonal_keys(lib):
    """(vii) keys along distinct axes: each state row follows its own scalar recurrence."""
    rng = np.random.default_rng(17)
    dk, dv, T = 8, 4, 8
    q, k, v, a, b, A_log, dtb, S0 = _rand_raw(rng, T, 1, 1, dk, dv, s0=1.0)
    k[:] = 0
    for t in range(T):
        k[0, t, 0, (3 * t) % dk] = 1.5  # T <= dk distinct axes (3 is coprime to 8)
    qh, kh, g, beta = oracle.prepare(q, k, a, b, A_log, dtb, lib=lib)
    _, S = oracle.core(qh, kh, v, g, beta, S0, lib=lib)
    ref = S0[0, 0].copy()
    for t in range(T):
        gam, bt, i = math.exp(g[0, t, 0]), beta[0, t, 0], (3 * t) % dk
        nk = float(kh[0, t, 0, i])  # 1 up to the norm epsilon
        ref *= gam
        ref[i] = ref[i] + nk * bt * (v[0, t, 0] - nk * ref[i])
    _close(S[0, 0], ref, 1e-12, "orthogonal keys")


def check_contraction(lib):
    """(viii) ||S_t||_F <= exp(g_t) ||S_{t-1}||_F + beta_t ||v_t|| every step (normalised keys)."""
    rng = np.random.default_rng(18)
    dk, dv, T = 16, 16, 40
    q, k, v, a, b, A_log, dtb, S0 = _rand_raw(rng, T, 1, 1, dk, dv, s0=1.0)
    qh, kh, g, beta = oracle.prepare(q, k, a, b, A_log, dtb, lib=lib)
    S = S0
    for t in range(T):
        sl = slice(t, t + 1)
        _, S1 = oracle.core(qh[:, sl], kh[:, sl], v[:, sl], g[:, sl], beta[:, sl], S, lib=lib)
        bound = math.exp(g[0, t, 0]) * np.linalg.norm(S) + beta[0, t, 0] * np.linalg.norm(
            v[0, t, 0])
        assert np.linalg.norm(S1) <= bound * (1 + 1e-12), f"contraction broken at t={t}"
        S = S1


def check_streaming_equals_recompute(lib):
    """(ix) prefill T1 then continue T2 steps from its final state == one pass over T1+T2."""
    rng = np.random.default_rng(19)
    dk, dv, T1, T2 = 8, 8, 23, 9
    q, k, v, a, b, A_log, dtb, S0 = _rand_raw(rng, T1 + T2, 2, 4, dk, dv)
    S0 = np.concatenate([S0] * 4, axis=1)[:, :4]
    o, S = oracle.forward(q, k, v, a, b, A_log, dtb, S0, lib=lib)
    p = slice(0, T1)
    c = slice(T1, T1 + T2)
    o1, S1 = oracle.forward(q[:, p], k[:, p], v[:, p], a[:, p], b[:, p], A_log, dtb, S0, lib=lib)
    o2, S2 = oracle.forward(q[:, c], k[:, c], v[:, c], a[:, c], b[:, c], A_log, dtb, S1, lib=lib)
    assert np.array_equal(np.concatenate([o1, o2], axis=1), o) and np.array_equal(S2, S)


def check_gate_values(lib):
    """(x) gate formula at points with known values, and its ranges."""
    # softplus(0) = ln 2, sigmoid(0) = 1/2: A_log = 0 gives g = -ln 2
    g, beta = oracle.gating(np.array([-0.5]), np.array([0.0]), 0.0, 0.5, lib=lib)
    assert abs(g[0] + math.log(2)) < 1e-15 and abs(beta[0] - 0.5) < 1e-15
    # A_log = ln 4 scales the rate by 4; sigmoid(ln 3) = 3/4
    g, beta = oracle.gating(np.array([0.0]), np.array([math.log(3)]), math.log(4), 0.0, lib=lib)
    assert abs(g[0] + 4 * math.log(2)) < 1e-14 and abs(beta[0] - 0.75) < 1e-15
    # softplus(x) -> x for large x, -> exp(x) for very negative x
    g, _ = oracle.gating(np.array([30.0, -30.0]), np.zeros(2), 0.0, 0.0, lib=lib)
    assert abs(g[0] + 30.0) < 1e-12 and abs(g[1] + math.exp(-30.0)) < 1e-25
    # ranges: g < 0, beta in (0, 1), over wide inputs
    rng = np.random.default_rng(20)
    a = rng.standard_normal(4000) * 8
    b = rng.standard_normal(4000) * 8
    for A_log in (0.0, 1.3, math.log(16)):
        g, beta = oracle.gating(a, b, A_log, -3.0, lib=lib)
        assert np.all(g < 0) and np.all(beta > 0) and np.all(beta < 1)


def check_normalisation_invariance(lib):
    """q and k enter only through their directions: scaling them by 2^m changes nothing."""
    rng = np.random.default_rng(21)
    dk, dv, T = 8, 4, 15
    q, k, v, a, b, A_log, dtb, S0 = _rand_raw(rng, T, 1, 1, dk, dv)
    o, S = oracle.forward(q, k, v, a, b, A_log, dtb, S0, lib=lib)
    o2, S2 = oracle.forward(q * 4, k * 0.5, v, a, b, A_log, dtb, S0, lib=lib)
    _close(o2, o, 1e-6, "q/k scale invariance (o)")
    _close(S2, S, 1e-6, "q/k scale invariance (S)")


def check_golden_hand_example(lib):
    """The hand-worked rational example in tests/golden (every step derived there)."""
    vals = {}
    with open(os.path.join(GOLDEN, "hand_example_dk4_dv2.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                key, *nums = line.split()
                vals[key] = np.array([float(x) for x in nums])
    dk, dv = int(vals["dk"][0]), int(vals["dv"][0])
    T = len(vals["a"])
    q = vals["q"].reshape(1, T, 1, dk).astype(np.float32)
    k = vals["k"].reshape(1, T, 1, dk).astype(np.float32)
    v = vals["v"].reshape(1, T, 1, dv).astype(np.float32)
    a = vals["a"].reshape(1, T, 1).astype(np.float32)
    b = vals["b"].reshape(1, T, 1).astype(np.float32)
    o, S = oracle.forward(q, k, v, a, b, vals["A_log"].astype(np.float32),
                          vals["dt_bias"].astype(np.float32), lib=lib)
    _close(o[0, :, 0], vals["o"].reshape(T, dv), 1e-6, "golden o")
    _close(S[0, 0], vals["S"].reshape(dk, dv), 1e-6, "golden S")


def check_grouped_heads_and_varlen(lib):
    """Value head h reads key head h // (Hv/Hk); packed sequences restart from their own state."""
    rng = np.random.default_rng(22)
    dk, dv, Hk, Hv = 4, 3, 2, 6
    lens = [5, 1, 9]
    T = sum(lens)
    q, k, v, a, b, A_log, dtb, S0 = _rand_raw(rng, T, Hk, Hv, dk, dv, nseq=3)
    cu = np.concatenate([[0], np.cumsum(lens)])
    o, S = oracle.forward(q, k, v, a, b, A_log, dtb, S0, cu_seqlens=cu, lib=lib)
    for s in range(3):
        sl = slice(cu[s], cu[s + 1])
        for h in range(Hv):
            kh = h // (Hv // Hk)
            o1, S1 = oracle.forward(q[:, sl, kh:kh + 1], k[:, sl, kh:kh + 1], v[:, sl, h:h + 1],
                                    a[:, sl, h:h + 1], b[:, sl, h:h + 1], A_log[h:h + 1],
                                    dtb[h:h + 1], S0[s:s + 1, h:h + 1], lib=lib)
            assert np.array_equal(o1[0, :, 0], o[0, sl, h]) and np.array_equal(S1[0, 0], S[s, h])


PINS = [check_bruteforce, check_gla, check_chunk_invariance, check_beta_one_retrieval,
        check_beta_zero_decay, check_full_decay_keeps_only_the_last_write, check_first_step,
        check_orthogonal_keys, check_contraction,
        check_streaming_equals_recompute, check_gate_values, check_normalisation_invariance,
        check_golden_hand_example, check_grouped_heads_and_varlen]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin, oracle_lib):
    pin(oracle_lib)


@pytest.mark.parametrize("mutation", oracle.MUTATIONS)
def test_planted_mistakes_are_caught(mutation):
    lib = oracle.load(oracle.build(defines=(mutation,)))
    failed = []
    for pin in PINS:
        try:
            pin(lib)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {mutation}"


def test_erase_matrix_is_a_contraction_only_with_normalised_keys():
    """Numeric policy (tessera PR #77, "Numerics finding"): with unit keys and beta in (0,1)
    the erase map I - beta k k^T has spectral norm <= 1; with raw N(0,1) keys it expands."""
    rng = np.random.default_rng(23)
    dk = 64
    grew = 0
    for _ in range(50):
        k = rng.standard_normal(dk)
        beta = rng.uniform(0.05, 0.95)
        khat = k / np.linalg.norm(k)
        assert np.linalg.norm(np.eye(dk) - beta * np.outer(khat, khat), 2) <= 1 + 1e-12
        grew += np.linalg.norm(np.eye(dk) - beta * np.outer(k, k), 2) > 1
    assert grew == 50


def test_bf16_rounding_is_round_to_nearest_even():
    from gated_delta_rule_145_b200 import synth

    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5], dtype=np.float32)
    r = synth.round_to_bf16(x)
    # 1 + 2^-8 is a tie -> even (1.0); 1 + 3*2^-8 is a tie -> even (1 + 2^-6)
    assert list(r) == [1.0, 1.0, 1.0 + 2 ** -6, 1.0, -2.5]
