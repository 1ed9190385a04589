"""fp64 CPU oracle for the gated delta rule forward pass.

TEST INFRASTRUCTURE ONLY: the test-suite, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / ``--impl reference`` legs are the only callers.  The
CUDA library and its Python binding never import this module, and this module never
imports them; the two share only the seeded input generator, which holds none of
the method's arithmetic.

Contents
  O1  ``forward`` / ``core`` / ``prepare`` -- the plain sequential recurrence in double
      precision, implemented in C (``gdr_oracle.c``) and reached through ctypes.
  O2  ``bruteforce_states`` -- every S_t as an explicit sum of products of dk x dk
      erase matrices exp(g_i)(I - beta_i k_i k_i^T); tiny sizes only.
  O3  ``gla_closed_form`` -- gated linear attention (no erase term) as a decay-masked
      causal attention sum.
  O4  ``chunked_ut`` -- the chunk-parallel UT-transform regrouping in fp64, for any
      chunk size; it exists to pin the chunk algebra, not as the GPU's reference.

Sources (page title and section):
  * Mila "GatedDeltaRule.ixx File Reference", Detailed Description -- the step
    S <- S exp(g); delta <- (v - k^T S) beta; S <- S + k (x) delta; o <- q^T S,
    q/k L2 normalisation, q scaled by 1/sqrt(dk), beta = sigmoid(b),
    g = -exp(A_log) softplus(a + dt_bias); the same section states that the chunked
    form is the same arithmetic regrouped, with one triangular solve per 32 tokens.
  * tessera PR #77 "Track L -- genuine gated delta rule + Mamba2 SSM", summary
    ("The core finding (L0)", "What landed"): the (I - beta k k^T) erase term, the
    independent brute-force check, erase=False being gated linear attention, and
    the chunked UT form, in which everything except the forward substitution for
    (I + A)^-1 is a matrix product.

Every function here is pinned by ``tests/test_oracle.py``; no function is
"parity unpinned".
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")

MUTATIONS = (
    "ORACLE_MUTATE_ERASE_SIGN",
    "ORACLE_MUTATE_DROP_QSCALE",
    "ORACLE_MUTATE_OUTPUT_BEFORE_UPDATE",
    "ORACLE_MUTATE_GATE_SIGN",
)


def build(defines=(), out_path=None) -> str:
    """Compile the C oracle (gcc -O2, no fast-math) and return the .so path.

    ``defines`` plants one of the ``MUTATIONS`` for the tests that check that the
    pins catch a wrong oracle; the default build has none.
    """
    if out_path is None:
        if defines:
            out_path = os.path.join(tempfile.mkdtemp(prefix="oracle_mut_"), "liboracle.so")
        else:
            out_path = _LIB_PATH
    os.makedirs(os.path.dirname(out_path), exist_ok=True)
    cmd = ["gcc", "-O2", "-std=c99", "-shared", "-fPIC", "-pthread", _SRC, "-o", out_path, "-lm"]
    cmd[1:1] = [f"-D{d}" for d in defines]
    subprocess.run(cmd, check=True)
    return out_path


_LIBS: dict = {}


def load(path=None):
    """Load (building if needed) the C oracle; returns a ctypes library."""
    if path is None:
        path = _LIB_PATH
        if not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(_SRC):
            build()
    if path in _LIBS:
        return _LIBS[path]
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I = ctypes.c_int
    lib.oracle_gdr_forward.argtypes = [P] * 11 + [I] * 7
    lib.oracle_gdr_forward.restype = I
    lib.oracle_gdr_core.argtypes = [P] * 9 + [I] * 7
    lib.oracle_gdr_core.restype = I
    lib.oracle_prepare.argtypes = [P] * 10 + [ctypes.c_int64, I, I, I]
    lib.oracle_prepare.restype = None
    lib.oracle_gating_array.argtypes = [I, P, P, ctypes.c_double, ctypes.c_double, P, P]
    lib.oracle_gating_array.restype = None
    _LIBS[path] = lib
    return lib


def _ptr(x):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p)


def _f32(x):
    return None if x is None else np.ascontiguousarray(x, dtype=np.float32)


def _f64(x):
    return None if x is None else np.ascontiguousarray(x, dtype=np.float64)


def _seqlens(n_tokens, B, T, cu_seqlens):
    if cu_seqlens is None:
        return np.arange(B + 1, dtype=np.int64) * T
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    assert cu[0] == 0 and cu[-1] == n_tokens and np.all(np.diff(cu) >= 0)
    return cu


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def forward(q, k, v, a, b, A_log, dt_bias, init_state=None, cu_seqlens=None, erase=True,
            nthreads=None, lib=None):
    """O1: the sequential recurrence from raw inputs, in fp64.

    Shapes: q, k [B, T, Hk, dk]; v [B, T, Hv, dv]; a, b [B, T, Hv]; A_log, dt_bias [Hv];
    init_state [Nseq, Hv, dk, dv] or None.  With ``cu_seqlens`` (length Nseq + 1) the
    tokens are packed (B == 1) and each sequence restarts from its own state.
    Returns (o [B, T, Hv, dv], final_state [Nseq, Hv, dk, dv]) as float64.
    """
    lib = lib or load()
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    N = B * T
    cu = _seqlens(N, B, T, cu_seqlens)
    nseq = len(cu) - 1
    qf, kf, vf, af, bf = (_f32(x) for x in (q, k, v, a, b))
    Al, dtb = _f32(A_log), _f32(dt_bias)
    S0 = _f64(init_state)
    if S0 is not None:
        assert S0.shape == (nseq, Hv, dk, dv)
    out = np.zeros((B, T, Hv, dv), dtype=np.float64)
    fin = np.zeros((nseq, Hv, dk, dv), dtype=np.float64)
    rc = lib.oracle_gdr_forward(_ptr(qf), _ptr(kf), _ptr(vf), _ptr(af), _ptr(bf), _ptr(Al),
                                _ptr(dtb), _ptr(S0), _ptr(out), _ptr(fin), _ptr(cu), nseq, Hk,
                                Hv, dk, dv, int(bool(erase)), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_gdr_forward: inconsistent sizes")
    return out, fin


def prepare(q, k, a, b, A_log, dt_bias, lib=None):
    """The preparation step of O1: (q_hat, k_hat, g, beta) in fp64, same shapes as inputs."""
    lib = lib or load()
    B, T, Hk, dk = q.shape
    Hv = a.shape[2]
    qf, kf, af, bf = (_f32(x) for x in (q, k, a, b))
    qh = np.zeros(q.shape, dtype=np.float64)
    kh = np.zeros(k.shape, dtype=np.float64)
    g = np.zeros(a.shape, dtype=np.float64)
    beta = np.zeros(a.shape, dtype=np.float64)
    lib.oracle_prepare(_ptr(qf), _ptr(kf), _ptr(af), _ptr(bf), _ptr(_f32(A_log)),
                       _ptr(_f32(dt_bias)), _ptr(qh), _ptr(kh), _ptr(g), _ptr(beta),
                       B * T, Hk, Hv, dk)
    return qh, kh, g, beta


def gating(a, b, A_log, dt_bias, lib=None):
    """O1's gate formula on 1-D arrays a, b of one head: returns (g, beta) in fp64."""
    lib = lib or load()
    a = _f64(a).ravel()
    b = _f64(b).ravel()
    g = np.zeros_like(a)
    beta = np.zeros_like(a)
    lib.oracle_gating_array(a.size, _ptr(a), _ptr(b), float(A_log), float(dt_bias), _ptr(g),
                            _ptr(beta))
    return g, beta


def core(qh, kh, v, g, beta, init_state=None, cu_seqlens=None, erase=True, nthreads=None,
         lib=None):
    """O1's recurrence from prepared inputs (q_hat, k_hat, g, beta), in fp64."""
    lib = lib or load()
    B, T, Hk, dk = qh.shape
    Hv, dv = v.shape[2], v.shape[3]
    N = B * T
    cu = _seqlens(N, B, T, cu_seqlens)
    nseq = len(cu) - 1
    S0 = _f64(init_state)
    out = np.zeros((B, T, Hv, dv), dtype=np.float64)
    fin = np.zeros((nseq, Hv, dk, dv), dtype=np.float64)
    rc = lib.oracle_gdr_core(_ptr(_f64(qh)), _ptr(_f64(kh)), _ptr(_f32(v)), _ptr(_f64(g)),
                             _ptr(_f64(beta)), _ptr(S0), _ptr(out), _ptr(fin), _ptr(cu), nseq,
                             Hk, Hv, dk, dv, int(bool(erase)), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_gdr_core: inconsistent sizes")
    return out, fin


# ----------------------------------------------------------------------------------------
# O2-O4: independent fp64 formulations on one (sequence, head): arrays are
# qh, kh [T, dk], v [T, dv], g, beta [T], S0 [dk, dv].
# ----------------------------------------------------------------------------------------


def bruteforce_states(qh, kh, v, g, beta, S0):
    """O2: S_t for every t from explicit products of erase matrices.

    With E_i = exp(g_i) (I - beta_i k_i k_i^T), the rule's step is S_i = E_i S_{i-1} +
    beta_i k_i v_i^T, so
        S_t = (E_t ... E_1) S0 + sum_{j<=t} (E_t ... E_{j+1}) beta_j k_j v_j^T .
    Each S_t is rebuilt from scratch by that sum (O(T^2) matrix products; tiny sizes).
    Returns (o [T, dv] with o_t = q_t^T S_t, states [T, dk, dv]).
    """
    T, dk = kh.shape
    E = [np.exp(g[i]) * (np.eye(dk) - beta[i] * np.outer(kh[i], kh[i])) for i in range(T)]
    states = np.zeros((T,) + S0.shape)
    for t in range(T):
        prod = np.eye(dk)
        for i in range(t, -1, -1):
            prod = prod @ E[i]
        acc = prod @ S0
        for j in range(t + 1):
            P = np.eye(dk)
            for i in range(t, j, -1):
                P = P @ E[i]
            acc = acc + P @ (beta[j] * np.outer(kh[j], v[j]))
        states[t] = acc
    o = np.einsum("tk,tkv->tv", qh, states)
    return o, states


def gla_closed_form(qh, kh, v, g, beta, S0):
    """O3: gated linear attention (no erase term) in closed form.

    With G_t = sum_{i<=t} g_i:
        o_t = exp(G_t) q_t^T S0 + sum_{j<=t} exp(G_t - G_j) beta_j (q_t . k_j) v_j
        S_T = exp(G_T) S0 + sum_j exp(G_T - G_j) beta_j k_j v_j^T
    Returns (o [T, dv], S_T [dk, dv]).
    """
    G = np.cumsum(g)
    T = len(G)
    o = np.zeros((T, v.shape[1]))
    for t in range(T):
        o[t] = np.exp(G[t]) * (qh[t] @ S0)
        for j in range(t + 1):
            o[t] += np.exp(G[t] - G[j]) * beta[j] * (qh[t] @ kh[j]) * v[j]
    S = np.exp(G[-1]) * S0
    for j in range(T):
        S = S + np.exp(G[-1] - G[j]) * beta[j] * np.outer(kh[j], v[j])
    return o, S


def chunked_ut(qh, kh, v, g, beta, S0, C):
    """O4: the chunk-parallel UT-transform form in fp64, any chunk size C >= 1.

    Inside one chunk with start state S0 and G_i = sum_{j<=i} g_j over the chunk,
    substituting the step into itself gives (I + A) Delta = diag(beta) V -
    diag(beta exp(G)) K S0 with A[i, j] = beta_i exp(G_i - G_j) (k_i . k_j) for j < i.
    With T = (I + A)^-1 (unit lower triangular; the forward substitution of the
    tessera page), U = T diag(beta) V and W = T diag(beta exp(G)) K:
        Delta = U - W S0
        O     = diag(exp(G)) Q S0 + (Q K^T * M) Delta,  M[i, j] = exp(G_i - G_j), j <= i
        S_C   = exp(G_C) S0 + (diag(exp(G_C - G)) K)^T Delta
    The last chunk may be shorter than C.  Returns (o [T, dv], S_T [dk, dv]).
    """
    T = kh.shape[0]
    S = S0.copy()
    o = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        c1 = min(T, c0 + C)
        Q, K, V = qh[c0:c1], kh[c0:c1], v[c0:c1]
        bt, G = beta[c0:c1], np.cumsum(g[c0:c1])
        n = c1 - c0
        causal = np.tril(np.ones((n, n), dtype=bool))  # j <= i
        strict = np.tril(causal, -1)  # j < i
        # exp(G_i - G_j) only where j <= i (there G_i - G_j <= 0); zero elsewhere
        decay = np.where(causal, np.exp(np.where(causal, G[:, None] - G[None, :], 0.0)), 0.0)
        A = np.where(strict, bt[:, None] * decay * (K @ K.T), 0.0)
        Tm = forward_substitution_inverse(A)
        U = Tm @ (bt[:, None] * V)
        W = Tm @ ((bt * np.exp(G))[:, None] * K)
        Delta = U - W @ S
        o[c0:c1] = np.exp(G)[:, None] * (Q @ S) + ((Q @ K.T) * decay) @ Delta
        S = np.exp(G[-1]) * S + (np.exp(G[-1] - G)[:, None] * K).T @ Delta
    return o, S


def forward_substitution_inverse(A):
    """(I + A)^-1 for strictly lower-triangular A, row by row (forward substitution)."""
    n = A.shape[0]
    Tm = np.eye(n)
    for i in range(1, n):
        # row i of (I + A) T = I:  T[i, :] = e_i - sum_{m < i} A[i, m] T[m, :]
        Tm[i, :i] = -(A[i, :i] @ Tm[:i, :i])
    return Tm
