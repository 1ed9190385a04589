"""Shared test helpers: device copies of synthetic inputs, oracle calls, the parity check.

Parity bar (written here once, used by every GPU test): the maximum over all elements of
|gpu - oracle| must not exceed tau * RMS(oracle), with RMS taken over the whole compared
tensor (outputs and final states separately); tau = 2e-3 for bf16 inputs and 1e-4 for
fp32 inputs.
"""

from __future__ import annotations

import numpy as np

TAU = {"bf16": 2e-3, "f32": 1e-4}


def rel_max_err(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    err = float(np.max(np.abs(x - ref))) if ref.size else 0.0
    return err / rms if rms > 0 else err, err, rms


def assert_parity(x, ref, tau, what):
    assert np.all(np.isfinite(x)), f"{what}: non-finite values"
    r, err, rms = rel_max_err(x, ref)
    assert r <= tau, f"{what}: max|err| {err:.3e} = {r:.2e} x RMS {rms:.3e} > {tau:.1e}"
    return r


def to_device(inp, device="cuda"):
    """torch tensors of an Inputs bundle (q, k, v, a, b in the storage dtype)."""
    import torch

    dt = torch.bfloat16 if inp.dtype == "bf16" else torch.float32

    def t(x, dtype):
        return torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dtype)

    d = dict(q=t(inp.q, dt), k=t(inp.k, dt), v=t(inp.v, dt), a=t(inp.a, dt), b=t(inp.b, dt),
             A_log=t(inp.A_log, torch.float32), dt_bias=t(inp.dt_bias, torch.float32))
    d["init_state"] = None if inp.init_state is None else t(inp.init_state, torch.float32)
    d["cu_seqlens"] = None if inp.cu_seqlens is None else t(inp.cu_seqlens, torch.int32)
    return d


def oracle_forward(inp, heads=None, nthreads=None, erase=True):
    """fp64 oracle on an Inputs bundle; optionally on a subset of value heads; erase=False
    gives gated linear attention.

    Returns (o, S) restricted to ``heads`` (value-head axis) when given.
    """
    from oracle import oracle

    q, k, v, a, b = inp.q, inp.k, inp.v, inp.a, inp.b
    A_log, dt_bias, S0 = inp.A_log, inp.dt_bias, inp.init_state
    Hk, Hv = q.shape[2], v.shape[2]
    if heads is not None:
        heads = list(heads)
        grp = Hv // Hk
        kh = [h // grp for h in heads]
        # present each selected value head with its own key head (Hk' = Hv' = len(heads))
        q, k = q[:, :, kh], k[:, :, kh]
        v, a, b = v[:, :, heads], a[:, :, heads], b[:, :, heads]
        A_log, dt_bias = A_log[heads], dt_bias[heads]
        S0 = None if S0 is None else S0[:, heads]
    return oracle.forward(q, k, v, a, b, A_log, dt_bias, S0, cu_seqlens=inp.cu_seqlens,
                          nthreads=nthreads, erase=erase)


class ParityAccumulator:
    """max|gpu - oracle| and RMS(oracle) over a whole tensor compared piece by piece (the
    oracle run on groups of value heads, to bound host memory at the largest sizes); the
    bar is the same as assert_parity's: max error <= tau * RMS over the whole tensor."""

    def __init__(self, what):
        self.what, self.err, self.sumsq, self.n = what, 0.0, 0.0, 0

    def add(self, x, ref):
        x = np.asarray(x, dtype=np.float64)
        ref = np.asarray(ref, dtype=np.float64)
        assert np.all(np.isfinite(x)), f"{self.what}: non-finite values"
        if ref.size:
            self.err = max(self.err, float(np.max(np.abs(x - ref))))
            self.sumsq += float(np.sum(ref * ref))
            self.n += ref.size

    def check(self, tau):
        rms = (self.sumsq / self.n) ** 0.5 if self.n else 0.0
        r = self.err / rms if rms > 0 else self.err
        assert r <= tau, (f"{self.what}: max|err| {self.err:.3e} = {r:.2e} x RMS {rms:.3e} "
                          f"> {tau:.1e}")
        return r


def check_all_heads(inp, o, S, tau, what, group=12, erase=True):
    """Every value head of a prefill's outputs o [B,T,Hv,dv] and final states S
    [Nseq,Hv,dk,dv] (host arrays) against the fp64 oracle, `group` heads per oracle run."""
    Hv = inp.v.shape[2]
    acc_o, acc_s = ParityAccumulator(f"{what} o"), ParityAccumulator(f"{what} final state")
    for h0 in range(0, Hv, group):
        heads = list(range(h0, min(Hv, h0 + group)))
        ro, rS = oracle_forward(inp, heads, erase=erase)
        acc_o.add(o[:, :, heads], ro)
        acc_s.add(S[:, heads], rS)
    return acc_o.check(tau), acc_s.check(tau)
