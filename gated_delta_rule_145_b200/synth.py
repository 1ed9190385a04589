"""Seeded synthetic inputs for the gated delta rule forward pass.

This module is the one piece shared by the CUDA path's harness and the fp64 oracle's
callers.  It draws random numbers and rounds them to the storage type; it holds none
of the method's arithmetic.

Workload shapes follow the pages: a 128 x 128 state per head (flashprove issue #32
"Qwen3.8-27B port", milestone M1: a single head with the full-size state), 48 value
heads (same issue, M2: the cost of all 48 heads is estimated from one) and 32-step
chunks (Mila "GatedDeltaRule.ixx File Reference": a triangular solve per 32 tokens).  No
dataset or trained weight is involved; every tensor is drawn here.

Recipe (numpy PCG64, ``default_rng(seed)``), drawn in this order:
  seqlens (varlen only, they fix the shapes), q, k, v, a, b, A_log, dt, S0
  q, k, v, a, b ~ N(0, 1) as float32, then rounded to bf16 (round to nearest even)
  when the workload is bf16; A_log ~ U(0, ln 16); dt ~ logU(1e-3, 1e-1);
  dt_bias = log(expm1(dt)) (the inverse softplus of dt); S0 ~ N(0, s0_std^2) fp32.
All arrays are returned as float32 holding the exact stored values (bf16 values
widen to float32 exactly); ``to_bf16_bits`` gives the raw bf16 encoding.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

LN16 = float(np.log(16.0))


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    return bf16_bits_to_f32(to_bf16_bits(x))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(
        np.float32)


@dataclass
class Inputs:
    """One workload's tensors (float32 arrays holding the stored values)."""

    q: np.ndarray  # [B, T, Hk, dk]
    k: np.ndarray  # [B, T, Hk, dk]
    v: np.ndarray  # [B, T, Hv, dv]
    a: np.ndarray  # [B, T, Hv]
    b: np.ndarray  # [B, T, Hv]
    A_log: np.ndarray  # [Hv] fp32
    dt_bias: np.ndarray  # [Hv] fp32
    init_state: np.ndarray | None  # [Nseq, Hv, dk, dv] fp32 or None (zeros)
    cu_seqlens: np.ndarray | None  # [Nseq + 1] int32 or None
    dtype: str  # "bf16" or "f32": storage type of q, k, v, a, b
    meta: dict = field(default_factory=dict)

    @property
    def shape(self):
        B, T, Hk, dk = self.q.shape
        return B, T, Hk, self.v.shape[2], dk, self.v.shape[3]

    @property
    def nseq(self):
        return self.q.shape[0] if self.cu_seqlens is None else len(self.cu_seqlens) - 1


def make_inputs(B, T, Hk, Hv, dk, dv, dtype="bf16", seed=0, s0_std=0.0, seqlens=None,
                seqlen_range=None, nseq=None) -> Inputs:
    """Draw one workload.

    Dense: B sequences of T tokens each.  Varlen: pass explicit ``seqlens`` or
    ``nseq`` with ``seqlen_range=(lo, hi)`` (lengths ~ U[lo, hi] integers); the tokens
    are then packed as B = 1, T = sum(lengths) with cu_seqlens.
    """
    rng = np.random.default_rng(seed)
    cu = None
    if seqlen_range is not None:
        lo, hi = seqlen_range
        seqlens = rng.integers(lo, hi + 1, nseq)
    if seqlens is not None:
        seqlens = np.asarray(seqlens, dtype=np.int64)
        cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
        B, T = 1, int(cu[-1])

    def normal(shape):
        x = rng.standard_normal(size=shape, dtype=np.float32)
        return round_to_bf16(x) if dtype == "bf16" else x

    q = normal((B, T, Hk, dk))
    k = normal((B, T, Hk, dk))
    v = normal((B, T, Hv, dv))
    a = normal((B, T, Hv))
    b = normal((B, T, Hv))
    A_log = rng.uniform(0.0, LN16, Hv).astype(np.float32)
    dt = np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), Hv))
    dt_bias = np.log(np.expm1(dt)).astype(np.float32)
    nseq_ = B if cu is None else len(cu) - 1
    S0 = None
    if s0_std > 0:
        S0 = (rng.standard_normal(size=(nseq_, Hv, dk, dv), dtype=np.float32) *
              np.float32(s0_std))
    return Inputs(q, k, v, a, b, A_log, dt_bias, S0, cu, dtype,
                  dict(seed=seed, B=B, T=T, Hk=Hk, Hv=Hv, dk=dk, dv=dv))


# The five workloads: the small fp32 reference case, the decode step, the prefill,
# the grouped-key varlen prefill and the long-context prefill + continuation.
WORKLOADS = {
    0: dict(name="fp32 reference case B=1 T=128 H=2 d=32", B=1, T=128, Hk=2, Hv=2, dk=32,
            dv=32, dtype="f32", chunk=32),
    1: dict(name="decode B=64 H=48 d=128 x256 steps", B=64, T=1, Hk=48, Hv=48, dk=128,
            dv=128, dtype="bf16", steps=256, s0_std=0.02),
    2: dict(name="chunked prefill B=1 T=8192 H=48 d=128 C=32", B=1, T=8192, Hk=48, Hv=48,
            dk=128, dv=128, dtype="bf16", chunk=32),
    3: dict(name="grouped-key varlen prefill 8 seqs U[256,4096] Hk=16 Hv=48 d=128 C=32",
            B=1, T=None, Hk=16, Hv=48, dk=128, dv=128, dtype="bf16", chunk=32, nseq=8,
            seqlen_range=(256, 4096)),
    4: dict(name="long context T=65536 + 512 decode steps H=48 d=128 C=32", B=1,
            T=65536 + 512, Hk=48, Hv=48, dk=128, dv=128, dtype="bf16", chunk=32,
            prefill_T=65536, decode_steps=512),
}


def workload(idx: int, seed=None, **overrides) -> Inputs:
    """Inputs of one of the five workloads (seed defaults to 1000 + idx).

    ``overrides`` change sizes (e.g. T, Hv) for reduced-size parity cases while
    keeping the recipe.  The decode workload returns per-step tensors stacked on the
    T axis: q [B, steps, Hk, dk] etc., with the fp32 initial state.
    """
    w = dict(WORKLOADS[idx])
    w.update(overrides)
    seed = 1000 + idx if seed is None else seed
    if idx == 1:
        return make_inputs(w["B"], w["steps"], w["Hk"], w["Hv"], w["dk"], w["dv"], w["dtype"],
                           seed, s0_std=w["s0_std"])
    if idx == 3:
        return make_inputs(1, 0, w["Hk"], w["Hv"], w["dk"], w["dv"], w["dtype"], seed,
                           seqlen_range=w["seqlen_range"], nseq=w["nseq"])
    return make_inputs(w["B"], w["T"], w["Hk"], w["Hv"], w["dk"], w["dv"], w["dtype"], seed,
                       s0_std=w.get("s0_std", 0.0))
