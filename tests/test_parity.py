"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle, element by
element on the same seeded inputs.  Bar: max|gpu - oracle| <= tau * RMS(oracle) with
tau = 2e-3 for bf16 inputs, 1e-4 for fp32 inputs (tests/helpers.py).

Reduced sizes span several chunks and dv slices and end on a ragged chunk; the full
workload sizes are checked on sampled heads (the oracle runs those heads in full)."""

import numpy as np
import pytest

import gated_delta_rule_145_b200 as gdr
from gated_delta_rule_145_b200 import synth

from .helpers import TAU, assert_parity, oracle_forward, to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().float().cpu().numpy()


def _run_prefill(inp, form="chunked", init=True):
    d = to_device(inp)
    out, fin = gdr.prefill(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                           d["init_state"] if init else None, d["cu_seqlens"], form=form)
    torch.cuda.synchronize()
    return _np(out), _np(fin)


def _check_prefill(inp, form="chunked", heads=None, tau=None):
    tau = tau or TAU[inp.dtype]
    o, S = _run_prefill(inp, form)
    ro, rS = oracle_forward(inp, heads)
    if heads is not None:
        o, S = o[:, :, heads], S[:, heads]
    e1 = assert_parity(o, ro, tau, f"{form} o")
    e2 = assert_parity(S, rS, tau, f"{form} final state")
    return e1, e2


# ------------------------------------------------------------------ reduced-size cases


@pytest.mark.parametrize("form", ["chunked", "recurrent"])
def test_fp32_reference_case(form):
    """The fp32 reference case in full: B=1, T=128, H=2, d=32, zero initial state."""
    _check_prefill(synth.workload(0), form)


@pytest.mark.parametrize("form", ["chunked", "recurrent"])
@pytest.mark.parametrize("d", [32, 64, 128])
def test_prefill_small_dense(form, d):
    """B=2 sequences, T=200 (6 full chunks + a ragged one), nonzero initial state."""
    inp = synth.make_inputs(2, 200, 3, 6, d, d, "bf16", seed=7, s0_std=0.05)
    _check_prefill(inp, form)


@pytest.mark.parametrize("form", ["chunked", "recurrent"])
def test_prefill_small_fp32_d128(form):
    inp = synth.make_inputs(1, 100, 2, 2, 128, 128, "f32", seed=8, s0_std=0.05)
    _check_prefill(inp, form)


@pytest.mark.parametrize("form", ["chunked", "recurrent"])
def test_prefill_varlen_grouped(form):
    """Packed sequences incl. length 0, 1 and exact chunk multiples; Hk=2 shared by Hv=6."""
    inp = synth.make_inputs(1, 0, 2, 6, 128, 128, "bf16", seed=9, s0_std=0.05,
                            seqlens=[37, 1, 0, 64, 100, 32])
    _check_prefill(inp, form)


def test_zero_length_returns_initial_state():
    inp = synth.make_inputs(3, 0, 2, 2, 128, 128, "bf16", seed=10, s0_std=0.1)
    for form in ("chunked", "recurrent"):
        _, S = _run_prefill(inp, form)
        assert np.array_equal(S, inp.init_state)


def test_init_state_may_alias_final_state():
    inp = synth.make_inputs(2, 70, 2, 4, 128, 128, "bf16", seed=11, s0_std=0.05)
    d = to_device(inp)
    out_ref, fin_ref = gdr.prefill(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"],
                                   d["dt_bias"], d["init_state"])
    st = d["init_state"].clone()
    out, fin = gdr.prefill(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                           st, final_state=st)
    torch.cuda.synchronize()
    assert torch.equal(out, out_ref) and torch.equal(st, fin_ref)


def test_decode_steps_small():
    """16 decode steps on B=3, Hk=2, Hv=4, d=128 against the oracle run over 16 tokens."""
    inp = synth.make_inputs(3, 16, 2, 4, 128, 128, "bf16", seed=12, s0_std=0.02)
    d = to_device(inp)
    state = d["init_state"].clone()
    outs = []
    for t in range(16):
        outs.append(gdr.decode_step(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(),
                                    d["v"][:, t].contiguous(), d["a"][:, t].contiguous(),
                                    d["b"][:, t].contiguous(), d["A_log"], d["dt_bias"], state))
    o = _np(torch.stack(outs, 1))
    ro, rS = oracle_forward(inp)
    assert_parity(o, ro, TAU["bf16"], "decode o")
    assert_parity(_np(state), rS, TAU["bf16"], "decode state")


def test_decode_fp32():
    inp = synth.make_inputs(2, 5, 2, 2, 32, 32, "f32", seed=13, s0_std=0.1)
    d = to_device(inp)
    state = d["init_state"].clone()
    outs = [gdr.decode_step(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(),
                            d["v"][:, t].contiguous(), d["a"][:, t].contiguous(),
                            d["b"][:, t].contiguous(), d["A_log"], d["dt_bias"], state)
            for t in range(5)]
    ro, rS = oracle_forward(inp)
    assert_parity(_np(torch.stack(outs, 1)), ro, TAU["f32"], "decode o (fp32)")
    assert_parity(_np(state), rS, TAU["f32"], "decode state (fp32)")


def test_chunked_equals_recurrent_small():
    inp = synth.make_inputs(1, 300, 2, 4, 128, 128, "bf16", seed=14, s0_std=0.05)
    o1, S1 = _run_prefill(inp, "chunked")
    o2, S2 = _run_prefill(inp, "recurrent")
    assert_parity(o1, o2, TAU["bf16"], "chunked vs recurrent o")
    assert_parity(S1, S2, TAU["bf16"], "chunked vs recurrent S")


# --------------------------------------------------------------- full workload sizes


@pytest.mark.slow
def test_full_prefill_T8192_sampled_heads():
    """The prefill workload in full (B=1, T=8192, H=48, d=128); the oracle checks 6 heads,
    and the GPU chunked form matches the GPU recurrent form on all 48."""
    inp = synth.workload(2)
    heads = [0, 9, 18, 27, 38, 47]
    o, S = _run_prefill(inp, "chunked")
    ro, rS = oracle_forward(inp, heads)
    assert_parity(o[:, :, heads], ro, TAU["bf16"], "T=8192 o")
    assert_parity(S[:, heads], rS, TAU["bf16"], "T=8192 S")
    o2, S2 = _run_prefill(inp, "recurrent")
    assert_parity(o, o2, TAU["bf16"], "T=8192 chunked vs recurrent o")
    assert_parity(S, S2, TAU["bf16"], "T=8192 chunked vs recurrent S")


@pytest.mark.slow
def test_full_varlen_grouped_sampled_heads():
    """8 packed sequences (lengths U[256, 4096]), Hk=16 shared by Hv=48."""
    inp = synth.workload(3)
    heads = [0, 1, 2, 25, 47]
    o, S = _run_prefill(inp, "chunked")
    ro, rS = oracle_forward(inp, heads)
    assert_parity(o[:, :, heads], ro, TAU["bf16"], "varlen o")
    assert_parity(S[:, heads], rS, TAU["bf16"], "varlen S")


@pytest.mark.slow
def test_full_decode_256_steps_sampled_batch():
    """The decode workload in full: B=64, H=48, d=128, 256 steps in place; the oracle runs
    every head of 3 batch rows over the 256 tokens."""
    inp = synth.workload(1)
    d = to_device(inp)
    steps = inp.q.shape[1]
    qs, ks, vs = (d[x].transpose(0, 1).contiguous() for x in ("q", "k", "v"))
    as_, bs = (d[x].transpose(0, 1).contiguous() for x in ("a", "b"))
    state = d["init_state"].clone()
    out = torch.empty((steps,) + tuple(vs.shape[1:]), device="cuda", dtype=torch.float32)
    for t in range(steps):
        gdr.decode_step(qs[t], ks[t], vs[t], as_[t], bs[t], d["A_log"], d["dt_bias"], state,
                        out=out[t])
    torch.cuda.synchronize()
    rows = [0, 31, 63]
    sub = synth.Inputs(inp.q[rows], inp.k[rows], inp.v[rows], inp.a[rows], inp.b[rows],
                       inp.A_log, inp.dt_bias, inp.init_state[rows], None, "bf16")
    ro, rS = oracle_forward(sub)
    o = _np(out.transpose(0, 1))[rows]
    assert_parity(o, ro, TAU["bf16"], "decode x256 o")
    assert_parity(_np(state)[rows], rS, TAU["bf16"], "decode x256 state")


@pytest.mark.slow
def test_full_long_context_continuation():
    """T=65536 chunked prefill, then 512 decode steps from its final state, equals the
    chunked prefill over all 66048 tokens; the oracle checks 2 heads over 66048 tokens."""
    inp = synth.workload(4)
    Tp = synth.WORKLOADS[4]["prefill_T"]
    d = to_device(inp)
    sl = slice(0, Tp)
    out_p, S = gdr.prefill(*(d[x][:, sl].contiguous() for x in ("q", "k", "v", "a", "b")),
                           d["A_log"], d["dt_bias"])
    outs = []
    for t in range(Tp, inp.q.shape[1]):
        outs.append(gdr.decode_step(*(d[x][:, t].contiguous() for x in ("q", "k", "v", "a", "b")),
                                    d["A_log"], d["dt_bias"], S))
    o_cont = torch.cat([out_p, torch.stack(outs, 1)], dim=1)
    o_all, S_all = gdr.prefill(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"])
    torch.cuda.synchronize()
    o_cont, S, o_all, S_all = _np(o_cont), _np(S), _np(o_all), _np(S_all)
    assert_parity(o_cont, o_all, TAU["bf16"], "continuation vs recompute o")
    assert_parity(S, S_all, TAU["bf16"], "continuation vs recompute S")
    heads = [5, 40]
    ro, rS = oracle_forward(inp, heads)
    assert_parity(o_all[:, :, heads], ro, TAU["bf16"], "T=66048 o")
    assert_parity(S_all[:, heads], rS, TAU["bf16"], "T=66048 S")
    assert_parity(o_cont[:, :, heads], ro, TAU["bf16"], "continued o")
