"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle, element by
element on the same seeded inputs.  Bar: max|gpu - oracle| <= tau * RMS(oracle) with
tau = 2e-3 for bf16 inputs, 1e-4 for fp32 inputs (tests/helpers.py).

Reduced sizes span several chunks and dv slices and end on a ragged chunk; every workload
is also checked at its full size on every head and batch row, in both forms."""

import numpy as np
import pytest

import gated_delta_rule_145_b200 as gdr
from gated_delta_rule_145_b200 import synth

from .helpers import (TAU, ParityAccumulator, assert_parity, check_all_heads,
                      oracle_forward, to_device)

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


@pytest.mark.parametrize("erase", [True, False])
def test_prefill_varlen_around_64_token_blocks(erase):
    """The tensor-core prefill steps its state 64 tokens at a time over two 32-token
    solves: packed sequences one short of, at, and one past one and two blocks (and of
    a solve), with Hk=3 key heads shared by Hv=6, nonzero initial states."""
    inp = synth.make_inputs(1, 0, 3, 6, 128, 128, "bf16", seed=15, s0_std=0.05,
                            seqlens=[63, 64, 65, 127, 128, 129, 31, 33, 2])
    d = to_device(inp)
    out, fin = gdr.prefill(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                           d["init_state"], d["cu_seqlens"], erase=erase)
    torch.cuda.synchronize()
    assert gdr.gdr_device_status() == gdr.GDR_OK
    ro, rS = oracle_forward(inp, erase=erase)
    assert_parity(_np(out), ro, TAU["bf16"], f"varlen 64-token edges o (erase={erase})")
    assert_parity(_np(fin), rS, TAU["bf16"], f"varlen 64-token edges S (erase={erase})")


@pytest.mark.parametrize("T", [64, 65, 191, 256])
def test_prefill_dense_block_multiples(T):
    """Dense batches of two sequences at and just past 64-token block multiples."""
    inp = synth.make_inputs(2, T, 2, 4, 128, 128, "bf16", seed=16 + T, s0_std=0.05)
    _check_prefill(inp, "chunked")


@pytest.mark.parametrize("erase", [True, False])
def test_prefill_one_key_head_for_eight_value_heads(erase):
    """The intra-block kernel computes a key head's tiles, Gram and norms once and then
    each of its value heads in turn: Hk=1 shared by Hv=8, a ragged dense batch."""
    inp = synth.make_inputs(2, 150, 1, 8, 128, 128, "bf16", seed=17, s0_std=0.05)
    d = to_device(inp)
    out, fin = gdr.prefill(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                           d["init_state"], erase=erase)
    torch.cuda.synchronize()
    assert gdr.gdr_device_status() == gdr.GDR_OK
    ro, rS = oracle_forward(inp, erase=erase)
    assert_parity(_np(out), ro, TAU["bf16"], f"Hk=1 Hv=8 o (erase={erase})")
    assert_parity(_np(fin), rS, TAU["bf16"], f"Hk=1 Hv=8 S (erase={erase})")


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
# Every config at its full size, every value head and batch row, both forms, against the
# fp64 oracle (run on groups of heads; the RMS is still taken over the whole tensor).


@pytest.mark.slow
@pytest.mark.parametrize("form", ["chunked", "recurrent"])
def test_full_prefill_T8192_all_heads(form):
    """The prefill workload in full (B=1, T=8192, Hk=Hv=48, d=128): all 48 heads."""
    inp = synth.workload(2)
    o, S = _run_prefill(inp, form)
    check_all_heads(inp, o, S, TAU["bf16"], f"T=8192 {form}")


@pytest.mark.slow
@pytest.mark.parametrize("form", ["chunked", "recurrent"])
def test_full_varlen_grouped_all_heads(form):
    """8 packed sequences (lengths U[256, 4096]), Hk=16 shared by Hv=48: all heads of all
    sequences, outputs and per-sequence final states."""
    inp = synth.workload(3)
    o, S = _run_prefill(inp, form)
    check_all_heads(inp, o, S, TAU["bf16"], f"varlen {form}")


@pytest.mark.slow
def test_full_decode_256_steps_all_rows():
    """The decode workload in full: B=64, H=48, d=128, 256 steps in place; every batch row
    and head against the oracle run over the same 256 tokens."""
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
    check_all_heads(inp, _np(out.transpose(0, 1)), _np(state), TAU["bf16"], "decode x256")


@pytest.mark.slow
def test_full_long_context_continuation():
    """T=65536 chunked prefill, then 512 decode steps from its final state: equal to the
    chunked prefill over all 66048 tokens, and both equal to the oracle on all 48 heads."""
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
    del out_p, outs
    o_all, S_all = gdr.prefill(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"])
    torch.cuda.synchronize()
    o_cont, S, o_all, S_all = _np(o_cont), _np(S), _np(o_all), _np(S_all)
    assert_parity(o_cont, o_all, TAU["bf16"], "continuation vs recompute o")
    assert_parity(S, S_all, TAU["bf16"], "continuation vs recompute S")
    Hv = inp.v.shape[2]
    accs = {n: ParityAccumulator(n) for n in ("T=66048 o", "T=66048 S", "continued o",
                                              "continued S")}
    for h0 in range(0, Hv, 8):
        heads = list(range(h0, min(Hv, h0 + 8)))
        ro, rS = oracle_forward(inp, heads)
        accs["T=66048 o"].add(o_all[:, :, heads], ro)
        accs["continued o"].add(o_cont[:, :, heads], ro)
        accs["T=66048 S"].add(S_all[:, heads], rS)
        accs["continued S"].add(S[:, heads], rS)
        del ro, rS
    for a in accs.values():
        a.check(TAU["bf16"])
