"""GPU parity on the method's degenerate inputs, which the seeded N(0,1) workloads never
reach: writes of strength exactly 1 or nearly 0, no decay and a decay that underflows fp32
in one token, jumps of hundreds of nats in the cumulative gate inside one block, zero q,
k or v rows, one key repeated, and rows scaled by 2^{+-40}, which the L2 normalisation
removes.  The gates and the normalisation are those of the Mila "GatedDeltaRule.ixx File
Reference", Detailed Description; beta = 0 reduces the rule to pure decay and beta = 1
with a repeated key to an overwrite of one direction.

Every form is compared with the fp64 oracle at the usual bar (max|gpu - oracle| <=
tau * RMS(oracle), tau = 2e-3 for bf16 inputs, 1e-4 for fp32): the chunked and recurrent
prefill, erase=False (gated linear attention) and the decode step.  A nonzero initial
state keeps the outputs nonzero where the writes vanish."""

import numpy as np
import pytest

import gated_delta_rule_145_b200 as gdr
from gated_delta_rule_145_b200 import synth

from .helpers import TAU, assert_parity, oracle_forward, to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = ["beta_one", "beta_zero", "no_decay", "full_decay", "mixed_gates", "zero_rows",
         "repeated_key", "scaled_rows"]
BIG = 40.0  # a gate input of +-40: sigmoid is 1 in fp32 (4e-18 below it), softplus 0 or ~40


def degenerate_inputs(case, dtype="bf16", B=2, T=200, Hk=2, Hv=4, d=128, seed=31):
    """Seeded inputs of one degenerate case (T = 200: three 64-token blocks and a ragged
    one; every stored value exactly representable in bf16)."""
    inp = synth.make_inputs(B, T, Hk, Hv, d, d, dtype, seed=seed, s0_std=0.05)
    rng = np.random.default_rng(seed + 1)
    if case == "beta_one":
        inp.b[:] = BIG
    elif case == "beta_zero":
        inp.b[:] = -BIG
    elif case == "no_decay":
        inp.a[:] = -BIG
    elif case == "full_decay":
        inp.a[:] = BIG
    elif case == "mixed_gates":
        # per (token, head): -40, as drawn or +40 with probabilities 0.2, 0.6, 0.2
        for x in (inp.a, inp.b):
            pick = rng.choice(3, size=x.shape, p=[0.2, 0.6, 0.2])
            x[pick == 0] = -BIG
            x[pick == 2] = BIG
    elif case == "zero_rows":
        for x in (inp.q, inp.k, inp.v):
            x[rng.random(x.shape[:3]) < 0.15] = 0.0
    elif case == "repeated_key":
        inp.k[:] = inp.k[:, :1]
        inp.b[:] = BIG
    elif case == "scaled_rows":
        for x in (inp.q, inp.k):
            x *= np.exp2(rng.choice([-40.0, 0.0, 40.0], size=x.shape[:3]))[..., None].astype(
                np.float32)
    else:
        raise ValueError(case)
    return inp


def _np(t):
    return t.detach().float().cpu().numpy()


def _prefill(inp, form, erase=True):
    d = to_device(inp)
    out, fin = gdr.prefill(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                           d["init_state"], form=form, erase=erase)
    torch.cuda.synchronize()
    assert gdr.gdr_device_status() == gdr.GDR_OK
    return _np(out), _np(fin)


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("form", ["chunked", "recurrent"])
def test_prefill_degenerate(case, form):
    inp = degenerate_inputs(case)
    o, S = _prefill(inp, form)
    ro, rS = oracle_forward(inp)
    assert_parity(o, ro, TAU["bf16"], f"{case} {form} o")
    assert_parity(S, rS, TAU["bf16"], f"{case} {form} final state")


@pytest.mark.parametrize("case", CASES)
def test_gla_degenerate(case):
    inp = degenerate_inputs(case)
    o, S = _prefill(inp, "chunked", erase=False)
    ro, rS = oracle_forward(inp, erase=False)
    assert_parity(o, ro, TAU["bf16"], f"{case} erase=False o")
    assert_parity(S, rS, TAU["bf16"], f"{case} erase=False final state")


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("form", ["chunked", "recurrent"])
def test_prefill_degenerate_fp32(case, form):
    inp = degenerate_inputs(case, dtype="f32")
    o, S = _prefill(inp, form)
    ro, rS = oracle_forward(inp)
    assert_parity(o, ro, TAU["f32"], f"{case} {form} fp32 o")
    assert_parity(S, rS, TAU["f32"], f"{case} {form} fp32 final state")


@pytest.mark.parametrize("case", CASES)
def test_decode_degenerate(case):
    """eight decode steps of each case, from its initial state, step by step"""
    inp = degenerate_inputs(case, T=8)
    d = to_device(inp)
    state = d["init_state"].clone()
    outs = []
    for t in range(8):
        outs.append(gdr.decode_step(*(d[n][:, t].contiguous() for n in ("q", "k", "v", "a", "b")),
                                    d["A_log"], d["dt_bias"], state))
    torch.cuda.synchronize()
    o = np.stack([_np(x) for x in outs], axis=1)
    ro, rS = oracle_forward(inp)
    assert_parity(o, ro, TAU["bf16"], f"{case} decode o")
    assert_parity(_np(state), rS, TAU["bf16"], f"{case} decode state")


@pytest.mark.parametrize("case", ["full_decay", "mixed_gates", "beta_one"])
@pytest.mark.parametrize("d", [32, 64])
def test_prefill_degenerate_small_heads(case, d):
    """the CUDA-core chunked kernel with bf16 inputs (head sizes below 128)"""
    inp = degenerate_inputs(case, d=d)
    o, S = _prefill(inp, "chunked")
    ro, rS = oracle_forward(inp)
    assert_parity(o, ro, TAU["bf16"], f"{case} d={d} o")
    assert_parity(S, rS, TAU["bf16"], f"{case} d={d} final state")


@pytest.mark.parametrize("case", ["full_decay", "mixed_gates", "no_decay"])
def test_context_parallel_degenerate(case):
    """one sequence in three segments: segment maps, their composition, then the prefill
    from the composed start states"""
    inp = degenerate_inputs(case, B=1, T=333)
    d = to_device(inp)
    out = torch.empty((1, 333, 4, 128), device="cuda")
    fin = torch.empty((1, 4, 128, 128), device="cuda")
    gdr.gdr_prefill_chunked_cp(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"],
                               d["dt_bias"], d["init_state"], out, fin, 333, 2, 4, 128, 128,
                               32, 3)
    torch.cuda.synchronize()
    assert gdr.gdr_device_status() == gdr.GDR_OK
    ro, rS = oracle_forward(inp)
    assert_parity(_np(out), ro, TAU["bf16"], f"{case} context-parallel o")
    assert_parity(_np(fin), rS, TAU["bf16"], f"{case} context-parallel final state")
