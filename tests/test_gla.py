"""erase=False (gated linear attention) through the same kernels: GPU parity against the
fp64 oracle run with erase=False, which tests/test_oracle.py pins to the closed-form
decay-masked attention sum (tessera PR #77 summary, "What landed": erase=False is gated
linear attention).  Same tolerance as the rule itself (tests/helpers.py)."""

import numpy as np
import pytest

import gated_delta_rule_145_b200 as gdr
from gated_delta_rule_145_b200 import synth

from .helpers import TAU, assert_parity, check_all_heads, oracle_forward, rel_max_err, to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().float().cpu().numpy()


def _check(inp, form, heads=None):
    d = to_device(inp)
    out, fin = gdr.prefill(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                           d["init_state"], d["cu_seqlens"], form=form, erase=False)
    torch.cuda.synchronize()
    assert gdr.gdr_device_status() == gdr.GDR_OK
    o, S = _np(out), _np(fin)
    ro, rS = oracle_forward(inp, heads, erase=False)
    if heads is not None:
        o, S = o[:, :, heads], S[:, heads]
    tau = TAU[inp.dtype]
    assert_parity(o, ro, tau, f"gla {form} o")
    assert_parity(S, rS, tau, f"gla {form} final state")
    return o, S


@pytest.mark.parametrize("form", ["chunked", "recurrent"])
@pytest.mark.parametrize("d", [32, 128])
def test_gla_prefill_dense(form, d):
    """B=2, T=200 (ragged last chunk), grouped heads, nonzero initial state; d=128 bf16 is
    the tensor-core path, d=32 the CUDA-core chunked kernel."""
    inp = synth.make_inputs(2, 200, 3, 6, d, d, "bf16", seed=31, s0_std=0.05)
    _check(inp, form)


@pytest.mark.parametrize("form", ["chunked", "recurrent"])
def test_gla_prefill_fp32(form):
    inp = synth.make_inputs(1, 100, 2, 2, 128, 128, "f32", seed=32, s0_std=0.05)
    _check(inp, form)


def test_gla_prefill_varlen():
    inp = synth.make_inputs(1, 0, 2, 6, 128, 128, "bf16", seed=33, s0_std=0.05,
                            seqlens=[37, 1, 0, 64, 100, 32])
    _check(inp, "chunked")


def test_gla_differs_from_the_rule():
    """The flag reaches the kernels: without the erase term the result moves far outside
    the tolerance."""
    inp = synth.make_inputs(1, 256, 2, 2, 128, 128, "bf16", seed=34, s0_std=0.05)
    o_gla, _ = _check(inp, "chunked")
    d = to_device(inp)
    out, _ = gdr.prefill(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                         d["init_state"], None, form="chunked")
    torch.cuda.synchronize()
    r, _, _ = rel_max_err(_np(out), o_gla)
    assert r > 100 * TAU["bf16"]


def test_gla_decode_steps():
    """8 in-place decode steps (B=4, H=4, d=128, bf16) against the oracle over the same
    8 tokens."""
    inp = synth.make_inputs(4, 8, 4, 4, 128, 128, "bf16", seed=35, s0_std=0.05)
    ro, rS = oracle_forward(inp, erase=False)
    d = to_device(inp)
    state = d["init_state"].clone()
    outs = []
    for t in range(8):
        outs.append(_np(gdr.decode_step(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(),
                                        d["v"][:, t].contiguous(), d["a"][:, t].contiguous(),
                                        d["b"][:, t].contiguous(), d["A_log"], d["dt_bias"],
                                        state, erase=False)))
    torch.cuda.synchronize()
    tau = TAU["bf16"]
    assert_parity(np.stack(outs, axis=1), ro, tau, "gla decode o")
    assert_parity(_np(state), rS, tau, "gla decode state")


@pytest.mark.slow
def test_gla_full_prefill_T8192_all_heads():
    """the bench's GLA workload (B=1, T=8192, H=48, d=128): every head and the whole state
    against the oracle's erase=False, with the same bound as the rule"""
    inp = synth.workload(2)
    d = to_device(inp)
    out, fin = gdr.prefill(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                           d["init_state"], d["cu_seqlens"], form="chunked", erase=False)
    torch.cuda.synchronize()
    assert gdr.gdr_device_status() == gdr.GDR_OK
    check_all_heads(inp, _np(out), _np(fin), TAU[inp.dtype], "gla T=8192", erase=False)
