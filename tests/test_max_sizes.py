"""GPU parity past 2^31 elements: every global offset the kernels form must be 64-bit.

Prefill: 4096 packed filler sequences of 1024 tokens (Hv = 4, dv = 128: exactly 2^31
output elements), then a 200-token sequence whose outputs all lie past element 2^31 of o.
The tail sequence, and the filler sequence that ends on the boundary, are compared with
the fp64 oracle run on each alone (packed sequences are independent: cu_seqlens
semantics, each with its own initial and final state).  Decode: B = 32769 sequences, so
the last one's state starts at element 2^31 of the state tensor.

About 27 GB on the device for the prefill (q, k 2.1 GB each, v 4.3 GB, o 8.6 GB, records
8.9 GB, states 2.1 GB) and 8.6 GB for decode.  Filler inputs are drawn on the device
(seeded torch generator, bf16); the compared sequences come from synth or are copied back.
"""

import numpy as np
import pytest

import gated_delta_rule_145_b200 as gdr
from gated_delta_rule_145_b200 import synth

from .helpers import TAU, assert_parity, oracle_forward

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

HK, HV, D = 2, 4, 128
NFILL, LFILL, LTAIL = 4096, 1024, 200


def _dev_normal(gen, shape):
    return torch.randn(shape, generator=gen, device="cuda", dtype=torch.bfloat16)


def _np(t):
    return t.detach().float().cpu().numpy()


@pytest.mark.parametrize("form", ["chunked", "recurrent"])
def test_prefill_outputs_past_2_31_elements(form):
    T_fill = NFILL * LFILL
    assert T_fill * HV * D == 2 ** 31
    T_all = T_fill + LTAIL
    tail = synth.make_inputs(1, LTAIL, HK, HV, D, D, "bf16", seed=91, s0_std=0.05)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(92)
    dev = {}
    for name, shape in (("q", (1, T_all, HK, D)), ("k", (1, T_all, HK, D)),
                        ("v", (1, T_all, HV, D)), ("a", (1, T_all, HV)), ("b", (1, T_all, HV))):
        x = _dev_normal(gen, shape)
        x[0, T_fill:] = torch.from_numpy(getattr(tail, name)[0]).to("cuda", torch.bfloat16)
        dev[name] = x
    A_log = torch.from_numpy(tail.A_log).cuda()
    dt_bias = torch.from_numpy(tail.dt_bias).cuda()
    cu = torch.arange(0, T_fill + 1, LFILL, dtype=torch.int32)
    cu = torch.cat([cu, torch.tensor([T_all], dtype=torch.int32)]).cuda()
    S0 = torch.zeros((NFILL + 1, HV, D, D), device="cuda")
    S0[NFILL] = torch.from_numpy(tail.init_state[0]).cuda()
    out, fin = gdr.prefill(dev["q"], dev["k"], dev["v"], dev["a"], dev["b"], A_log, dt_bias, S0,
                           cu, form=form)
    torch.cuda.synchronize()
    assert gdr.gdr_device_status() == gdr.GDR_OK
    # the tail: outputs at elements [2^31, 2^31 + 200 * 512)
    ro, rS = oracle_forward(tail)
    assert_parity(_np(out[0, T_fill:])[None], ro, TAU["bf16"], f"{form} tail o")
    assert_parity(_np(fin[NFILL])[None], rS, TAU["bf16"], f"{form} tail final state")
    # the last filler sequence, whose outputs end on the boundary
    sl = slice(T_fill - LFILL, T_fill)
    last = synth.Inputs(*(_np(dev[n][:, sl]) for n in ("q", "k", "v", "a", "b")),
                        tail.A_log, tail.dt_bias, None, None, "bf16")
    ro, rS = oracle_forward(last)
    assert_parity(_np(out[0, sl])[None], ro, TAU["bf16"], f"{form} boundary o")
    assert_parity(_np(fin[NFILL - 1])[None], rS, TAU["bf16"], f"{form} boundary final state")


def test_decode_state_past_2_31_elements():
    B = 32769
    assert (B - 1) * HV * D * D == 2 ** 31
    one = synth.make_inputs(1, 2, HK, HV, D, D, "bf16", seed=93, s0_std=0.05)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(94)
    state = torch.zeros((B, HV, D, D), device="cuda")
    state[-1] = torch.from_numpy(one.init_state[0]).cuda()
    A_log = torch.from_numpy(one.A_log).cuda()
    dt_bias = torch.from_numpy(one.dt_bias).cuda()
    outs = []
    for t in range(2):
        step = {}
        for name, shape in (("q", (B, HK, D)), ("k", (B, HK, D)), ("v", (B, HV, D)),
                            ("a", (B, HV)), ("b", (B, HV))):
            x = _dev_normal(gen, shape)
            x[-1] = torch.from_numpy(getattr(one, name)[0, t]).to("cuda", torch.bfloat16)
            step[name] = x
        outs.append(gdr.decode_step(step["q"], step["k"], step["v"], step["a"], step["b"],
                                    A_log, dt_bias, state)[-1].clone())
    torch.cuda.synchronize()
    ro, rS = oracle_forward(one)
    o = np.stack([_np(x) for x in outs])[None]
    assert_parity(o, ro, TAU["bf16"], "decode o of the last sequence")
    assert_parity(_np(state[-1])[None], rS, TAU["bf16"], "decode state of the last sequence")
