"""Out-of-bounds writes and cross-CTA interference, checked without a sanitizer (none runs
on the GPUs these tests are for): every output of every call sits between two guard
ranges filled with a marker value, which must be untouched afterwards; the inputs must be
unchanged; and a sequence must give bit-identical results alone and inside a batch (the
kernels' CTAs own disjoint (sequence, head, column-slice) units, so a neighbour can change
nothing).  Shapes are small, with ragged tails and empty sequences."""

import numpy as np
import pytest

import gated_delta_rule_145_b200 as gdr
from gated_delta_rule_145_b200 import synth

from .helpers import to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GUARD = 4096          # elements on each side (16-byte aligned views for every dtype here)
MARK = -1234.5        # exactly representable in fp32 and bf16


class Guarded:
    """a tensor of `shape` in the middle of a buffer whose ends hold MARK"""

    def __init__(self, shape, dtype=None, fill=MARK):
        dtype = dtype or torch.float32
        self.n = int(np.prod(shape))
        self.buf = torch.full((self.n + 2 * GUARD,), MARK, dtype=dtype, device="cuda")
        self.t = self.buf[GUARD:GUARD + self.n].view(shape)
        if fill is not None:
            self.t.fill_(fill)

    def check(self, what):
        lo, hi = self.buf[:GUARD], self.buf[GUARD + self.n:]
        assert bool((lo == MARK).all()) and bool((hi == MARK).all()), f"{what}: guard written"


def _snapshot(d):
    return {k: (None if v is None else v.clone()) for k, v in d.items()}


def _unchanged(d, snap):
    for k, v in d.items():
        if v is not None:
            assert torch.equal(v, snap[k]), f"input {k} was modified"


@pytest.mark.parametrize("case", ["tc_dense", "tc_varlen", "gla", "recurrent_d64", "noalloc"])
def test_prefill_writes_only_its_outputs(case):
    if case == "tc_varlen":
        inp = synth.make_inputs(1, 0, 2, 4, 128, 128, "bf16", seed=81, s0_std=0.05,
                                seqlens=[70, 0, 129, 1])
    elif case == "recurrent_d64":
        inp = synth.make_inputs(2, 77, 2, 4, 64, 64, "bf16", seed=82, s0_std=0.05)
    else:
        inp = synth.make_inputs(2, 150, 2, 4, 128, 128, "bf16", seed=83, s0_std=0.05)
    d = to_device(inp)
    snap = _snapshot(d)
    nseq = inp.init_state.shape[0]
    tokens = inp.q.shape[0] * inp.q.shape[1]
    Hv, dk, dv = inp.v.shape[2], inp.q.shape[3], inp.v.shape[3]
    out = Guarded((tokens, Hv, dv))
    fin = Guarded((nseq, Hv, dk, dv))
    B = inp.q.shape[0] if inp.cu_seqlens is None else nseq
    T = inp.q.shape[1]
    Hk = inp.q.shape[2]
    args = (d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"], d["init_state"],
            out.t, fin.t, d["cu_seqlens"], B, T, Hk, Hv, dk, dv)
    if case == "gla":
        gdr.gdr_gla_prefill_chunked(*args, 32)
    elif case == "recurrent_d64":
        gdr.gdr_prefill_recurrent(*args)
    elif case == "noalloc":
        gdr.gdr_prefill_chunked_noalloc(*args, 32)
    else:
        gdr.gdr_prefill_chunked(*args, 32)
    torch.cuda.synchronize()
    assert gdr.gdr_device_status() == gdr.GDR_OK
    out.check("o")
    fin.check("final state")
    assert bool(torch.isfinite(out.t).all()) and bool(torch.isfinite(fin.t).all())
    _unchanged(d, snap)


def test_decode_writes_only_its_outputs():
    inp = synth.make_inputs(3, 1, 2, 4, 128, 128, "bf16", seed=84, s0_std=0.05)
    d = to_device(inp)
    state = Guarded(inp.init_state.shape, fill=None)
    state.t.copy_(d["init_state"])
    out = Guarded((3, 4, 128))
    snap = _snapshot({k: d[k] for k in ("q", "k", "v", "a", "b", "A_log", "dt_bias")})
    gdr.gdr_decode_step(d["q"][:, 0].contiguous(), d["k"][:, 0].contiguous(),
                        d["v"][:, 0].contiguous(), d["a"][:, 0].contiguous(),
                        d["b"][:, 0].contiguous(), d["A_log"], d["dt_bias"], state.t, out.t,
                        3, 2, 4, 128, 128)
    torch.cuda.synchronize()
    state.check("state")
    out.check("o")
    _unchanged({k: d[k] for k in snap}, snap)


def test_segment_calls_write_only_their_outputs():
    inp = synth.make_inputs(1, 0, 2, 4, 128, 128, "bf16", seed=85, s0_std=0.05,
                            seqlens=[100, 64, 37])
    d = to_device(inp)
    snap = _snapshot(d)
    phi, nmap = Guarded((3, 4, 128, 128)), Guarded((3, 4, 128, 128))
    gdr.gdr_prefill_segment_maps(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"],
                                 d["dt_bias"], phi.t, nmap.t, d["cu_seqlens"], 3, 201, 2, 4, 128,
                                 128, 32)
    seg, fin = Guarded((3, 4, 128, 128)), Guarded((1, 4, 128, 128))
    S0 = torch.randn((1, 4, 128, 128), device="cuda")
    gdr.gdr_segment_combine(phi.t, nmap.t, S0, seg.t, fin.t, 3, 4, 128, 128)
    torch.cuda.synchronize()
    assert gdr.gdr_device_status() == gdr.GDR_OK
    for g, what in ((phi, "phi"), (nmap, "nmap"), (seg, "seg_init"), (fin, "final")):
        g.check(what)
    _unchanged(d, snap)
    # the one-device context-parallel call on one sequence
    one = synth.make_inputs(1, 333, 2, 4, 128, 128, "bf16", seed=86, s0_std=0.05)
    e = to_device(one)
    snap = _snapshot(e)
    out, fin = Guarded((333, 4, 128)), Guarded((1, 4, 128, 128))
    gdr.gdr_prefill_chunked_cp(e["q"], e["k"], e["v"], e["a"], e["b"], e["A_log"],
                               e["dt_bias"], e["init_state"], out.t, fin.t, 333, 2, 4, 128, 128,
                               32, 3)
    torch.cuda.synchronize()
    assert gdr.gdr_device_status() == gdr.GDR_OK
    out.check("cp o")
    fin.check("cp final state")
    _unchanged(e, snap)


@pytest.mark.parametrize("T", [100, 300])  # the per-thread and the TMA-fed convolution
def test_mixer_io_writes_only_its_outputs(T):
    B, C = 2, 136  # 8 channels in the last 128-channel tile
    x = torch.randn((B, T, C), device="cuda").to(torch.bfloat16)
    w = torch.randn((C, 4), device="cuda")
    bias = torch.randn((C,), device="cuda")
    st_in = torch.randn((B, C, 3), device="cuda")
    snap = _snapshot(dict(x=x, w=w, bias=bias, st_in=st_in))
    y = Guarded((B, T, C), dtype=torch.bfloat16)
    st = Guarded((B, C, 3))
    gdr.gdr_short_conv_silu(x, w, bias, st_in, st.t, y.t, B, T, C)
    torch.cuda.synchronize()
    assert gdr.gdr_device_status() == gdr.GDR_OK
    y.check("y")
    st.check("conv state")
    _unchanged(dict(x=x, w=w, bias=bias, st_in=st_in), snap)
    rows = B * T
    o = torch.randn((rows, 128), device="cuda")
    z = torch.randn((rows, 128), device="cuda").to(torch.bfloat16)
    wt = torch.rand((128,), device="cuda")
    yn = Guarded((rows, 128))
    gdr.gdr_gated_rmsnorm(o, z, wt, yn.t, rows, 128)
    torch.cuda.synchronize()
    yn.check("norm y")


@pytest.mark.parametrize("form", ["chunked", "recurrent"])
@pytest.mark.parametrize("erase", [True, False])
def test_a_sequence_alone_equals_it_inside_a_batch(form, erase):
    """bit-identical outputs and final state for sequence 1 of a batch of three and for
    the same sequence run alone"""
    inp = synth.make_inputs(3, 130, 2, 4, 128, 128, "bf16", seed=87, s0_std=0.05)
    d = to_device(inp)
    out, fin = gdr.prefill(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                           d["init_state"], form=form, erase=erase)
    one = {k: (v[1:2].contiguous() if k in ("q", "k", "v", "a", "b", "init_state") else v)
           for k, v in d.items()}
    out1, fin1 = gdr.prefill(one["q"], one["k"], one["v"], one["a"], one["b"], one["A_log"],
                             one["dt_bias"], one["init_state"], form=form, erase=erase)
    torch.cuda.synchronize()
    assert torch.equal(out[1:2], out1)
    assert torch.equal(fin[1:2], fin1)
