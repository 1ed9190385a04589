"""The steps around the rule on the GPU (gdr_short_conv_silu, gdr_gated_rmsnorm) against
the fp64 oracle of oracle/mixer_io.py, through the C ABI.

conv + SiLU writes bf16: each output must equal the oracle's value rounded to bf16, or
its bf16 neighbour (the kernel computes in fp32, so a value near a rounding boundary
may round the other way); the carried state is copies of inputs and must be exact.
gated RMSNorm is fp32 throughout: max |gpu - oracle| <= 1e-4 RMS(oracle)."""

import numpy as np
import pytest

import gated_delta_rule_145_b200 as gdr
from gated_delta_rule_145_b200 import synth

from .helpers import TAU, assert_parity

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
RNG = np.random.default_rng(4242)


def _bf16(x):
    return torch.from_numpy(synth.round_to_bf16(np.asarray(x, np.float32))).cuda().bfloat16()


def _f32(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def _ulp_close(got_bf16, ref64, mag=None):
    """every element equals the oracle rounded to bf16 or one bf16 step away; where the
    convolution's terms cancel, the kernel's fp32 sum carries an absolute error of a few fp32
    ulps of their magnitudes `mag` (|bias| + sum |w x|), which may exceed that step"""
    ref = synth.round_to_bf16(ref64.astype(np.float32))
    got = got_bf16.float().cpu().numpy()
    # one bf16 step at the reference's magnitude
    step = np.abs(ref) * 2.0 ** -7 + 1e-30
    if mag is not None:
        step = step + 2.0 ** -20 * mag
    bad = np.abs(got - ref) > step
    assert not bad.any(), f"{bad.sum()} outputs differ by more than one bf16 step"
    return float((got == ref).mean())


def _conv_case(B, T, C, with_state, with_bias):
    from oracle import mixer_io as mio
    x = synth.round_to_bf16(RNG.standard_normal((B, T, C)).astype(np.float32))
    w = RNG.standard_normal((C, 4)).astype(np.float32) * 0.5
    b = RNG.standard_normal(C).astype(np.float32) * 0.1 if with_bias else None
    st = RNG.standard_normal((B, C, 3)).astype(np.float32) if with_state else None
    ry, rs = mio.short_conv_silu(x, w, b, st)
    return x, w, b, st, ry, rs


def _conv_mag(x, w, b, st):
    """|bias| + sum_i |w_i x_{t-3+i}| per output, in fp64"""
    B, T, C = x.shape
    hist = np.concatenate([np.zeros((B, 3, C)) if st is None else np.swapaxes(st, 1, 2), x],
                          axis=1).astype(np.float64)
    mag = np.zeros((B, T, C)) + (0.0 if b is None else np.abs(b.astype(np.float64)))
    for i in range(4):
        mag += np.abs(w[:, i].astype(np.float64)) * np.abs(hist[:, i:i + T, :])
    return mag


# T >= 256 takes the TMA-fed kernel (tiles of 64 tokens x 128 channels, time segments per
# CTA), shorter inputs the per-thread one: both with ragged tails; C = 1160 leaves 8
# channels in the last 128-channel tile, C = 18432 is the q|k|v width of 48 heads
@pytest.mark.parametrize("B,T,C,with_state,with_bias", [
    (2, 300, 96, True, True), (2, 300, 96, False, False), (2, 300, 96, True, False),
    (2, 200, 96, True, True), (3, 777, 1160, True, True), (1, 512, 18432, True, False)])
def test_conv_silu_matches_oracle(B, T, C, with_state, with_bias):
    x, w, b, st, ry, rs = _conv_case(B, T, C, with_state, with_bias)
    y = torch.empty((B, T, C), device="cuda", dtype=torch.bfloat16)
    so = torch.full((B, C, 3), float("nan"), device="cuda")
    gdr.gdr_short_conv_silu(_bf16(x), _f32(w), None if b is None else _f32(b),
                            None if st is None else _f32(st), so, y, B, T, C)
    torch.cuda.synchronize()
    exact = _ulp_close(y, ry, _conv_mag(x, w, b, st))
    assert exact > 0.99
    assert np.array_equal(so.cpu().numpy(), rs.astype(np.float32))


@pytest.mark.parametrize("T0", [200, 600])
def test_conv_silu_streams_like_one_call_and_updates_in_place(T0):
    """prefill T0 tokens, then three 1-token decode calls on a state updated in place,
    equal one call over T0 + 3 tokens"""
    B, T, C = 3, T0 + 3, 64
    x, w, b, st, ry, rs = _conv_case(B, T, C, True, True)
    wt, bt = _f32(w), _f32(b)
    state = _f32(st).clone()
    outs = []
    y1 = torch.empty((B, T0, C), device="cuda", dtype=torch.bfloat16)
    gdr.gdr_short_conv_silu(_bf16(x[:, :T0]), wt, bt, state, state, y1, B, T0, C)
    outs.append(y1)
    for t in range(T0, T):
        yt = torch.empty((B, 1, C), device="cuda", dtype=torch.bfloat16)
        gdr.gdr_short_conv_silu(_bf16(x[:, t:t + 1]), wt, bt, state, state, yt, B, 1, C)
        outs.append(yt)
    torch.cuda.synchronize()
    _ulp_close(torch.cat(outs, dim=1), ry, _conv_mag(x, w, b, st))
    assert np.array_equal(state.cpu().numpy(), rs.astype(np.float32))


@pytest.mark.parametrize("d,zf32", [(128, False), (64, True), (32, False)])
def test_gated_rmsnorm_matches_oracle(d, zf32):
    from oracle import mixer_io as mio
    rows = 3000
    o = RNG.standard_normal((rows, d)).astype(np.float32) * 2.0
    z = RNG.standard_normal((rows, d)).astype(np.float32)
    if not zf32:
        z = synth.round_to_bf16(z)
    w = RNG.uniform(0.5, 1.5, d).astype(np.float32)
    ref = mio.gated_rmsnorm(o, z, w, 1e-6)
    y = torch.full((rows, d), float("nan"), device="cuda")
    fn = gdr.gdr_gated_rmsnorm_f32 if zf32 else gdr.gdr_gated_rmsnorm
    fn(_f32(o), _f32(z) if zf32 else _bf16(z), _f32(w), y, rows, d, 1e-6)
    torch.cuda.synchronize()
    assert_parity(y.cpu().numpy(), ref, TAU["f32"], f"gated rmsnorm d={d}")


def test_gated_rmsnorm_on_the_rule_output():
    """the step after the rule on a real prefill output (B=1, T=256, H=4, d=128)"""
    from oracle import mixer_io as mio
    from .helpers import oracle_forward, to_device
    inp = synth.make_inputs(1, 256, 4, 4, 128, 128, "bf16", seed=77)
    d = to_device(inp)
    out, _ = gdr.prefill(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"])
    z = synth.round_to_bf16(RNG.standard_normal((1, 256, 4, 128)).astype(np.float32))
    w = RNG.uniform(0.5, 1.5, 128).astype(np.float32)
    y = torch.empty_like(out)
    gdr.gdr_gated_rmsnorm(out, _bf16(z), _f32(w), y, 256 * 4, 128, 1e-6)
    torch.cuda.synchronize()
    ro, _ = oracle_forward(inp)
    assert_parity(y.cpu().numpy(), mio.gated_rmsnorm(ro, z, w, 1e-6), TAU["bf16"],
                  "rule + gated rmsnorm")
