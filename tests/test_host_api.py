"""gdr_prefill_chunked_host: the chunked prefill from and to host memory, the copies
overlapped with the kernels in chunk-aligned segments.

CPU: argument errors, caught before anything is enqueued.
GPU: the results in host memory against the fp64 oracle, for several sequences, an
initial state, a ragged last segment and a ragged last chunk, the default and a small
segment size; and against the device-resident call.
"""

import numpy as np
import pytest

import gated_delta_rule_145_b200 as gdr
from gated_delta_rule_145_b200 import synth

from .helpers import TAU, assert_parity, oracle_forward, to_device

A = 1 << 20  # fake addresses for the refusals (never dereferenced)


def _fake(**kw):
    args = dict(q=A, k=A + 256, v=A + 512, a=A + 768, b=A + 1024, A_log=A + 1280,
                dt_bias=A + 1536, init_state=None, out=A + 2048, final_state=None, B=1, T=64,
                Hk=4, Hv=4, dk=128, dv=128, chunk=32, seg_tokens=64)
    args.update(kw)
    return gdr.gdr_prefill_chunked_host(**args, stream=0, check=False)


def test_host_prefill_argument_errors():
    assert _fake(seg_tokens=40) == gdr.GDR_ERR_SHAPE   # not chunk-aligned
    assert _fake(seg_tokens=-32) == gdr.GDR_ERR_SHAPE
    assert _fake(Hv=6) == gdr.GDR_ERR_SHAPE            # Hv % Hk != 0
    assert _fake(B=0) == gdr.GDR_ERR_SHAPE
    assert _fake(chunk=64) == gdr.GDR_ERR_UNSUPPORTED
    assert _fake(dk=96, dv=96) == gdr.GDR_ERR_UNSUPPORTED
    assert _fake(q=None) == gdr.GDR_ERR_NULL
    assert _fake(A_log=None) == gdr.GDR_ERR_NULL


def _pinned(x, dtype):
    import torch

    return torch.from_numpy(np.ascontiguousarray(x)).to(dtype).pin_memory()


@pytest.mark.gpu
# 96: ten full segments and a ragged one; 0: the default (256 here); 512: the last segment
# cut in two, twice (512, 224, 128, 136 tokens)
@pytest.mark.parametrize("seg", [96, 0, 512])
def test_host_prefill_matches_oracle_and_device_call(seg):
    torch = pytest.importorskip("torch")
    B, T, Hk, Hv = 2, 1000, 2, 6  # 1000 = 10 segments of 96 + 40; ragged last chunk
    inp = synth.make_inputs(B, T, Hk, Hv, 128, 128, "bf16", seed=88, s0_std=0.05)
    h = {n: _pinned(getattr(inp, n), torch.bfloat16) for n in ("q", "k", "v", "a", "b")}
    Al, dtb = _pinned(inp.A_log, torch.float32), _pinned(inp.dt_bias, torch.float32)
    S0 = _pinned(inp.init_state, torch.float32)
    out = torch.full((B, T, Hv, 128), float("nan")).pin_memory()
    fin = torch.full((B, Hv, 128, 128), float("nan")).pin_memory()
    stream = torch.cuda.current_stream()
    gdr.gdr_prefill_chunked_host(h["q"], h["k"], h["v"], h["a"], h["b"], Al, dtb, S0, out, fin,
                                 B, T, Hk, Hv, 128, 128, 32, seg, stream=stream)
    stream.synchronize()
    assert gdr.gdr_device_status() == gdr.GDR_OK
    ro, rS = oracle_forward(inp)
    assert_parity(out.numpy(), ro, TAU["bf16"], f"host prefill seg={seg} o")
    assert_parity(fin.numpy(), rS, TAU["bf16"], f"host prefill seg={seg} final state")
    # the device-resident call on the same inputs
    d = to_device(inp)
    od = torch.empty((B, T, Hv, 128), device="cuda")
    fd = torch.empty((B, Hv, 128, 128), device="cuda")
    gdr.gdr_prefill_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                            d["init_state"], od, fd, None, B, T, Hk, Hv, 128, 128, 32)
    torch.cuda.synchronize()
    assert_parity(out.numpy(), od.cpu().numpy(), TAU["bf16"], "host vs device o")


@pytest.mark.gpu
def test_host_prefill_small_heads_and_no_state():
    torch = pytest.importorskip("torch")
    B, T, H = 1, 300, 3
    inp = synth.make_inputs(B, T, H, H, 64, 64, "bf16", seed=89)
    h = {n: _pinned(getattr(inp, n), torch.bfloat16) for n in ("q", "k", "v", "a", "b")}
    out = torch.full((B, T, H, 64), float("nan")).pin_memory()
    gdr.gdr_prefill_chunked_host(h["q"], h["k"], h["v"], h["a"], h["b"],
                                 _pinned(inp.A_log, torch.float32),
                                 _pinned(inp.dt_bias, torch.float32), None, out, None, B, T, H,
                                 H, 64, 64, 32, 64)
    torch.cuda.current_stream().synchronize()
    ro, _ = oracle_forward(inp)
    assert_parity(out.numpy(), ro, TAU["bf16"], "host prefill d=64 o")
