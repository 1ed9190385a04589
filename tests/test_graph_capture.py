"""Decode steps and prefill calls captured in a CUDA graph: the C-ABI calls enqueue only
kernels on the caller's stream (host-side checks, no synchronisation, no allocation on the
decode path), so a serving loop can capture them; a replay must give the bit-identical
outputs and state of the same calls made directly."""

import numpy as np
import pytest

import gated_delta_rule_145_b200 as gdr
from gated_delta_rule_145_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


# B=64, H=48: a grid of several waves, launched with programmatic stream serialization
@pytest.mark.parametrize("B,H,n", [(2, 4, 8), (64, 48, 4)])
def test_decode_steps_replayed_from_a_graph_match_direct_calls(B, H, n):
    D = 128
    inp = synth.make_inputs(B, n, H, H, D, D, "bf16", seed=71, s0_std=0.05)
    dev = torch.device("cuda", 0)

    def steps_first(x):
        return torch.from_numpy(np.ascontiguousarray(np.swapaxes(x, 0, 1))).to(dev).to(
            torch.bfloat16)

    q, k, v, a, b = (steps_first(getattr(inp, m)) for m in ("q", "k", "v", "a", "b"))
    A_log = torch.from_numpy(inp.A_log).to(dev)
    dt_bias = torch.from_numpy(inp.dt_bias).to(dev)
    S0 = torch.from_numpy(inp.init_state).to(dev)

    def run(state, outs, stream):
        for t in range(n):
            gdr.gdr_decode_step(q[t], k[t], v[t], a[t], b[t], A_log, dt_bias, state, outs[t],
                                B, H, H, D, D, stream=stream)

    # direct calls
    S_direct = S0.clone()
    o_direct = torch.empty((n, B, H, D), device=dev)
    run(S_direct, o_direct, None)
    torch.cuda.synchronize()
    # the same calls captured once, then replayed from the initial state
    S_graph = S0.clone()
    o_graph = torch.full((n, B, H, D), float("nan"), device=dev)
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=cap):
        run(S_graph, o_graph, cap)
    S_graph.copy_(S0)  # capture does not execute: start the replay from S0
    torch.cuda.current_stream().wait_stream(cap)
    graph.replay()
    torch.cuda.synchronize()
    assert gdr.gdr_device_status() == gdr.GDR_OK
    assert torch.equal(o_graph, o_direct)
    assert torch.equal(S_graph, S_direct)


def test_prefill_replayed_from_a_graph_matches_a_direct_call():
    """the tensor-core prefill takes its workspace from a stream-ordered pool, which graph
    capture records as graph-owned allocations; the replay must match the direct call"""
    inp = synth.make_inputs(1, 300, 2, 4, 128, 128, "bf16", seed=72, s0_std=0.05)
    dev = torch.device("cuda", 0)
    t = lambda x: torch.from_numpy(x).to(dev).to(torch.bfloat16)
    q, k, v, a, b = (t(getattr(inp, m)) for m in ("q", "k", "v", "a", "b"))
    A_log = torch.from_numpy(inp.A_log).to(dev)
    dt_bias = torch.from_numpy(inp.dt_bias).to(dev)
    S0 = torch.from_numpy(inp.init_state).to(dev)
    out_d = torch.empty((1, 300, 4, 128), device=dev)
    fin_d = torch.empty((1, 4, 128, 128), device=dev)
    gdr.gdr_prefill_chunked(q, k, v, a, b, A_log, dt_bias, S0, out_d, fin_d, None, 1, 300, 2, 4,
                            128, 128, 32)
    torch.cuda.synchronize()
    out_g = torch.full_like(out_d, float("nan"))
    fin_g = torch.full_like(fin_d, float("nan"))
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=cap):
        gdr.gdr_prefill_chunked(q, k, v, a, b, A_log, dt_bias, S0, out_g, fin_g, None, 1, 300,
                                2, 4, 128, 128, 32, stream=cap)
    torch.cuda.current_stream().wait_stream(cap)
    graph.replay()
    torch.cuda.synchronize()
    assert gdr.gdr_device_status() == gdr.GDR_OK
    assert torch.equal(out_g, out_d)
    assert torch.equal(fin_g, fin_d)
    del graph
