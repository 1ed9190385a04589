"""Context-parallel prefill: one sequence cut into segments whose state maps are composed.

The rule's update is affine in the state, so a segment maps its start state S to its end
state as Phi S + N, with Phi the run from S = I with v = 0 and N the run from S = 0.

CPU (no GPU):
* the decomposition itself, on the fp64 oracle: composing the segments' maps gives the
  whole sequence's final state, and each segment rerun from its composed start state
  gives the whole sequence's outputs for its tokens;
* two gloo ranks, one segment each: the all-gather of the maps (shard.exchange_segment_maps)
  delivers them in rank order, and the composition matches the single-process oracle;
* argument errors of the three calls, caught before any launch.

GPU (through the C ABI):
* gdr_prefill_segment_maps against the oracle's Phi and N;
* gdr_segment_combine against the composition written out in fp64;
* gdr_prefill_chunked_cp against the oracle's whole-sequence outputs and final state,
  with and without an initial state, for several segment counts and a ragged tail.
"""

import os
import socket

import numpy as np
import pytest

import gated_delta_rule_145_b200 as gdr
from gated_delta_rule_145_b200 import synth

from .helpers import TAU, assert_parity, to_device


def _oracle_maps(inp, cu):
    """(Phi, N) of every segment of cu by the fp64 oracle (dk == dv)."""
    from oracle import oracle

    nseg = len(cu) - 1
    Hv, dk = inp.v.shape[2], inp.q.shape[3]
    eye = np.broadcast_to(np.eye(dk), (nseg, Hv, dk, dk)).copy()
    _, phi = oracle.forward(inp.q, inp.k, np.zeros_like(inp.v), inp.a, inp.b, inp.A_log,
                            inp.dt_bias, eye, cu_seqlens=cu)
    _, nmap = oracle.forward(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias, None,
                             cu_seqlens=cu)
    return phi, nmap


def _compose(phi, nmap, S0):
    """seg_init[s] and the final state, in fp64 (the composition written out)."""
    G, Hv, dk, _ = phi.shape
    cur = np.zeros(nmap.shape[1:]) if S0 is None else np.asarray(S0, np.float64).reshape(
        nmap.shape[1:])
    seg = []
    for s in range(G):
        seg.append(cur)
        cur = np.einsum("hij,hjk->hik", phi[s], cur) + nmap[s]
    return np.stack(seg), cur


def _one_sequence(T, Hk, Hv, d, dtype, seed, s0_std):
    return synth.make_inputs(1, T, Hk, Hv, d, d, dtype, seed=seed, s0_std=s0_std)


@pytest.mark.parametrize("lens", [[13, 9, 18], [40], [1, 31, 8]])
def test_segment_maps_compose_to_the_whole_sequence(lens):
    from oracle import oracle

    inp = _one_sequence(sum(lens), 2, 4, 8, "f32", 5, 0.2)
    ro, rS = oracle.forward(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                            inp.init_state)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    phi, nmap = _oracle_maps(inp, cu)
    seg_init, final = _compose(phi, nmap, inp.init_state)
    np.testing.assert_allclose(final, rS[0], rtol=1e-10, atol=1e-12)
    o, _ = oracle.forward(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias, seg_init,
                          cu_seqlens=cu)
    np.testing.assert_allclose(o, ro, rtol=1e-10, atol=1e-12)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import torch
    import torch.distributed as dist

    from gated_delta_rule_145_b200.shard import exchange_segment_maps

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from oracle import oracle

        lens = [23, 17]  # rank r holds segment r
        inp = _one_sequence(sum(lens), 2, 4, 8, "f32", 9, 0.2)
        cu = np.array([0, lens[0], sum(lens)], dtype=np.int32)
        t0, t1 = int(cu[rank]), int(cu[rank + 1])
        seg = synth.Inputs(**{**inp.__dict__, "q": inp.q[:, t0:t1], "k": inp.k[:, t0:t1],
                              "v": inp.v[:, t0:t1], "a": inp.a[:, t0:t1], "b": inp.b[:, t0:t1],
                              "init_state": None, "cu_seqlens": None})
        phi, nmap = _oracle_maps(seg, np.array([0, t1 - t0], dtype=np.int32))
        pa, na = exchange_segment_maps(torch.from_numpy(phi), torch.from_numpy(nmap))
        seg_init, final = _compose(pa.numpy(), na.numpy(), inp.init_state)
        ro, rS = oracle.forward(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                                inp.init_state)
        o, _ = oracle.forward(seg.q, seg.k, seg.v, seg.a, seg.b, seg.A_log, seg.dt_bias,
                              seg_init[rank:rank + 1])
        ok = np.allclose(final, rS[0], rtol=1e-10, atol=1e-12)
        ok &= np.allclose(o, ro[:, t0:t1], rtol=1e-10, atol=1e-12)
        ok &= pa.shape[0] == world and np.array_equal(pa[rank].numpy(), phi[0])
        res = [None] * world
        dist.all_gather_object(res, bool(ok))
        if rank == 0:
            q.put(all(res))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_exchange_segment_maps_in_rank_order():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    assert q.get(timeout=10) is True


# fake, 256-byte aligned addresses for the host-side refusals (never dereferenced)
A = 1 << 20


def test_context_parallel_argument_errors():
    P = dict(q=A, k=A + 256, v=A + 512, a=A + 768, b=A + 1024, A_log=A + 1280, dt_bias=A + 1536)
    cp = dict(P, init_state=None, out=A + 2048, final_state=None, T=64, Hk=4, Hv=4, dk=128,
              dv=128, chunk=32, nseg=2)

    def call_cp(**kw):
        return gdr.gdr_prefill_chunked_cp(**{**cp, **kw}, stream=0, check=False)

    assert call_cp(nseg=0) == gdr.GDR_ERR_SHAPE
    assert call_cp(dk=64, dv=64) == gdr.GDR_ERR_UNSUPPORTED
    assert call_cp(chunk=64) == gdr.GDR_ERR_UNSUPPORTED
    assert call_cp(q=None) == gdr.GDR_ERR_NULL
    assert call_cp(out=A + 2056) == gdr.GDR_ERR_ALIGN
    maps = dict(P, phi=A + 4096, nmap=A + 8192, cu_seqlens=None, B=2, T=64, Hk=4, Hv=4, dk=128,
                dv=128, chunk=32)

    def call_maps(**kw):
        return gdr.gdr_prefill_segment_maps(**{**maps, **kw}, stream=0, check=False)

    assert call_maps(phi=None) == gdr.GDR_ERR_NULL
    assert call_maps(nmap=A + 8200) == gdr.GDR_ERR_ALIGN
    assert call_maps(T=0) == gdr.GDR_ERR_UNSUPPORTED
    assert call_maps(Hv=6) == gdr.GDR_ERR_SHAPE
    comb = dict(phi=A, nmap=A + 4096, init_state=None, seg_init=A + 8192, final_state=None, G=3,
                Hv=4, dk=128, dv=128)

    def call_comb(**kw):
        return gdr.gdr_segment_combine(**{**comb, **kw}, stream=0, check=False)

    assert call_comb(G=0) == gdr.GDR_ERR_SHAPE
    assert call_comb(phi=None) == gdr.GDR_ERR_NULL
    assert call_comb(dk=64, dv=64) == gdr.GDR_ERR_UNSUPPORTED
    assert call_comb(seg_init=A + 8196) == gdr.GDR_ERR_ALIGN


# ------------------------------------------------------------------------------ GPU


@pytest.mark.gpu
def test_segment_maps_match_oracle():
    torch = pytest.importorskip("torch")
    inp = synth.make_inputs(1, 700, 2, 4, 128, 128, "bf16", seed=41,
                            seqlens=[300, 37, 363])
    d = to_device(inp)
    G, Hv = 3, 4
    phi = torch.full((G, Hv, 128, 128), float("nan"), device="cuda")
    nmap = torch.full_like(phi, float("nan"))
    gdr.gdr_prefill_segment_maps(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"],
                                 d["dt_bias"], phi, nmap, d["cu_seqlens"], G, 700, 2, Hv, 128,
                                 128, 32)
    torch.cuda.synchronize()
    assert gdr.gdr_device_status() == gdr.GDR_OK
    rphi, rn = _oracle_maps(inp, inp.cu_seqlens)
    assert_parity(phi.cpu().numpy(), rphi, TAU["bf16"], "Phi")
    assert_parity(nmap.cpu().numpy(), rn, TAU["bf16"], "N")


@pytest.mark.gpu
@pytest.mark.parametrize("Hv", [3, 12, 30, 48])  # slices of 8, 16, 32, 64 columns on 148 SMs
def test_segment_combine_matches_composition(Hv):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(7 + Hv)
    G, d = 5, 128
    # contractive maps, as the rule's are (|Phi| <= 1): scaled random matrices
    phi = rng.standard_normal((G, Hv, d, d)) * (0.9 / np.sqrt(d))
    nmap = rng.standard_normal((G, Hv, d, d))
    S0 = rng.standard_normal((1, Hv, d, d))
    seg, fin = _compose(phi, nmap, S0)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()
    phi_d, n_d, s0_d = t(phi), t(nmap), t(S0)
    seg_d = torch.full((G, Hv, d, d), float("nan"), device="cuda")
    fin_d = torch.full((1, Hv, d, d), float("nan"), device="cuda")
    gdr.gdr_segment_combine(phi_d, n_d, s0_d, seg_d, fin_d, G, Hv, d, d)
    torch.cuda.synchronize()
    # fp32 products over 128 terms against fp64 on fp32-rounded inputs
    ref_seg, ref_fin = _compose(phi.astype(np.float32).astype(np.float64),
                                nmap.astype(np.float32).astype(np.float64),
                                S0.astype(np.float32).astype(np.float64))
    assert_parity(seg_d.cpu().numpy(), ref_seg, 1e-5, "seg_init")
    assert_parity(fin_d.cpu().numpy()[0], ref_fin, 1e-5, "final")
    # without an initial state the first segment starts from zero
    gdr.gdr_segment_combine(phi_d, n_d, None, seg_d, None, G, Hv, d, d)
    torch.cuda.synchronize()
    assert float(seg_d[0].abs().max()) == 0.0


@pytest.mark.gpu
@pytest.mark.parametrize("nseg,s0", [(1, 0.0), (3, 0.05), (7, 0.0), (40, 0.05)])
def test_prefill_chunked_cp_matches_oracle(nseg, s0):
    torch = pytest.importorskip("torch")
    T, Hk, Hv = 1000, 2, 6  # ragged: 1000 = 31 chunks + 8 tokens
    inp = _one_sequence(T, Hk, Hv, 128, "bf16", 50 + nseg, s0)
    d = to_device(inp)
    out = torch.full((1, T, Hv, 128), float("nan"), device="cuda")
    fin = torch.full((1, Hv, 128, 128), float("nan"), device="cuda")
    gdr.gdr_prefill_chunked_cp(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                               d["init_state"], out, fin, T, Hk, Hv, 128, 128, 32, nseg)
    torch.cuda.synchronize()
    assert gdr.gdr_device_status() == gdr.GDR_OK
    from .helpers import oracle_forward

    ro, rS = oracle_forward(inp)
    assert_parity(out.cpu().numpy(), ro, TAU["bf16"], f"cp nseg={nseg} o")
    assert_parity(fin.cpu().numpy(), rS, TAU["bf16"], f"cp nseg={nseg} final state")


def _cp_rank_worker(rank, world, port, lens, q):
    """One rank of shard.prefill_context_parallel on GPU 0 under a gloo group: segment
    `rank` of one sequence in, its outputs and the sequence's final state out (to rank 0)."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import torch
    import torch.distributed as dist

    from gated_delta_rule_145_b200.shard import prefill_context_parallel

    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        Hk, Hv = 2, 6
        inp = _one_sequence(sum(lens), Hk, Hv, 128, "bf16", 60, 0.05)
        d = to_device(inp)
        t0 = sum(lens[:rank])
        t1 = t0 + lens[rank]
        seg = {n: d[n][:, t0:t1].contiguous() for n in ("q", "k", "v", "a", "b")}
        out = torch.full((1, t1 - t0, Hv, 128), float("nan"), device="cuda")
        final = prefill_context_parallel(seg["q"], seg["k"], seg["v"], seg["a"], seg["b"],
                                         d["A_log"], d["dt_bias"], d["init_state"], out, Hk, Hv)
        torch.cuda.synchronize()
        status = gdr.gdr_device_status()
        parts = [None] * world
        dist.all_gather_object(parts, (out.cpu().numpy(), final.cpu().numpy(), status))
        if rank == 0:
            q.put(parts)
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_multirank_context_parallel_driver_matches_oracle():
    """shard.prefill_context_parallel run by two processes on one GPU (gloo exchanges the
    maps through host memory): the ranks' outputs, concatenated in rank order, and the
    final state each rank returns equal the oracle's over the whole sequence."""
    import torch.multiprocessing as mp

    lens = [517, 400]  # ragged segments: 16 chunks + 5 tokens, 12 chunks + 16 tokens
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_rank_worker, args=(r, 2, port, lens, q)) for r in range(2)]
    for p in procs:
        p.start()
    import queue
    import time

    parts, deadline = None, time.time() + 600
    while parts is None and time.time() < deadline:
        try:
            parts = q.get(timeout=5)
        except queue.Empty:
            if any(p.exitcode not in (None, 0) for p in procs):
                break  # a rank failed: stop waiting for the result
    for p in procs:
        p.join(timeout=120)
        if p.is_alive():
            p.kill()
        assert p.exitcode == 0
    assert parts is not None
    assert all(st == gdr.GDR_OK for _, _, st in parts)
    from .helpers import oracle_forward

    inp = _one_sequence(sum(lens), 2, 6, 128, "bf16", 60, 0.05)
    ro, rS = oracle_forward(inp)
    o = np.concatenate([p[0] for p in parts], axis=1)
    assert_parity(o, ro, TAU["bf16"], "multi-rank cp o")
    for r, (_, fin, _) in enumerate(parts):
        assert_parity(fin, rS, TAU["bf16"], f"multi-rank cp final state (rank {r})")
