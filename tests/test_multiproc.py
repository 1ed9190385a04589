"""The N > 1 path without GPUs: two gloo ranks on CPU.

* head sharding: each rank runs the fp64 oracle on its key-head block; the gathered
  blocks equal the single-process result exactly (no exchange is needed on the data path);
* the max-over-ranks timing reduction used by bench.py.
"""

import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

from gated_delta_rule_145_b200.shard import head_shard  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from gated_delta_rule_145_b200 import synth
        from oracle import oracle

        inp = synth.make_inputs(2, 40, 4, 8, 8, 8, "f32", seed=31, s0_std=0.1)
        (k0, k1), (v0, v1) = head_shard(4, 8, world, rank)
        o, S = oracle.forward(inp.q[:, :, k0:k1], inp.k[:, :, k0:k1], inp.v[:, :, v0:v1],
                              inp.a[:, :, v0:v1], inp.b[:, :, v0:v1], inp.A_log[v0:v1],
                              inp.dt_bias[v0:v1], inp.init_state[:, v0:v1], nthreads=1)
        parts = [None] * world
        dist.all_gather_object(parts, (v0, v1, o, S))
        # bench.py's reduction of the timed region: max over ranks
        import bench

        d = bench.Dist()
        d.pg = dist
        t = d.max(float(rank + 1))
        if rank == 0:
            ro, rS = oracle.forward(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                                    inp.init_state, nthreads=1)
            ok = t == float(world)
            for v0_, v1_, o_, S_ in parts:
                ok &= np.array_equal(o_, ro[:, :, v0_:v1_]) and np.array_equal(S_, rS[:, v0_:v1_])
            covered = sorted((p[0], p[1]) for p in parts)
            ok &= covered[0][0] == 0 and covered[-1][1] == 8 and all(
                covered[i][1] == covered[i + 1][0] for i in range(len(covered) - 1))
            q.put(bool(ok))
    finally:
        dist.destroy_process_group()


def test_head_shard_ranges():
    assert head_shard(48, 48, 8, 0) == ((0, 6), (0, 6))
    assert head_shard(16, 48, 3, 2) == ((11, 16), (33, 48))
    cover = [head_shard(5, 10, 3, r)[1] for r in range(3)]
    assert cover == [(0, 4), (4, 8), (8, 10)]
    assert head_shard(2, 4, 4, 3) == ((2, 2), (4, 4))
    with pytest.raises(ValueError):
        head_shard(3, 4, 2, 0)


def test_two_gloo_ranks_shard_heads_without_exchange():
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
