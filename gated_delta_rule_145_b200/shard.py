"""Splitting the gated delta rule across GPUs.

Heads (no exchange).  Every (sequence, value head) state evolves on its own, and value
heads that share a key head read the same q and k, so the natural unit is a (sequence,
key-head group) pair.  `head_shard` gives each rank a contiguous block of key-head
groups (and their value heads) for all sequences; the outputs of the ranks are disjoint
slices of o and of the final state, so no collective is needed on the data path.

Context (one exchange).  One long sequence cut into consecutive segments, one per rank
in rank order: each rank computes its segment's state map S_end = Phi S_start + N
(gdr_prefill_segment_maps), the maps are all-gathered (`exchange_segment_maps`), every
rank composes them (gdr_segment_combine) into its segment's start state, and runs the
prefill of its segment from there (`prefill_context_parallel`).
"""

from __future__ import annotations


def head_shard(Hk: int, Hv: int, world: int, rank: int):
    """Key heads [k0, k1) and value heads [v0, v1) owned by `rank` (contiguous, balanced).

    Value head h reads key head h // (Hv // Hk).  Ranks beyond the number of key heads
    get empty ranges.
    """
    if Hk < 1 or Hv % Hk != 0 or world < 1 or not 0 <= rank < world:
        raise ValueError("bad shard arguments")
    group = Hv // Hk
    base, extra = divmod(Hk, world)
    k0 = rank * base + min(rank, extra)
    k1 = k0 + base + (1 if rank < extra else 0)
    return (k0, k1), (k0 * group, k1 * group)


def exchange_segment_maps(phi, nmap, group=None):
    """All-gather of every rank's segment map, in rank order: (phi_all, nmap_all) with a
    leading dimension of world size, on the device phi and nmap ([1, Hv, dk, dk] and
    [1, Hv, dk, dv]) live on.  With NCCL the maps travel device to device; a gloo group
    cannot gather device tensors, so there they are staged through host memory."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    stage = phi.is_cuda and dist.get_backend(group) != "nccl"
    out = []
    for t in (phi, nmap):
        src = t.detach().cpu() if stage else t.contiguous()
        parts = [torch.empty_like(src) for _ in range(world)]
        dist.all_gather(parts, src.contiguous(), group=group)
        res = torch.cat(parts, 0)
        out.append(res.to(t.device) if stage else res)
    return out[0], out[1]


def prefill_context_parallel(q, k, v, a, b, A_log, dt_bias, init_state, out, Hk, Hv,
                             group=None):
    """Context-parallel prefill of ONE sequence whose tokens are split across the ranks of
    `group` in rank order.  This rank holds its segment's q, k ([1, T_r, Hk, 128]), v
    ([1, T_r, Hv, 128]), a, b ([1, T_r, Hv]) as bf16 CUDA tensors and writes that
    segment's outputs into out ([1, T_r, Hv, 128] fp32).  init_state ([1, Hv, 128, 128]
    fp32 or None) is the sequence's initial state, the same on every rank.  Returns the
    sequence's final state (computed on every rank).  Every rank needs T_r >= 1.

    The library calls run on the current stream, which the collective follows."""
    import gated_delta_rule_145_b200 as gdr
    import torch
    import torch.distributed as dist

    T_r, d = q.shape[1], 128
    phi = torch.empty((1, Hv, d, d), device=q.device, dtype=torch.float32)
    nmap = torch.empty_like(phi)
    gdr.gdr_prefill_segment_maps(q, k, v, a, b, A_log, dt_bias, phi, nmap, None, 1, T_r, Hk,
                                 Hv, d, d, 32)
    phi_all, nmap_all = exchange_segment_maps(phi, nmap, group)
    G = phi_all.shape[0]
    seg_init = torch.empty_like(phi_all)
    final = torch.empty((1, Hv, d, d), device=q.device, dtype=torch.float32)
    gdr.gdr_segment_combine(phi_all, nmap_all, init_state, seg_init, final, G, Hv, d, d)
    r = dist.get_rank(group)
    gdr.gdr_prefill_chunked(q, k, v, a, b, A_log, dt_bias, seg_init[r:r + 1], out, None, None,
                            1, T_r, Hk, Hv, d, d, 32)
    return final
