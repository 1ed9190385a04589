"""Splitting one batch of the gated delta rule across GPUs without any exchange.

Every (sequence, value head) state evolves on its own, and value heads that share a key
head read the same q and k, so the natural unit is a (sequence, key-head group) pair.
`head_shard` gives each rank a contiguous block of key-head groups (and their value
heads) for all sequences; the outputs of the ranks are disjoint slices of o and of the
final state, so no collective is needed on the data path.
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
