"""The chunked prefill entry point that allocates no memory (gdr_prefill_chunked_noalloc).

Some callers cannot allocate device memory during a call -- their framework's allocator
already owns the memory, or the call sits on a path where an allocation's possible
device synchronisation or failure is not acceptable.  For them the library offers a
variant of the chunked prefill that keeps its per-chunk records in a fixed 64 MiB scratch
array compiled into the library.  This file checks, through the C ABI, that the variant
returns what gdr_prefill_chunked returns on two calls in a row (the scratch is shared
between calls, so the second call must not see the first one's records), and that calls
needing more than the fixed scratch are refused before any work is enqueued.

The file is named so that pytest collects it last.
"""

import numpy as np
import pytest

import gated_delta_rule_145_b200 as gdr
from gated_delta_rule_145_b200 import synth

from .helpers import TAU, assert_parity, to_device

# fake, 256-byte aligned addresses for the host-side refusals (never dereferenced)
A = 1 << 20


def _fake(**kw):
    args = dict(q=A, k=A + 256, v=A + 512, a=A + 768, b=A + 1024, A_log=A + 1280,
                dt_bias=A + 1536, init_state=None, out=A + 2048, final_state=None,
                cu_seqlens=None, B=1, T=64, Hk=4, Hv=4, dk=128, dv=128, chunk=32)
    args.update(kw)
    return gdr.gdr_prefill_chunked_noalloc(**args, stream=0, check=False)


def test_noalloc_refuses_what_does_not_fit():
    # 64 blocks of 64 tokens x 48 heads = 3072 records of 33808 bytes > 64 MiB
    assert _fake(T=4096, Hk=48, Hv=48) == gdr.GDR_ERR_TOO_LARGE
    # just past the limit: 42 blocks x 48 heads = 2016 records > 1984 = 64 MiB / 33808
    assert _fake(T=2625, Hk=48, Hv=48) == gdr.GDR_ERR_TOO_LARGE
    # the tensor-core variant only: other head sizes, chunk sizes or empty inputs are
    # left to gdr_prefill_chunked
    assert _fake(dk=64, dv=64) == gdr.GDR_ERR_UNSUPPORTED
    assert _fake(chunk=64) == gdr.GDR_ERR_UNSUPPORTED
    assert _fake(T=0, q=None, k=None, v=None, a=None, b=None, out=None) == \
        gdr.GDR_ERR_UNSUPPORTED
    assert _fake(q=None) == gdr.GDR_ERR_NULL
    assert gdr.gdr_status_string(gdr.GDR_ERR_TOO_LARGE).startswith("GDR_ERR_TOO_LARGE")


def _pair(inp, init):
    """(noalloc, pooled) outputs and final states for the same inputs."""
    torch = pytest.importorskip("torch")
    d = to_device(inp)
    nseq = inp.nseq
    T = inp.q.shape[1]
    Bq = inp.q.shape[0]  # 1 in varlen mode
    Hk, Hv = inp.q.shape[2], inp.v.shape[2]
    res = []
    for name in ("gdr_prefill_chunked_noalloc", "gdr_prefill_chunked"):
        out = torch.full((Bq, T, Hv, 128), float("nan"), device="cuda")
        fin = torch.full((nseq, Hv, 128, 128), float("nan"), device="cuda")
        rc = getattr(gdr, name)(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"],
                                d["dt_bias"], d["init_state"] if init else None, out, fin,
                                d["cu_seqlens"], nseq, T, Hk, Hv, 128, 128, 32)
        assert rc == gdr.GDR_OK
        torch.cuda.synchronize()
        res.append((out.cpu().numpy(), fin.cpu().numpy()))
    assert gdr.gdr_device_status() == gdr.GDR_OK
    return res


def _same(x, ref, what):
    """Both calls run the same kernels on the same inputs, so they agree bit for bit; a
    record left over from an earlier call would show up as a difference.  The tolerance
    check is kept for its message."""
    assert_parity(x, ref, TAU["bf16"], what)
    assert np.array_equal(x, ref), f"{what}: not bitwise equal to gdr_prefill_chunked"


@pytest.mark.gpu
def test_noalloc_matches_pooled_on_two_calls_in_a_row():
    pytest.importorskip("torch")
    tau = TAU["bf16"]
    # first call: 2 sequences x 1000 tokens (ragged last chunk), 24 heads, initial state
    first = synth.make_inputs(2, 1000, 24, 24, 128, 128, "bf16", seed=71, s0_std=0.05)
    (o1, s1), (r1, rs1) = _pair(first, init=True)
    _same(o1, r1, "noalloc call 1 o")
    _same(s1, rs1, "noalloc call 1 final state")
    # second call, other shapes and no initial state: nothing of call 1 may leak in
    second = synth.make_inputs(1, 2500, 16, 48, 128, 128, "bf16", seed=72)
    (o2, s2), (r2, rs2) = _pair(second, init=False)
    _same(o2, r2, "noalloc call 2 o")
    _same(s2, rs2, "noalloc call 2 final state")
    assert np.isfinite(o2).all() and np.isfinite(s2).all()
    assert tau > 0


@pytest.mark.gpu
def test_noalloc_packed_sequences_after_a_larger_call():
    """Packed sequences (cu_seqlens) after a larger dense call: the varlen record count is
    only bounded from above, so a stale record of the bigger call would be read if the
    indexing were off."""
    pytest.importorskip("torch")
    big = synth.make_inputs(1, 2400, 16, 48, 128, 128, "bf16", seed=73, s0_std=0.05)
    (o1, s1), (r1, rs1) = _pair(big, init=True)
    _same(o1, r1, "noalloc dense 2400 o")
    _same(s1, rs1, "noalloc dense 2400 final state")
    packed = synth.make_inputs(1, 0, 8, 24, 128, 128, "bf16", seed=74, s0_std=0.05,
                               seqlens=[300, 1, 0, 64, 517, 33, 200])
    (o2, s2), (r2, rs2) = _pair(packed, init=True)
    _same(o2, r2, "noalloc packed o")
    _same(s2, rs2, "noalloc packed final states")
