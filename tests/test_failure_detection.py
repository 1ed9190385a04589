"""Failure detection on the GPU without a fault: the kernels' waits on shared-memory
barriers are bounded (2 s); a wait that runs out records a timeout, lets its kernel exit
and is reported by gdr_device_status.  The self-test kernel makes one such wait run out
(a barrier that nothing completes); the context must stay usable afterwards."""

import time

import pytest

import gated_delta_rule_145_b200 as gdr
from gated_delta_rule_145_b200 import synth

from .helpers import TAU, assert_parity, oracle_forward, to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_is_reported():
    assert gdr.gdr_device_status() == gdr.GDR_OK
    t0 = time.monotonic()
    assert gdr.gdr_selftest_bounded_wait() == gdr.GDR_OK
    assert gdr.gdr_device_status() == gdr.GDR_ERR_TIMEOUT
    waited = time.monotonic() - t0
    assert 1.5 < waited < 30.0, waited
    # reading the status clears it, and the same context still runs the prefill
    assert gdr.gdr_device_status() == gdr.GDR_OK
    inp = synth.make_inputs(1, 100, 2, 4, 128, 128, "bf16", seed=17, s0_std=0.05)
    d = to_device(inp)
    out, fin = gdr.prefill(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                           d["init_state"])
    torch.cuda.synchronize()
    assert gdr.gdr_device_status() == gdr.GDR_OK
    ro, rS = oracle_forward(inp)
    assert_parity(out.float().cpu().numpy(), ro, TAU["bf16"], "o after a timed-out wait")
    assert_parity(fin.float().cpu().numpy(), rS, TAU["bf16"], "S after a timed-out wait")
