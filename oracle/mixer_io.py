"""fp64 CPU oracle for the steps on either side of the gated delta rule in its mixer.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: the test-suite and the
benchmark's ``cpu_baseline`` leg are the only callers; the CUDA library never imports
this module and this module imports nothing from it.

  short_conv_silu   the step before the rule: a short causal depthwise convolution over
                    time, kept as a ring buffer of the last taps, then SiLU.
  gated_rmsnorm     the step after the rule: RMS normalisation of each head's output,
                    times a per-channel weight, gated by SiLU of a gate input.

Sources (page title and section):
  * flashprove issue #32 "Qwen3.8-27B port": the tracking list names a four-tap short
    convolution and sigmoid gates among the operators a port needs; the registered M2
    design decisions scope one head from the input projections to the normalised,
    gated output, with the short convolution and SiLU before the rule and a gated RMS
    normalisation of the rule's output after it.
  * PLENA_Simulator PR #113, "Mamba + KDA support: common state engine, hybrid DSE",
    commit notes: the short convolution is kept as a ring buffer (a shift, a per-channel
    weight stride, a bias), and a convolution whose only non-zero tap is the newest one
    passes its input through.

The pages give no formulas; the readings taken here:
  * conv: y_t[c] = bias[c] + sum_{i=0}^{W-1} w[c, i] x_{t-W+1+i}[c], so w[c, W-1] is the
    newest tap; inputs before the call come from the state (the previous W-1 inputs,
    oldest first), zeros if there is none; the state after the call holds the last W-1
    inputs.  Activation SiLU(y) = y sigmoid(y).  W = 4.
  * gated RMSNorm over the head dimension d of each (token, head):
    y = o / sqrt(mean(o^2) + eps) * weight * SiLU(z), weight shared by all heads,
    eps = 1e-6.

Every function here is pinned by ``tests/test_oracle_mixer_io.py``.
"""

from __future__ import annotations

import numpy as np


def silu(x):
    """SiLU(x) = x / (1 + exp(-x)) in fp64, written to avoid overflow for large |x|."""
    x = np.asarray(x, dtype=np.float64)
    e = np.exp(-np.abs(x))
    sig = np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))
    return x * sig


def short_conv_silu(x, weight, bias=None, state=None):
    """Short causal depthwise convolution over time, then SiLU.

    x       [B, T, C]   inputs (any float dtype; used exactly)
    weight  [C, W]      per-channel taps; weight[:, W-1] multiplies the newest input
    bias    [C] or None
    state   [B, C, W-1] the W-1 inputs before x, oldest first, or None (zeros)
    Returns (y [B, T, C] fp64, new_state [B, C, W-1] fp64).
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(weight, dtype=np.float64)
    B, T, C = x.shape
    W = w.shape[1]
    if state is None:
        state = np.zeros((B, C, W - 1))
    hist = np.concatenate([np.swapaxes(np.asarray(state, dtype=np.float64), 1, 2), x], axis=1)
    # hist[:, j] is the input at time j - (W - 1)
    y = np.zeros((B, T, C))
    for t in range(T):
        for i in range(W):
            y[:, t, :] += w[:, i] * hist[:, t + i, :]
    if bias is not None:
        y += np.asarray(bias, dtype=np.float64)
    new_state = np.swapaxes(hist[:, hist.shape[1] - (W - 1):, :], 1, 2).copy()
    return silu(y), new_state


def gated_rmsnorm(o, z, weight, eps=1e-6):
    """Gated RMS normalisation over the last axis (the head dimension d).

    o [..., d] the rule's output, z [..., d] the gate input, weight [d].
    Returns o / sqrt(mean(o^2) + eps) * weight * SiLU(z) in fp64.
    """
    o = np.asarray(o, dtype=np.float64)
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    return o / rms * np.asarray(weight, dtype=np.float64) * silu(z)
