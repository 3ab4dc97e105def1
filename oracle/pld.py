"""fp64 oracle of Progressive Layer Dropping over a stack of encoder layers.

TEST INFRASTRUCTURE ONLY (see the package docstring): never imported by the
product path.

"Progressive Layer Dropping" page, schedule section: the keep level theta
starts at 1 and decays towards a target theta_bar with the global step t,
theta(t) = (1 - theta_bar) exp(-gamma t) + theta_bar; at each step some
layers are skipped (identity in forward and backward), and the skipping
grows along two axes, time (the schedule) and depth.  Readings taken where
the page is silent:
  * depth profile: linear, layer l of L (0-based) is kept with probability
    1 - (l + 1) / L * (1 - theta(t)); the last layer's keep probability is
    theta(t) itself;
  * the random draw: Philox4x32-10 with counter (t mod 2^32, t div 2^32, 3,
    l) and key (seed mod 2^32, seed div 2^32), the layer kept when output
    word 0 (a 32-bit unsigned integer) is below floor(p * 2^32);
  * a skipped layer produces no parameter gradients (None here).

Pins: tests/test_oracle_pld.py (schedule endpoints and half-life, the depth
profile's mean, kept-frequency statistics, the identity of a skipped layer,
finite differences through a two-layer stack).
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

from .layer import LayerConfig, layer_backward, layer_forward, philox4x32_10

SITE_PLD = 3


def pld_theta(theta_bar: float, gamma: float, step: int) -> float:
    """Keep level at global step `step` (Python float arithmetic, libm exp)."""
    return (1.0 - theta_bar) * math.exp(-gamma * float(step)) + theta_bar


def pld_keep_prob(layer: int, num_layers: int, theta: float) -> float:
    """Probability that layer `layer` (0-based) of `num_layers` runs."""
    assert 0 <= layer < num_layers
    return 1.0 - (layer + 1) / num_layers * (1.0 - theta)


def pld_keep(seed: int, step: int, layer: int, num_layers: int, theta: float) -> bool:
    """Whether the layer runs at this step (see the module docstring)."""
    p = pld_keep_prob(layer, num_layers, theta)
    if p >= 1.0:
        return True
    if not p > 0.0:
        return False
    thr = math.floor(p * 4294967296.0)
    w = philox4x32_10(step & 0xFFFFFFFF, (step >> 32) & 0xFFFFFFFF, SITE_PLD, layer,
                      seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    return int(w[0]) < thr


def stack_forward_backward(cfg: LayerConfig, x, mask, weights: list, dy, keep: list,
                           seq_index=None, storage_rounded=False) -> dict:
    """A stack of len(weights) layers of configuration `cfg`, layer l with
    philox_offset = l; layers with keep[l] False are the identity.  Runs the
    forward through the kept layers, then the backward in reverse.  Returns
    dict(y, dx, grads: list (None for skipped layers), inputs: each layer's
    input, dys: each layer's upstream gradient)."""
    nl = len(weights)
    assert len(keep) == nl
    inputs, saved = [], []
    h = np.asarray(x, dtype=np.float64)
    for l in range(nl):
        inputs.append(h)
        if keep[l]:
            c = dataclasses.replace(cfg, philox_offset=l)
            h, sv = layer_forward(c, h, mask, weights[l], seq_index=seq_index, storage_rounded=storage_rounded)
            saved.append((c, sv))
        else:
            saved.append(None)
    y = h
    grads = [None] * nl
    dys = [None] * nl
    g = np.asarray(dy, dtype=np.float64)
    for l in reversed(range(nl)):
        dys[l] = g
        if saved[l] is not None:
            c, sv = saved[l]
            g, grads[l] = layer_backward(c, sv, g)
    return dict(y=y, dx=g, grads=grads, inputs=inputs, dys=dys)
