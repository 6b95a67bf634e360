"""Pins of the oracle's prologue (q, k L2-normalised; g = -5 sigmoid(z)).

The definitions are checked through properties a plausible slip would break
(a sign in the exponent, a missing factor, normalising over the wrong axis,
dividing a zero vector), not by retyping them.
"""
import numpy as np
import torch

import oracle
from linear_attention_07_b200.inputs import prefill_inputs, raw_inputs


def test_gate_values_and_symmetry():
    z = np.array([0.0, 1.0, -1.0, 3.0, -3.0, 30.0, -30.0, 800.0, -800.0])
    _, _, g = oracle.prologue(np.ones((1, 1, 9)), np.ones((1, 1, 9)), z.reshape(1, 1, 9))
    g = g.ravel()
    assert g[0] == -2.5                                       # sigmoid(0) = 1/2
    assert np.all(g <= 0.0) and np.all(g >= -5.0)             # the bound of the pages
    assert abs(g[7] + 5.0) < 1e-300 and g[8] == 0.0           # saturation, no overflow fault
    # sigmoid(-z) = 1 - sigmoid(z)  =>  g(-z) = -5 - g(z)
    for a, b in ((1, 2), (3, 4), (5, 6)):
        assert abs(g[b] - (-5.0 - g[a])) < 1e-14
    assert g[1] < g[0] < g[2]                                 # larger z decays faster


def test_normalisation_axis_zero_rows_and_scale():
    x = raw_inputs((2, 5, 3, 16), (2, 5, 3, 8), (2, 5, 3), seed=3, zero_rows=2)
    q, k, _ = oracle.prologue(x["q"], x["k"], x["z"])
    nq = np.sqrt((q * q).sum(-1))
    assert np.allclose(nq[:, 2:], 1.0, atol=1e-13)            # unit over the key channels
    assert np.all(q[:, :2] == 0.0) and np.all(k[:, :2] == 0.0)  # zero vectors stay zero
    q2, _, _ = oracle.prologue(3.5 * x["q"].double(), x["k"], x["z"])
    assert np.allclose(q2, q, atol=1e-14)                      # scale invariant
    # direction kept: q is a positive multiple of the raw vector
    raw = x["q"].double().numpy()[:, 2:]
    cos = (raw * q[:, 2:]).sum(-1) / np.sqrt((raw * raw).sum(-1))
    assert np.allclose(cos, 1.0, atol=1e-13)


def test_raw_forward_equals_forward_on_prepared_inputs():
    """fwd_raw on raw inputs = fwd on the prologue's outputs, and on inputs
    that are already unit vectors with z chosen for a given g it is fwd."""
    x = prefill_inputs(1, 40, 2, 16, 16, seed=5, h0_std=0.1)
    g = x["g"].double().numpy()
    z = -np.log(-5.0 / g - 1.0)                                # inverse of g = -5 sigmoid(z)
    o1, h1 = oracle.fwd_raw(x["q"], x["k"], x["v"], z, x["beta"], x["h0"])
    q, k, g2 = oracle.prologue(x["q"], x["k"], z)
    assert np.allclose(g2, g, atol=1e-12)
    o2, h2 = oracle.fwd(q, k, x["v"], g2, x["beta"], x["h0"])
    assert np.array_equal(o1, o2) and np.array_equal(h1, h2)
    o3, h3 = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
    # the generator's q, k are unit vectors rounded to bf16: normalising again
    # moves them by at most the bf16 rounding
    assert np.abs(o1 - o3).max() <= 2e-2 * np.sqrt((o3 * o3).mean()) + 1e-12
