"""The oracle against values fixed by the definition, not by itself (CPU)."""
import json
import math
import os

import numpy as np
import pytest
import torch

import pins


@pytest.mark.parametrize("name", sorted(pins.ALL_PINS))
def test_pin(oracle_mod, name):
    fn, tol = pins.ALL_PINS[name]
    err = fn(oracle_mod.default())
    assert err <= tol, f"{name}: discrepancy {err:.3e} > {tol:.0e}"


def test_decay_bound_arithmetic():
    """With g >= -5, a 16-token tile scales by at most exp(80), which bf16
    represents ('T11E1: K3 tech report' transcript, log-decay-bound turn)."""
    with open(os.path.join(pins.GOLDEN, "decay_bound.json")) as f:
        fx = json.load(f)
    bf16_max = torch.finfo(torch.bfloat16).max
    assert math.isclose(math.log(bf16_max), fx["ln_bf16_max"], rel_tol=1e-12)
    worst = -fx["g_min"] * fx["tile"]
    assert worst == fx["max_log_scaling"] == 80.0
    assert worst < math.log(bf16_max)
    up = torch.tensor(math.exp(worst)).to(torch.bfloat16)
    down = torch.tensor(math.exp(-worst)).to(torch.bfloat16)
    assert torch.isfinite(up) and float(up) > 1e34
    assert float(down) >= torch.finfo(torch.bfloat16).smallest_normal
    # the largest tile length that still fits, and the first that does not
    n = fx["largest_tile_within_bound"]
    assert -fx["g_min"] * n < math.log(bf16_max) < -fx["g_min"] * (n + 1)
    assert not torch.isfinite(torch.tensor(math.exp(-fx["g_min"] * (n + 1))).to(torch.bfloat16))


def test_empty_and_degenerate(oracle_mod):
    """T = 0 returns h0 unchanged; a single head with dk = dv = 1 is scalar."""
    h0 = np.arange(6, dtype=np.float64).reshape(1, 2, 3)
    e = np.zeros((1, 0, 2))
    o, hT = oracle_mod.heads(e, e, np.zeros((1, 0, 3)), e, np.zeros((1, 0)), h0)
    assert o.shape == (1, 0, 3) and np.array_equal(hT, h0)
    # scalar: s <- e^g s; u = b(v - s); s += u; o = q s  (k = 1)
    s, out = 0.5, []
    qv, vv, gv, bv = [0.3, -1.0], [2.0, 1.0], [-0.5, -1.5], [0.25, 0.75]
    for t in range(2):
        s = math.exp(gv[t]) * s
        s = s + bv[t] * (vv[t] - s)
        out.append(qv[t] * s)
    o, hT = oracle_mod.heads(np.array(qv).reshape(1, 2, 1), np.ones((1, 2, 1)),
                             np.array(vv).reshape(1, 2, 1), np.array(gv).reshape(1, 2, 1),
                             np.array(bv).reshape(1, 2), np.array([[[0.5]]]))
    assert np.allclose(o.ravel(), out, rtol=1e-15, atol=0) and math.isclose(hT.item(), s, rel_tol=1e-15)


def test_decode_wrapper_matches_closed_form(oracle_mod):
    """decode_step's marshalling: N x H single-token updates, closed form."""
    rng = np.random.default_rng(12)
    N, H, dk, dv = 3, 2, 6, 5
    q = rng.standard_normal((N, H, dk)); q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rng.standard_normal((N, H, dk)); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((N, H, dv)); beta = rng.uniform(0, 1, (N, H))
    g = -rng.uniform(0, 5, (N, H, dk)); S = rng.standard_normal((N, H, dk, dv))
    o, S1 = oracle_mod.decode_step(q, k, v, g, beta, S)
    for n in range(N):
        for h in range(H):
            DS = np.exp(g[n, h])[:, None] * S[n, h]
            u = beta[n, h] * (v[n, h] - DS.T @ k[n, h])
            assert np.allclose(o[n, h], DS.T @ q[n, h] + u * (k[n, h] @ q[n, h]), rtol=1e-13, atol=1e-15)
            assert np.allclose(S1[n, h], DS + np.outer(k[n, h], u), rtol=1e-13, atol=1e-15)


def test_threads_do_not_change_results(oracle_mod):
    rng = np.random.default_rng(13)
    q, k, v, g, beta, S0 = pins._rand_problem(rng, 33, 8, 8, n=9)
    a = oracle_mod.heads(q, k, v, g, beta, S0, n_threads=1)
    b = oracle_mod.heads(q, k, v, g, beta, S0, n_threads=4)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
