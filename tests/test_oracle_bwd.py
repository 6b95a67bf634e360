"""The backward oracle against values fixed by the forward recurrence (CPU)."""
import numpy as np
import pytest

import pins_bwd
from pins import _rand_problem, _rel


@pytest.mark.parametrize("name", sorted(pins_bwd.ALL_PINS))
def test_pin(oracle_mod, name):
    fn, tol = pins_bwd.ALL_PINS[name]
    err = fn(oracle_mod.default())
    assert err <= tol, f"{name}: discrepancy {err:.3e} > {tol:.0e}"


def test_empty_sequence_passes_state_adjoint(oracle_mod):
    """T = 0: hT = h0, so dh0 = dhT and there is nothing else."""
    dhT = np.arange(6, dtype=np.float64).reshape(1, 2, 3)
    e = np.zeros((1, 0, 2))
    out = oracle_mod.heads_bwd(e, e, np.zeros((1, 0, 3)), e, np.zeros((1, 0)),
                               np.ones((1, 2, 3)), None, dhT)
    assert all(x.size == 0 for x in out[:5]) and np.array_equal(out[5], dhT)


def test_missing_cotangents_are_zero(oracle_mod):
    """dO = None and dhT = None mean zero cotangents; the gradients are
    linear in (dO, dhT)."""
    rng = np.random.default_rng(31)
    q, k, v, g, beta, h0 = _rand_problem(rng, 20, 5, 4, n=2)
    dO = rng.standard_normal((2, 20, 4))
    dhT = rng.standard_normal((2, 5, 4))
    only_o = oracle_mod.heads_bwd(q, k, v, g, beta, h0, dO, None)
    only_s = oracle_mod.heads_bwd(q, k, v, g, beta, h0, None, dhT)
    both = oracle_mod.heads_bwd(q, k, v, g, beta, h0, dO, dhT)
    for a, b, c in zip(only_o, only_s, both):
        assert _rel(a + b, c) < 1e-13
    zero = oracle_mod.heads_bwd(q, k, v, g, beta, h0, None, None)
    assert all(not np.any(x) for x in zero)


def test_threads_do_not_change_results(oracle_mod):
    rng = np.random.default_rng(32)
    q, k, v, g, beta, h0 = _rand_problem(rng, 70, 6, 6, n=7)
    dO = rng.standard_normal((7, 70, 6))
    a = oracle_mod.heads_bwd(q, k, v, g, beta, h0, dO, None, n_threads=1)
    b = oracle_mod.heads_bwd(q, k, v, g, beta, h0, dO, None, n_threads=4)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))


def test_prologue_chain_rule_finite_differences(oracle_mod):
    """bwd_raw (raw q, k and gate pre-activation z) against central finite
    differences of fwd_raw, the forward with the fused prologue."""
    rng = np.random.default_rng(33)
    B, T, H, dk, dv = 1, 5, 2, 4, 3
    qr = rng.standard_normal((B, T, H, dk)) * 2.0
    kr = rng.standard_normal((B, T, H, dk)) * 0.5
    z = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    beta = rng.uniform(0.1, 0.9, (B, T, H))
    h0 = 0.3 * rng.standard_normal((B, H, dk, dv))
    dO = rng.standard_normal((B, T, H, dv))
    dhT = rng.standard_normal((B, H, dk, dv))
    x = [qr, kr, v, z, beta, h0]
    grads = oracle_mod.bwd_raw(*x, dO=dO, dhT=dhT)

    def loss(y):
        o, hT = oracle_mod.fwd_raw(*y)
        return float((o * dO).sum() + (hT * dhT).sum())

    eps = 1e-6
    for a, G in enumerate(grads):
        fd = np.zeros_like(x[a])
        for idx in np.ndindex(x[a].shape):
            xp = [y.copy() for y in x]
            xm = [y.copy() for y in x]
            xp[a][idx] += eps
            xm[a][idx] -= eps
            fd[idx] = (loss(xp) - loss(xm)) / (2 * eps)
        assert _rel(G, fd) < 1e-7, f"input {a}: {_rel(G, fd):.2e}"


def test_prologue_chain_rule_special_cases(oracle_mod):
    """A zero raw vector has zero gradient; the gradient of a normalised
    vector is orthogonal to it (length is not seen); z far in the tails has
    vanishing gate gradient."""
    rng = np.random.default_rng(34)
    r = rng.standard_normal((3, 4, 2, 8))
    r[0, 1, 1] = 0.0
    d = rng.standard_normal(r.shape)
    z = np.zeros(r.shape)
    z[1, 2, 0] = 80.0
    z[2, 3, 1] = -80.0
    dq_raw, dk_raw, dz = oracle_mod.prologue_bwd(r, r, z, d, d, np.ones(r.shape))
    assert not np.any(dq_raw[0, 1, 1]) and not np.any(dk_raw[0, 1, 1])
    assert np.max(np.abs((dq_raw * r).sum(axis=-1))) < 1e-14
    assert np.allclose(dz[0, 0, 0], -5.0 * 0.25, rtol=0, atol=1e-15)
    assert np.max(np.abs(dz[1, 2, 0])) < 1e-30 and np.max(np.abs(dz[2, 3, 1])) < 1e-30


def test_tiled_scheme_is_finite_in_fp32_at_the_floor(oracle_mod):
    """g = -5 on every channel over 64 tokens: a factor 1/gamma relative to
    the chunk start would reach e^155 (inf in fp32); the GPU backward's tile
    references keep every factor at or below e^80, so its scheme run in fp32
    stays finite and close to the fp64 oracle."""
    from pins import _rand_problem
    rng = np.random.default_rng(31)
    T, dk, dv = 64, 16, 8
    q, k, v, g, beta, h0 = _rand_problem(rng, T, dk, dv, n=1)
    g = np.full_like(g, -5.0)
    dO = rng.standard_normal((1, T, dv))
    dhT = rng.standard_normal((1, dk, dv))
    got = pins_bwd.tiled_chunk_bwd(q[0], k[0], v[0], g[0], beta[0], h0[0], dO[0], dhT[0], dtype=np.float32)
    want = oracle_mod.heads_bwd(q, k, v, g, beta, h0, dO, dhT)
    for x, w in zip(got, want):
        assert np.all(np.isfinite(x))
        w = w[0]
        scale = np.sqrt(np.mean(w * w)) + np.abs(w)
        assert np.max(np.abs(x - w) / np.where(scale > 0, scale, 1.0)) <= 1e-3   # dg: fp32 rounding of a cancelling sum
