"""KDA backward on the GPU (kda_chunk_bwd) against the fp64 backward oracle.

The gradients are those of L = sum(dO * o) + sum(dhT * hT) with respect to
q, k, v, g, beta and h0.  The pages give the forward recurrence only; the
oracle (oracle/kda_oracle_bwd.c) is its exact derivative, pinned on the CPU
by finite differences, autograd of a dense-product forward, closed forms and
the transpose and split identities (tests/test_oracle_bwd.py).  bf16 outputs
use the same error report as o (plain, floor, relaxed, excess) and the
relaxed form at 1e-2; dh0 is fp32 and held to the stated max/rms metric.
"""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_07_b200 as kda
from linear_attention_07_b200.inputs import prefill_inputs
from tolerance import TOL_BF16, check_out, err_state

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)
NAMES = ("dq", "dk", "dv", "dg", "dbeta")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from linear_attention_07_b200 import build
    build.build()
    kda.load_library()
    torch.cuda.init()


def cotangents(B, T, H, seed, dhT_std=0.1):
    gen = torch.Generator().manual_seed(seed)
    dO = torch.randn((B, T, H, 128), generator=gen).to(torch.bfloat16)
    dhT = torch.randn((B, H, 128, 128), generator=gen) * dhT_std if dhT_std > 0 else None
    return dO, dhT


def run_bwd(x, dO, dhT):
    d = {k: (None if t is None else t.to(DEV)) for k, t in x.items()}
    got = kda.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"], dO.to(DEV),
                        None if dhT is None else dhT.to(DEV))
    torch.cuda.synchronize()
    assert kda.device_status() == kda.KDA_OK
    return got


def check_grads(x, dO, dhT, got, tol=TOL_BF16, dh0_tol=1e-3):
    want = oracle.bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], dO, dhT)
    for name, gval, wval in zip(NAMES, got[:5], want[:5]):
        assert torch.isfinite(gval).all(), name
        check_out(gval, wval, tol, what=name)
    e = err_state(got[5], want[5])
    assert e <= dh0_tol, f"dh0: {e:.3e}"


@pytest.mark.parametrize("T", [1, 31, 32, 33, 300])
def test_bwd_ragged_lengths(T):
    x = prefill_inputs(2, T, 3, 128, 128, seed=4000 + T, h0_std=0.1)
    dO, dhT = cotangents(2, T, 3, seed=4100 + T)
    check_grads(x, dO, dhT, run_bwd(x, dO, dhT))


@pytest.mark.parametrize("case", ["g_min", "g_zero", "beta_zero", "pinned"])
def test_bwd_degenerate_gates(case):
    x = prefill_inputs(1, 200, 2, 128, 128, seed=4200, h0_std=0.1,
                       pin_frac=0.1 if case == "pinned" else 0.0)
    if case == "g_min":
        x["g"] = torch.full_like(x["g"], -5.0)
    elif case == "g_zero":
        x["g"] = torch.zeros_like(x["g"])
    elif case == "beta_zero":
        x["beta"] = torch.zeros_like(x["beta"])
    dO, dhT = cotangents(1, 200, 2, seed=4201)
    check_grads(x, dO, dhT, run_bwd(x, dO, dhT))


def test_bwd_without_h0_and_dhT():
    x = prefill_inputs(1, 100, 2, 128, 128, seed=4300)
    dO, _ = cotangents(1, 100, 2, seed=4301)
    check_grads(x, dO, None, run_bwd(x, dO, None))


def test_bwd_t0_passes_dhT_through():
    x = prefill_inputs(2, 0, 2, 128, 128, seed=4400, h0_std=0.1)
    dO, dhT = cotangents(2, 0, 2, seed=4401)
    got = run_bwd(x, dO, dhT)
    assert torch.equal(got[5].cpu(), dhT)


def test_bwd_deterministic():
    x = prefill_inputs(1, 150, 2, 128, 128, seed=4500, h0_std=0.1)
    dO, dhT = cotangents(1, 150, 2, seed=4501)
    a = run_bwd(x, dO, dhT)
    b = run_bwd(x, dO, dhT)
    for u, w in zip(a, b):
        assert torch.equal(u, w)


def test_bwd_full_8k_head():
    """One head over the 8K pre-training length, two heads in the batch."""
    x = prefill_inputs(1, 8192, 2, 128, 128, seed=4600, h0_std=0.1)
    dO, dhT = cotangents(1, 8192, 2, seed=4601)
    check_grads(x, dO, dhT, run_bwd(x, dO, dhT))


def test_bwd_matches_split_identity():
    """dh0 of the second part of a split sequence is the dhT of the first:
    the backward of two halves joined this way equals the whole backward."""
    T, cut = 200, 96
    x = prefill_inputs(1, T, 2, 128, 128, seed=4700, h0_std=0.1)
    dO, dhT = cotangents(1, T, 2, seed=4701)
    d = {k: (None if t is None else t.to(DEV)) for k, t in x.items()}
    names = ("q", "k", "v", "g", "beta")
    A = [d[n][:, :cut].contiguous() for n in names]
    Bp = [d[n][:, cut:].contiguous() for n in names]
    _, h_cut = kda.chunk_fwd(*A, d["h0"])
    g2 = kda.chunk_bwd(*Bp, h_cut, dO[:, cut:].contiguous().to(DEV), dhT.to(DEV))
    g1 = kda.chunk_bwd(*A, d["h0"], dO[:, :cut].contiguous().to(DEV), g2[5])
    torch.cuda.synchronize()
    joined = [torch.cat([u, w], 1) for u, w in zip(g1[:5], g2[:5])] + [g1[5]]
    check_grads(x, dO, dhT, joined, dh0_tol=2e-3)


@pytest.mark.parametrize("B,H,T", [(1, 2, 77), (2, 3, 300)])
def test_bwd_through_fused_prologue(B, H, T):
    """kda_chunk_bwd_raw against the oracle's backward through the prologue
    (q, k normalised, g = -5 sigmoid(z); zero q/k rows; ragged lengths)."""
    from linear_attention_07_b200.inputs import raw_inputs
    x = raw_inputs((B, T, H, 128), (B, T, H, 128), (B, T, H), seed=4800 + T, zero_rows=2)
    gen = torch.Generator().manual_seed(4801 + T)
    h0 = torch.randn((B, H, 128, 128), generator=gen) * 0.1
    dO = torch.randn((B, T, H, 128), generator=gen).to(torch.bfloat16)
    dhT = torch.randn((B, H, 128, 128), generator=gen) * 0.1
    d = {k: t.to(DEV) for k, t in x.items()}
    got = kda.chunk_bwd_raw(d["q"], d["k"], d["v"], d["z"], d["beta"], h0.to(DEV), dO.to(DEV), dhT.to(DEV))
    torch.cuda.synchronize()
    assert kda.device_status() == kda.KDA_OK
    want = oracle.bwd_raw(x["q"], x["k"], x["v"], x["z"], x["beta"], h0, dO, dhT)
    for name, gval, wval in zip(("dq_raw", "dk_raw", "dv", "dz", "dbeta"), got[:5], want[:5]):
        assert torch.isfinite(gval).all(), name
        check_out(gval, wval, TOL_BF16, what=name)
    assert err_state(got[5], want[5]) <= 1e-3
    assert not got[0][:, :2].float().abs().max() > 0, "zero q rows must have a zero gradient"
