"""Failure detection on the real prefill and backward kernels, without any
GPU fault.

Every wait between the roles of a prefill kernel (input loads, MMA
completion, slot hand-overs between the CTAs of a cluster) is bounded; the
limit is 2 s, and KDA_WAIT_LIMIT_NS=0 makes every wait a single
non-blocking check, so the first wait for an input load (or, in the cluster
variant, for a chunk pushed by another SM) gives up.  The kernel must
then wind down on its own: no new MMA or copy, every barrier rendezvous
kept, in-flight copies and MMAs drained, o and hT filled with NaN, and
KDA_ERR_TIMEOUT in the status word that kda_device_status reads.  The
context stays usable: the same prefill with the normal limit is correct.
The backward's chunk-local kernel waits (bounded the same way) for its two
groups of tensor-core products; when the first wait gives up it issues no
second group, lets the first finish before releasing tensor memory, and
writes NaN for the chunk's dq, dk, dv, dg and dbeta.
"""
import pytest
import torch

import oracle
import linear_attention_07_b200 as kda
from linear_attention_07_b200.inputs import prefill_inputs
from tolerance import TOL_BF16, check_out, err_state

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from linear_attention_07_b200 import build
    build.build()
    kda.load_library()
    torch.cuda.init()


@pytest.mark.parametrize("variant", ["fused", "cluster"])
def test_prefill_own_waits_expire(monkeypatch, variant):
    monkeypatch.setenv("KDA_PREFILL_VARIANT", variant)
    x = prefill_inputs(1, 200, 2, 128, 128, seed=5000, h0_std=0.1)
    d = {k: (None if t is None else t.to(DEV)) for k, t in x.items()}
    assert kda.device_status() == kda.KDA_OK
    monkeypatch.setenv("KDA_WAIT_LIMIT_NS", "0")
    o, hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    torch.cuda.synchronize()
    assert kda.device_status() == kda.KDA_ERR_TIMEOUT
    assert kda.device_status() == kda.KDA_OK            # read and cleared
    assert torch.isnan(hT).all(), "hT of a timed-out prefill must be NaN"
    assert torch.isnan(o.float()).all(), "o of a timed-out prefill must be NaN"
    monkeypatch.delenv("KDA_WAIT_LIMIT_NS")
    o, hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    torch.cuda.synchronize()
    assert kda.device_status() == kda.KDA_OK
    o_ref, hT_ref = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
    check_out(o, o_ref, TOL_BF16)
    assert err_state(hT, hT_ref) <= TOL_BF16


def test_backward_own_waits_expire(monkeypatch):
    x = prefill_inputs(1, 100, 2, 128, 128, seed=5100, h0_std=0.1)
    d = {k: (None if t is None else t.to(DEV)) for k, t in x.items()}
    gen = torch.Generator().manual_seed(5101)
    dO = torch.randn((1, 100, 2, 128), generator=gen).to(torch.bfloat16)
    dhT = torch.randn((1, 2, 128, 128), generator=gen) * 0.1
    assert kda.device_status() == kda.KDA_OK
    monkeypatch.setenv("KDA_WAIT_LIMIT_NS", "0")
    got = kda.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"], dO.to(DEV), dhT.to(DEV))
    torch.cuda.synchronize()
    assert kda.device_status() == kda.KDA_ERR_TIMEOUT
    assert kda.device_status() == kda.KDA_OK            # read and cleared
    for name, t in zip(("dq", "dk", "dv", "dg", "dbeta"), got[:5]):
        assert torch.isnan(t.float()).all(), f"{name} of a timed-out backward must be NaN"
    monkeypatch.delenv("KDA_WAIT_LIMIT_NS")
    got = kda.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"], dO.to(DEV), dhT.to(DEV))
    torch.cuda.synchronize()
    assert kda.device_status() == kda.KDA_OK
    want = oracle.bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], dO, dhT)
    for name, gval, wval in zip(("dq", "dk", "dv", "dg", "dbeta"), got[:5], want[:5]):
        check_out(gval, wval, TOL_BF16, what=name)
    assert err_state(got[5], want[5]) <= 1e-3
