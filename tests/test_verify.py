"""Multi-token verify and rollback (speculative decoding) on the GPU.

kda_verify_fwd runs K drafted tokens per request from a checkpoint state and
keeps the state after every token.  After acceptance a request continues
from the state after its last accepted token, found two ways: the snapshot
written by the verify call, or a replay of the accepted tokens from the
checkpoint ("177: Kimi K3 in Detail" episode notes, Deep dive 23: rollback
keeps a checkpoint and replays the accepted steps).  Every check is against
the fp64 oracle on the same inputs; the two rollback routes must agree bit
for bit when the replay uses the decode kernel (the same per-token
arithmetic as the verify kernel).
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


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from linear_attention_07_b200 import build
    build.build()
    kda.load_library()
    torch.cuda.init()


def _prefix_states(x, h0, K):
    """Oracle states after each of the K tokens: [N, K, H, dk, dv]."""
    out = []
    for t in range(1, K + 1):
        _, hT = oracle.fwd(*(x[n][:, :t] for n in ("q", "k", "v", "g", "beta")), h0)
        out.append(hT)
    return np.stack(out, axis=1)


@pytest.mark.parametrize("N,K,H,dk,dv", [(3, 8, 2, 128, 128), (2, 5, 3, 64, 128), (4, 1, 2, 128, 32),
                                         (1, 64, 1, 32, 32)])
def test_verify_against_oracle(N, K, H, dk, dv):
    x = prefill_inputs(N, K, H, dk, dv, seed=3000 + N * K + dk, h0_std=0.1)
    d = {k: (None if t is None else t.to(DEV)) for k, t in x.items()}
    h0_before = d["h0"].clone()
    o, states = kda.verify_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    torch.cuda.synchronize()
    assert torch.equal(d["h0"], h0_before), "verify must not modify the checkpoint"
    o_ref, _ = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
    check_out(o, o_ref, TOL_BF16)
    st_ref = _prefix_states(x, x["h0"], K)
    e = err_state(states, st_ref)
    assert e <= 1e-5, f"states: {e:.3e}"          # fp32 arithmetic throughout


def test_verify_zero_start_state():
    x = prefill_inputs(2, 6, 2, 128, 128, seed=3100)
    d = {k: (None if t is None else t.to(DEV)) for k, t in x.items()}
    o, states = kda.verify_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], None)
    torch.cuda.synchronize()
    o_ref, hT_ref = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None)
    check_out(o, o_ref, TOL_BF16)
    assert err_state(states[:, -1], hT_ref) <= 1e-5


def test_verify_snapshots_equal_decode_replay_bitwise():
    """Replaying the first j tokens with kda_decode_step from the checkpoint
    gives the verify call's o and states[:, j - 1] bit for bit."""
    N, K, H = 3, 7, 4
    x = prefill_inputs(N, K, H, 128, 128, seed=3200, h0_std=0.1)
    d = {k: (None if t is None else t.to(DEV)) for k, t in x.items()}
    o, states = kda.verify_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    S = d["h0"].clone()
    for t in range(K):
        od = kda.decode_step(*(d[n][:, t].contiguous() for n in ("q", "k", "v", "g", "beta")), S)
        torch.cuda.synchronize()
        assert torch.equal(od, o[:, t]), f"o differs at token {t}"
        assert torch.equal(S, states[:, t]), f"state differs after token {t + 1}"


def test_serving_flow_verify_rollback_replay_continue():
    """Prefill 4096 tokens (the checkpoint), verify 8 drafted tokens, accept
    j_n of them per request (5, 0 and 8), roll back by snapshot and by
    replay from the checkpoint (decode kernel: bit for bit; prefill kernel:
    within tolerance), then decode 3 more tokens; everything against the
    oracle on the whole accepted sequence."""
    N, H, P, K, extra = 3, 2, 4096, 8, 3
    accept = [5, 0, 8]
    x = prefill_inputs(N, P + K + extra, H, 128, 128, seed=3300, h0_std=0.1)
    d = {k: (None if t is None else t.to(DEV)) for k, t in x.items()}
    sl = lambda t, a, b: t[:, a:b].contiguous()
    names = ("q", "k", "v", "g", "beta")
    # 1. prefill: the checkpoint
    _, ckpt = kda.chunk_fwd(*(sl(d[n], 0, P) for n in names), d["h0"])
    # 2. verify K drafted tokens from the checkpoint
    o_ver, states = kda.verify_fwd(*(sl(d[n], P, P + K) for n in names), ckpt)
    # 3a. rollback by snapshot: request n continues from states[n, j_n - 1]
    S_snap = torch.stack([states[n, j - 1] if j > 0 else ckpt[n] for n, j in enumerate(accept)])
    # 3b. rollback by replay of the accepted tokens from the checkpoint
    S_rep = ckpt.clone()
    for t in range(max(accept)):
        live = [n for n, j in enumerate(accept) if t < j]
        xt = [d[n][live, P + t].contiguous() for n in names]
        Sl = S_rep[live].contiguous()
        kda.decode_step(*xt, Sl)
        S_rep[live] = Sl
    torch.cuda.synchronize()
    assert torch.equal(S_snap, S_rep), "snapshot and decode replay differ"
    # 3c. replay through the prefill kernel (tensor cores): within tolerance
    for n, j in enumerate(accept):
        if j == 0:
            continue
        _, S_pf = kda.chunk_fwd(*(d[m][n:n + 1, P:P + j].contiguous() for m in names), ckpt[n:n + 1])
        torch.cuda.synchronize()
        _, h_ref = oracle.fwd(*(x[m][n:n + 1, :P + j] for m in names), x["h0"][n:n + 1])
        assert err_state(S_pf, h_ref) <= TOL_BF16
    # 4. continue decoding `extra` tokens after each request's accepted prefix
    S = S_snap.clone()
    outs = []
    for t in range(extra):
        xt = [torch.stack([d[m][n, P + accept[n] + t] for n in range(N)]) for m in names]
        outs.append(kda.decode_step(*xt, S))
    torch.cuda.synchronize()
    # oracle over each request's accepted sequence
    for n, j in enumerate(accept):
        T_n = P + j + extra
        o_ref, h_ref = oracle.fwd(*(x[m][n:n + 1, :T_n] for m in names), x["h0"][n:n + 1])
        if j > 0:
            check_out(o_ver[n:n + 1, :j], o_ref[:, P:P + j], TOL_BF16, what="verify o")
        check_out(torch.stack([outs[t][n] for t in range(extra)])[None], o_ref[:, P + j:], TOL_BF16,
                  what="decode o after rollback")
        assert err_state(S[n:n + 1], h_ref) <= TOL_BF16
