"""Context parallelism: one sequence split into blocks joined through their
transitions.

CPU: the collective orchestration on a 2-rank gloo group, with the per-rank
steps done by the fp64 oracle, against the oracle on the whole sequence.
GPU: the two joining kernels (kda_chunk_transition, kda_state_chain) against
their definitions, three blocks composed as the ranks compose them, and the
module end to end on a one-rank NCCL group.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from linear_attention_07_b200.inputs import prefill_inputs
from tolerance import TOL_BF16, check_out, err_state


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The per-rank steps in fp64 on the host (oracle), for the CPU test."""

    @staticmethod
    def block_fwd(q, k, v, g, beta, h0):
        o, hT = oracle.fwd(q, k, v, g, beta, h0)
        return torch.from_numpy(np.ascontiguousarray(o)), torch.from_numpy(np.ascontiguousarray(hT))

    @staticmethod
    def transition(q, k, g, beta):
        B, T, H, d = q.shape
        eye = torch.eye(d, dtype=torch.float64).expand(B, H, d, d).contiguous()
        _, M = oracle.fwd(q, k, torch.zeros_like(q), g, beta, eye, want_o=False)
        return torch.from_numpy(np.ascontiguousarray(M))

    @staticmethod
    def state_chain(M, N, h0):
        B, P, H, d, _ = N.shape
        S = torch.zeros_like(N[:, 0]) if h0 is None else h0.to(N.dtype).clone()
        S_start = torch.empty_like(N)
        for p in range(P):
            S_start[:, p] = S
            S = M[:, p] @ S + N[:, p]
        return S_start, S


def _cpu_worker(rank, world, port, seed, errs, cuts=None, with_h0=True):
    import torch.distributed as dist
    from linear_attention_07_b200.context_parallel import chunk_fwd_context_parallel
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        B, T, H, d = 2, 96, 2, 16
        x = prefill_inputs(B, T, H, d, d, seed=seed, h0_std=0.1 if with_h0 else 0.0)
        cuts = cuts or [T * r // world for r in range(world + 1)]
        lo, hi = cuts[rank], cuts[rank + 1]
        blk = {n: x[n][:, lo:hi].contiguous() for n in ("q", "k", "v", "g", "beta")}
        h0 = None if x["h0"] is None else x["h0"].double()
        o, hT = chunk_fwd_context_parallel(blk["q"], blk["k"], blk["v"], blk["g"], blk["beta"], h0,
                                           ops=OracleOps)
        o_ref, hT_ref = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
        eo = float(np.abs(o.numpy() - o_ref[:, lo:hi]).max())
        eh = float(np.abs(hT.numpy() - hT_ref).max())
        errs[rank] = max(eo, eh)
    finally:
        dist.destroy_process_group()


def _run_ranks(world, seed, cuts=None, with_h0=True):
    ctx = mp.get_context("spawn")
    errs = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_cpu_worker, args=(r, world, port, seed, errs, cuts, with_h0))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert sorted(errs.keys()) == list(range(world))
    return dict(errs)


def test_context_parallel_orchestration_gloo():
    """Two ranks, one sequence: each rank's o and the final state equal the
    whole-sequence oracle (fp64 throughout, so to rounding)."""
    errs = _run_ranks(2, 1301)
    assert max(errs.values()) < 1e-9, errs


def test_context_parallel_uneven_blocks_three_ranks():
    """Three ranks with blocks of 17, 50 and 29 tokens and no start state:
    the exchanged (M, N) have fixed shapes, so the blocks need not match."""
    errs = _run_ranks(3, 1302, cuts=[0, 17, 67, 96], with_h0=False)
    assert max(errs.values()) < 1e-9, errs


# ----------------------------------------------------------------- GPU ---

DEV = torch.device("cuda", 0)


@pytest.fixture(scope="module")
def kda_lib():
    import linear_attention_07_b200 as kda
    from linear_attention_07_b200 import build
    build.build()
    kda.load_library()
    return kda


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,T", [(1, 2, 700), (2, 3, 64), (1, 1, 0)])
def test_transition_kernel(kda_lib, B, H, T):
    kda = kda_lib
    x = prefill_inputs(B, max(T, 1), H, 128, 128, seed=1400 + T)
    x = {n: (None if t is None else t[:, :T].contiguous()) for n, t in x.items() if n != "h0"}
    # slow decay (g scaled by 0.01, still in [-5, 0]): with the usual gates the
    # transition over tens of tokens is below fp32's range (about e^-160)
    x["g"] = (x["g"].float() * 0.01).to(torch.bfloat16)
    d = {n: t.to(DEV) for n, t in x.items()}
    M = kda.chunk_transition(d["q"], d["k"], d["g"], d["beta"])
    torch.cuda.synchronize()
    eye = torch.eye(128, dtype=torch.float64).expand(B, H, 128, 128).contiguous()
    if T == 0:
        assert torch.equal(M.cpu().double(), eye)
        return
    _, M_ref = oracle.fwd(x["q"], x["k"], torch.zeros_like(x["q"]), x["g"], x["beta"], eye, want_o=False)
    assert err_state(M, M_ref) <= TOL_BF16


@pytest.mark.gpu
def test_state_chain_kernel(kda_lib):
    kda = kda_lib
    B, P, H = 2, 5, 3
    gen = torch.Generator().manual_seed(1500)
    M = (torch.randn(B, P, H, 128, 128, generator=gen) * 0.08).float()
    N = torch.randn(B, P, H, 128, 128, generator=gen).float()
    h0 = torch.randn(B, H, 128, 128, generator=gen).float()
    S_start, hT = kda.state_chain(M.to(DEV), N.to(DEV), h0.to(DEV))
    torch.cuda.synchronize()
    S = h0.double()
    for p in range(P):
        assert torch.allclose(S_start[:, p].cpu().double(), S, rtol=1e-5, atol=1e-5)
        S = M[:, p].double() @ S + N[:, p].double()
    assert torch.allclose(hT.cpu().double(), S, rtol=1e-5, atol=1e-5)


@pytest.mark.gpu
def test_three_blocks_composed_as_ranks_do(kda_lib):
    """Blocks run independently and joined through their transitions give
    the whole sequence's o and final state (oracle parity)."""
    kda = kda_lib
    B, H, L, W = 1, 2, 1024, 3
    x = prefill_inputs(B, W * L, H, 128, 128, seed=1600, h0_std=0.1)
    d = {n: t.to(DEV) for n, t in x.items()}
    blk = lambda t, p: t[:, p * L:(p + 1) * L].contiguous()
    Ms, Ns = [], []
    for p in range(W):
        _, N = kda.chunk_fwd(blk(d["q"], p), blk(d["k"], p), blk(d["v"], p), blk(d["g"], p), blk(d["beta"], p), None)
        Ns.append(N)
        Ms.append(kda.chunk_transition(blk(d["q"], p), blk(d["k"], p), blk(d["g"], p), blk(d["beta"], p)))
    S_start, hT = kda.state_chain(torch.stack(Ms, 1).contiguous(), torch.stack(Ns, 1).contiguous(), d["h0"])
    o = torch.cat([kda.chunk_fwd(blk(d["q"], p), blk(d["k"], p), blk(d["v"], p), blk(d["g"], p), blk(d["beta"], p),
                                 S_start[:, p].contiguous())[0] for p in range(W)], 1)
    torch.cuda.synchronize()
    o_ref, hT_ref = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
    check_out(o, o_ref, TOL_BF16)
    assert err_state(hT, hT_ref) <= TOL_BF16


@pytest.mark.gpu
def test_module_on_one_rank_nccl(kda_lib):
    """chunk_fwd_context_parallel end to end on the kernels (a one-rank NCCL
    group: the exchange is a copy, the steps are the real ones)."""
    import torch.distributed as dist
    from linear_attention_07_b200.context_parallel import chunk_fwd_context_parallel
    kda = kda_lib
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        x = prefill_inputs(1, 800, 2, 128, 128, seed=1700, h0_std=0.1)
        d = {n: t.to(DEV) for n, t in x.items()}
        o, hT = chunk_fwd_context_parallel(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    o_ref, hT_ref = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
    check_out(o, o_ref, TOL_BF16)
    assert err_state(hT, hT_ref) <= TOL_BF16
