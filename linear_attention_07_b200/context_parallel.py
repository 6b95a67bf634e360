"""KDA prefill of one long sequence split across the ranks of a process group
(context parallelism with one exchange step).

Rank r holds the r-th contiguous block of tokens of every sequence (the blocks
in rank order make up the sequence), with the same B and H on every rank;
block lengths may differ between ranks, since M and N do not depend on them.  The recurrence is affine in the state, so a block run from a
start state S ends at M S + N, with M the block's transition (the product of
its per-token (I - b k k^T) Diag(exp g)) and N the state it reaches from zero.
Each rank

  1. runs its block from zero (N_r) and computes its transition (M_r);
  2. all-gathers (M_r, N_r) over the group in one collective: 2 x 64 KB per
     (b, h) per rank;
  3. chains S_{p+1} = M_p S_p + N_p from h0 over the blocks (every rank the
     same small computation), which gives its own start state S_r and the
     final state hT;
  4. reruns its block from S_r, writing its part of o.

Steps 1, 3 and 4 run in the library's kernels (kda_chunk_fwd,
kda_chunk_transition, kda_state_chain); step 2 is a torch.distributed
all-gather (NCCL over NVLink between GPUs).  The same construction inside one
GPU is kda_chunk_fwd's segment scan.
"""
import torch
import torch.distributed as dist

import linear_attention_07_b200 as kda


class KernelOps:
    """The per-rank steps, on the library's kernels."""

    @staticmethod
    def block_fwd(q, k, v, g, beta, h0):
        return kda.chunk_fwd(q, k, v, g, beta, h0)

    @staticmethod
    def transition(q, k, g, beta):
        return kda.chunk_transition(q, k, g, beta)

    @staticmethod
    def state_chain(M, N, h0):
        return kda.state_chain(M, N, h0)


def chunk_fwd_context_parallel(q, k, v, g, beta, h0=None, *, group=None, ops=KernelOps):
    """This rank's block of one sequence batch: q, k, g [B, L, H, dk]; v
    [B, L, H, dv]; beta [B, L, H]; h0 [B, H, dk, dv] (the sequence's start
    state, the same on every rank) or None.  Returns (o of this block,
    hT of the whole sequence)."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    _, N = ops.block_fwd(q, k, v, g, beta, None)
    M = ops.transition(q, k, g, beta)
    if M.shape != N.shape:
        raise ValueError("the exchange step needs d_k == d_v, got M %s and N %s"
                         % (tuple(M.shape), tuple(N.shape)))
    MN = torch.stack([M, N])                       # [2, B, H, dk, dv]
    parts = [torch.empty_like(MN) for _ in range(world)]
    dist.all_gather(parts, MN, group=group)
    Ms = torch.stack([p[0] for p in parts], 1).contiguous()
    Ns = torch.stack([p[1] for p in parts], 1).contiguous()
    S_start, hT = ops.state_chain(Ms, Ns, h0)
    o, _ = ops.block_fwd(q, k, v, g, beta, S_start[:, rank].contiguous())
    return o, hT
