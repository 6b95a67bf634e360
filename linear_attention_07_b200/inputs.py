"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds no arithmetic of the method itself: it only draws random
tensors with the distributions of the workloads and rounds them to the
storage dtype.  Both sides of every parity check consume the exact tensors
produced here (the oracle widens the stored bf16/fp32 values to fp64).

Recipe (all draws from one seeded ``torch.Generator``, in this order):
  q, k  ~ N(0, 1) in fp32, each L2-normalised over d_k per (token, head),
         with no epsilon, then rounded to the storage dtype;
  v     ~ N(0, 1);
  beta  = sigmoid(N(0, 1))              (write strength in (0, 1));
  g     = -5 * sigmoid(N(0, 1))         (channel-wise log-decay in (-5, 0));
  h0    ~ N(0, sigma^2) fp32 when requested (sigma = 0.1, variance 0.01);
  pinned channels (optional): per (b, h) a seeded permutation of the d_k
         channels; the first round(frac * d_k) get g = -5 at every token and
         the next round(frac * d_k) get g = 0 at every token.
The -5 floor and the sigmoid shape of the decay follow the K3 pages ("T11E1:
K3 tech report" transcript, the log-decay-bound turn; "Kimi K3 goes
trillion-scale ..." subtitles, cue 14: a lower-bounded sigmoid decay).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                  # "prefill" or "decode"
    B: int                     # batch (prefill) or requests (decode)
    T: int                     # tokens per sequence (prefill) or decode steps
    H: int
    dk: int
    dv: int
    dtype: torch.dtype
    seed: int
    h0_std: float = 0.0        # 0 -> h0 = None (zero state)
    pin_frac: float = 0.0      # fraction of g channels pinned at -5 and at 0
    note: str = field(default="", compare=False)


# The five workloads: a tiny fp32 case, an 8K prefill, a batch of 64K
# pre-training sequences, a million-token prefill and a batched decode run;
# plus a profiling size for the one-SM-per-head prefill path (the 64K batch
# scaled down in T so that a full profiler capture stays at about 1 GB) and a
# million-token context with only two heads (the segment-scan path).
WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", "prefill", 1, 64, 2, 32, 32,
                          torch.float32, 1001,
                          note="B1 H2 T64 d32 fp32, h0=0, 16-token tiles"),
    "prefill_8k": Workload("prefill_8k", "prefill", 1, 8192, 32, 128, 128,
                           torch.bfloat16, 1002, h0_std=0.1,
                           note="B1 H32 T8192 d128 bf16, h0~N(0,0.01)"),
    "pretrain_64k": Workload("pretrain_64k", "prefill", 4, 65536, 32, 128, 128,
                             torch.bfloat16, 1003, pin_frac=0.1,
                             note="B4 H32 T65536 d128 bf16, 10%+10% of g "
                                  "channels pinned at -5 and 0, h0=0"),
    "prefill_1m": Workload("prefill_1m", "prefill", 1, 1048576, 32, 128, 128,
                           torch.bfloat16, 1004,
                           note="B1 H32 T1048576 d128 bf16, h0=0"),
    "pretrain_8k_b4": Workload("pretrain_8k_b4", "prefill", 4, 8192, 32, 128, 128,
                               torch.bfloat16, 1006, pin_frac=0.1,
                               note="B4 H32 T8192 d128 bf16, 10%+10% of g channels "
                                    "pinned at -5 and 0, h0=0 (profiling size)"),
    "prefill_1m_h2": Workload("prefill_1m_h2", "prefill", 1, 1048576, 2, 128, 128,
                              torch.bfloat16, 1007,
                              note="B1 H2 T1048576 d128 bf16, h0=0 (few heads, long "
                                   "context: the segment-scan path)"),
    "decode_256": Workload("decode_256", "decode", 256, 1000, 32, 128, 128,
                           torch.bfloat16, 1005, h0_std=0.1,
                           note="256 requests x H32 d128, fp32 state "
                                "~N(0,0.01), 1000 single-token steps"),
}


def _normalised(shape, gen, device):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    x = x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)
    return x


def prefill_inputs(B: int, T: int, H: int, dk: int, dv: int, *, seed: int,
                   dtype: torch.dtype = torch.bfloat16, device="cpu",
                   h0_std: float = 0.0, pin_frac: float = 0.0):
    """Return dict(q, k, v, g, beta, h0) in the library layout.

    q, k, g: [B, T, H, dk]; v: [B, T, H, dv]; beta: [B, T, H] (all `dtype`);
    h0: [B, H, dk, dv] fp32, or None when h0_std == 0.
    """
    gen = torch.Generator(device=device).manual_seed(int(seed))
    q = _normalised((B, T, H, dk), gen, device).to(dtype)
    k = _normalised((B, T, H, dk), gen, device).to(dtype)
    v = torch.randn((B, T, H, dv), generator=gen, device=device,
                    dtype=torch.float32).to(dtype)
    beta = torch.sigmoid(torch.randn((B, T, H), generator=gen, device=device,
                                     dtype=torch.float32)).to(dtype)
    g = (-5.0 * torch.sigmoid(torch.randn((B, T, H, dk), generator=gen,
                                          device=device,
                                          dtype=torch.float32))).to(dtype)
    if pin_frac > 0.0:
        n_pin = int(round(pin_frac * dk))
        for b in range(B):
            for h in range(H):
                perm = torch.randperm(dk, generator=gen, device=device)
                g[b, :, h, perm[:n_pin]] = -5.0
                g[b, :, h, perm[n_pin:2 * n_pin]] = 0.0
    h0 = None
    if h0_std > 0.0:
        h0 = torch.randn((B, H, dk, dv), generator=gen, device=device,
                         dtype=torch.float32) * h0_std
    return dict(q=q, k=k, v=v, g=g, beta=beta, h0=h0)


def raw_inputs(shape_qk, shape_v, shape_beta, *, seed: int, device="cpu", zero_rows: int = 0):
    """Inputs for the fused prologue: q and k as drawn (N(0, 1), not
    normalised), the gate pre-activation z ~ N(0, 1) (the gate is
    g = -5 sigmoid(z)), v ~ N(0, 1) and beta = sigmoid(N(0, 1)), all bf16.
    q, k, z: shape_qk; v: shape_v; beta: shape_beta.  The first `zero_rows`
    entries along the second axis of q and k are zero vectors (the degenerate
    case of the normalisation)."""
    gen = torch.Generator(device=device).manual_seed(int(seed))
    f32 = dict(generator=gen, device=device, dtype=torch.float32)
    q = torch.randn(shape_qk, **f32)
    k = torch.randn(shape_qk, **f32)
    if zero_rows > 0:
        q[:, :zero_rows] = 0.0
        k[:, :zero_rows] = 0.0
    z = torch.randn(shape_qk, **f32)
    v = torch.randn(shape_v, **f32)
    beta = torch.sigmoid(torch.randn(shape_beta, **f32))
    bf = lambda t: t.to(torch.bfloat16)
    return dict(q=bf(q), k=bf(k), z=bf(z), v=bf(v), beta=bf(beta))


def decode_inputs(N: int, H: int, dk: int, dv: int, steps: int, *, seed: int,
                  dtype: torch.dtype = torch.bfloat16, device="cpu",
                  state_std: float = 0.1):
    """Per-step decode inputs stacked on a leading step axis.

    q, k, g: [steps, N, H, dk]; v: [steps, N, H, dv]; beta: [steps, N, H];
    state: [N, H, dk, dv] fp32 ~ N(0, state_std^2).
    """
    gen = torch.Generator(device=device).manual_seed(int(seed))
    state = torch.randn((N, H, dk, dv), generator=gen, device=device,
                        dtype=torch.float32) * state_std
    q = _normalised((steps, N, H, dk), gen, device).to(dtype)
    k = _normalised((steps, N, H, dk), gen, device).to(dtype)
    v = torch.randn((steps, N, H, dv), generator=gen, device=device,
                    dtype=torch.float32).to(dtype)
    beta = torch.sigmoid(torch.randn((steps, N, H), generator=gen,
                                     device=device,
                                     dtype=torch.float32)).to(dtype)
    g = (-5.0 * torch.sigmoid(torch.randn((steps, N, H, dk), generator=gen,
                                          device=device,
                                          dtype=torch.float32))).to(dtype)
    return dict(q=q, k=k, v=v, g=g, beta=beta, state=state)


def workload_inputs(w: Workload, device="cpu", B: Optional[int] = None,
                    T: Optional[int] = None):
    """Inputs of a named workload, optionally with a smaller B or T."""
    B = w.B if B is None else B
    T = w.T if T is None else T
    if w.kind == "decode":
        return decode_inputs(B, w.H, w.dk, w.dv, T, seed=w.seed, dtype=w.dtype,
                             device=device, state_std=w.h0_std)
    return prefill_inputs(B, T, w.H, w.dk, w.dv, seed=w.seed, dtype=w.dtype,
                          device=device, h0_std=w.h0_std, pin_frac=w.pin_frac)
