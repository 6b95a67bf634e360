"""Independent checks that pin the KDA backward oracle.

The pages give the forward recurrence only (the gated delta rule of Kimi
Delta Attention: "T11E1: K3 tech report" transcript, the KDA turn; "Kimi K3
goes trillion-scale with sparse MoE efficiency" subtitles, cue 14); its
backward is the derivative of that recurrence, so every pin here ties the
oracle's reverse sweep to the forward recurrence by a route other than the
reverse sweep itself: finite differences of the (separately pinned) forward
oracle, reverse-mode autograd of a forward loop written here in the dense
product form, closed forms, an exact transpose identity and the split
identity of the backward chain.  ``chunked_bwd`` is the chunked (WY) form of
the same derivative, the algebra a tensor-core backward follows.

Every pin computes the gradients of L = sum(dO * o) + sum(dhT * hT).
"""
from __future__ import annotations

import numpy as np

from pins import _rand_problem, _rel

NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dh0")


def _cotangents(rng, n, T, dv, dk):
    return rng.standard_normal((n, T, dv)), rng.standard_normal((n, dk, dv))


def _grad_rel(got, want):
    return max(_rel(a, b) for a, b in zip(got, want))


def _loss(orc, x, dO, dhT):
    o, hT = orc.heads(*x)
    return float((o * dO).sum() + (hT * dhT).sum())


# -- 1. central finite differences of the forward oracle --------------------
def finite_differences(orc, seed=21, eps=1e-6):
    """Every input element of a small problem (with h0, both cotangents)."""
    rng = np.random.default_rng(seed)
    n, T, dk, dv = 2, 7, 4, 3
    x = list(_rand_problem(rng, T, dk, dv, n=n))
    dO, dhT = _cotangents(rng, n, T, dv, dk)
    grads = orc.heads_bwd(*x, dO=dO, dhT=dhT)
    # x = (q, k, v, g, beta, h0); gradient order (dq, dk, dv, dg, dbeta, dh0)
    err = 0.0
    for a, G in enumerate(grads):
        fd = np.zeros_like(x[a])
        for idx in np.ndindex(x[a].shape):
            xp = [y.copy() for y in x]
            xm = [y.copy() for y in x]
            xp[a][idx] += eps
            xm[a][idx] -= eps
            fd[idx] = (_loss(orc, xp, dO, dhT) - _loss(orc, xm, dO, dhT)) / (2 * eps)
        err = max(err, _rel(G, fd))
    return err


# -- 2. autograd of the dense product form, long enough to cross the oracle's
#       internal recompute segments ---------------------------------------
def _autograd_dense(q, k, v, g, beta, h0, dO, dhT):
    import torch
    ts = [torch.tensor(x, dtype=torch.float64, requires_grad=True)
          for x in (q, k, v, g, beta, h0)]
    tq, tk, tv, tg, tb, th = ts
    T, dk = q.shape
    eye = torch.eye(dk, dtype=torch.float64)
    S = th
    loss = torch.zeros((), dtype=torch.float64)
    dO_t = torch.tensor(dO)
    for t in range(T):
        M = (eye - tb[t] * torch.outer(tk[t], tk[t])) @ torch.diag(torch.exp(tg[t]))
        S = M @ S + tb[t] * torch.outer(tk[t], tv[t])
        loss = loss + (S.T @ tq[t] * dO_t[t]).sum()
    loss = loss + (S * torch.tensor(dhT)).sum()
    loss.backward()
    return [x.grad.numpy() for x in ts]


def autograd_dense_form(orc, seed=22, lengths=(1, 63, 64, 65, 150)):
    rng = np.random.default_rng(seed)
    dk, dv = 5, 4
    err = 0.0
    for T in lengths:
        q, k, v, g, beta, h0 = _rand_problem(rng, T, dk, dv, n=2)
        dO, dhT = _cotangents(rng, 2, T, dv, dk)
        got = orc.heads_bwd(q, k, v, g, beta, h0, dO, dhT)
        for h in range(2):
            want = _autograd_dense(q[h], k[h], v[h], g[h], beta[h], h0[h], dO[h], dhT[h])
            err = max(err, _grad_rel([x[h] for x in got], want))
    return err


# -- 3. one token: closed forms in matrix form ------------------------------
def single_token_closed_form(orc, seed=23):
    """With G = q dO^T + dhT, Sd = Diag(exp g) h0 and w = G^T k:
    L = <G, Sd> + beta w.v - beta w.(Sd^T k), so
      dv = beta w,  dbeta = w.(v - Sd^T k),  dq = (Sd + k u^T) dO,
      dk = beta G v - beta (G Sd^T + Sd G^T) k,
      dSd = G - beta k w^T,  dh0 = Diag(exp g) dSd,  dg = rowsum(dSd * Sd)."""
    rng = np.random.default_rng(seed)
    n, dk, dv = 3, 6, 5
    q, k, v, g, beta, h0 = _rand_problem(rng, 1, dk, dv, n=n)
    dO, dhT = _cotangents(rng, n, 1, dv, dk)
    got = orc.heads_bwd(q, k, v, g, beta, h0, dO, dhT)
    err = 0.0
    for h in range(n):
        qq, kk, vv, b = q[h, 0], k[h, 0], v[h, 0], beta[h, 0]
        a = np.exp(g[h, 0])
        Sd = a[:, None] * h0[h]
        G = np.outer(qq, dO[h, 0]) + dhT[h]
        w = G.T @ kk
        u = b * (vv - Sd.T @ kk)
        dSd = G - b * np.outer(kk, w)
        want = [
            ((Sd + np.outer(kk, u)) @ dO[h, 0])[None],
            (b * G @ vv - b * (G @ Sd.T + Sd @ G.T) @ kk)[None],
            (b * w)[None],
            (dSd * Sd).sum(axis=1)[None],
            np.array([w @ (vv - Sd.T @ kk)]),
            a[:, None] * dSd,
        ]
        err = max(err, _grad_rel([x[h] for x in got], want))
    return err


# -- 4. beta = 0: pure decay of h0, closed forms ----------------------------
def beta_zero_closed_form(orc, seed=24):
    """beta = 0 leaves S_t = Diag(exp Gam_t) h0 (Gam_t the running sum of g).
    With Lam_t = dL/dS_t = sum_{s>=t} Diag(exp(Gam_s - Gam_t)) q_s dO_s^T
    + Diag(exp(Gam_T - Gam_t)) dhT:
      dq_t = S_t dO_t, dk = 0, dv = 0, dbeta_t = (Lam_t^T k_t).(v_t - S_t^T k_t),
      dg_t = sum_{s>=t} c_s with c_s[i] = exp Gam_s[i] (q_s[i] h0[i].dO_s
      + [s = T] h0[i].dhT[i]),
      dh0 = sum_t Diag(exp Gam_t) q_t dO_t^T + Diag(exp Gam_T) dhT."""
    rng = np.random.default_rng(seed)
    n, T, dk, dv = 2, 70, 6, 5
    q, k, v, g, beta, h0 = _rand_problem(rng, T, dk, dv, n=n)
    beta = np.zeros_like(beta)
    dO, dhT = _cotangents(rng, n, T, dv, dk)
    got = orc.heads_bwd(q, k, v, g, beta, h0, dO, dhT)
    err = 0.0
    for h in range(n):
        Gam = np.cumsum(g[h], axis=0)
        E = np.exp(Gam)                                   # [T, dk]
        S = E[:, :, None] * h0[h][None]                   # [T, dk, dv]
        dq = np.einsum("tij,tj->ti", S, dO[h])
        c = E * q[h] * (h0[h] @ dO[h].T).T                # [T, dk]
        c[-1] += E[-1] * (h0[h] * dhT[h]).sum(axis=1)
        dg = np.cumsum(c[::-1], axis=0)[::-1]
        dh0 = np.einsum("ti,tj->ij", E * q[h], dO[h]) + E[-1][:, None] * dhT[h]
        dbeta = np.zeros(T)
        for t in range(T):
            lam = (np.exp(Gam[t:] - Gam[t])[:, :, None]
                   * (q[h][t:, :, None] * dO[h][t:, None, :])).sum(axis=0)
            lam += np.exp(Gam[-1] - Gam[t])[:, None] * dhT[h]
            dbeta[t] = (lam.T @ k[h, t]) @ (v[h, t] - S[t].T @ k[h, t])
        want = [dq, np.zeros((T, dk)), np.zeros((T, dv)), dg, dbeta, dh0]
        for x, y in zip([x[h] for x in got], want):
            scale = max(float(np.max(np.abs(y))), 1.0)
            err = max(err, float(np.max(np.abs(x - y))) / scale)
    return err


# -- 5. the map (v, h0) -> (o, hT) is linear: its adjoint is its transpose --
def transpose_identity(orc, seed=25):
    """<dO, o(dv', dh0')> + <dhT, hT(dv', dh0')> = <dv, dv'> + <dh0, dh0'>
    for any direction (dv', dh0'), with q, k, g, beta fixed."""
    rng = np.random.default_rng(seed)
    n, T, dk, dv = 2, 90, 7, 6
    q, k, v, g, beta, h0 = _rand_problem(rng, T, dk, dv, n=n)
    dO, dhT = _cotangents(rng, n, T, dv, dk)
    _, _, gv, _, _, gh = orc.heads_bwd(q, k, v, g, beta, h0, dO, dhT)
    err = 0.0
    for _ in range(3):
        pv = rng.standard_normal(v.shape)
        ph = rng.standard_normal(h0.shape)
        o, hT = orc.heads(q, k, pv, g, beta, ph)
        lhs = (dO * o).sum(axis=(1, 2)) + (dhT * hT).sum(axis=(1, 2))
        rhs = (gv * pv).sum(axis=(1, 2)) + (gh * ph).sum(axis=(1, 2))
        scale = np.abs(dO * o).sum(axis=(1, 2)) + np.abs(gv * pv).sum(axis=(1, 2))
        err = max(err, float(np.max(np.abs(lhs - rhs) / scale)))
    return err


# -- 6. split: the state adjoint carries the backward across a cut ---------
def split_resume_bwd(orc, seed=26, T=150, cut=97):
    """Backward of [cut, T) from the forward state at `cut` gives dL/dS_cut;
    feeding that as dhT to the backward of [0, cut) reproduces the whole
    backward."""
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, h0 = _rand_problem(rng, T, 6, 5, n=2)
    dO, dhT = _cotangents(rng, 2, T, 5, 6)
    full = orc.heads_bwd(q, k, v, g, beta, h0, dO, dhT)
    A = lambda x: x[:, :cut]
    Bq = lambda x: x[:, cut:]
    _, h_cut = orc.heads(A(q), A(k), A(v), A(g), A(beta), h0, want_o=False)
    second = orc.heads_bwd(Bq(q), Bq(k), Bq(v), Bq(g), Bq(beta), h_cut, Bq(dO), dhT)
    first = orc.heads_bwd(A(q), A(k), A(v), A(g), A(beta), h0, A(dO), second[5])
    joined = [np.concatenate([a, b], axis=1) for a, b in zip(first[:5], second[:5])]
    joined.append(first[5])
    return _grad_rel(full, joined)


# -- 7. the library layout: [B, T, H, d] marshalling of the backward -------
def batch_layout_bwd(orc, seed=27):
    """bwd in the library layout against heads_bwd on each (b, h) slice."""
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 2, 5, 3, 4, 3
    q = rng.standard_normal((B, T, H, dk)); k = rng.standard_normal((B, T, H, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    g = -rng.uniform(0, 5, (B, T, H, dk))
    beta = rng.uniform(0.1, 0.9, (B, T, H))
    h0 = rng.standard_normal((B, H, dk, dv))
    dO = rng.standard_normal((B, T, H, dv))
    dhT = rng.standard_normal((B, H, dk, dv))
    got = orc.bwd(q, k, v, g, beta, h0, dO, dhT)
    err = 0.0
    for b in range(B):
        for h in range(H):
            one = orc.heads_bwd(q[b:b + 1, :, h], k[b:b + 1, :, h], v[b:b + 1, :, h],
                                g[b:b + 1, :, h], beta[b:b + 1, :, h], h0[b:b + 1, h],
                                dO[b:b + 1, :, h], dhT[b:b + 1, h])
            mine = [got[0][b, :, h], got[1][b, :, h], got[2][b, :, h], got[3][b, :, h],
                    got[4][b, :, h], got[5][b, h]]
            err = max(err, _grad_rel(mine, [x[0] for x in one]))
    return err


# -- 8. chunked (WY) form of the backward, fp64, any chunk size ------------
def chunked_bwd(q, k, v, g, beta, S0, dO, dhT, C):
    """One head: the derivative of the chunked forward taken chunk by chunk.

    Forward per chunk (start state S0; Gam the in-chunk running sum of g,
    gam = exp(Gam), gC = gam of the last token):
      Kt = K*gam, Qt = Q*gam, Kh = K/gam, Kb = K*gC/gam,
      A = diag(beta) strict_lower(Kt Kh^T), X = (I + A)^-1, Tm = X diag(beta),
      W = Tm Kt, U = Tm V - W S0, P = lower_incl(Qt Kh^T),
      O = Qt S0 + P U,  S_C = Diag(gC) S0 + Kb^T U.
    Backward per chunk, last chunk first, with dS = dL/dS_C:
      dU  = P^T dO + Kb dS
      dS0 = Diag(gC) dS - W^T (Kb dS) + (Qt - P W)^T dO     (the state chain)
    then the chunk-local gradients of Kt, Qt, Kh, Kb, V, beta and through
    them q, k, v, beta and g.  Returns (dq, dk, dv, dg, dbeta, dh0,
    chain_gap) where chain_gap is the largest difference between dS0 taken
    in the state-chain form above and dS0 taken term by term.
    """
    T, dk = q.shape
    dv = v.shape[1]
    starts = list(range(0, T, C))
    S = S0.copy()
    S_start = []
    for c0 in starts:                      # forward: the state at each chunk start
        S_start.append(S.copy())
        Q, K, V, G, Bt = (x[c0:c0 + C] for x in (q, k, v, g, beta))
        Gam = np.cumsum(G, axis=0)
        gam = np.exp(Gam)
        Kt, Kh = K * gam, K / gam
        Kb = K * np.exp(Gam[-1][None, :] - Gam)
        n = Q.shape[0]
        A = np.tril(Kt @ Kh.T, -1) * Bt[:, None]
        Tm = np.linalg.solve(np.eye(n) + A, np.diag(Bt))
        U = Tm @ (V - Kt @ S)
        S = np.exp(Gam[-1])[:, None] * S + Kb.T @ U
    dq = np.zeros_like(q); dk_ = np.zeros_like(k); dv_ = np.zeros_like(v)
    dg = np.zeros_like(g); dbeta = np.zeros_like(beta)
    dS = dhT.copy()
    gap = 0.0
    for c0, S0c in zip(reversed(starts), reversed(S_start)):
        sl = slice(c0, c0 + C)
        Q, K, V, G, Bt, dOc = q[sl], k[sl], v[sl], g[sl], beta[sl], dO[sl]
        n = Q.shape[0]
        Gam = np.cumsum(G, axis=0)
        gam = np.exp(Gam)
        gC = gam[-1]
        Kt, Qt, Kh = K * gam, Q * gam, K / gam
        Kb = K * (gC[None, :] / gam)
        low = np.tril(np.ones((n, n)), -1)
        incl = np.tril(np.ones((n, n)))
        Araw = Kt @ Kh.T
        X = np.linalg.inv(np.eye(n) + low * Araw * Bt[:, None])
        Tm = X * Bt[None, :]
        W = Tm @ Kt
        U = Tm @ V - W @ S0c
        P = incl * (Qt @ Kh.T)
        dU = P.T @ dOc + Kb @ dS
        dS0 = Qt.T @ dOc + gC[:, None] * dS - W.T @ dU
        chain = gC[:, None] * dS - W.T @ (Kb @ dS) + (Qt - P @ W).T @ dOc
        gap = max(gap, _rel(chain, dS0))
        dPm = incl * (dOc @ U.T)
        dQt = dOc @ S0c.T + dPm @ Kh
        dKh = dPm.T @ Qt
        dKb = U @ dS.T
        dW = -dU @ S0c.T
        dTm = dW @ Kt.T + dU @ V.T
        dKt = Tm.T @ dW
        dV = Tm.T @ dU
        dX = dTm * Bt[None, :]
        dB = (dTm * X).sum(axis=0)
        dA = -(X.T @ dX @ X.T) * low
        dB += (dA * Araw).sum(axis=1)
        dAr = dA * Bt[:, None]
        dKt += dAr @ Kh
        dKh += dAr.T @ Kt
        dk_[sl] = dKt * gam + dKh / gam + dKb * (gC[None, :] / gam)
        dq[sl] = dQt * gam
        dv_[sl] = dV
        dbeta[sl] = dB
        dGam = dKt * Kt - dKh * Kh + dQt * Qt - dKb * Kb
        dGam[-1] += (dKb * Kb).sum(axis=0) + (dS * S0c).sum(axis=1) * gC
        dg[sl] = np.cumsum(dGam[::-1], axis=0)[::-1]
        dS = dS0
    return dq, dk_, dv_, dg, dbeta, dS, gap


def chunked_bwd_form(orc, seed=28, T=77, chunks=(1, 2, 4, 8, 16, 32, 64)):
    rng = np.random.default_rng(seed)
    dk, dv = 12, 9
    q, k, v, g, beta, h0 = _rand_problem(rng, T, dk, dv, n=2)
    dO, dhT = _cotangents(rng, 2, T, dv, dk)
    got = orc.heads_bwd(q, k, v, g, beta, h0, dO, dhT)
    err = 0.0
    for C in chunks:
        for h in range(2):
            *mine, gap = chunked_bwd(q[h], k[h], v[h], g[h], beta[h], h0[h], dO[h], dhT[h], C)
            err = max(err, gap, _grad_rel([x[h] for x in got], mine))
    return err


ALL_PINS = {
    "finite_differences": (finite_differences, 1e-7),
    "autograd_dense_form": (autograd_dense_form, 1e-12),
    "single_token_closed_form": (single_token_closed_form, 1e-13),
    "beta_zero_closed_form": (beta_zero_closed_form, 1e-12),
    "transpose_identity": (transpose_identity, 1e-13),
    "split_resume_bwd": (split_resume_bwd, 1e-12),
    "batch_layout_bwd": (batch_layout_bwd, 1e-14),
    "chunked_bwd_form": (chunked_bwd_form, 1e-9),
}


# -- 9. the GPU backward's scheme: 16-token tile references, row/column roles --
def _tile_factors(Gam, tile):
    """Row factor a_r = exp(Gam_r - Gam_ref(r)) (<= 1), same-tile column factor
    b_i = exp(Gam_ref(i) - Gam_i) (<= e^{5 tile}), cross column factor
    c_i = exp(Gam_{tile-1} - Gam_i) for the first tile (<= 1); ref(r) is Gam
    just before r's tile."""
    n = Gam.shape[0]
    ref = np.zeros_like(Gam)
    for r in range(n):
        t0 = (r // tile) * tile
        if t0 > 0:
            ref[r] = Gam[t0 - 1]
    a = np.exp(Gam - ref)
    b = np.exp(ref - Gam)
    c = np.exp(Gam[min(tile, n) - 1][None, :] - Gam)
    return a, b, c


def _pairs(L, R, a, b, c, tile, incl):
    """G[r, i] = sum_ch L[r] R[i] exp(Gam_r - Gam_i) for i < r (or i <= r)."""
    n = L.shape[0]
    G = np.zeros((n, n), L.dtype)
    for r in range(n):
        for i in range(r + 1 if incl else r):
            f = b[i] if i // tile == r // tile else c[i]
            G[r, i] = np.sum(L[r] * a[r] * R[i] * f)
    return G


def _row_role(dG, R, a, b, c, tile):
    """out[r] = a_r * sum_i dG[r, i] R[i] f_i  (= sum_i dG[r, i] R[i] exp(Gam_r - Gam_i))."""
    n = dG.shape[0]
    out = np.zeros_like(R)
    for r in range(n):
        for i in range(n):
            if dG[r, i] != 0:
                out[r] += dG[r, i] * R[i] * (b[i] if i // tile == r // tile else c[i])
        out[r] *= a[r]
    return out


def _col_role(dG, L, a, b, c, tile):
    """out[i] = sum_r dG[r, i] L[r] exp(Gam_r - Gam_i)."""
    n = dG.shape[0]
    out = np.zeros_like(L)
    for i in range(n):
        same = np.zeros(L.shape[1], L.dtype)
        cross = np.zeros(L.shape[1], L.dtype)
        for r in range(n):
            if dG[r, i] != 0:
                if r // tile == i // tile:
                    same += dG[r, i] * L[r] * a[r]
                else:
                    cross += dG[r, i] * L[r] * a[r]
        out[i] = same * b[i] + cross * c[i]
    return out


def tiled_chunk_bwd(q, k, v, g, beta, h0, dO, dhT, C=32, tile=16, dtype=np.float64):
    """One head, in the order of the GPU backward: per-chunk operands (pair
    products with tile references, X = (I + A)^-1, W, U', Z = Qt - P W, Kb),
    the forward state chain, the reverse state chain, then the chunk-local
    gradients, whose decayed pair terms split into row and column roles
    (dk += row(dAr, K) + col(dAr, K) + col(dP, Q), dq += row(dP, K), and
    dGam += k row(dAr, K) + q row(dP, K) - k col(...)).  No factor 1/gam
    relative to the chunk start is ever formed.  Returns (dq, dk, dv, dg,
    dbeta, dh0)."""
    T = q.shape[0]
    n_ch = (T + C - 1) // C
    pad = n_ch * C - T
    P = lambda x: np.concatenate([x, np.zeros((pad,) + x.shape[1:])]).astype(dtype)
    q, k, v, g, beta, dO = (P(x) for x in (q, k, v, g, beta, dO))
    recs = []
    for ch in range(n_ch):
        sl = slice(ch * C, (ch + 1) * C)
        Q, K, V, G, Bt = q[sl], k[sl], v[sl], g[sl], beta[sl]
        Gam = np.cumsum(G, axis=0)
        a, b, c = _tile_factors(Gam, tile)
        Kt, Qt, Kb = K * np.exp(Gam), Q * np.exp(Gam), K * np.exp(Gam[-1][None, :] - Gam)
        Araw = _pairs(K, K, a, b, c, tile, incl=False)
        Praw = _pairs(Q, K, a, b, c, tile, incl=True)
        X = np.linalg.inv(np.eye(C, dtype=dtype) + Araw * Bt[:, None])
        Tm = X * Bt[None, :]
        W = Tm @ Kt
        recs.append(dict(Gam=Gam, a=a, b=b, c=c, Kt=Kt, Qt=Qt, Kb=Kb, Araw=Araw, P=Praw, X=X, Tm=Tm, W=W,
                         Up=Tm @ V, Z=Qt - Praw @ W, gC=np.exp(Gam[-1])))
    S = h0.astype(dtype)
    S0 = []
    for r in recs:                                    # forward chain
        S0.append(S)
        S = r["gC"][:, None] * S + r["Kb"].T @ (r["Up"] - r["W"] @ S)
    dS = dhT.astype(dtype)
    dS_end = [None] * n_ch
    for ch in reversed(range(n_ch)):                  # reverse chain
        r = recs[ch]
        dS_end[ch] = dS
        dS = r["gC"][:, None] * dS - r["W"].T @ (r["Kb"] @ dS) + r["Z"].T @ dO[ch * C:(ch + 1) * C]
    dh0 = dS
    dq, dk, dv, dg, db = (np.zeros_like(x) for x in (q, k, v, g, beta))
    for ch, r in enumerate(recs):                     # chunk-local gradients
        sl = slice(ch * C, (ch + 1) * C)
        Q, K, V, dOc, Bt = q[sl], k[sl], v[sl], dO[sl], beta[sl]
        a, b, c, X, Tm = r["a"], r["b"], r["c"], r["X"], r["Tm"]
        U = Tm @ V - r["W"] @ S0[ch]
        dU = r["P"].T @ dOc + r["Kb"] @ dS_end[ch]
        dP = np.tril(dOc @ U.T)
        dQt = dOc @ S0[ch].T
        dKb = U @ dS_end[ch].T
        dW = -dU @ S0[ch].T
        dTm = dW @ r["Kt"].T + dU @ V.T
        dKt = Tm.T @ dW
        dB = (dTm * X).sum(axis=0)
        dA = -(X.T @ (dTm * Bt[None, :]) @ X.T) * np.tril(np.ones((C, C)), -1)
        dB = dB + (dA * r["Araw"]).sum(axis=1)
        dAr = dA * Bt[:, None]
        rowK = _row_role(dAr, K, a, b, c, tile)
        rowQ = _row_role(dP, K, a, b, c, tile)
        colK = _col_role(dAr, K, a, b, c, tile) + _col_role(dP, Q, a, b, c, tile)
        gam, kbf = np.exp(r["Gam"]), np.exp(r["Gam"][-1][None, :] - r["Gam"])
        dk[sl] = dKt * gam + rowK + colK + dKb * kbf
        dq[sl] = dQt * gam + rowQ
        dv[sl] = Tm.T @ dU
        db[sl] = dB
        dGam = dKt * r["Kt"] + dQt * r["Qt"] - dKb * r["Kb"] + K * rowK + Q * rowQ - K * colK
        dGam[-1] += (dKb * r["Kb"]).sum(axis=0) + (dS_end[ch] * S0[ch]).sum(axis=1) * r["gC"]
        dg[sl] = np.cumsum(dGam[::-1], axis=0)[::-1]
    cut = lambda x: x[:T]
    return cut(dq), cut(dk), cut(dv), cut(dg), cut(db), dh0


def tiled_scheme_form(orc, seed=29, lengths=(1, 16, 31, 33, 70)):
    """The GPU backward's scheme against the oracle (fp64, decays down to the
    -5 floor so every tile reference matters)."""
    rng = np.random.default_rng(seed)
    dk, dv = 12, 9
    err = 0.0
    for T in lengths:
        q, k, v, g, beta, h0 = _rand_problem(rng, T, dk, dv, n=1)
        g = -5.0 * rng.uniform(0.0, 1.0, g.shape)
        dO, dhT = _cotangents(rng, 1, T, dv, dk)
        got = tiled_chunk_bwd(q[0], k[0], v[0], g[0], beta[0], h0[0], dO[0], dhT[0])
        want = orc.heads_bwd(q, k, v, g, beta, h0, dO, dhT)
        err = max(err, _grad_rel(got, [w[0] for w in want]))
    return err


ALL_PINS["tiled_scheme_form"] = (tiled_scheme_form, 1e-10)
