"""Independent checks that pin the KDA oracle to things other than itself.

Each function takes a loaded oracle (``oracle.Oracle``) and returns the
largest discrepancy it found against a value fixed by the definition of the
recurrence, by a hand-worked example, or by an independent formulation
written here in numpy.  The recurrence being pinned is the gated delta rule
of Kimi Delta Attention,

    S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T,
    o_t = S_t^T q_t,

("T11E1: K3 tech report" transcript, the KDA turn; "Kimi K3 goes
trillion-scale with sparse MoE efficiency" subtitles, cue 14).

The same functions are run against deliberately broken builds of the
oracle (``test_oracle_mutants.py``) to show that each plausible mistake is
caught by at least one of them.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _unit(rng, *shape):
    x = rng.standard_normal(shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_problem(rng, T, dk, dv, n=1, h0=True):
    q = _unit(rng, n, T, dk)
    k = _unit(rng, n, T, dk)
    v = rng.standard_normal((n, T, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((n, T))))
    g = -5.0 / (1.0 + np.exp(-rng.standard_normal((n, T, dk))))
    S0 = 0.3 * rng.standard_normal((n, dk, dv)) if h0 else None
    return q, k, v, g, beta, S0


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    scale = max(float(np.max(np.abs(b))), 1e-300)
    return float(np.max(np.abs(a - b))) / scale


# -- 1. one token, zero state: o = beta (q.k) v, hT = beta k v^T ------------
def single_token_zero_state(orc, seed=1):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, _ = _rand_problem(rng, 1, 16, 12, n=3, h0=False)
    o, hT = orc.heads(q, k, v, g, beta, None)
    err = 0.0
    for h in range(3):
        o_cf = beta[h, 0] * float(q[h, 0] @ k[h, 0]) * v[h, 0]
        hT_cf = beta[h, 0] * np.outer(k[h, 0], v[h, 0])
        err = max(err, _rel(o[h, 0], o_cf), _rel(hT[h], hT_cf))
    return err


# -- 2. one token, nonzero state: o = (D S0)^T q + beta (v - (D S0)^T k)(k.q)
def single_token_with_state(orc, seed=2):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, S0 = _rand_problem(rng, 1, 8, 5, n=2)
    o, hT = orc.heads(q, k, v, g, beta, S0)
    err = 0.0
    for h in range(2):
        DS = np.exp(g[h, 0])[:, None] * S0[h]
        u = beta[h, 0] * (v[h, 0] - DS.T @ k[h, 0])
        o_cf = DS.T @ q[h, 0] + u * float(k[h, 0] @ q[h, 0])
        hT_cf = DS + np.outer(k[h, 0], u)
        err = max(err, _rel(o[h, 0], o_cf), _rel(hT[h], hT_cf))
    return err


# -- 3. beta = 0: pure channel-wise decay of h0 -----------------------------
def beta_zero_pure_decay(orc, seed=3):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, S0 = _rand_problem(rng, 11, 6, 7, n=2)
    beta = np.zeros_like(beta)
    o, hT = orc.heads(q, k, v, g, beta, S0)
    err = 0.0
    for h in range(2):
        Gam = np.cumsum(g[h], axis=0)               # [T, dk]
        for t in range(11):
            St = np.exp(Gam[t])[:, None] * S0[h]
            err = max(err, _rel(o[h, t], St.T @ q[h, t]))
        err = max(err, _rel(hT[h], np.exp(Gam[-1])[:, None] * S0[h]))
    return err


# -- 4. g = 0: the plain delta rule, written as a prediction-error update ---
def g_zero_plain_delta_rule(orc, seed=4):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, S0 = _rand_problem(rng, 40, 10, 6, n=2)
    g = np.zeros_like(g)
    o, hT = orc.heads(q, k, v, g, beta, S0)
    err = 0.0
    for h in range(2):
        W = S0[h].T.copy()                           # W = S^T: maps keys to values
        for t in range(40):
            pred = W @ k[h, t]
            W = W + beta[h, t] * np.outer(v[h, t] - pred, k[h, t])
            err = max(err, _rel(o[h, t], W @ q[h, t]))
        err = max(err, _rel(hT[h], W.T))
    return err


# -- 5. dense d_k x d_k transition products (short sequences) --------------
def dense_product_form(orc, seed=5):
    rng = np.random.default_rng(seed)
    T, dk, dv = 16, 7, 5
    q, k, v, g, beta, S0 = _rand_problem(rng, T, dk, dv, n=2)
    o, hT = orc.heads(q, k, v, g, beta, S0)
    err = 0.0
    for h in range(2):
        M = [(np.eye(dk) - beta[h, t] * np.outer(k[h, t], k[h, t]))
             @ np.diag(np.exp(g[h, t])) for t in range(T)]
        for t in range(T):
            # S_t = M_t ... M_1 S0 + sum_{s<=t} M_t ... M_{s+1} beta_s k_s v_s^T
            prod = np.eye(dk)
            St = np.zeros((dk, dv))
            for s in range(t, -1, -1):
                St += prod @ (beta[h, s] * np.outer(k[h, s], v[h, s]))
                prod = prod @ M[s]
            St += prod @ S0[h]
            err = max(err, _rel(o[h, t], St.T @ q[h, t]))
            if t == T - 1:
                err = max(err, _rel(hT[h], St))
    return err


# -- 6. chunked (WY / UT-transform) formulation, fp64, any chunk size -------
def chunked_wy(q, k, v, g, beta, S0, C):
    """One head: q, k, g [T, dk]; v [T, dv]; beta [T]; S0 [dk, dv].

    Within a chunk, with Gam_r = sum_{i<=r} g_i (per channel) and
    gamma = exp(Gam):
      A = diag(beta) strictly_lower((K*gamma)(K/gamma)^T)
      Tm = (I + A)^-1 diag(beta)
      U = Tm (V - (K*gamma) S0)
      O = (Q*gamma) S0 + lower_incl((Q*gamma)(K/gamma)^T) U
      S = Diag(gamma_C) S0 + (K*gamma_C/gamma)^T U
    """
    T, dk = q.shape
    S = S0.copy()
    O = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        Q, K, V, G, Bt = (x[c0:c0 + C] for x in (q, k, v, g, beta))
        n = Q.shape[0]
        Gam = np.cumsum(G, axis=0)
        gam = np.exp(Gam)
        Kt, Qt, Kh = K * gam, Q * gam, K / gam
        Kb = K * np.exp(Gam[-1][None, :] - Gam)
        A = np.tril(Kt @ Kh.T, -1) * Bt[:, None]
        Tm = np.linalg.solve(np.eye(n) + A, np.diag(Bt))
        U = Tm @ (V - Kt @ S)
        O[c0:c0 + n] = Qt @ S + np.tril(Qt @ Kh.T) @ U
        S = np.exp(Gam[-1])[:, None] * S + Kb.T @ U
    return O, S


def chunked_form(orc, seed=6, T=77, chunks=(1, 2, 4, 8, 16, 32, 64)):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, S0 = _rand_problem(rng, T, 12, 9, n=2)
    o, hT = orc.heads(q, k, v, g, beta, S0)
    err = 0.0
    for C in chunks:
        for h in range(2):
            O, S = chunked_wy(q[h], k[h], v[h], g[h], beta[h], S0[h], C)
            err = max(err, _rel(o[h], O), _rel(hT[h], S))
    return err


# -- 7. associative memory: orthonormal keys, no forgetting, beta = 1 ------
def associative_recall(orc, seed=7):
    """Writing (e_j, v_j) with beta = 1 and g = 0 stores v_j exactly in row
    j; reading with q = e_j returns it; a second write to the same key
    replaces the first."""
    rng = np.random.default_rng(seed)
    dk, dv = 6, 4
    vals = rng.standard_normal((dk + 2, dv))
    keys = [np.eye(dk)[j] for j in range(dk)] + [np.eye(dk)[2], np.eye(dk)[4]]
    T = len(keys) + dk                      # writes, then read-only tokens
    q = np.zeros((1, T, dk)); k = np.zeros((1, T, dk)); v = np.zeros((1, T, dv))
    beta = np.zeros((1, T)); g = np.zeros((1, T, dk))
    for t, key in enumerate(keys):
        k[0, t] = key; v[0, t] = vals[t]; beta[0, t] = 1.0; q[0, t] = key
    for j in range(dk):                     # reads: beta = 0, k = 0
        q[0, len(keys) + j] = np.eye(dk)[j]
    o, hT = orc.heads(q, k, v, g, beta, None)
    expect_final = {j: vals[j] for j in range(dk)}
    expect_final[2] = vals[dk]
    expect_final[4] = vals[dk + 1]
    err = 0.0
    for t in range(len(keys)):              # each write reads back its value
        err = max(err, float(np.max(np.abs(o[0, t] - vals[t]))))
    for j in range(dk):
        err = max(err, float(np.max(np.abs(o[0, len(keys) + j] - expect_final[j]))))
        err = max(err, float(np.max(np.abs(hT[0, j] - expect_final[j]))))
    return err


# -- 8. linearity in (v, h0) jointly ---------------------------------------
def linearity(orc, seed=8):
    rng = np.random.default_rng(seed)
    q, k, v1, g, beta, h1 = _rand_problem(rng, 23, 9, 6)
    v2 = rng.standard_normal(v1.shape)
    h2 = rng.standard_normal(h1.shape)
    a = 0.7
    o1, s1 = orc.heads(q, k, v1, g, beta, h1)
    o2, s2 = orc.heads(q, k, v2, g, beta, h2)
    o3, s3 = orc.heads(q, k, a * v1 + v2, g, beta, a * h1 + h2)
    return max(_rel(o3, a * o1 + o2), _rel(s3, a * s1 + s2))


# -- 9. split and resume: run(T1) -> hT -> run(T2) equals run(T1 + T2) -----
def split_resume(orc, seed=9):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, S0 = _rand_problem(rng, 50, 8, 8)
    o, hT = orc.heads(q, k, v, g, beta, S0)
    oa, ha = orc.heads(q[:, :19], k[:, :19], v[:, :19], g[:, :19], beta[:, :19], S0)
    ob, hb = orc.heads(q[:, 19:], k[:, 19:], v[:, 19:], g[:, 19:], beta[:, 19:], ha)
    return max(_rel(o, np.concatenate([oa, ob], axis=1)), _rel(hT, hb))


# -- 10. the hand-worked example -------------------------------------------
def hand_worked(orc):
    with open(os.path.join(GOLDEN, "hand_worked_d2_t3.json")) as f:
        fx = json.load(f)
    ln2 = math.log(2.0)
    gv = {"0": 0.0, "-ln2": -ln2}
    toks = fx["tokens"]
    T = len(toks)
    q = np.array([[t["q"] for t in toks]], np.float64)
    k = np.array([[t["k"] for t in toks]], np.float64)
    v = np.array([[t["v"] for t in toks]], np.float64)
    beta = np.array([[t["beta"] for t in toks]], np.float64)
    g = np.array([[[gv[x] for x in t["g"]] for t in toks]], np.float64)
    h0 = np.array([fx["h0"]], np.float64)
    o, hT = orc.heads(q, k, v, g, beta, h0)
    assert o.shape == (1, T, 2)
    return max(float(np.max(np.abs(o[0] - np.array(fx["o"])))),
               float(np.max(np.abs(hT[0] - np.array(fx["hT"])))))


# -- 11. layout marshalling: [B, T, H, d] batch vs independent heads -------
def batch_layout(orc, seed=11):
    """Single-token closed form evaluated per (b, h) in the library layout,
    so a transposed or mis-strided batch axis shows up."""
    rng = np.random.default_rng(seed)
    B, H, dk, dv = 2, 3, 5, 4
    q = _unit(rng, B, 1, H, dk); k = _unit(rng, B, 1, H, dk)
    v = rng.standard_normal((B, 1, H, dv))
    beta = rng.uniform(0.1, 0.9, (B, 1, H))
    g = -rng.uniform(0, 5, (B, 1, H, dk))
    h0 = rng.standard_normal((B, H, dk, dv))
    o, hT = orc.fwd(q, k, v, g, beta, h0)
    err = 0.0
    for b in range(B):
        for h in range(H):
            DS = np.exp(g[b, 0, h])[:, None] * h0[b, h]
            u = beta[b, 0, h] * (v[b, 0, h] - DS.T @ k[b, 0, h])
            err = max(err, _rel(o[b, 0, h], DS.T @ q[b, 0, h] + u * float(k[b, 0, h] @ q[b, 0, h])))
            err = max(err, _rel(hT[b, h], DS + np.outer(k[b, 0, h], u)))
    return err


ALL_PINS = {
    "single_token_zero_state": (single_token_zero_state, 1e-14),
    "single_token_with_state": (single_token_with_state, 1e-13),
    "beta_zero_pure_decay": (beta_zero_pure_decay, 1e-13),
    "g_zero_plain_delta_rule": (g_zero_plain_delta_rule, 1e-12),
    "dense_product_form": (dense_product_form, 1e-12),
    "chunked_form": (chunked_form, 1e-10),
    "associative_recall": (associative_recall, 1e-14),
    "linearity": (linearity, 1e-12),
    "split_resume": (split_resume, 1e-13),
    "hand_worked": (hand_worked, 1e-14),
    "batch_layout": (batch_layout, 1e-13),
}
