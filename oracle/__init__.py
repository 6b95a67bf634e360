"""KDA oracle: the fp64 token-by-token recurrence, for tests only.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package.  The
product library never does, and this package imports nothing from it.

The arithmetic lives in ``kda_oracle.c`` (plain C, fp64, one head per host
thread); this module only builds that file with gcc, loads it and marshals
arrays.  The recurrence it evaluates is

    S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T,
    o_t = S_t^T q_t,

the delta-rule recurrence with a channel-wise forget gate of Kimi Delta
Attention ("Kimi K3 goes trillion-scale with sparse MoE efficiency"
subtitles, cue 14; "T11E1: K3 tech report" transcript, the KDA turn).

Layouts follow the library: q, k, g are [B, T, H, dk]; v and o are
[B, T, H, dv]; beta is [B, T, H]; states are [B, H, dk, dv].

``kda_oracle_bwd.c`` (plain C, fp64) is the reverse-mode derivative of the
same recurrence: the gradients of sum(dO * o) + sum(dhT * hT) with respect
to q, k, v, g, beta and h0, by a token-by-token reverse sweep.  The pages
give no backward pass; its pins tie it to the forward recurrence (finite
differences, autograd of a dense-product forward, closed forms).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "kda_oracle.c")
SOURCE_BWD = os.path.join(_HERE, "kda_oracle_bwd.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_LIB_BWD_PATH = os.path.join(_HERE, "libkda_oracle_bwd.so")
_default = None


def compile_c(src: str, out: str) -> str:
    """gcc -O2 a C file of the oracle into a shared library at `out`."""
    tmp = out + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
           "-o", tmp, src, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _build_one(src: str, out: str, force: bool) -> str:
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    return compile_c(src, out)


def build(force: bool = False) -> str:
    """Compile kda_oracle.c and kda_oracle_bwd.c into shared libraries
    beside them (each only if stale).  Returns the forward library's path."""
    _build_one(SOURCE_BWD, _LIB_BWD_PATH, force)
    return _build_one(SOURCE, _LIB_PATH, force)


def _f64(x):
    """Any array-like (numpy, torch of any float dtype) -> contiguous float64."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor, possibly bf16 and/or on a device
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


class Oracle:
    """A loaded build of the oracle's C files (the default ones, or a test's
    deliberately altered copy).  `bwd_lib_path` is the backward file's
    library; without it only the forward functions work."""

    def __init__(self, lib_path: str, bwd_lib_path: str | None = None):
        lib = ctypes.CDLL(lib_path)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.kda_oracle_heads.argtypes = [
            ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
            dp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int]
        lib.kda_oracle_heads.restype = ctypes.c_int
        lib.kda_oracle_num_cores.argtypes = []
        lib.kda_oracle_num_cores.restype = ctypes.c_int
        self.lib = lib
        self.bwd_lib = None
        if bwd_lib_path is not None:
            bl = ctypes.CDLL(bwd_lib_path)
            bl.kda_oracle_heads_bwd.argtypes = (
                [ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int]
                + [dp] * 14 + [ctypes.c_int])
            bl.kda_oracle_heads_bwd.restype = ctypes.c_int
            self.bwd_lib = bl

    def num_cores(self) -> int:
        return int(self.lib.kda_oracle_num_cores())

    def heads(self, q, k, v, g, beta, h0=None, want_o=True, n_threads=0):
        """n independent heads stacked on axis 0.

        q, k, g: [n, T, dk]; v: [n, T, dv]; beta: [n, T]; h0: [n, dk, dv]
        or None.  Returns (o [n, T, dv] or None, hT [n, dk, dv]) in float64.
        """
        q, k, v, g, beta, h0 = map(_f64, (q, k, v, g, beta, h0))
        n, T, dk = q.shape
        dv = v.shape[2]
        assert k.shape == (n, T, dk) and g.shape == (n, T, dk)
        assert v.shape == (n, T, dv) and beta.shape == (n, T)
        if h0 is not None:
            assert h0.shape == (n, dk, dv)
        o = np.empty((n, T, dv), np.float64) if want_o else None
        hT = np.empty((n, dk, dv), np.float64)
        rc = self.lib.kda_oracle_heads(n, T, dk, dv, _ptr(q), _ptr(k), _ptr(v),
                                       _ptr(g), _ptr(beta), _ptr(h0), _ptr(o),
                                       _ptr(hT), int(n_threads))
        if rc != 0:
            raise RuntimeError("kda oracle failed with code %d" % rc)
        return o, hT

    def fwd(self, q, k, v, g, beta, h0=None, want_o=True, n_threads=0):
        """Whole-batch prefill in the library layout.

        q, k, g: [B, T, H, dk]; v: [B, T, H, dv]; beta: [B, T, H];
        h0: [B, H, dk, dv] or None (zero state).
        Returns (o [B, T, H, dv] or None, hT [B, H, dk, dv]) in float64.
        """
        q, k, v, g, beta, h0 = map(_f64, (q, k, v, g, beta, h0))
        B, T, H, dk = q.shape
        dv = v.shape[3]

        def per_head(x):
            return np.ascontiguousarray(
                x.transpose(0, 2, 1, 3).reshape(B * H, T, x.shape[3]))

        o, hT = self.heads(
            per_head(q), per_head(k), per_head(v), per_head(g),
            np.ascontiguousarray(beta.transpose(0, 2, 1).reshape(B * H, T)),
            None if h0 is None else h0.reshape(B * H, dk, dv),
            want_o=want_o, n_threads=n_threads)
        if o is not None:
            o = o.reshape(B, H, T, dv).transpose(0, 2, 1, 3)
        return o, hT.reshape(B, H, dk, dv)

    def heads_bwd(self, q, k, v, g, beta, h0=None, dO=None, dhT=None, n_threads=0):
        """Gradients of L = sum(dO * o) + sum(dhT * hT) for n stacked heads
        (layouts as in `heads`; dO [n, T, dv] and dhT [n, dk, dv] may each be
        None, meaning zero).  Returns (dq, dk, dv, dg, dbeta, dh0) in float64
        with the shapes of q, k, v, g, beta and [n, dk, dv]."""
        if self.bwd_lib is None:
            raise RuntimeError("this oracle build has no backward library")
        q, k, v, g, beta, h0, dO, dhT = map(_f64, (q, k, v, g, beta, h0, dO, dhT))
        n, T, dk = q.shape
        dv = v.shape[2]
        assert k.shape == (n, T, dk) and g.shape == (n, T, dk)
        assert v.shape == (n, T, dv) and beta.shape == (n, T)
        for x, shp in ((h0, (n, dk, dv)), (dO, (n, T, dv)), (dhT, (n, dk, dv))):
            if x is not None:
                assert x.shape == shp
        dq = np.empty_like(q); dk_ = np.empty_like(k); dv_ = np.empty_like(v)
        dg = np.empty_like(g); dbeta = np.empty_like(beta)
        dh0 = np.empty((n, dk, dv), np.float64)
        rc = self.bwd_lib.kda_oracle_heads_bwd(
            n, T, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
            _ptr(h0), _ptr(dO), _ptr(dhT), _ptr(dq), _ptr(dk_), _ptr(dv_),
            _ptr(dg), _ptr(dbeta), _ptr(dh0), int(n_threads))
        if rc != 0:
            raise RuntimeError("kda backward oracle failed with code %d" % rc)
        return dq, dk_, dv_, dg, dbeta, dh0

    def bwd(self, q, k, v, g, beta, h0=None, dO=None, dhT=None, n_threads=0):
        """Whole-batch backward in the library layout (q, k, g [B, T, H, dk];
        v, dO [B, T, H, dv]; beta [B, T, H]; h0, dhT [B, H, dk, dv]).
        Returns (dq, dk, dv, dg, dbeta, dh0) in that layout, float64."""
        q, k, v, g, beta, h0, dO, dhT = map(_f64, (q, k, v, g, beta, h0, dO, dhT))
        B, T, H, dk = q.shape
        dv = v.shape[3]

        def per_head(x):
            if x is None:
                return None
            return np.ascontiguousarray(
                x.transpose(0, 2, 1, 3).reshape(B * H, T, x.shape[3]))

        def back(x):
            return x.reshape(B, H, T, x.shape[2]).transpose(0, 2, 1, 3)

        dq, dk_, dv_, dg, dbeta, dh0 = self.heads_bwd(
            per_head(q), per_head(k), per_head(v), per_head(g),
            np.ascontiguousarray(beta.transpose(0, 2, 1).reshape(B * H, T)),
            None if h0 is None else h0.reshape(B * H, dk, dv),
            per_head(dO),
            None if dhT is None else dhT.reshape(B * H, dk, dv),
            n_threads=n_threads)
        return (back(dq), back(dk_), back(dv_), back(dg),
                dbeta.reshape(B, H, T).transpose(0, 2, 1),
                dh0.reshape(B, H, dk, dv))

    def decode_step(self, q, k, v, g, beta, state, n_threads=0):
        """One token per request: the same recurrence applied once.

        q, k, g: [N, H, dk]; v: [N, H, dv]; beta: [N, H];
        state: [N, H, dk, dv].  Returns (o [N, H, dv], new state) in float64.
        """
        q, k, v, g, beta, state = map(_f64, (q, k, v, g, beta, state))
        N, H, dk = q.shape
        dv = v.shape[2]
        o, hT = self.heads(q.reshape(N * H, 1, dk), k.reshape(N * H, 1, dk),
                           v.reshape(N * H, 1, dv), g.reshape(N * H, 1, dk),
                           beta.reshape(N * H, 1), state.reshape(N * H, dk, dv),
                           n_threads=n_threads)
        return o.reshape(N, H, dv), hT.reshape(N, H, dk, dv)


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build(), _LIB_BWD_PATH)
    return _default


def num_cores() -> int:
    """Host cores the oracle's thread pool uses by default."""
    return default().num_cores()


def heads(*a, **kw):
    return default().heads(*a, **kw)


def fwd(*a, **kw):
    return default().fwd(*a, **kw)


def decode_step(*a, **kw):
    return default().decode_step(*a, **kw)


def heads_bwd(*a, **kw):
    return default().heads_bwd(*a, **kw)


def bwd(*a, **kw):
    return default().bwd(*a, **kw)


def prologue(q_raw, k_raw, z):
    """The fused prologue by its definition, in fp64: q and k L2-normalised
    over the key channels for every (token, head) (a zero vector stays zero),
    and the log-decay g = -5 sigmoid(z) (the lower-bounded sigmoid decay of
    the "Kimi K3 goes trillion-scale ..." subtitles, cue 14, with the -5 floor
    of the "T11E1: K3 tech report" transcript).  Returns (q, k, g) in fp64.
    """
    q, k, z = map(_f64, (q_raw, k_raw, z))

    def unit(x):
        n = np.sqrt((x * x).sum(axis=-1, keepdims=True))
        return np.where(n > 0.0, x / np.where(n > 0.0, n, 1.0), 0.0)

    with np.errstate(over="ignore"):
        g = -5.0 / (1.0 + np.exp(-z))
    return unit(q), unit(k), g


def fwd_raw(q_raw, k_raw, v, z, beta, h0=None, **kw):
    """fwd after the prologue: raw q, k and gate pre-activation z."""
    q, k, g = prologue(q_raw, k_raw, z)
    return fwd(q, k, v, g, beta, h0, **kw)


def decode_step_raw(q_raw, k_raw, v, z, beta, state, **kw):
    """decode_step after the prologue."""
    q, k, g = prologue(q_raw, k_raw, z)
    return decode_step(q, k, v, g, beta, state, **kw)


def prologue_bwd(q_raw, k_raw, z, dq, dk, dg):
    """Chain rule through the prologue, in fp64: given the gradients with
    respect to the normalised q, k and the log-decay g, return those with
    respect to q_raw, k_raw and z.  For x = r / |r|,
    dr = (dx - x (x . dx)) / |r| (zero where r = 0); for g = -5 sigmoid(z),
    dz = -5 sigmoid(z) (1 - sigmoid(z)) dg."""
    q_raw, k_raw, z, dq, dk, dg = map(_f64, (q_raw, k_raw, z, dq, dk, dg))

    def unit_bwd(r, dx):
        n = np.sqrt((r * r).sum(axis=-1, keepdims=True))
        safe = np.where(n > 0.0, n, 1.0)
        x = r / safe
        dr = (dx - x * (x * dx).sum(axis=-1, keepdims=True)) / safe
        return np.where(n > 0.0, dr, 0.0)

    with np.errstate(over="ignore"):
        s = 1.0 / (1.0 + np.exp(-z))
    return unit_bwd(q_raw, dq), unit_bwd(k_raw, dk), -5.0 * s * (1.0 - s) * dg


def bwd_raw(q_raw, k_raw, v, z, beta, h0=None, dO=None, dhT=None, **kw):
    """bwd through the prologue: gradients with respect to (q_raw, k_raw, v,
    z, beta, h0)."""
    q, k, g = prologue(q_raw, k_raw, z)
    dq, dk, dv, dg, dbeta, dh0 = bwd(q, k, v, g, beta, h0, dO, dhT, **kw)
    dq_raw, dk_raw, dz = prologue_bwd(q_raw, k_raw, z, dq, dk, dg)
    return dq_raw, dk_raw, dv, dz, dbeta, dh0
