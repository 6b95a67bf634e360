"""Kimi Delta Attention (KDA) prefill and decode on NVIDIA B200 (sm_100a).

Thin ctypes binding over ``libkda.so`` (the C ABI declared in
``include/kda.h``).  Every step of the computation runs in the library's
CUDA kernels; this module only checks tensors and passes pointers, sizes
and the current CUDA stream of the tensors' device, which it makes the
current device for the call.  PyTorch is used for device memory and streams.

Raw C functions are exposed under their C names (every name in
``EXPORTED``).  The tensor-level helpers wrap them: ``chunk_fwd``,
``chunk_fwd_raw`` (prologue fused), ``chunk_fwd_noalloc``,
``chunk_fwd_states`` (intermediate states), ``chunk_transition`` and
``state_chain`` (the pieces of a split sequence), ``chunk_fwd_f32``,
``decode_step``, ``decode_step_raw``, ``verify_fwd`` (several tokens
per request with the state after each) and ``chunk_bwd`` (the gradients).  They accept only contiguous CUDA
tensors of the documented dtypes and shapes.

If the library is missing or cannot be loaded, every call raises
``KdaLibraryError``: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda.so")

KDA_OK = 0
KDA_ERR_INVALID_ARG = -1
KDA_ERR_UNSUPPORTED = -2
KDA_ERR_CUDA = -3
KDA_ERR_TIMEOUT = -4
KDA_ERR_NO_MEMORY = -5

EXPORTED = ("kda_chunk_fwd", "kda_chunk_fwd_noalloc", "kda_chunk_fwd_states", "kda_chunk_fwd_f32",
            "kda_chunk_transition", "kda_state_chain", "kda_chunk_fwd_raw", "kda_decode_step",
            "kda_decode_step_raw", "kda_verify_fwd", "kda_chunk_bwd", "kda_chunk_bwd_raw",
            "kda_device_status", "kda_selftest_bounded_wait",
            "kda_status_string", "kda_launch_count", "kda_prefill_path", "kda_version")


class KdaLibraryError(RuntimeError):
    pass


class KdaError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__("%s failed: %s (%d)" % (fn, status_string(status), status))


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libkda.so (once) and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise KdaLibraryError(
            "libkda.so not found at %s; build it with "
            "`python -m linear_attention_07_b200.build`" % path)
    try:
        lib = ctypes.CDLL(path)
    except OSError as e:  # pragma: no cover - depends on the machine
        raise KdaLibraryError("cannot load %s: %s" % (path, e)) from e
    vp, fp, i = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int
    lib.kda_chunk_fwd.argtypes = [vp, vp, vp, vp, vp, fp, vp, fp, i, i, i, i, i, vp]
    lib.kda_chunk_fwd.restype = i
    lib.kda_chunk_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, fp, vp, fp, i, i, i, i, i, vp]
    lib.kda_chunk_fwd_noalloc.restype = i
    lib.kda_chunk_fwd_states.argtypes = [vp, vp, vp, vp, vp, fp, vp, fp, fp, i, i, i, i, i, i, vp]
    lib.kda_chunk_fwd_states.restype = i
    lib.kda_chunk_transition.argtypes = [vp, vp, vp, vp, fp, i, i, i, i, vp]
    lib.kda_chunk_transition.restype = i
    lib.kda_state_chain.argtypes = [fp, fp, fp, fp, fp, i, i, i, i, i, vp]
    lib.kda_state_chain.restype = i
    lib.kda_chunk_fwd_f32.argtypes = [fp, fp, fp, fp, fp, fp, fp, fp, i, i, i, i, i, vp]
    lib.kda_chunk_fwd_f32.restype = i
    lib.kda_decode_step.argtypes = [vp, vp, vp, vp, vp, fp, vp, i, i, i, i, vp]
    lib.kda_decode_step.restype = i
    lib.kda_chunk_fwd_raw.argtypes = [vp, vp, vp, vp, vp, fp, vp, fp, i, i, i, i, i, vp]
    lib.kda_chunk_fwd_raw.restype = i
    lib.kda_decode_step_raw.argtypes = [vp, vp, vp, vp, vp, fp, vp, i, i, i, i, vp]
    lib.kda_decode_step_raw.restype = i
    lib.kda_chunk_bwd.argtypes = [vp, vp, vp, vp, vp, fp, vp, fp, vp, vp, vp, vp, vp, fp,
                                  i, i, i, i, i, vp]
    lib.kda_chunk_bwd.restype = i
    lib.kda_chunk_bwd_raw.argtypes = lib.kda_chunk_bwd.argtypes
    lib.kda_chunk_bwd_raw.restype = i
    lib.kda_verify_fwd.argtypes = [vp, vp, vp, vp, vp, fp, vp, fp, i, i, i, i, i, vp]
    lib.kda_verify_fwd.restype = i
    lib.kda_device_status.argtypes = [vp]
    lib.kda_device_status.restype = i
    lib.kda_selftest_bounded_wait.argtypes = [ctypes.c_uint64, vp]
    lib.kda_selftest_bounded_wait.restype = i
    lib.kda_status_string.argtypes = [i]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_launch_count.argtypes = []
    lib.kda_launch_count.restype = ctypes.c_uint64
    lib.kda_prefill_path.argtypes = [i, i, i]
    lib.kda_prefill_path.restype = i
    lib.kda_version.argtypes = []
    lib.kda_version.restype = i
    _lib = lib
    return lib


def __getattr__(name):
    # raw C entry points under their C names, resolved on first use
    if name in EXPORTED:
        return getattr(load_library(), name)
    raise AttributeError(name)


def status_string(status: int) -> str:
    return load_library().kda_status_string(int(status)).decode()


def device_status(device=None) -> int:
    """KDA_OK or KDA_ERR_TIMEOUT (a bounded device wait expired since the
    last call); synchronises the current stream and clears the flag."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return int(load_library().kda_device_status(_stream(dev)))


PREFILL_PATHS = ("one SM per head", "cluster of four SMs per head", "segment scan")


def prefill_path(B: int, T: int, H: int) -> str:
    """The path a bf16 prefill of this shape takes on the current device."""
    p = int(load_library().kda_prefill_path(int(B), int(T), int(H)))
    if p < 0:
        raise KdaError("kda_prefill_path", p)
    return PREFILL_PATHS[p]


def launch_count() -> int:
    """Kernels launched by libkda.so so far in this process."""
    return int(load_library().kda_launch_count())


# ---------------------------------------------------------------- tensors --

def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _require_cuda(t, name="inputs"):
    if t.device.type != "cuda":
        raise ValueError("%s must be CUDA tensors, got %s" % (name, t.device))
    return t.device


def _check(t, name, dtype, shape, device):
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    if t.device != device:
        raise ValueError("%s must be on %s, got %s" % (name, device, t.device))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def _prefill(fn_name, dtype, q, k, v, g, beta, h0, o, hT, output_final_state):
    import torch
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev = _require_cuda(q)
    for name, t, shp in (("q", q, (B, T, H, dk)), ("k", k, (B, T, H, dk)),
                         ("g", g, (B, T, H, dk)), ("v", v, (B, T, H, dv)),
                         ("beta", beta, (B, T, H))):
        _check(t, name, dtype, shp, dev)
    if h0 is not None:
        _check(h0, "h0", torch.float32, (B, H, dk, dv), dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dtype, device=dev)
    _check(o, "o", dtype, (B, T, H, dv), dev)
    if hT is None and output_final_state:
        hT = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    if hT is not None:
        _check(hT, "hT", torch.float32, (B, H, dk, dv), dev)
    fn = getattr(load_library(), fn_name)
    with torch.cuda.device(dev):
        st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0), _ptr(o),
                _ptr(hT), B, T, H, dk, dv, _stream(dev))
    if st != KDA_OK:
        raise KdaError(fn_name, st)
    return o, hT


def chunk_fwd(q, k, v, g, beta, h0=None, *, o=None, hT=None, output_final_state=True):
    """KDA prefill, bf16 in/out, fp32 state (kda_chunk_fwd).

    q, k, g: [B, T, H, dk]; v: [B, T, H, dv]; beta: [B, T, H] (bf16, CUDA,
    contiguous); h0: [B, H, dk, dv] fp32 or None.  Returns (o, hT).
    hT may be passed as h0 to update a state in place.
    """
    import torch
    return _prefill("kda_chunk_fwd", torch.bfloat16, q, k, v, g, beta, h0, o,
                    hT, output_final_state)


def chunk_fwd_raw(q_raw, k_raw, v, z, beta, h0=None, *, o=None, hT=None, output_final_state=True):
    """chunk_fwd with the prologue fused in (kda_chunk_fwd_raw): q_raw, k_raw
    unnormalised, z the gate pre-activation (g = -5 sigmoid(z) in the kernel)."""
    import torch
    return _prefill("kda_chunk_fwd_raw", torch.bfloat16, q_raw, k_raw, v, z, beta, h0, o,
                    hT, output_final_state)


def chunk_fwd_noalloc(q, k, v, g, beta, h0=None, *, o=None, hT=None, output_final_state=True):
    """chunk_fwd without any allocation in the library (kda_chunk_fwd_noalloc):
    the segment-scan path uses the library's fixed device scratch."""
    import torch
    return _prefill("kda_chunk_fwd_noalloc", torch.bfloat16, q, k, v, g, beta, h0, o,
                    hT, output_final_state)


def chunk_fwd_states(q, k, v, g, beta, h0=None, *, state_every, o=None, hT=None, states=None):
    """chunk_fwd that also returns the fp32 state after every `state_every`
    tokens (kda_chunk_fwd_states): (o, hT, states), states [B, H, T //
    state_every, dk, dv]."""
    import torch
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    _require_cuda(q)
    n = T // state_every if state_every > 0 else 0
    if states is None:
        states = torch.empty((B, H, n, dk, dv), dtype=torch.float32, device=q.device)
    _check(states, "states", torch.float32, (B, H, n, dk, dv), q.device)
    if o is None:
        o = torch.empty_like(v)
    if hT is None:
        hT = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    for name, t, shp in (("q", q, (B, T, H, dk)), ("k", k, (B, T, H, dk)), ("g", g, (B, T, H, dk)),
                         ("v", v, (B, T, H, dv)), ("beta", beta, (B, T, H)), ("o", o, (B, T, H, dv))):
        _check(t, name, torch.bfloat16, shp, q.device)
    _check(hT, "hT", torch.float32, (B, H, dk, dv), q.device)
    if h0 is not None:
        _check(h0, "h0", torch.float32, (B, H, dk, dv), q.device)
    with torch.cuda.device(q.device):
        st = load_library().kda_chunk_fwd_states(
            _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0), _ptr(o), _ptr(hT),
            _ptr(states) if n > 0 else None, int(state_every), B, T, H, dk, dv,
            _stream(q.device))
    if st != KDA_OK:
        raise KdaError("kda_chunk_fwd_states", st)
    return o, hT, states


def chunk_transition(q, k, g, beta, *, M=None):
    """Transition M [B, H, dk, dk] (fp32) of each whole sequence
    (kda_chunk_transition): running it from S0 ends at M S0 + (its state from zero)."""
    import torch
    B, T, H, dk = q.shape
    dev = _require_cuda(q)
    for name, t, shp in (("q", q, (B, T, H, dk)), ("k", k, (B, T, H, dk)), ("g", g, (B, T, H, dk)),
                         ("beta", beta, (B, T, H))):
        _check(t, name, torch.bfloat16, shp, dev)
    if M is None:
        M = torch.empty((B, H, dk, dk), dtype=torch.float32, device=dev)
    _check(M, "M", torch.float32, (B, H, dk, dk), dev)
    with torch.cuda.device(dev):
        st = load_library().kda_chunk_transition(_ptr(q), _ptr(k), _ptr(g), _ptr(beta), _ptr(M),
                                                 B, T, H, dk, _stream(dev))
    if st != KDA_OK:
        raise KdaError("kda_chunk_transition", st)
    return M


def state_chain(M, N, h0=None, *, S_start=None, hT=None):
    """S_0 = h0, S_{p+1} = M_p S_p + N_p over P segments (kda_state_chain).
    M: [B, P, H, dk, dk]; N: [B, P, H, dk, dv]; h0: [B, H, dk, dv] or None.
    Returns (S_start [B, P, H, dk, dv], hT [B, H, dk, dv])."""
    import torch
    B, P, H, dk, dv = N.shape
    dev = _require_cuda(N)
    _check(M, "M", torch.float32, (B, P, H, dk, dk), dev)
    _check(N, "N", torch.float32, (B, P, H, dk, dv), dev)
    if h0 is not None:
        _check(h0, "h0", torch.float32, (B, H, dk, dv), dev)
    if S_start is None:
        S_start = torch.empty_like(N)
    if hT is None:
        hT = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    _check(S_start, "S_start", torch.float32, (B, P, H, dk, dv), dev)
    _check(hT, "hT", torch.float32, (B, H, dk, dv), dev)
    with torch.cuda.device(dev):
        st = load_library().kda_state_chain(_ptr(M), _ptr(N), _ptr(h0), _ptr(S_start), _ptr(hT),
                                            B, P, H, dk, dv, _stream(dev))
    if st != KDA_OK:
        raise KdaError("kda_state_chain", st)
    return S_start, hT


def chunk_fwd_f32(q, k, v, g, beta, h0=None, *, o=None, hT=None, output_final_state=True):
    """KDA prefill with fp32 inputs/outputs and fp32 arithmetic."""
    import torch
    return _prefill("kda_chunk_fwd_f32", torch.float32, q, k, v, g, beta, h0, o,
                    hT, output_final_state)


def _decode(fn_name, q, k, v, g, beta, state, o):
    import torch
    N, H, dk = q.shape
    dv = v.shape[-1]
    dev = _require_cuda(q)
    for name, t, shp in (("q", q, (N, H, dk)), ("k", k, (N, H, dk)),
                         ("g", g, (N, H, dk)), ("v", v, (N, H, dv)),
                         ("beta", beta, (N, H))):
        _check(t, name, torch.bfloat16, shp, dev)
    _check(state, "state", torch.float32, (N, H, dk, dv), dev)
    if o is None:
        o = torch.empty((N, H, dv), dtype=torch.bfloat16, device=dev)
    _check(o, "o", torch.bfloat16, (N, H, dv), dev)
    with torch.cuda.device(dev):
        st = getattr(load_library(), fn_name)(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                            _ptr(state), _ptr(o), N, H, dk, dv, _stream(dev))
    if st != KDA_OK:
        raise KdaError(fn_name, st)
    return o


def decode_step(q, k, v, g, beta, state, *, o=None):
    """One decode token per request; `state` [N, H, dk, dv] fp32 is updated
    in place.  q, k, g: [N, H, dk]; v: [N, H, dv]; beta: [N, H] (bf16).
    Returns o [N, H, dv] bf16."""
    return _decode("kda_decode_step", q, k, v, g, beta, state, o)


def decode_step_raw(q_raw, k_raw, v, z, beta, state, *, o=None):
    """decode_step with the prologue fused in (kda_decode_step_raw): q_raw,
    k_raw unnormalised, z the gate pre-activation."""
    return _decode("kda_decode_step_raw", q_raw, k_raw, v, z, beta, state, o)




VERIFY_MAX_TOKENS = 64


def verify_fwd(q, k, v, g, beta, h0=None, *, o=None, states=None):
    """K tokens per request from the start states h0, keeping the state after
    every token (kda_verify_fwd).  q, k, g: [N, K, H, dk]; v: [N, K, H, dv];
    beta: [N, K, H] (bf16); h0: [N, H, dk, dv] fp32 or None (read only).
    Returns (o [N, K, H, dv] bf16, states [N, K, H, dk, dv] fp32), with
    states[n, t] the state of request n after its token t + 1."""
    import torch
    N, K, H, dk = q.shape
    dv = v.shape[-1]
    dev = _require_cuda(q)
    for name, t, shp in (("q", q, (N, K, H, dk)), ("k", k, (N, K, H, dk)),
                         ("g", g, (N, K, H, dk)), ("v", v, (N, K, H, dv)),
                         ("beta", beta, (N, K, H))):
        _check(t, name, torch.bfloat16, shp, dev)
    if h0 is not None:
        _check(h0, "h0", torch.float32, (N, H, dk, dv), dev)
    if o is None:
        o = torch.empty((N, K, H, dv), dtype=torch.bfloat16, device=dev)
    if states is None:
        states = torch.empty((N, K, H, dk, dv), dtype=torch.float32, device=dev)
    _check(o, "o", torch.bfloat16, (N, K, H, dv), dev)
    _check(states, "states", torch.float32, (N, K, H, dk, dv), dev)
    with torch.cuda.device(dev):
        st = load_library().kda_verify_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                           _ptr(h0), _ptr(o), _ptr(states), N, K, H, dk, dv,
                                           _stream(dev))
    if st != KDA_OK:
        raise KdaError("kda_verify_fwd", st)
    return o, states


def _bwd(fn_name, q, k, v, g, beta, h0, dO, dhT, want_dh0):
    import torch
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev = _require_cuda(q)
    for name, t, shp in (("q", q, (B, T, H, dk)), ("k", k, (B, T, H, dk)),
                         ("g", g, (B, T, H, dk)), ("v", v, (B, T, H, dv)),
                         ("beta", beta, (B, T, H)), ("dO", dO, (B, T, H, dv))):
        _check(t, name, torch.bfloat16, shp, dev)
    for name, t in (("h0", h0), ("dhT", dhT)):
        if t is not None:
            _check(t, name, torch.float32, (B, H, dk, dv), dev)
    gq, gk, gg = (torch.empty((B, T, H, dk), dtype=torch.bfloat16, device=dev) for _ in range(3))
    gv = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device=dev)
    gb = torch.empty((B, T, H), dtype=torch.bfloat16, device=dev)
    gh = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev) if want_dh0 else None
    with torch.cuda.device(dev):
        st = getattr(load_library(), fn_name)(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                                              _ptr(dO), _ptr(dhT), _ptr(gq), _ptr(gk), _ptr(gv), _ptr(gg),
                                              _ptr(gb), _ptr(gh), B, T, H, dk, dv, _stream(dev))
    if st != KDA_OK:
        raise KdaError(fn_name, st)
    return gq, gk, gv, gg, gb, gh


def chunk_bwd(q, k, v, g, beta, h0, dO, dhT=None, *, want_dh0=True):
    """Gradients of chunk_fwd (kda_chunk_bwd): with L = sum(dO * o) +
    sum(dhT * hT), returns (dq, dk, dv, dg, dbeta, dh0); dq, dk, dg, dv,
    dbeta bf16 in the input layouts, dh0 [B, H, dk, dv] fp32 (None if
    want_dh0 is False).  dO: [B, T, H, dv] bf16; dhT: [B, H, dk, dv] fp32 or
    None; h0 as for chunk_fwd."""
    return _bwd("kda_chunk_bwd", q, k, v, g, beta, h0, dO, dhT, want_dh0)


def chunk_bwd_raw(q_raw, k_raw, v, z, beta, h0, dO, dhT=None, *, want_dh0=True):
    """Gradients of chunk_fwd_raw (kda_chunk_bwd_raw): (dq_raw, dk_raw, dv,
    dz, dbeta, dh0), the prologue and its chain rule inside the kernels."""
    return _bwd("kda_chunk_bwd_raw", q_raw, k_raw, v, z, beta, h0, dO, dhT, want_dh0)
