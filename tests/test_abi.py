"""The C ABI: library loads, exports what include/kda.h declares, and rejects
bad arguments on the host before any launch (no GPU needed)."""
import ctypes
import os
import re

import pytest

import linear_attention_07_b200 as kda
from linear_attention_07_b200 import build as kbuild

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "kda.h")


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load_library()


def declared_functions():
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_\w+)\s*\(", text)))


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("kda_chunk_fwd", "kda_chunk_fwd_f32", "kda_decode_step", "kda_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(kda.EXPORTED) >= set(declared_functions())


def test_status_strings(lib):
    assert kda.status_string(0) == "KDA_OK"
    assert kda.status_string(-1) == "KDA_ERR_INVALID_ARG"
    assert kda.status_string(-2) == "KDA_ERR_UNSUPPORTED"
    assert kda.status_string(-3) == "KDA_ERR_CUDA"
    assert kda.status_string(12345) == "KDA_ERR_UNKNOWN"
    assert lib.kda_version() >> 16 == 1


# Fake, never-dereferenced addresses: every call below fails a host check
# first, so nothing is launched and no address is touched.
A = ctypes.c_void_p(0x10000)
A2 = ctypes.c_void_p(0x20000)
MIS = ctypes.c_void_p(0x10008)   # 8-byte aligned only
NUL = None


def prefill(lib, fn, q=A, k=A, v=A, g=A, beta=A2, h0=NUL, o=A, hT=NUL,
            B=1, T=16, H=2, dk=128, dv=128):
    return getattr(lib, fn)(q, k, v, g, beta, h0, o, hT, B, T, H, dk, dv, None)


@pytest.mark.parametrize("fn", ["kda_chunk_fwd", "kda_chunk_fwd_f32"])
def test_prefill_argument_errors(lib, fn):
    n0 = lib.kda_launch_count()
    assert prefill(lib, fn, q=NUL) == kda.KDA_ERR_INVALID_ARG
    assert prefill(lib, fn, o=NUL) == kda.KDA_ERR_INVALID_ARG
    assert prefill(lib, fn, beta=NUL) == kda.KDA_ERR_INVALID_ARG
    assert prefill(lib, fn, k=MIS) == kda.KDA_ERR_INVALID_ARG
    assert prefill(lib, fn, h0=MIS) == kda.KDA_ERR_INVALID_ARG
    assert prefill(lib, fn, hT=MIS) == kda.KDA_ERR_INVALID_ARG
    assert prefill(lib, fn, B=-1) == kda.KDA_ERR_INVALID_ARG
    assert prefill(lib, fn, T=-5) == kda.KDA_ERR_INVALID_ARG
    assert prefill(lib, fn, dk=0) == kda.KDA_ERR_INVALID_ARG
    assert prefill(lib, fn, dk=96) == kda.KDA_ERR_UNSUPPORTED
    assert prefill(lib, fn, dv=256) == kda.KDA_ERR_UNSUPPORTED
    assert prefill(lib, fn, H=70000) == kda.KDA_ERR_UNSUPPORTED
    assert prefill(lib, fn, B=1 << 30, T=1 << 30, H=1 << 10) == kda.KDA_ERR_INVALID_ARG
    # nothing to do: returns OK without a launch
    assert prefill(lib, fn, B=0) == kda.KDA_OK
    assert prefill(lib, fn, H=0) == kda.KDA_OK
    assert prefill(lib, fn, T=0, q=NUL, k=NUL, v=NUL, g=NUL, beta=NUL, o=NUL) == kda.KDA_OK
    assert lib.kda_launch_count() == n0


def test_states_argument_errors(lib):
    """kda_chunk_fwd_states: the block length and the states buffer are checked
    on the host; nothing is launched on a bad argument."""
    n0 = lib.kda_launch_count()
    f = lib.kda_chunk_fwd_states
    args = lambda states, every, T=64: (A, A, A, A, A2, NUL, A, NUL, states, every, 1, T, 2, 128, 128, None)
    assert f(*args(A, 0)) == kda.KDA_ERR_INVALID_ARG          # no block length
    assert f(*args(A, 48)) == kda.KDA_ERR_INVALID_ARG         # not a multiple of 32
    assert f(*args(A, -32)) == kda.KDA_ERR_INVALID_ARG
    assert f(*args(NUL, 32)) == kda.KDA_ERR_INVALID_ARG       # two states to write, no buffer
    assert f(*args(MIS, 32)) == kda.KDA_ERR_INVALID_ARG       # misaligned buffer
    assert f(*args(A, 32, T=64)[:1] + (NUL,) + args(A, 32)[2:]) == kda.KDA_ERR_INVALID_ARG   # k missing
    assert lib.kda_launch_count() == n0


def test_raw_entry_points_argument_errors(lib):
    """The fused-prologue entry points check their arguments like the plain
    ones; nothing is launched."""
    n0 = lib.kda_launch_count()
    assert prefill(lib, "kda_chunk_fwd_raw", q=NUL) == kda.KDA_ERR_INVALID_ARG
    assert prefill(lib, "kda_chunk_fwd_raw", g=MIS) == kda.KDA_ERR_INVALID_ARG
    assert prefill(lib, "kda_chunk_fwd_raw", dk=64, dv=64) == kda.KDA_ERR_UNSUPPORTED
    assert prefill(lib, "kda_chunk_fwd_raw", B=0) == kda.KDA_OK
    dec = lib.kda_decode_step_raw
    assert dec(A, A, A, A, A2, A, A, 4, 2, 96, 128, None) == kda.KDA_ERR_UNSUPPORTED
    assert dec(A, A, A, NUL, A2, A, A, 4, 2, 128, 128, None) == kda.KDA_ERR_INVALID_ARG
    assert dec(A, A, A, A, A2, A, A, 0, 2, 128, 128, None) == kda.KDA_OK
    assert lib.kda_launch_count() == n0


def test_joining_entry_points_argument_errors(lib):
    """kda_chunk_transition and kda_state_chain: host checks, no launch."""
    n0 = lib.kda_launch_count()
    tr = lib.kda_chunk_transition
    assert tr(A, A, A, A2, NUL, 1, 16, 2, 128, None) == kda.KDA_ERR_INVALID_ARG     # no M
    assert tr(A, A, A, A2, MIS, 1, 16, 2, 128, None) == kda.KDA_ERR_INVALID_ARG     # misaligned M
    assert tr(NUL, A, A, A2, A, 1, 16, 2, 128, None) == kda.KDA_ERR_INVALID_ARG
    assert tr(A, A, A, A2, A, 1, 16, 2, 64, None) == kda.KDA_ERR_UNSUPPORTED
    assert tr(A, A, A, A2, A, 0, 16, 2, 128, None) == kda.KDA_OK                    # nothing to do
    ch = lib.kda_state_chain
    assert ch(NUL, A, NUL, A, NUL, 1, 3, 2, 128, 128, None) == kda.KDA_ERR_INVALID_ARG
    assert ch(A, A, NUL, MIS, NUL, 1, 3, 2, 128, 128, None) == kda.KDA_ERR_INVALID_ARG
    assert ch(A, A, MIS, A, NUL, 1, 3, 2, 128, 128, None) == kda.KDA_ERR_INVALID_ARG
    assert ch(A, A, NUL, A, NUL, 1, 3, 2, 64, 64, None) == kda.KDA_ERR_UNSUPPORTED
    assert ch(A, A, NUL, A, NUL, 1, -1, 2, 128, 128, None) == kda.KDA_ERR_INVALID_ARG
    assert ch(NUL, NUL, NUL, NUL, NUL, 1, 0, 2, 128, 128, None) == kda.KDA_OK      # no segments
    assert lib.kda_launch_count() == n0


def test_bf16_prefill_shape_support(lib):
    # the tensor-core path is specialised to d_k = d_v = 128
    assert prefill(lib, "kda_chunk_fwd", dk=64, dv=64) == kda.KDA_ERR_UNSUPPORTED
    assert prefill(lib, "kda_chunk_fwd", dk=128, dv=64) == kda.KDA_ERR_UNSUPPORTED


def test_decode_argument_errors(lib):
    n0 = lib.kda_launch_count()

    def dec(q=A, k=A, v=A, g=A, beta=A2, state=A, o=A, N=4, H=2, dk=128, dv=128):
        return lib.kda_decode_step(q, k, v, g, beta, state, o, N, H, dk, dv, None)

    assert dec(state=NUL) == kda.KDA_ERR_INVALID_ARG
    assert dec(state=MIS) == kda.KDA_ERR_INVALID_ARG
    assert dec(o=NUL) == kda.KDA_ERR_INVALID_ARG
    assert dec(beta=ctypes.c_void_p(0x20001)) == kda.KDA_ERR_INVALID_ARG
    assert dec(N=-1) == kda.KDA_ERR_INVALID_ARG
    assert dec(dk=48) == kda.KDA_ERR_UNSUPPORTED
    assert dec(N=0) == kda.KDA_OK
    assert dec(H=0, q=NUL) == kda.KDA_OK
    assert lib.kda_launch_count() == n0


def test_backward_argument_errors(lib):
    """kda_chunk_bwd: host checks, no launch."""
    n0 = lib.kda_launch_count()

    def bwd(q=A, dO=A, dhT=NUL, dq=A, dk=A, dv=A, dg=A, dbeta=A2, dh0=A, B=1, T=64, H=2, d_k=128, d_v=128):
        return lib.kda_chunk_bwd(q, A, A, A, A2, NUL, dO, dhT, dq, dk, dv, dg, dbeta, dh0,
                                 B, T, H, d_k, d_v, None)

    assert bwd(q=NUL) == kda.KDA_ERR_INVALID_ARG
    assert bwd(dO=NUL) == kda.KDA_ERR_INVALID_ARG
    assert bwd(dq=NUL) == kda.KDA_ERR_INVALID_ARG
    assert bwd(dg=MIS) == kda.KDA_ERR_INVALID_ARG
    assert bwd(dbeta=NUL) == kda.KDA_ERR_INVALID_ARG
    assert bwd(dbeta=ctypes.c_void_p(0x20001)) == kda.KDA_ERR_INVALID_ARG
    assert bwd(dh0=MIS) == kda.KDA_ERR_INVALID_ARG
    assert bwd(dhT=MIS) == kda.KDA_ERR_INVALID_ARG
    assert bwd(T=-1) == kda.KDA_ERR_INVALID_ARG
    assert bwd(d_k=64, d_v=64) == kda.KDA_ERR_UNSUPPORTED
    assert bwd(B=0) == kda.KDA_OK
    assert bwd(T=0, dh0=NUL) == kda.KDA_OK                 # nothing to write
    raw = lib.kda_chunk_bwd_raw
    assert raw(A, A, A, A, A2, NUL, NUL, NUL, A, A, A, A, A2, A, 1, 64, 2, 128, 128, None) == kda.KDA_ERR_INVALID_ARG
    assert raw(A, A, A, A, A2, NUL, A, NUL, A, A, A, A, A2, A, 1, 64, 2, 64, 64, None) == kda.KDA_ERR_UNSUPPORTED
    assert raw(A, A, A, A, A2, NUL, A, NUL, A, A, A, A, A2, A, 0, 64, 2, 128, 128, None) == kda.KDA_OK
    assert lib.kda_launch_count() == n0


def test_verify_argument_errors(lib):
    """kda_verify_fwd: host checks, no launch."""
    n0 = lib.kda_launch_count()

    def ver(q=A, k=A, v=A, g=A, beta=A2, h0=NUL, o=A, states=A, N=3, K=8, H=2, dk=128, dv=128):
        return lib.kda_verify_fwd(q, k, v, g, beta, h0, o, states, N, K, H, dk, dv, None)

    assert ver(states=NUL) == kda.KDA_ERR_INVALID_ARG
    assert ver(states=MIS) == kda.KDA_ERR_INVALID_ARG
    assert ver(h0=MIS) == kda.KDA_ERR_INVALID_ARG
    assert ver(o=NUL) == kda.KDA_ERR_INVALID_ARG
    assert ver(beta=ctypes.c_void_p(0x20001)) == kda.KDA_ERR_INVALID_ARG
    assert ver(K=-1) == kda.KDA_ERR_INVALID_ARG
    assert ver(K=kda.VERIFY_MAX_TOKENS + 1) == kda.KDA_ERR_UNSUPPORTED
    assert ver(dk=96) == kda.KDA_ERR_UNSUPPORTED
    assert ver(K=0, q=NUL, states=NUL) == kda.KDA_OK
    assert ver(N=0) == kda.KDA_OK
    assert lib.kda_launch_count() == n0


def test_verify_max_tokens_matches_header(lib):
    with open(HEADER) as f:
        m = re.search(r"#define\s+KDA_VERIFY_MAX_TOKENS\s+(\d+)", f.read())
    assert m and int(m.group(1)) == kda.VERIFY_MAX_TOKENS


def test_prefill_path_query(lib):
    """kda_prefill_path launches nothing; without a GPU the SM count falls
    back to the B200's 148."""
    n0 = lib.kda_launch_count()
    assert lib.kda_prefill_path(-1, 16, 2) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_prefill_path(4, 65536, 32) == 0          # 128 heads: one SM per head
    assert lib.kda_prefill_path(1, 8192, 32) == 1           # 32 heads: clusters of four SMs
    assert lib.kda_prefill_path(1, 1 << 20, 2) == 2         # two heads, long: segment scan
    assert lib.kda_launch_count() == n0


def test_selftest_limit_checked_on_host(lib):
    n0 = lib.kda_launch_count()
    assert lib.kda_selftest_bounded_wait(0, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_selftest_bounded_wait(2_000_000_000, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_launch_count() == n0


def test_binding_requires_cuda_tensors(lib):
    """Every tensor-level wrapper refuses host tensors before any launch:
    the library takes device pointers only."""
    import torch
    n0 = lib.kda_launch_count()
    x = torch.zeros(1, 64, 1, 128, dtype=torch.bfloat16)
    b = torch.zeros(1, 64, 1, dtype=torch.bfloat16)
    xf = torch.zeros(1, 64, 1, 128)
    bf = torch.zeros(1, 64, 1)
    d = torch.zeros(2, 1, 128, dtype=torch.bfloat16)
    db = torch.zeros(2, 1, dtype=torch.bfloat16)
    st = torch.zeros(2, 1, 128, 128)
    M = torch.zeros(1, 2, 1, 128, 128)
    calls = [
        lambda: kda.chunk_fwd(x, x, x, x, b),
        lambda: kda.chunk_fwd_raw(x, x, x, x, b),
        lambda: kda.chunk_fwd_noalloc(x, x, x, x, b),
        lambda: kda.chunk_fwd_states(x, x, x, x, b, state_every=32),
        lambda: kda.chunk_transition(x, x, x, b),
        lambda: kda.state_chain(M, M),
        lambda: kda.chunk_fwd_f32(xf, xf, xf, xf, bf),
        lambda: kda.decode_step(d, d, d, d, db, st),
        lambda: kda.decode_step_raw(d, d, d, d, db, st),
        lambda: kda.verify_fwd(x, x, x, x, b),
        lambda: kda.chunk_bwd(x, x, x, x, b, None, x),
        lambda: kda.chunk_bwd_raw(x, x, x, x, b, None, x),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="CUDA"):
            call()
    assert lib.kda_launch_count() == n0


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(kda.KdaLibraryError):
        import importlib
        mod = importlib.import_module("linear_attention_07_b200")
        saved = mod._lib
        mod._lib = None
        try:
            mod.load_library(str(tmp_path / "nope.so"))
        finally:
            mod._lib = saved
