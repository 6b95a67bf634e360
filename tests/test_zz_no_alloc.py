"""kda_chunk_fwd_noalloc: the prefill without any allocation in the library.

The segment scan (very few heads on a long sequence) needs workspace for
three fp32 state arrays per segment-head.  kda_chunk_fwd takes it from the
stream-ordered pool; kda_chunk_fwd_noalloc uses a fixed scratch array in the
library's device memory instead, checks its size before launching anything,
and otherwise computes the same thing bit for bit.
"""
import ctypes

import pytest
import torch

import oracle
import linear_attention_07_b200 as kda
from linear_attention_07_b200.inputs import prefill_inputs
from tolerance import TOL_BF16, check_out, err_state

DEV = torch.device("cuda", 0)
SCRATCH_BYTES = 3 * 148 * 128 * 128 * 4

A = ctypes.c_void_p(0x10000)
A2 = ctypes.c_void_p(0x20000)


@pytest.fixture(scope="module")
def lib():
    from linear_attention_07_b200 import build
    build.build()
    return kda.load_library()


def test_declared_and_exported(lib):
    assert hasattr(lib, "kda_chunk_fwd_noalloc")
    assert "kda_chunk_fwd_noalloc" in kda.EXPORTED
    assert kda.status_string(kda.KDA_ERR_NO_MEMORY) == "KDA_ERR_NO_MEMORY"


def test_argument_errors_before_any_launch(lib):
    """Host checks as in kda_chunk_fwd; fake addresses are never touched."""
    n0 = lib.kda_launch_count()
    f = lib.kda_chunk_fwd_noalloc
    assert f(None, A, A, A, A2, None, A, None, 1, 16, 2, 128, 128, None) == kda.KDA_ERR_INVALID_ARG
    assert f(A, A, A, A, A2, None, A, None, 1, 16, 2, 64, 64, None) == kda.KDA_ERR_UNSUPPORTED
    assert f(A, A, A, A, A2, None, A, None, 0, 16, 2, 128, 128, None) == kda.KDA_OK
    assert lib.kda_launch_count() == n0


def _pool_used_high():
    """High-water mark of the device's default (stream-ordered) memory pool,
    reset to zero; None when the runtime bindings are not importable."""
    try:
        from cuda.bindings import driver as dr
        from cuda.bindings import runtime as rt
    except Exception:
        return None
    err, pool = rt.cudaDeviceGetDefaultMemPool(0)
    assert err == rt.cudaError_t.cudaSuccess

    def read():
        err, v = rt.cudaMemPoolGetAttribute(pool, rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemHigh)
        assert err == rt.cudaError_t.cudaSuccess
        return int(v)

    def reset():
        (err,) = rt.cudaMemPoolSetAttribute(pool, rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemHigh,
                                            dr.cuuint64_t(0))
        assert err == rt.cudaError_t.cudaSuccess
    return read, reset


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,T", [(1, 1, 5000), (1, 2, 4173)])
def test_segment_scan_without_allocation(lib, B, H, T):
    """The segment scan through the fixed scratch: oracle parity, the same
    bits as kda_chunk_fwd, and no growth of the stream-ordered pool."""
    x = prefill_inputs(B, T, H, 128, 128, seed=950 + T, h0_std=0.1)
    d = {k: (None if t is None else t.to(DEV)) for k, t in x.items()}
    pool = _pool_used_high()
    torch.cuda.synchronize()
    if pool is not None:
        pool[1]()
    n0 = lib.kda_launch_count()
    o, hT = kda.chunk_fwd_noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    torch.cuda.synchronize()
    assert lib.kda_launch_count() - n0 == 4          # pass 1 (twice), segment chain, pass 3
    if pool is not None:
        assert pool[0]() == 0, "the no-allocation entry point used the memory pool"
    assert kda.device_status() == kda.KDA_OK
    o_ref, hT_ref = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
    eh = err_state(hT, hT_ref)
    check_out(o, o_ref, TOL_BF16)
    assert eh <= TOL_BF16, f"err_hT={eh:.3e}"
    o2, hT2 = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    torch.cuda.synchronize()
    if pool is not None:
        assert pool[0]() > 0, "the pool check does not see the allocating entry point"
    assert torch.equal(o, o2) and torch.equal(hT, hT2)


@pytest.mark.gpu
def test_scratch_too_small_is_reported_before_launch(lib, monkeypatch):
    """Forcing the segment scan on 128 heads needs 3 * 256 segment-heads of
    state: more than the fixed scratch.  KDA_ERR_NO_MEMORY, nothing written."""
    monkeypatch.setenv("KDA_PREFILL_VARIANT", "segmented")
    B, H, T = 4, 32, 512
    assert 3 * B * 2 * H * 128 * 128 * 4 > SCRATCH_BYTES
    x = prefill_inputs(B, T, H, 128, 128, seed=960)
    d = {k: (None if t is None else t.to(DEV)) for k, t in x.items()}
    o = torch.full((B, T, H, 128), 7.0, dtype=torch.bfloat16, device=DEV)
    n0 = lib.kda_launch_count()
    with pytest.raises(kda.KdaError) as ei:
        kda.chunk_fwd_noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], None, o=o)
    torch.cuda.synchronize()
    assert ei.value.status == kda.KDA_ERR_NO_MEMORY
    assert lib.kda_launch_count() == n0
    assert bool((o == 7.0).all())


@pytest.mark.gpu
def test_other_paths_unchanged(lib):
    """Paths without the segment scan take no scratch and give the same bits."""
    x = prefill_inputs(1, 1000, 32, 128, 128, seed=970, h0_std=0.1)
    d = {k: (None if t is None else t.to(DEV)) for k, t in x.items()}
    o, hT = kda.chunk_fwd_noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    o2, hT2 = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(hT, hT2)
    o_ref, hT_ref = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
    check_out(o, o_ref, TOL_BF16)
    assert err_state(hT, hT_ref) <= TOL_BF16
