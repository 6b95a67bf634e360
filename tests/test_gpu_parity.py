"""GPU parity: libkda.so against the fp64 oracle on the same seeded inputs.

Every call goes through the C ABI (via the ctypes binding).  Tolerances:
fp32 entry point <= 1e-4, bf16 entry points <= 1e-2, with the metrics of
tests/tolerance.py (err_state for fp32 outputs, err_out for bf16 outputs).
"""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_07_b200 as kda
from linear_attention_07_b200.inputs import WORKLOADS, prefill_inputs, decode_inputs
from tolerance import TOL_BF16, TOL_F32, check_out, err_out, err_state

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from linear_attention_07_b200 import build
    build.build()
    kda.load_library()
    torch.cuda.init()


def to_dev(x):
    return {k: (None if t is None else t.to(DEV)) for k, t in x.items()}


def run_prefill(x, fn=kda.chunk_fwd):
    d = to_dev(x)
    o, hT = fn(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    torch.cuda.synchronize()
    return o, hT


def check_prefill(x, o, hT, tol, bf16_out=True):
    o_ref, hT_ref = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
    eh = err_state(hT, hT_ref)
    if bf16_out:
        eo = check_out(o, o_ref, tol)[2]
    else:
        eo = err_state(o, o_ref)
    assert eo <= tol and eh <= tol, f"err_o={eo:.3e} err_hT={eh:.3e} tol={tol:.0e}"
    return eo, eh


# ----------------------------------------------------------- fp32 path ----

def test_tiny_fp32_workload():
    w = WORKLOADS["tiny_fp32"]
    x = prefill_inputs(w.B, w.T, w.H, w.dk, w.dv, seed=w.seed, dtype=torch.float32)
    o, hT = run_prefill(x, kda.chunk_fwd_f32)
    check_prefill(x, o, hT, TOL_F32, bf16_out=False)


@pytest.mark.parametrize("dk,dv,T", [(32, 32, 1), (64, 128, 37), (128, 64, 100), (128, 128, 70)])
def test_fp32_shapes(dk, dv, T):
    x = prefill_inputs(2, T, 3, dk, dv, seed=dk + dv + T, dtype=torch.float32, h0_std=0.1)
    o, hT = run_prefill(x, kda.chunk_fwd_f32)
    check_prefill(x, o, hT, TOL_F32, bf16_out=False)


# ----------------------------------------------------------- bf16 path ----

@pytest.mark.parametrize("T", [1, 15, 16, 17, 64, 200, 1000])
def test_bf16_ragged_lengths(T):
    x = prefill_inputs(2, T, 4, 128, 128, seed=100 + T, h0_std=0.1)
    o, hT = run_prefill(x)
    check_prefill(x, o, hT, TOL_BF16)


def test_bf16_zero_h0_and_pinned_channels():
    x = prefill_inputs(1, 512, 4, 128, 128, seed=7, pin_frac=0.1)
    o, hT = run_prefill(x)
    check_prefill(x, o, hT, TOL_BF16)


@pytest.mark.parametrize("case", ["g_min", "g_zero", "beta_zero"])
def test_bf16_degenerate_gates(case):
    x = prefill_inputs(1, 160, 2, 128, 128, seed=11, h0_std=0.1)
    if case == "g_min":
        x["g"] = torch.full_like(x["g"], -5.0)
    elif case == "g_zero":
        x["g"] = torch.zeros_like(x["g"])
    else:
        x["beta"] = torch.zeros_like(x["beta"])
    o, hT = run_prefill(x)
    o_ref, hT_ref = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
    check_out(o, o_ref, TOL_BF16)
    assert err_state(hT, hT_ref) <= TOL_BF16


def test_bf16_t0_copies_state_and_inplace_update():
    x = prefill_inputs(1, 0, 2, 128, 128, seed=3, h0_std=0.1)
    d = to_dev(x)
    o, hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    torch.cuda.synchronize()
    assert o.shape[1] == 0 and torch.equal(hT, d["h0"])
    # hT == h0: in-place state update
    x = prefill_inputs(1, 48, 2, 128, 128, seed=4, h0_std=0.1)
    d = to_dev(x)
    S = d["h0"].clone()
    kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S, hT=S)
    torch.cuda.synchronize()
    _, hT_ref = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
    assert err_state(S, hT_ref) <= TOL_BF16


def test_bf16_guard_bands_untouched():
    x = prefill_inputs(1, 33, 3, 128, 128, seed=5, h0_std=0.1)
    d = to_dev(x)
    n_o = 33 * 3 * 128
    n_s = 3 * 128 * 128
    pad = 4096
    o_buf = torch.full((n_o + 2 * pad,), 12345.0, dtype=torch.bfloat16, device=DEV)
    s_buf = torch.full((n_s + 2 * pad,), float("nan"), dtype=torch.float32, device=DEV)
    o = o_buf[pad:pad + n_o].view(1, 33, 3, 128)
    hT = s_buf[pad:pad + n_s].view(1, 3, 128, 128)
    kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"], o=o, hT=hT)
    torch.cuda.synchronize()
    assert torch.all(o_buf[:pad] == 12345.0) and torch.all(o_buf[-pad:] == 12345.0)
    assert torch.all(torch.isnan(s_buf[:pad])) and torch.all(torch.isnan(s_buf[-pad:]))
    assert torch.isfinite(o).all() and torch.isfinite(hT).all()


def test_bf16_split_resume_and_determinism():
    x = prefill_inputs(1, 300, 4, 128, 128, seed=21, h0_std=0.1)
    d = to_dev(x)
    o_a, h_a = kda.chunk_fwd(*(d[k][:, :123] for k in ("q", "k", "v", "g", "beta")), d["h0"])
    o_b, h_b = kda.chunk_fwd(*(d[k][:, 123:].contiguous() for k in ("q", "k", "v", "g", "beta")), h_a)
    o1, h1 = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    o2, h2 = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(h1, h2), "not deterministic"
    o_ref, h_ref = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
    check_out(torch.cat([o_a, o_b], 1), o_ref, TOL_BF16)
    assert err_state(h_b, h_ref) <= TOL_BF16


@pytest.mark.parametrize("variant", ["fused", "cluster"])
@pytest.mark.parametrize("T", [1, 31, 33, 95, 300])
def test_bf16_both_prefill_variants(monkeypatch, variant, T):
    """The one-SM-per-head kernel and the three-SM cluster kernel, each forced."""
    monkeypatch.setenv("KDA_PREFILL_VARIANT", variant)
    x = prefill_inputs(2, T, 3, 128, 128, seed=500 + T, h0_std=0.1)
    o, hT = run_prefill(x)
    check_prefill(x, o, hT, TOL_BF16)
    assert kda.device_status() == kda.KDA_OK


@pytest.mark.parametrize("variant", ["fused", "cluster"])
@pytest.mark.parametrize("scale", [1e-3, 30.0])
def test_bf16_input_scale(monkeypatch, variant, scale):
    """v and h0 scaled down (states of order 1e-3, still normal fp16 numbers)
    and up (|U| and |S| of order 100): the cluster kernel's fp16 state
    products keep the stated error at both ends of the documented range,
    like the all-tf32 one-SM kernel."""
    monkeypatch.setenv("KDA_PREFILL_VARIANT", variant)
    x = prefill_inputs(1, 300, 3, 128, 128, seed=620, h0_std=0.1)
    x["v"] = (x["v"].float() * scale).to(torch.bfloat16)
    x["h0"] = x["h0"] * scale
    o, hT = run_prefill(x)
    check_prefill(x, o, hT, TOL_BF16)
    assert kda.device_status() == kda.KDA_OK


# ------------------------------------------------------ segment scan ---

@pytest.mark.parametrize("B,H,T,pin", [(1, 1, 5000, 0.0), (1, 2, 4096, 0.1), (2, 1, 6173, 0.0)])
def test_bf16_segment_scan_chosen(B, H, T, pin):
    """Very few heads on a long sequence: the segment scan is chosen by itself
    (pass 1 from S = 0 and from S = I with v = 0, the segment chain, pass 3)."""
    x = prefill_inputs(B, T, H, 128, 128, seed=700 + T + H, h0_std=0.0 if pin else 0.1, pin_frac=pin)
    o, hT = run_prefill(x)
    check_prefill(x, o, hT, TOL_BF16)
    assert kda.device_status() == kda.KDA_OK


@pytest.mark.parametrize("T", [512, 1000, 2048, 3000])
def test_bf16_segment_scan_forced(monkeypatch, T):
    """Forced at more heads: segments that end on the last token and ragged
    last segments; the per-pass kernel is the cluster variant (up to 37
    segment-heads) or the one-SM variant."""
    monkeypatch.setenv("KDA_PREFILL_VARIANT", "segmented")
    x = prefill_inputs(2, T, 3, 128, 128, seed=800 + T, h0_std=0.1)
    o, hT = run_prefill(x)
    check_prefill(x, o, hT, TOL_BF16)
    assert kda.device_status() == kda.KDA_OK


@pytest.mark.slow
def test_workload_prefill_1m_h2_sampled():
    """A million-token context with two heads (segment scan, 74 segments per
    head): one head checked over the full length."""
    w = WORKLOADS["prefill_1m_h2"]
    x = prefill_inputs(w.B, w.T, w.H, w.dk, w.dv, seed=w.seed, device=DEV)
    o, hT = kda.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
    torch.cuda.synchronize()
    assert kda.device_status() == kda.KDA_OK
    eo, eh = _sampled_heads_check(w, x, o, hT, [(0, 1)])
    assert eo <= TOL_BF16 and eh <= TOL_BF16, f"err_o={eo:.3e} err_hT={eh:.3e}"


def test_bf16_segment_scan_inplace_state():
    """hT = h0 (in-place state update) through the segment scan."""
    x = prefill_inputs(1, 4500, 1, 128, 128, seed=901, h0_std=0.1)
    d = to_dev(x)
    S = d["h0"].clone()
    o, _ = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S, hT=S)
    torch.cuda.synchronize()
    check_prefill(x, o, S, TOL_BF16)


# -------------------------------------------------- intermediate states ---

def _check_states(x, states, every, tol=TOL_BF16):
    """states[:, :, s] against the oracle's final state on the prefix of
    (s + 1) * every tokens."""
    T = x["q"].shape[1]
    assert states.shape[2] == T // every
    pre = lambda t, n: t[:, :n]
    for s in range(T // every):
        n = (s + 1) * every
        _, hT_ref = oracle.fwd(pre(x["q"], n), pre(x["k"], n), pre(x["v"], n), pre(x["g"], n),
                               pre(x["beta"], n), x["h0"])
        e = err_state(states[:, :, s], hT_ref)
        assert e <= tol, f"state {s} (after {n} tokens): err={e:.3e}"


@pytest.mark.parametrize("variant,B,H,T,every", [
    ("fused", 2, 3, 1000, 256), ("cluster", 2, 3, 1000, 256), ("cluster", 1, 2, 300, 32),
    ("segmented", 2, 3, 2000, 512), ("segmented", 1, 1, 1100, 96)])
def test_bf16_intermediate_states(monkeypatch, variant, B, H, T, every):
    """kda_chunk_fwd_states on every path: each state against the oracle on the
    matching prefix; o and hT as kda_chunk_fwd's, bit for bit."""
    monkeypatch.setenv("KDA_PREFILL_VARIANT", variant)
    x = prefill_inputs(B, T, H, 128, 128, seed=1100 + T + every, h0_std=0.1)
    d = to_dev(x)
    o, hT, st = kda.chunk_fwd_states(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"], state_every=every)
    o2, hT2 = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    torch.cuda.synchronize()
    assert kda.device_status() == kda.KDA_OK
    assert torch.equal(o, o2) and torch.equal(hT, hT2)
    _check_states(x, st.cpu(), every)
    if T % every == 0:
        assert torch.equal(st[:, :, -1], hT)


def test_bf16_intermediate_states_chosen_segment_scan():
    """Few heads on a long sequence (segment scan chosen by itself): states
    come from pass 3, which starts each segment from its true state."""
    x = prefill_inputs(1, 4608, 1, 128, 128, seed=1200, h0_std=0.1)
    d = to_dev(x)
    o, hT, st = kda.chunk_fwd_states(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"], state_every=512)
    torch.cuda.synchronize()
    check_prefill(x, o, hT, TOL_BF16)
    _check_states(x, st.cpu(), 512)
    assert torch.equal(st[:, :, -1], hT)


# ------------------------------------------------------- fused prologue ---

def _raw_prefill(B, T, H, seed, zero_rows=2):
    from linear_attention_07_b200.inputs import raw_inputs
    x = raw_inputs((B, T, H, 128), (B, T, H, 128), (B, T, H), seed=seed, zero_rows=zero_rows)
    gen = torch.Generator().manual_seed(seed + 1)
    x["h0"] = torch.randn((B, H, 128, 128), generator=gen) * 0.1
    return x


@pytest.mark.parametrize("variant,B,H,T", [("fused", 2, 3, 1000), ("fused", 1, 2, 77), ("cluster", 2, 3, 1000),
                                           ("cluster", 1, 2, 77), ("segmented", 1, 2, 2100)])
def test_bf16_fused_prologue(monkeypatch, variant, B, H, T):
    """kda_chunk_fwd_raw (q, k normalised and g = -5 sigmoid(z) in the
    kernel) against the oracle's prologue + recurrence, with zero q/k
    vectors and ragged tails (g stays 0 past the end)."""
    monkeypatch.setenv("KDA_PREFILL_VARIANT", variant)
    x = _raw_prefill(B, T, H, seed=1800 + T + H)
    d = to_dev(x)
    o, hT = kda.chunk_fwd_raw(d["q"], d["k"], d["v"], d["z"], d["beta"], d["h0"])
    torch.cuda.synchronize()
    assert kda.device_status() == kda.KDA_OK
    o_ref, hT_ref = oracle.fwd_raw(x["q"], x["k"], x["v"], x["z"], x["beta"], x["h0"])
    eh = err_state(hT, hT_ref)
    check_out(o, o_ref, TOL_BF16)
    assert eh <= TOL_BF16, f"err_hT={eh:.3e}"


def test_bf16_fused_prologue_decode():
    """kda_decode_step_raw over 6 steps (state in place) against the oracle."""
    from linear_attention_07_b200.inputs import raw_inputs
    N, H, steps = 5, 3, 6
    x = raw_inputs((steps, N, H, 128), (steps, N, H, 128), (steps, N, H), seed=1900, zero_rows=1)
    gen = torch.Generator().manual_seed(1901)
    state0 = torch.randn((N, H, 128, 128), generator=gen) * 0.1
    S = state0.to(DEV)
    S_ref = state0.double().numpy()
    for t in range(steps):
        o = kda.decode_step_raw(x["q"][t].to(DEV), x["k"][t].to(DEV), x["v"][t].to(DEV), x["z"][t].to(DEV),
                                x["beta"][t].to(DEV), S)
        o_ref, S_ref = oracle.decode_step_raw(x["q"][t], x["k"][t], x["v"][t], x["z"][t], x["beta"][t], S_ref)
        torch.cuda.synchronize()
        check_out(o, o_ref, TOL_BF16)
    assert err_state(S, S_ref) <= TOL_BF16


# ------------------------------------------------------- full workloads ---

def _sampled_heads_check(w, d, o, hT, heads):
    """Run the oracle on a few whole (b, h) sequences and compare them."""
    errs_o, errs_h = [], []
    sel = lambda t, b, h: t[b:b + 1, :, h:h + 1]
    for b, h in heads:
        xs = {k: sel(d[k], b, h).cpu() for k in ("q", "k", "v", "g", "beta")}
        h0 = None if d["h0"] is None else d["h0"][b:b + 1, h:h + 1].cpu()
        o_ref, hT_ref = oracle.fwd(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], h0)
        errs_o.append(check_out(sel(o, b, h), o_ref, TOL_BF16, what="o[%d, :, %d]" % (b, h))[2])
        errs_h.append(err_state(hT[b:b + 1, h:h + 1], hT_ref))
    return max(errs_o), max(errs_h)


def test_workload_prefill_8k_full():
    w = WORKLOADS["prefill_8k"]
    x = prefill_inputs(w.B, w.T, w.H, w.dk, w.dv, seed=w.seed, h0_std=w.h0_std)
    o, hT = run_prefill(x)
    check_prefill(x, o, hT, TOL_BF16)
    assert kda.device_status() == kda.KDA_OK


def test_workload_pretrain_64k_sampled():
    w = WORKLOADS["pretrain_64k"]
    d = prefill_inputs(w.B, w.T, w.H, w.dk, w.dv, seed=w.seed, device=DEV, pin_frac=w.pin_frac)
    o, hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and torch.isfinite(hT).all()
    eo, eh = _sampled_heads_check(w, d, o, hT, [(0, 0), (1, 7), (2, 19), (3, 31)])
    assert eo <= TOL_BF16 and eh <= TOL_BF16, (eo, eh)


@pytest.mark.slow
def test_workload_prefill_1m_sampled():
    w = WORKLOADS["prefill_1m"]
    d = prefill_inputs(w.B, w.T, w.H, w.dk, w.dv, seed=w.seed, device=DEV)
    o, hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    torch.cuda.synchronize()
    assert torch.isfinite(hT).all()
    eo, eh = _sampled_heads_check(w, d, o, hT, [(0, 5)])
    assert eo <= TOL_BF16 and eh <= TOL_BF16, (eo, eh)


# --------------------------------------------------------------- decode ---

@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 32), (32, 32)])
def test_decode_shapes_several_steps(dk, dv):
    x = decode_inputs(5, 3, dk, dv, 4, seed=dk * dv)
    d = to_dev(x)
    S = d["state"].clone()
    S_ref = x["state"]
    for t in range(4):
        o = kda.decode_step(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], S)
        o_ref, S_ref = oracle.decode_step(x["q"][t], x["k"][t], x["v"][t], x["g"][t],
                                          x["beta"][t], S_ref)
        torch.cuda.synchronize()
        check_out(o, o_ref, TOL_BF16)
    assert err_state(S, S_ref) <= 1e-5   # fp32 arithmetic throughout


def test_decode_continues_prefill():
    x = prefill_inputs(1, 40, 2, 128, 128, seed=31, h0_std=0.1)
    d = to_dev(x)
    _, S = kda.chunk_fwd(*(d[k][:, :32].contiguous() for k in ("q", "k", "v", "g", "beta")), d["h0"])
    outs = []
    for t in range(32, 40):
        outs.append(kda.decode_step(*(d[k][:, t].contiguous() for k in ("q", "k", "v", "g", "beta")), S))
    torch.cuda.synchronize()
    o_ref, h_ref = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
    check_out(torch.stack(outs, 1), o_ref[:, 32:], TOL_BF16)
    assert err_state(S, h_ref) <= TOL_BF16


def test_workload_decode_256_sampled():
    w = WORKLOADS["decode_256"]
    steps = w.T
    d = decode_inputs(w.B, w.H, w.dk, w.dv, steps, seed=w.seed, device=DEV, state_std=w.h0_std)
    reqs = [0, 97, 255]
    S0 = d["state"][reqs].cpu()
    S = d["state"]
    o_all = torch.empty((steps, len(reqs), w.H, w.dv), dtype=torch.bfloat16, device=DEV)
    for t in range(steps):
        o = kda.decode_step(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], S)
        o_all[t] = o[reqs]
    torch.cuda.synchronize()
    # oracle over the sampled requests: same inputs, as a prefill of `steps`
    # tokens whose final state must equal the decoded state
    sel = lambda t: t[:, reqs].transpose(0, 1).cpu()
    o_ref, S_ref = oracle.fwd(sel(d["q"]), sel(d["k"]), sel(d["v"]), sel(d["g"]),
                              sel(d["beta"]), S0)
    check_out(o_all.transpose(0, 1), o_ref, TOL_BF16)
    assert err_state(S[reqs], S_ref) <= 1e-4


# ---------------------------------------------------- failure detection ---

def test_bounded_wait_expiry_is_reported_and_context_survives():
    """A device wait that nothing satisfies gives up after its limit, the
    status word reports KDA_ERR_TIMEOUT once, and the context keeps working."""
    stream = torch.cuda.current_stream(DEV)
    assert kda.device_status() == kda.KDA_OK
    lib = kda.load_library()
    import ctypes
    assert lib.kda_selftest_bounded_wait(20_000_000, ctypes.c_void_p(stream.cuda_stream)) == kda.KDA_OK
    assert kda.device_status() == kda.KDA_ERR_TIMEOUT
    assert kda.device_status() == kda.KDA_OK            # read and cleared
    x = prefill_inputs(1, 40, 2, 128, 128, seed=41, h0_std=0.1)
    o, hT = run_prefill(x)
    check_prefill(x, o, hT, TOL_BF16)
    assert kda.device_status() == kda.KDA_OK


# ------------------------------------------------------- several devices ---

@pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs two visible GPUs")
def test_prefill_on_two_devices_in_one_process():
    """Kernel attributes are set per device: a prefill on cuda:0 and then on
    cuda:1 (no peer access) both launch and both match the oracle."""
    x = prefill_inputs(1, 100, 2, 128, 128, seed=61, h0_std=0.1)
    o_ref, hT_ref = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
    for dev in (torch.device("cuda", 0), torch.device("cuda", 1)):
        d = {k: (None if t is None else t.to(dev)) for k, t in x.items()}
        o, hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
        torch.cuda.synchronize(dev)
        check_out(o, o_ref, TOL_BF16)
        assert err_state(hT, hT_ref) <= TOL_BF16
