"""bench.py's end-to-end loop on the CPU: CUDA stream semantics simulated.

The pipelined loop puts uploads, the prefill and downloads of successive
steps on three streams.  Here every stream operation is recorded with its
stream order and event waits; the test then requires that every two
operations on one buffer (at least one writing) are ordered, and that all
timed work lies between the two timing events.  Planted mistakes (a missing
wait) are caught by the same check.
"""
import contextlib
import itertools

import pytest
import torch

import bench


class _Sim:
    def __init__(self):
        self.ops = []             # (stream, deps, reads, writes, label)

    def enqueue(self, stream, reads, writes, label):
        deps = set(stream.pending)
        if stream.last is not None:
            deps.add(stream.last)
        self.ops.append((stream.name, deps, set(reads), set(writes), label))
        stream.last = len(self.ops) - 1
        stream.pending = set()
        return stream.last

    def host_sync(self, *a):
        self.ops.append(("host", set(), set(), set(), "sync"))

    def happens_before(self):
        before, last_sync = [], -1
        for i, (st, deps, _, _, _) in enumerate(self.ops):
            if st == "host":
                before.append(set(range(i)))
                last_sync = i
                continue
            b = set()
            for d in deps:
                b |= before[d] | {d}
            if last_sync >= 0:
                b |= before[last_sync] | {last_sync}
            before.append(b)
        return before


def _install(monkeypatch, sim, fail_streams=False):
    class Stream:
        n = 0

        def __init__(self, device=None, name=None):
            if name is None:                          # a side stream: side1, side2, ...
                if fail_streams:
                    raise RuntimeError("no side streams")
                Stream.n += 1
                name = "side%d" % Stream.n
            self.name = name
            self.last, self.pending, self.cuda_stream = None, set(), 0

        def wait_event(self, ev):
            if ev.op is not None:
                self.pending.add(ev.op)

    comp = Stream(name="comp")
    cur = [comp]

    class Event:
        def __init__(self, enable_timing=False, **kw):
            self.op = None

        def record(self, stream=None):
            self.op = sim.enqueue(stream or cur[-1], (), (), "record")

        def wait(self, stream=None):
            (stream or cur[-1]).wait_event(self)

        def elapsed_time(self, other):
            return 1.0

    @contextlib.contextmanager
    def stream_ctx(s):
        cur.append(s)
        try:
            yield
        finally:
            cur.pop()

    copy = torch.Tensor.copy_

    def copy_(self, src, non_blocking=False):
        sim.enqueue(cur[-1], [src.data_ptr()], [self.data_ptr()], "copy")
        return copy(self, src)

    empty, empty_like = torch.empty, torch.empty_like

    def host(kw):
        d = kw.get("device")
        if d is not None and torch.device(d).type == "cuda":
            kw = dict(kw, device="cpu")
        return kw

    monkeypatch.setattr(torch.cuda, "Stream", Stream)
    monkeypatch.setattr(torch.cuda, "Event", Event)
    monkeypatch.setattr(torch.cuda, "stream", stream_ctx)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a: cur[-1])
    monkeypatch.setattr(torch.cuda, "synchronize", sim.host_sync)
    monkeypatch.setattr(torch, "empty", lambda *a, **kw: empty(*a, **host(kw)))
    monkeypatch.setattr(torch, "empty_like", lambda *a, **kw: empty_like(*a, **host(kw)))
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    monkeypatch.setattr(torch.Tensor, "copy_", copy_)

    def fwd(q, k, v, g, beta, h0=None, *, o=None, hT=None):
        sim.enqueue(cur[-1], [t.data_ptr() for t in (q, k, v, g, beta, h0) if t is not None],
                    [o.data_ptr(), hT.data_ptr()], "fwd")
        return o, hT

    return fwd


def _run(monkeypatch, h0_std, fail_streams=False, steps=5):
    from linear_attention_07_b200.inputs import prefill_inputs
    sim = _Sim()
    fwd = _install(monkeypatch, sim, fail_streams)
    sets = [prefill_inputs(1, 64, 2, 128, 128, seed=s, h0_std=h0_std) for s in (1, 2)]

    class Args:
        pass
    Args.steps, Args.warmup = steps, 3
    res = bench.bench_e2e(Args, None, sets, torch.device("cuda", 0), 1, 64, 1, fwd, torch.bfloat16)
    return sim, res


def _verify(sim, steps, uploads):
    before = sim.happens_before()
    mem = [(i, r, w) for i, (st, d, r, w, lab) in enumerate(sim.ops) if r or w]
    races = [(a, b) for (a, ra, wa), (b, rb, wb) in itertools.combinations(mem, 2)
             if ((wa & (rb | wb)) or (wb & ra)) and a not in before[b] and b not in before[a]]
    syncs = [i for i, op in enumerate(sim.ops) if op[0] == "host"]
    lo, hi = syncs[-2], syncs[-1]                       # the timed region's two host waits
    timed = [i for i in range(lo + 1, hi) if sim.ops[i][0] != "host"]
    marks = [i for i in timed if sim.ops[i][4] == "record" and sim.ops[i][0] == "comp"]
    e0, e1 = min(marks), max(marks)
    work = [i for i in timed if sim.ops[i][4] in ("copy", "fwd")]
    assert not races, "unordered accesses to one buffer: %s" % races[:5]
    assert len(work) == steps * (uploads + 1 + 2)       # uploads, the prefill, 2 downloads
    assert sum(sim.ops[i][4] == "fwd" for i in work) == steps
    assert all(e0 in before[i] for i in work) and all(i in before[e1] for i in work)


@pytest.mark.parametrize("h0_std,uploads", [(0.1, 6), (0.0, 5)])
def test_pipelined_e2e_is_ordered_and_timed(monkeypatch, h0_std, uploads):
    sim, res = _run(monkeypatch, h0_std)
    assert res["mode"].startswith("pipelined")
    assert res["h2d_bytes_per_step"] > 0 and res["d2h_bytes_per_step"] > 0
    _verify(sim, 5, uploads)


def test_serial_fallback_is_ordered_and_says_so(monkeypatch):
    sim, res = _run(monkeypatch, 0.1, fail_streams=True)
    assert res["mode"].startswith("serial (pipelined loop failed")
    _verify(sim, 5, 6)


def test_a_missing_wait_is_caught(monkeypatch):
    """The check is not vacuous: when uploads ignore every event (so one can
    overwrite a buffer the previous kernel still reads), it reports races."""
    from linear_attention_07_b200.inputs import prefill_inputs
    sim = _Sim()
    fwd = _install(monkeypatch, sim)
    Stream = torch.cuda.Stream
    wait = Stream.wait_event

    def uploads_ignore_events(self, ev):
        if self.name != "side1":                      # side1: the first side stream, uploads
            wait(self, ev)
    monkeypatch.setattr(Stream, "wait_event", uploads_ignore_events)
    sets = [prefill_inputs(1, 64, 2, 128, 128, seed=s, h0_std=0.1) for s in (1, 2)]

    class Args:
        steps, warmup = 5, 3
    res = bench.bench_e2e(Args, None, sets, torch.device("cuda", 0), 1, 64, 1, fwd, torch.bfloat16)
    assert res["mode"].startswith("pipelined")
    with pytest.raises(AssertionError, match="unordered"):
        _verify(sim, 5, 6)


def test_tensor_fraction_uses_each_products_own_peak():
    """tensor_frac_mma: the state products on the fp16 peak for the cluster
    kernel and everything on the tf32 peak (half of it) otherwise; the
    one-peak fractions stay as they were."""
    B, T, H, d = 1, 8192, 32, 128
    alg = bench.prefill_alg_flops(B, T, H, d, d)
    state = bench.prefill_state_flops(B, T, H, d, d)
    assert state == B * T * H * 6 * d * d and 0 < state < alg
    peak, ms = 1600.0, 0.5
    one_sm = bench.tensor_fractions(alg, state, ms, peak, "one SM per head")
    cluster = bench.tensor_fractions(alg, state, ms, peak, "cluster of four SMs per head")
    sec = ms / 1e3
    assert one_sm["tensor_frac_mma"] == pytest.approx(alg / (peak / 2 * 1e12) / sec, rel=1e-3)
    assert one_sm["tensor_frac_mma"] == one_sm["tensor_frac_tf32"]
    want = ((alg - state) / (peak / 2 * 1e12) + state / (peak * 1e12)) / sec
    assert cluster["tensor_frac_mma"] == pytest.approx(want, rel=1e-3)
    assert cluster["tensor_frac_bf16"] < cluster["tensor_frac_mma"] < cluster["tensor_frac_tf32"]
    assert "fp16" in cluster["mma_kinds"] and "fp16" not in one_sm["mma_kinds"]
