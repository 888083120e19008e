"""The persistent sweep (qg_sweep_plan / qg_sweep_run) vs the oracle and the
single calls.

A sweep is the chain of S=1 calls a decode step makes, run as one launch.  An
all-int8 plan whose rows hold whole 512-code steps runs on the stream kernel:
its results are within the oracle's bound (teacher-forced on the x each stage
actually read) and bit-identical from run to run (a fixed summation order per
row), though not in the single calls' summation order.  Other plans run on
the general persistent kernels, whose results are bit-identical to the same
calls enqueued one by one.  The chains below read earlier stages' outputs (o
reads fp16 q, down reads the SwiGLU output, a head reads a GEMV's fp16
output), so a stage that read its x before the previous stage finished would
differ.  Shapes cover ragged row counts and both item sizes of the stream
kernel (one and two rows), and every ring variant of the general kernels."""
import gc

import numpy as np
import pytest
import torch

import oracle
from helpers import assert_within_bound, oracle_gemv
from int4_quantized_decode_b200 import qgemv as qg
from int4_quantized_decode_b200 import workloads as wl
from int4_quantized_decode_b200.sweep import DecodeSweep

pytestmark = pytest.mark.gpu
I8, I4 = qg.FMT_I8_B32, qg.FMT_I4_G64
SAMPLE = 64


class Chain:
    """A list of stages with their own output buffers, runnable as a sweep or
    as single calls."""

    def __init__(self, dev, body_fmt):
        self.dev, self.body = dev, body_fmt
        self.ops = []       # (kind, weights, x producer, outputs)
        self.bufs = {}
        self.seed = 1
        self.x0 = wl.act_fp16(1024, 11, dev)
        self.x1 = wl.act_fp16(1024, 12, dev)

    def weight(self, n, k, fmt):
        self.seed += 1
        w = wl.weight_fp32(n, k, 9000 + self.seed, self.dev)
        q = qg.quantize(w, fmt)
        del w
        return q

    def gemv(self, name, n, k, x, fp16_out=False):
        W = self.weight(n, k, self.body)
        self.ops.append(("gemv", name, (W,), x, fp16_out))
        return name

    def swiglu(self, name, n, k, x):
        self.ops.append(("swiglu", name, (self.weight(n, k, self.body),
                                          self.weight(n, k, self.body)), x, False))
        return name

    def head(self, name, n, k, x):
        self.ops.append(("head", name, (self.weight(n, k, I8),), x, False))
        return name

    def _x(self, src, outs):
        if isinstance(src, torch.Tensor):
            return src
        name, length = src                      # an earlier stage's fp16 output
        return outs[name][-1][:length]

    def _alloc(self):
        outs = {}
        for kind, name, Ws, _, fp16_out in self.ops:
            n = Ws[0].n
            if kind == "gemv":
                y = torch.full((n,), float("nan"), dtype=torch.float32, device=self.dev)
                y16 = torch.empty(n, dtype=torch.float16, device=self.dev) if fp16_out else None
                outs[name] = (y, y16) if fp16_out else (y,)
            elif kind == "swiglu":
                outs[name] = (torch.empty(n, dtype=torch.float16, device=self.dev),)
            else:
                outs[name] = (torch.full((n,), float("nan"), dtype=torch.float32,
                                         device=self.dev),
                              torch.full((1,), -1, dtype=torch.int32, device=self.dev))
        return outs

    def run_calls(self):
        outs = self._alloc()
        ws = qg.head_workspace(1, self.dev)
        for kind, name, Ws, src, _ in self.ops:
            x, o = self._x(src, outs), outs[name]
            if kind == "gemv":
                qg.qg_gemv_s1(Ws[0], x, o[0], o[1] if len(o) > 1 else None)
            elif kind == "swiglu":
                qg.qg_gate_up_swiglu(Ws[0], Ws[1], x, o[0])
            else:
                qg.qg_head_argmax(Ws[0], x, o[1], ws, o[0])
        qg.qg_stream_check()
        return outs

    def stages(self, outs):
        st = []
        for kind, name, Ws, src, _ in self.ops:
            x, o = self._x(src, outs), outs[name]
            if kind == "gemv":
                st.append(qg.stage_gemv(Ws[0], x, o[0], o[1] if len(o) > 1 else None))
            elif kind == "swiglu":
                st.append(qg.stage_swiglu(Ws[0], Ws[1], x, o[0]))
            else:
                st.append(qg.stage_head(Ws[0], x, o[1], o[0]))
        return st


def build_chain(dev, body):
    """qkv -> o -> gate/up -> down, then larger and smaller projections and three
    heads; row counts pick every variant (1/2/4 rows per warp item)."""
    c = Chain(dev, body)
    qkv = c.gemv("qkv", 1536, 1024, c.x0, fp16_out=True)
    c.gemv("o", 1024, 1024, (qkv, 1024))
    h = c.swiglu("gate_up", 5120, 1024, c.x0)
    down = c.gemv("down", 1024, 5120, (h, 5120), fp16_out=True)
    big = c.gemv("big", 20001, 1024, (down, 1024), fp16_out=True)
    c.gemv("mid", 6000, 1024, c.x1)
    h2 = c.swiglu("gate_up_small", 1536, 1024, (big, 1024))
    c.gemv("down_small", 1000, 1536, (h2, 1536))
    c.head("head_mid", 5003, 1024, (big, 1024))
    c.head("head_big", 20003, 1024, c.x1)
    c.head("head_small", 1000, 1024, (qkv, 1024))
    return c


def _equal(a, b):
    return torch.equal(a.view(torch.int32) if a.dtype == torch.float32 else a,
                       b.view(torch.int32) if b.dtype == torch.float32 else b)


STREAM = 2  # qg_sweep.kernel of the stream kernel


def _counter_bytes(plan):
    """Workspace bytes that hold the grid counters of the plan's kernel."""
    n = plan.n_stages
    return 4 * (n * 8 * 32 + 32) if plan.sweep.kernel == STREAM else 4 * (n + 1)


@pytest.mark.parametrize("body", [I8, I4])
def test_sweep_chain_bitwise_and_oracle(cuda, body):
    c = build_chain(cuda, body)
    ref = c.run_calls()
    outs = c._alloc()
    plan = qg.SweepPlan(c.stages(outs), [], cuda)
    assert plan.sweep.kernel == (STREAM if body == I8 else 1)
    first = None
    for rep in range(3):                      # counters reset after every run
        for o in outs.values():
            for t in o:
                t.fill_(0 if t.dtype != torch.float32 else float("nan"))
        plan.run()
        qg.qg_stream_check()
        # the general kernels equal the single calls; the stream kernel equals
        # itself from run to run
        expect = ref if plan.sweep.kernel != STREAM else first
        if expect is not None:
            for kind, name, Ws, src, _ in c.ops:
                for a, b in zip(outs[name], expect[name]):
                    assert _equal(a, b), (rep, name)
        if first is None:
            first = {k: [t.clone() for t in v] for k, v in outs.items()}
        ctr = plan.workspace[256:256 + _counter_bytes(plan)]
        assert int(ctr.sum().item()) == 0
    # every stage within the oracle's bound (teacher-forced on its actual x)
    for kind, name, Ws, src, _ in c.ops:
        x = c._x(src, outs)
        n = Ws[0].n
        rows = None if n <= 6000 else wl.sample_rows(n, SAMPLE, n).tolist()
        if kind == "swiglu":
            gr, mg = oracle_gemv(Ws[0], x, rows)
            ur, mu = oracle_gemv(Ws[1], x, rows)
            hr, hb = oracle.swiglu(gr, ur, mg, mu, oracle.GEMV_TOL)
            hd = outs[name][0].cpu().numpy().astype(np.float64)
            hd = hd if rows is None else hd[rows]
            assert np.all(np.abs(hd - hr) <= hb), name
        else:
            yr, mag = oracle_gemv(Ws[0], x, rows)
            y = outs[name][0].cpu().numpy()
            assert_within_bound(y if rows is None else y[rows], yr, mag)
            if kind == "head":
                full, _ = oracle_gemv(Ws[0], x)
                assert oracle.argmax_ok(int(outs[name][1].item()), full), name


def test_sweep_in_graph_matches_eager(cuda):
    c = build_chain(cuda, I8)
    outs = c._alloc()
    plan = qg.SweepPlan(c.stages(outs), [], cuda)
    plan.run()
    qg.qg_stream_check()
    snap = {k: [t.clone() for t in v] for k, v in outs.items()}
    s = torch.cuda.Stream(device=cuda)
    s.wait_stream(torch.cuda.current_stream(cuda))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        plan.run()
        plan.run()
    for t in (t for v in outs.values() for t in v):
        t.zero_()
    g.replay()
    qg.qg_stream_check()
    for k, v in outs.items():
        for a, b in zip(v, snap[k]):
            assert _equal(a, b), k


def test_sweep_plan_rejects(cuda):
    c = build_chain(cuda, I8)
    outs = c._alloc()
    st = c.stages(outs)
    ws = torch.zeros(qg.qg_sweep_workspace_bytes(len(st)) + 512, dtype=torch.uint8, device=cuda)
    off = (-ws.data_ptr()) % 256
    aligned = ws[off:]
    with pytest.raises(qg.QgError, match="QG_ERR_WORKSPACE"):
        qg.qg_sweep_plan(st, aligned[:64])
    with pytest.raises(qg.QgError, match="QG_ERR_ALIGN"):
        qg.qg_sweep_plan(st, aligned[16:])
    bad = list(st)
    bad[1] = qg.CStage(7, 0, bad[1].w, bad[1].w_up, bad[1].x, bad[1].y, None, None, None, None)
    with pytest.raises(qg.QgError, match="QG_ERR_FORMAT"):
        qg.qg_sweep_plan(bad, aligned)
    # int4 projections with an int4 head: not a layout the int4 kernel holds
    c4 = Chain(cuda, I4)
    W4 = c4.weight(64, 1024, I4)
    idx = torch.zeros(1, dtype=torch.int32, device=cuda)
    with pytest.raises(qg.QgError, match="QG_ERR_FORMAT"):
        qg.qg_sweep_plan([qg.stage_head(W4, c4.x0, idx)], aligned)
    # k that is not a multiple of 8 scales per row
    W8 = c.weight(64, 96, I8)
    y = torch.empty(64, dtype=torch.float32, device=cuda)
    with pytest.raises(qg.QgError, match="QG_ERR_SHAPE"):
        qg.qg_sweep_plan([qg.stage_gemv(W8, wl.act_fp16(96, 1, cuda), y)], aligned)


def test_sweep_wrong_plan_and_expired_wait_are_reported(cuda):
    """A run whose descriptor does not match the workspace exits at once
    (QG_ERR_PLAN); a stage barrier that can never complete gives up after its
    bounded wait (QG_ERR_TIMEOUT) and leaves the context usable."""
    c = build_chain(cuda, I8)
    outs = c._alloc()
    plan = qg.SweepPlan(c.stages(outs), [], cuda)
    plan.run()
    qg.qg_stream_check()
    clean = {k: [t.clone() for t in v] for k, v in outs.items()}
    wrong = qg.CSweep(plan.sweep.n_stages, 1)
    qg.qg_sweep_run(wrong, plan.workspace)
    with pytest.raises(qg.QgError, match="QG_ERR_PLAN"):
        qg.qg_stream_check()
    # Counter of stage 0 set to 2^32 - 1: the first arrival wraps it to 0, so
    # after every CTA has arrived it holds grid - 1 and the wait of stage 1
    # can never see grid arrivals.  Each CTA gives up after its bounded wait.
    plan.workspace[256:260].fill_(255)
    plan.run()
    with pytest.raises(qg.QgError, match="QG_ERR_TIMEOUT"):
        qg.qg_stream_check()
    plan.sweep = qg.qg_sweep_plan(c.stages(outs), plan.workspace)   # plan again
    for t in (t for v in outs.values() for t in v):
        t.zero_()
    plan.run()
    qg.qg_stream_check()
    for k, v in outs.items():
        for a, b in zip(v, clean[k]):
            assert _equal(a, b), k


@pytest.mark.parametrize("dec,body", [(wl.QWEN3VL_2B, I8), (wl.QWEN3VL_4B, I4),
                                      (wl.DENSE_27B, I8)])
def test_decode_sweep_persistent(cuda, dec, body):
    """The full-size sweep bench.py times: one persistent launch per sweep.
    Two sweeps captured in a graph leave every buffer (last layer's outputs,
    logits, token) bit-identical to one eager persistent sweep; the general
    int4 kernel also equals the launch path bit for bit; and the last layer
    and the head are within the oracle's bound on sampled rows, teacher-forced
    on the x each stage read, with the token passing the margin rule."""
    sw = DecodeSweep(dec, body, I8, S=1, device=cuda, keep_logits=True)
    try:
        bufs = [sw.y_qkv, sw.y16_qkv, sw.y_o, sw.h, sw.y_down, sw.logits, sw.idx]
        sw.step()
        qg.qg_stream_check()
        launches = [b.clone() for b in bufs]
        sw.step(persistent=True)
        qg.qg_stream_check()
        ref = [b.clone() for b in bufs]
        for b in bufs:
            b.zero_()
        g = sw.capture(sweeps_per_graph=2, persistent=True)
        g.replay()
        qg.qg_stream_check()
        for a, b in zip(bufs, ref):
            assert _equal(a, b)
        if sw.make_plan().sweep.kernel != STREAM:
            for a, b in zip(ref, launches):
                assert _equal(a, b)
        assert int(sw.ws.sum().item()) == 0
        L, d = sw.layers[-1], dec
        x = sw.x[-1]
        for W, xin, y in [(L.qkv, x, sw.y_qkv[0]), (L.o, sw.y16_qkv[: d.q_dim], sw.y_o[0]),
                          (L.down, sw.h[0], sw.y_down[0])]:
            rows = wl.sample_rows(W.n, SAMPLE, W.n).tolist()
            yr, mag = oracle_gemv(W, xin, rows)
            assert_within_bound(y.cpu().numpy()[rows], yr, mag)
        rows = wl.sample_rows(L.gate.n, SAMPLE, 7).tolist()
        gr, mg = oracle_gemv(L.gate, x, rows)
        ur, mu = oracle_gemv(L.up, x, rows)
        hr, hb = oracle.swiglu(gr, ur, mg, mu, oracle.GEMV_TOL)
        assert np.all(np.abs(sw.h[0].cpu().numpy().astype(np.float64)[rows] - hr) <= hb)
        full, mag = oracle_gemv(sw.head, sw.head_input())
        assert_within_bound(sw.logits.cpu().numpy(), full, mag)
        assert oracle.argmax_ok(int(sw.idx.item()), full)
    finally:
        del sw
        gc.collect()
        torch.cuda.empty_cache()


def test_stream_sweep_short_plans(cuda):
    """Plans with fewer rows than CTAs (most CTAs own no rows of a stage, and
    every CTA still takes part in each stage boundary), a one-stage plan, and
    rows that exactly fill the stream kernel's 32 KB chunks (a SwiGLU stage of
    k = 16384: one gate row and one up row per chunk) run on the stream kernel
    and stay within the oracle's bound, teacher-forced on the x each read."""
    c = Chain(cuda, I8)
    a = c.gemv("a", 1, 512, c.x0[:512], fp16_out=True)
    c.swiglu("b", 3, 512, c.x1[:512])
    c.head("c", 147, 1024, c.x0)
    big_x = wl.act_fp16(16384, 13, cuda)
    c.swiglu("d", 300, 16384, big_x)
    c.gemv("e", 149, 1024, c.x1)
    outs = c._alloc()
    plan = qg.SweepPlan(c.stages(outs), [], cuda)
    assert plan.sweep.kernel == STREAM
    for _ in range(2):
        plan.run()
        qg.qg_stream_check()
    for kind, name, Ws, src, _ in c.ops:
        x = c._x(src, outs)
        if kind == "swiglu":
            gr, mg = oracle_gemv(Ws[0], x)
            ur, mu = oracle_gemv(Ws[1], x)
            hr, hb = oracle.swiglu(gr, ur, mg, mu, oracle.GEMV_TOL)
            hd = outs[name][0].cpu().numpy().astype(np.float64)
            assert np.all(np.abs(hd - hr) <= hb), name
        else:
            yr, mag = oracle_gemv(Ws[0], x)
            assert_within_bound(outs[name][0].cpu().numpy(), yr, mag)
            if kind == "head":
                assert oracle.argmax_ok(int(outs[name][1].item()), yr), name
    # one stage
    c1 = Chain(cuda, I8)
    c1.head("h", 5003, 2048, wl.act_fp16(2048, 14, cuda))
    o1 = c1._alloc()
    p1 = qg.SweepPlan(c1.stages(o1), [], cuda)
    assert p1.sweep.kernel == STREAM
    p1.run()
    qg.qg_stream_check()
    Wh = c1.ops[0][2][0]
    yr, mag = oracle_gemv(Wh, c1._x(c1.ops[0][3], o1))
    assert_within_bound(o1["h"][0].cpu().numpy(), yr, mag)
    assert oracle.argmax_ok(int(o1["h"][1].item()), yr)
