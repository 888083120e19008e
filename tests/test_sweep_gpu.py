"""Full-size decoder sweeps, built and launched exactly as bench.py does, vs the
oracle on sampled rows.

For the first, middle and last layer of each workload: the codes of sampled
rows of every projection are bit-exact with the oracle's quantization of the
same seeded fp32 rows, and every sampled output row is within the bound,
teacher-forced on the device's actual inputs (o reads the device's fp16 q,
down the device's SwiGLU output).  The head's argmax over the full vocabulary
passes the margin rule, and the graph replay gives the eager result bit for
bit.
"""
import gc

import numpy as np
import pytest
import torch

import oracle
from helpers import assert_within_bound, bits, host_weight, oracle_gemv, oracle_quantize
from int4_quantized_decode_b200 import qgemv as qg
from int4_quantized_decode_b200 import workloads as wl
from int4_quantized_decode_b200.sweep import DecodeSweep

pytestmark = pytest.mark.gpu
I8, I4 = qg.FMT_I8_B32, qg.FMT_I4_G64
SAMPLE = 48


def _check_codes(sw, W, l, parts, rows):
    """parts: [(proj name, row offset, row count)] of the fused weight W."""
    d = sw.dec
    for name, off, cnt in parts:
        sel = [r - off for r in rows if off <= r < off + cnt]
        if not sel:
            continue
        w = wl.weight_fp32(cnt, W.k, d.weight_seed(l, name), sw.device)
        wr = w.index_select(0, torch.as_tensor(sel, device=sw.device)).cpu().numpy()
        del w
        if W.fmt == qg.FMT_F16:  # plain fp16 weights: the IEEE RNE of the draw
            dc, _, _ = host_weight(W, [r for r in rows if off <= r < off + cnt])
            assert np.array_equal(dc, oracle.f32_to_f16_bits(wr)), (name, l)
            continue
        oc, os_, ob = oracle_quantize(W.fmt, wr)
        dc, ds, db = host_weight(W, [r for r in rows if off <= r < off + cnt])
        assert np.array_equal(dc, oc), (name, l)
        assert np.array_equal(ds, os_), (name, l)
        if ob is not None:
            assert np.array_equal(db, ob), (name, l)


def _rows_out(Y, rows, s=0):
    return Y[s].cpu().numpy()[rows] if Y.dim() == 2 else Y.cpu().numpy()[rows]


def _check_layer(sw, l):
    d, L, S = sw.dec, sw.layers[l], sw.S
    sw.run_layer(l)
    qg.qg_stream_check()
    seed = 1000 * l + 7
    # q|(gate)|k|v
    rows = wl.sample_rows(d.qkv_rows, SAMPLE, seed).tolist()
    parts, off = [], 0
    for name, cnt in d.qkv_parts():
        parts.append((name, off, cnt))
        off += cnt
    _check_codes(sw, L.qkv, l, parts, rows)
    tokens = range(S) if S == 1 else (0, 7, S - 1)
    for s in tokens:
        x = sw.x[l] if S == 1 else sw.x[l][s]
        yr, mag = oracle_gemv(L.qkv, x, rows)
        assert_within_bound(_rows_out(sw.y_qkv, rows, s), yr, mag)
    if S == 1:
        y16 = bits(sw.y16_qkv)
        assert np.array_equal(y16, oracle.f32_to_f16_bits(sw.y_qkv[0].cpu().numpy()))
    # o (teacher-forced on the device's fp16 q or the seeded stand-in chunk)
    rows = wl.sample_rows(d.hidden, SAMPLE, seed + 1).tolist()
    _check_codes(sw, L.o, l, [("o", 0, d.hidden)], rows)
    for s in tokens:
        xo = sw.y16_qkv[: d.q_dim] if S == 1 else sw.x_o[l][s]
        yr, mag = oracle_gemv(L.o, xo, rows)
        assert_within_bound(_rows_out(sw.y_o, rows, s), yr, mag)
    # gate/up + SwiGLU
    rows = wl.sample_rows(d.inter, SAMPLE, seed + 2).tolist()
    _check_codes(sw, L.gate, l, [("gate", 0, d.inter)], rows)
    _check_codes(sw, L.up, l, [("up", 0, d.inter)], rows)
    for s in tokens:
        x = sw.x[l] if S == 1 else sw.x[l][s]
        gr, mg = oracle_gemv(L.gate, x, rows)
        ur, mu = oracle_gemv(L.up, x, rows)
        hr, hb = oracle.swiglu(gr, ur, mg, mu, oracle.GEMV_TOL)
        hd = sw.h[s].cpu().numpy().astype(np.float64)[rows]
        assert np.all(np.abs(hd - hr) <= hb), (l, s)
    # down (teacher-forced on the device's h)
    rows = wl.sample_rows(d.hidden, SAMPLE, seed + 3).tolist()
    _check_codes(sw, L.down, l, [("down", 0, d.hidden)], rows)
    for s in tokens:
        yr, mag = oracle_gemv(L.down, sw.h[s], rows)
        assert_within_bound(_rows_out(sw.y_down, rows, s), yr, mag)


def _check_sweep(dec, body_fmt, head_fmt, S, cuda):
    sw = DecodeSweep(dec, body_fmt, head_fmt, S=S, device=cuda, keep_logits=True)
    try:
        sw.capture(sweeps_per_graph=2)
        sw.graph.replay()
        qg.qg_stream_check()
        idx_graph = int(sw.idx.item())
        logits_graph = sw.logits.clone()
        sw.step()
        qg.qg_stream_check()
        assert int(sw.idx.item()) == idx_graph
        assert torch.equal(sw.logits, logits_graph), "graph replay differs from eager"
        assert int(sw.ws.sum().item()) == 0
        # head: sampled rows' codes, full logits bound and the greedy token
        rows = wl.sample_rows(dec.vocab, SAMPLE, 99).tolist()
        _check_codes(sw, sw.head, -1, [("head", 0, dec.vocab)], rows)
        yr, mag = oracle_gemv(sw.head, sw.head_input())
        assert_within_bound(sw.logits.cpu().numpy(), yr, mag)
        assert oracle.argmax_ok(idx_graph, yr)
        for l in sorted({0, dec.layers // 2, dec.layers - 1}):
            _check_layer(sw, l)
    finally:
        del sw
        gc.collect()
        torch.cuda.empty_cache()


def test_single_gemv_2048(cuda):
    """Single 2048 x 2048 int8 GEMV (W seed 0), checked on every row."""
    cfg = wl.GEMV_2048
    w = wl.weight_fp32(cfg["n"], cfg["k"], cfg["w_seed"], cuda)
    W = qg.quantize(w, I8)
    x = wl.act_fp16(cfg["k"], cfg["x_seed"], cuda)
    y = torch.empty(cfg["n"], dtype=torch.float32, device=cuda)
    qg.qg_gemv_s1(W, x, y)
    qg.qg_stream_check()
    codes, scales = oracle.quantize_block32(w.cpu().numpy())
    assert np.array_equal(codes, W.codes.cpu().numpy())
    assert np.array_equal(scales, bits(W.scales))
    yr, mag = oracle.matvec(0, codes, scales, None, bits(x))
    assert_within_bound(y.cpu().numpy(), yr, mag)


def test_sweep_2b_int8(cuda):
    _check_sweep(wl.QWEN3VL_2B, I8, I8, 1, cuda)


def test_sweep_2b_int8_tied_fp16_head(cuda):
    """The int8lin bundle: int8 body, the fp16 embedding table as the head."""
    _check_sweep(wl.QWEN3VL_2B, I8, qg.FMT_F16, 1, cuda)


def test_sweep_4b_int8(cuda):
    _check_sweep(wl.QWEN3VL_4B, I8, I8, 1, cuda)


def test_sweep_4b_int4_body(cuda):
    _check_sweep(wl.QWEN3VL_4B, I4, I8, 1, cuda)


def test_sweep_8b_int8(cuda):
    _check_sweep(wl.QWEN3VL_8B, I8, I8, 1, cuda)


def test_sweep_8b_s16_chunk(cuda):
    _check_sweep(wl.QWEN3VL_8B, I8, I8, 16, cuda)


def test_sweep_27b_int8(cuda):
    _check_sweep(wl.DENSE_27B, I8, I8, 1, cuda)


def test_sweep_8b_int4_body(cuda):
    _check_sweep(wl.QWEN3VL_8B, I4, I8, 1, cuda)


def test_sweep_27b_int4_body_and_head(cuda):
    """The 27B 'int4lin' option: every matrix int4 group-64, the head too."""
    _check_sweep(wl.DENSE_27B, I4, I4, 1, cuda)
