"""The decode step around the weight stream: embedding gather, RMSNorm fused
into the S=1 calls, residual adds, vs the fp64 oracle (teacher-forced on the
device's own hidden state and on the device's own fp16 x).

The device rounds the RMSNorm to fp16 from fp32, so its x is checked apart,
within one fp16 ulp of the oracle's fp64 RMSNorm rounded to fp16; the fused
calls are then checked at the plain 2e-3 bound against the oracle on that x
(qg_rmsnorm_f16 returns it), and bit for bit against the plain calls given
the same x, which shows the fused calls staged exactly that x."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_within_bound, bits, oracle_gemv
from int4_quantized_decode_b200 import qgemv as qg
from int4_quantized_decode_b200 import workloads as wl

pytestmark = pytest.mark.gpu
I8, I4, F16 = qg.FMT_I8_B32, qg.FMT_I4_G64, qg.FMT_F16
EPS = 1e-6
TOL = oracle.GEMV_TOL


def _weight(fmt, n, k, seed, dev):
    w = wl.weight_fp32(n, k, seed, dev)
    return qg.QWeight.fp16(w.half()) if fmt == F16 else qg.quantize(w, fmt)


def _hidden(k, seed, dev, scale=3.0):
    return (wl.weight_fp32(1, k, seed, dev)[0] * (scale / 0.02)).contiguous()


def _gamma(k, seed, dev):
    return (1.0 + 0.1 * wl.act_fp16(k, seed, dev).float()).half()


def _x_ref(h, gamma, dev):
    xb, _ = oracle.rmsnorm(h.cpu().numpy(), bits(gamma), EPS)
    return torch.from_numpy(xb.view(np.int16)).to(dev).view(torch.float16)


def _x_dev(h, gamma, dev):
    """The device's x = fp16(RMSNorm(h)), checked within one fp16 ulp of the
    oracle's (fp64 RMSNorm rounded to fp16)."""
    x = torch.empty(h.numel(), dtype=torch.float16, device=dev)
    qg.qg_rmsnorm_f16(h, gamma, EPS, x)
    qg.qg_stream_check()
    xr = _x_ref(h, gamma, dev).cpu().numpy().astype(np.float64)
    xd = x.cpu().numpy().astype(np.float64)
    ulp = np.spacing(np.abs(xr).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(xd - xr) <= ulp), "device RMSNorm off by more than one fp16 ulp"
    return x


def _same(a, b):
    return torch.equal(a.view(torch.int32) if a.dtype == torch.float32 else a,
                       b.view(torch.int32) if b.dtype == torch.float32 else b)


@pytest.mark.parametrize("fmt,n,k", [(I8, 300, 2048), (I8, 4096, 2560), (I4, 1000, 2560),
                                     (I8, 2048, 6144), (F16, 777, 4096), (I8, 20001, 5120)])
def test_rmsnorm_gemv(cuda, fmt, n, k):
    W = _weight(fmt, n, k, 800 + n % 7, cuda)
    h, gam = _hidden(k, 801, cuda), _gamma(k, 802, cuda)
    y = torch.full((n,), float("nan"), dtype=torch.float32, device=cuda)
    y16 = torch.empty(n, dtype=torch.float16, device=cuda)
    qg.qg_rmsnorm_gemv_s1(W, h, gam, EPS, y, y16)
    qg.qg_stream_check()
    x = _x_dev(h, gam, cuda)
    yr, mag = oracle_gemv(W, x)
    yd = y.cpu().numpy()
    assert_within_bound(yd, yr, mag, TOL)
    assert np.array_equal(bits(y16), oracle.f32_to_f16_bits(yd))
    y1 = torch.empty_like(y)
    qg.qg_gemv_s1(W, x, y1)
    qg.qg_stream_check()
    assert _same(y, y1), "the fused call did not multiply by the device's x"


@pytest.mark.parametrize("fmt,n,k", [(I8, 2048, 2048), (I4, 2560, 9728), (I8, 5120, 17408)])
def test_residual_add(cuda, fmt, n, k):
    W = _weight(fmt, n, k, 810, cuda)
    x = wl.act_fp16(k, 811, cuda)
    h0 = _hidden(n, 812, cuda)
    h = h0.clone()
    qg.qg_gemv_s1_residual(W, x, h)
    qg.qg_stream_check()
    yr, mag = oracle_gemv(W, x)
    hn, ho = h.cpu().numpy().astype(np.float64), h0.cpu().numpy().astype(np.float64)
    err = np.abs(hn - (ho + yr))
    assert np.all(err <= oracle.GEMV_TOL * mag + np.spacing(np.abs(hn).astype(np.float32)))


@pytest.mark.parametrize("fmt,n,k", [(I8, 6144, 2048), (I4, 9728, 2560)])
def test_rmsnorm_gate_up_swiglu(cuda, fmt, n, k):
    Wg, Wu = _weight(fmt, n, k, 820, cuda), _weight(fmt, n, k, 821, cuda)
    h, gam = _hidden(k, 822, cuda), _gamma(k, 823, cuda)
    H = torch.empty(n, dtype=torch.float16, device=cuda)
    qg.qg_rmsnorm_gate_up_swiglu(Wg, Wu, h, gam, EPS, H)
    qg.qg_stream_check()
    x = _x_dev(h, gam, cuda)
    gr, mg = oracle_gemv(Wg, x)
    ur, mu = oracle_gemv(Wu, x)
    hr, hb = oracle.swiglu(gr, ur, mg, mu, TOL)
    assert np.all(np.abs(H.cpu().numpy().astype(np.float64) - hr) <= hb)
    H1 = torch.empty_like(H)
    qg.qg_gate_up_swiglu(Wg, Wu, x, H1)
    qg.qg_stream_check()
    assert _same(H, H1), "the fused call did not multiply by the device's x"


@pytest.mark.parametrize("fmt,V,k", [(I8, 151936, 2048), (F16, 151936, 2048), (I4, 20000, 2560)])
def test_rmsnorm_head_argmax(cuda, fmt, V, k):
    W = _weight(fmt, V, k, 830, cuda)
    h, gam = _hidden(k, 831, cuda), _gamma(k, 832, cuda)
    idx = torch.full((1,), -1, dtype=torch.int32, device=cuda)
    logits = torch.empty(V, dtype=torch.float32, device=cuda)
    ws = qg.head_workspace(V, cuda)
    qg.qg_rmsnorm_head_argmax(W, h, gam, EPS, idx, ws, logits)
    qg.qg_stream_check()
    x = _x_dev(h, gam, cuda)
    yr, mag = oracle_gemv(W, x)
    assert_within_bound(logits.cpu().numpy(), yr, mag, TOL)
    assert oracle.argmax_ok(int(idx.item()), yr)
    assert int(ws.sum().item()) == 0
    logits1 = torch.empty_like(logits)
    idx1 = torch.full_like(idx, -1)
    qg.qg_head_argmax(W, x, idx1, ws, logits1)
    qg.qg_stream_check()
    assert _same(logits, logits1) and int(idx1.item()) == int(idx.item())


def test_embedding_gather_exact_and_out_of_range(cuda):
    V, H = 151936, 2048
    E = wl.weight_fp32(V, H, 840, cuda).half()
    h = torch.full((H,), float("nan"), dtype=torch.float32, device=cuda)
    for t in (0, 12345, V - 1):
        tok = torch.tensor([t], dtype=torch.int32, device=cuda)
        qg.qg_embedding_gather(E, tok, h)
        qg.qg_stream_check()
        assert torch.equal(h, E[t].float())
    before = h.clone()
    for bad in (V, -1):
        qg.qg_embedding_gather(E, torch.tensor([bad], dtype=torch.int32, device=cuda), h)
        with pytest.raises(qg.QgError, match="QG_ERR_SHAPE"):
            qg.qg_stream_check()
        assert torch.equal(h, before)


def test_decode_step_chain_2b(cuda):
    """The 2B-shaped decode step minus attention, teacher-forced op by op on the
    device's own state: gather, every norm-fused projection of the first and
    the last layer (sampled rows), the residual stream, the head's argmax; then
    the graph of two chained steps equals two eager steps bit for bit, and the
    second step starts from the first step's token."""
    import gc
    from int4_quantized_decode_b200.sweep import DecodeSweep
    d = wl.QWEN3VL_2B
    sw = DecodeSweep(d, I8, I8, S=1, device=cuda, keep_logits=True, decode_step=True)
    try:
        tok0 = int(sw.idx.item())
        sw.run_embed()
        qg.qg_stream_check()
        assert torch.equal(sw.hstate, sw.embed[tok0].float())
        rows = wl.sample_rows(d.hidden, 64, 5).tolist()
        for l in range(d.layers):
            L = sw.layers[l]
            check = l in (0, d.layers - 1)
            h0 = sw.hstate.clone()
            qg.qg_rmsnorm_gemv_s1(L.qkv, sw.hstate, sw.gamma_attn[l], sw.eps, sw.y_qkv[0],
                                  sw.y16_qkv)
            if check:
                x = _x_dev(h0, sw.gamma_attn[l], cuda)
                r = wl.sample_rows(d.qkv_rows, 64, 6).tolist()
                yr, mag = oracle_gemv(L.qkv, x, r)
                assert_within_bound(sw.y_qkv[0].cpu().numpy()[r], yr, mag, TOL)
            xo = sw.y16_qkv[: d.q_dim].clone()
            qg.qg_gemv_s1_residual(L.o, sw.y16_qkv[: d.q_dim], sw.hstate)
            if check:
                yr, mag = oracle_gemv(L.o, xo, rows)
                dh = (sw.hstate.cpu().numpy().astype(np.float64) - h0.cpu().numpy())[rows]
                assert np.all(np.abs(dh - yr) <= oracle.GEMV_TOL * mag +
                              np.spacing(np.abs(sw.hstate.cpu().numpy()[rows])))
            h1 = sw.hstate.clone()
            qg.qg_rmsnorm_gate_up_swiglu(L.gate, L.up, sw.hstate, sw.gamma_mlp[l], sw.eps,
                                         sw.h[0])
            if check:
                x = _x_dev(h1, sw.gamma_mlp[l], cuda)
                r = wl.sample_rows(d.inter, 64, 7).tolist()
                gr, mg = oracle_gemv(L.gate, x, r)
                ur, mu = oracle_gemv(L.up, x, r)
                hr, hb = oracle.swiglu(gr, ur, mg, mu, TOL)
                assert np.all(np.abs(sw.h[0].cpu().numpy().astype(np.float64)[r] - hr) <= hb)
            hh = sw.h[0].clone()
            qg.qg_gemv_s1_residual(L.down, sw.h[0], sw.hstate)
            if check:
                yr, mag = oracle_gemv(L.down, hh, rows)
                dh = (sw.hstate.cpu().numpy().astype(np.float64) - h1.cpu().numpy())[rows]
                assert np.all(np.abs(dh - yr) <= oracle.GEMV_TOL * mag +
                              np.spacing(np.abs(sw.hstate.cpu().numpy()[rows])))
        hf = sw.hstate.clone()
        sw.run_head()
        qg.qg_stream_check()
        assert np.all(np.isfinite(hf.cpu().numpy()))
        yr, mag = oracle_gemv(sw.head, _x_dev(hf, sw.gamma_final, cuda))
        assert_within_bound(sw.logits.cpu().numpy(), yr, mag, TOL)
        tok1 = int(sw.idx.item())
        assert oracle.argmax_ok(tok1, yr)
        # two chained steps in one graph == two eager steps from the same start
        sw.idx.fill_(tok0)
        sw.step()
        sw.step()
        qg.qg_stream_check()
        eager = (int(sw.idx.item()), sw.hstate.clone(), sw.logits.clone())
        g = sw.capture(sweeps_per_graph=2)
        sw.idx.fill_(tok0)
        g.replay()
        qg.qg_stream_check()
        assert int(sw.idx.item()) == eager[0]
        assert torch.equal(sw.hstate, eager[1]) and torch.equal(sw.logits, eager[2])
        sw.idx.fill_(tok0)
        sw.step()
        qg.qg_stream_check()
        assert int(sw.idx.item()) == tok1  # the first step alone chooses tok1 again
    finally:
        del sw
        gc.collect()
        torch.cuda.empty_cache()


def _u16(t):
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("dec,ctx", [(wl.QWEN3VL_2B, 300), (wl.QWEN3VL_8B, 1025)])
def test_decode_step_with_attention(cuda, dec, ctx):
    """The whole decode step with RoPE + GQA attention over each layer's K/V
    cache (2 and 4 query heads per kv head): the attention of the first two
    layers, teacher-forced on the layer's own q|k|v output and the cache as it
    stood, is within its bound and appends the oracle's rows; the next
    projection reads the attention output; the step's argmax is the oracle's
    on the final hidden state; a graph of the step equals the eager step."""
    import gc
    from int4_quantized_decode_b200.sweep import DecodeSweep
    sw = DecodeSweep(dec, I8, I8, S=1, device=cuda, keep_logits=True, decode_step=True,
                     context=ctx)
    hd = dec.head_dim
    hq, hkv, pos = dec.q_dim // hd, dec.kv_dim // hd, ctx - 1
    try:
        tok0 = int(sw.idx.item())
        sw.run_embed()
        for l in range(2):  # op by op, as run_layer enqueues them
            L = sw.layers[l]
            kc0, vc0 = _u16(sw.kcache[l]), _u16(sw.vcache[l])
            qg.qg_rmsnorm_gemv_s1(L.qkv, sw.hstate, sw.gamma_attn[l], sw.eps, sw.y_qkv[0],
                                  sw.y16_qkv)
            qg.qg_decode_attention(sw.y_qkv[0], sw.kcache[l], sw.vcache[l], sw.pos,
                                   sw.attn_out, sw.attn_ws)
            qg.qg_stream_check()
            o_ref, mag, kn, vn = oracle.decode_attention(
                sw.y_qkv[0].cpu().numpy(), hq, hkv, hd, kc0, vc0, pos, qg.ROPE_THETA)
            od = sw.attn_out.cpu().float().numpy().astype(np.float64)
            ulp = np.array([oracle.ulp_f16(v) for v in o_ref])
            assert np.all(np.abs(od - o_ref) <= 1e-3 * mag + ulp)
            assert np.array_equal(_u16(sw.vcache[l])[:, pos, :].reshape(-1), vn)
            kd = _u16(sw.kcache[l])[:, pos, :].reshape(-1).astype(np.int32)
            assert np.all(np.abs(kd - kn.astype(np.int32)) <= 1)
            assert np.array_equal(_u16(sw.kcache[l])[:, :pos], kc0[:, :pos])
            # o adds W_o (attention output) into the residual stream
            h0 = sw.hstate.clone()
            qg.qg_gemv_s1_residual(L.o, sw.attn_out, sw.hstate)
            qg.qg_stream_check()
            rows = wl.sample_rows(dec.hidden, 32, l).tolist()
            yr, ymag = oracle_gemv(L.o, sw.attn_out, rows)
            hn = sw.hstate.cpu().numpy()
            dh = (hn.astype(np.float64) - h0.cpu().numpy())[rows]
            assert np.all(np.abs(dh - yr) <= oracle.GEMV_TOL * ymag + np.spacing(np.abs(hn[rows])))
            qg.qg_rmsnorm_gate_up_swiglu(L.gate, L.up, sw.hstate, sw.gamma_mlp[l], sw.eps,
                                         sw.h[0])
            qg.qg_gemv_s1_residual(L.down, sw.h[0], sw.hstate)
        for l in range(2, dec.layers):
            sw.run_layer(l)
        hf = sw.hstate.clone()
        sw.run_head()
        qg.qg_stream_check()
        yr, mag = oracle_gemv(sw.head, _x_dev(hf, sw.gamma_final, cuda))
        assert oracle.argmax_ok(int(sw.idx.item()), yr)
        tok1 = int(sw.idx.item())
        # the graph of one step equals the eager step from the same token
        g = sw.capture(sweeps_per_graph=1)
        sw.idx.fill_(tok0)
        sw.step()
        qg.qg_stream_check()
        eager = (int(sw.idx.item()), sw.hstate.clone(), sw.logits.clone(), sw.attn_out.clone())
        assert eager[0] == tok1
        sw.idx.fill_(tok0)
        g.replay()
        qg.qg_stream_check()
        assert int(sw.idx.item()) == eager[0]
        assert torch.equal(sw.hstate, eager[1]) and torch.equal(sw.logits, eager[2])
        assert torch.equal(sw.attn_out, eager[3])
    finally:
        del sw
        gc.collect()
        torch.cuda.empty_cache()
