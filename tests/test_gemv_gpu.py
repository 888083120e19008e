"""S=1 GEMV, fused gate/up SwiGLU and fused head argmax vs the fp64 oracle.

Shapes span several tiles, ragged row tails (n not a multiple of the rows per
warp), K that is not a multiple of a stage (partial last stage), K whose
scale windows are not 16-byte aligned (scales loaded by the lanes), the
smallest legal shapes, and every rows-per-warp variant the launcher picks.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_codes_equal, assert_within_bound, bits, host_weight, oracle_gemv
from int4_quantized_decode_b200 import qgemv as qg
from int4_quantized_decode_b200 import workloads as wl

pytestmark = pytest.mark.gpu

I8, I4 = qg.FMT_I8_B32, qg.FMT_I4_G64

SHAPES_I8 = [(1, 32), (7, 96), (33, 544), (300, 2048), (1000, 2080), (4103, 512),
             (2048, 6144), (9473, 2560), (20000, 1024), (64, 17408),
             # three rows per warp item would cut the busiest warp's rows, but their
             # ring does not fit beside this x: the launcher falls back to fewer rows
             (6144, 17408),
             # rows of exactly three whole steps (the whole-step loop's copy cursor
             # moves to the next item at each item's first step), 3-4 items per warp
             (30000, 1536)]
SHAPES_I4 = [(1, 64), (9, 192), (41, 1088), (300, 2560), (1000, 1536), (4103, 1024),
             (20000, 2048), (64, 9728),
             # rows of 32 x + 16 lane granules with 2 and 4 rows per warp item
             # (the last step of each row pair packed into one warp step)
             (4103, 2560), (6001, 1536), (3000, 9728),
             # three whole int4 steps per row, 1-2 items per warp
             (12000, 3072)]


def _weight(fmt, n, k, seed, dev):
    w = wl.weight_fp32(n, k, seed, dev)
    return w, qg.quantize(w, fmt)


@pytest.mark.parametrize("fmt,n,k", [(I8, n, k) for n, k in SHAPES_I8] +
                         [(I4, n, k) for n, k in SHAPES_I4])
def test_gemv_s1_parity(cuda, fmt, n, k):
    w, W = _weight(fmt, n, k, 100 + n % 97, cuda)
    x = wl.act_fp16(k, 200 + k % 89, cuda)
    y = torch.full((n,), float("nan"), dtype=torch.float32, device=cuda)
    y16 = torch.empty(n, dtype=torch.float16, device=cuda)
    qg.qg_gemv_s1(W, x, y, y16)
    qg.qg_stream_check()
    assert_codes_equal(W, w)
    yr, mag = oracle_gemv(W, x)
    yd = y.cpu().numpy()
    assert_within_bound(yd, yr, mag)
    # y16 is the fp16 rounding (RNE) of the fp32 result
    assert np.array_equal(bits(y16), oracle.f32_to_f16_bits(yd))


@pytest.mark.parametrize("fmt", [I8, I4])
def test_gemv_y16_only_and_repeat(cuda, fmt):
    n, k = 513, 1024
    _, W = _weight(fmt, n, k, 5, cuda)
    x = wl.act_fp16(k, 6, cuda)
    y = torch.empty(n, dtype=torch.float32, device=cuda)
    qg.qg_gemv_s1(W, x, y)
    y16 = torch.empty(n, dtype=torch.float16, device=cuda)
    qg.qg_gemv_s1(W, x, None, y16)
    y2 = torch.empty_like(y)
    qg.qg_gemv_s1(W, x, y2)
    qg.qg_stream_check()
    assert torch.equal(y, y2), "repeated calls must be bitwise deterministic"
    assert np.array_equal(bits(y16), oracle.f32_to_f16_bits(y.cpu().numpy()))


def test_gemv_one_hot_and_ones_closed_forms(cuda):
    n, k = 257, 2048
    _, W = _weight(I8, n, k, 9, cuda)
    c, s, _ = host_weight(W)
    sf = s.view(np.float16).astype(np.float64)
    y = torch.empty(n, dtype=torch.float32, device=cuda)
    for j in (0, 17, 1023, 2047):
        e = torch.zeros(k, dtype=torch.float16, device=cuda)
        e[j] = 1.0
        qg.qg_gemv_s1(W, e, y)
        assert np.array_equal(y.cpu().numpy().astype(np.float64), c[:, j] * sf[:, j // 32])
    # constant weight c, x = 1: y = 127 s K sign(c), exact in fp32
    w = torch.full((4, k), -0.013, dtype=torch.float32, device=cuda)
    Wc = qg.quantize(w, I8)
    qg.qg_gemv_s1(Wc, torch.ones(k, dtype=torch.float16, device=cuda), y[:4])
    s0 = bits(Wc.scales)[0, 0:1].view(np.float16).astype(np.float64)[0]
    assert np.all(y[:4].cpu().numpy() == -127 * s0 * k)


@pytest.mark.parametrize("fmt,n,k", [(I8, 1, 32), (I8, 45, 2048), (I8, 6144, 2048),
                                     (I8, 3000, 2080), (I4, 77, 2560), (I4, 9728, 2560),
                                     (I8, 17408, 5120), (I8, 6144, 12288), (I8, 9000, 1536),
                                     (I4, 5000, 3072)])
def test_gate_up_swiglu_s1(cuda, fmt, n, k):
    wg, Wg = _weight(fmt, n, k, 31, cuda)
    wu, Wu = _weight(fmt, n, k, 32, cuda)
    x = wl.act_fp16(k, 33, cuda)
    h = torch.empty(n, dtype=torch.float16, device=cuda)
    qg.qg_gate_up_swiglu(Wg, Wu, x, h)
    qg.qg_stream_check()
    gr, mg = oracle_gemv(Wg, x)
    ur, mu = oracle_gemv(Wu, x)
    hr, hb = oracle.swiglu(gr, ur, mg, mu, oracle.GEMV_TOL)
    err = np.abs(h.cpu().numpy().astype(np.float64) - hr)
    assert np.all(err <= hb), f"worst {np.max(err / hb)}"
    # gate and up alone through the plain GEMV are within their own bounds
    g = torch.empty(n, dtype=torch.float32, device=cuda)
    qg.qg_gemv_s1(Wg, x, g)
    assert_within_bound(g.cpu().numpy(), gr, mg)


def test_swiglu_zero_gate(cuda):
    """g = 0 (all-zero gate weight) gives h = 0 exactly."""
    n, k = 100, 512
    Wg = qg.quantize(torch.zeros((n, k), dtype=torch.float32, device=cuda), I8)
    _, Wu = _weight(I8, n, k, 3, cuda)
    h = torch.full((n,), 1.0, dtype=torch.float16, device=cuda)
    qg.qg_gate_up_swiglu(Wg, Wu, wl.act_fp16(k, 4, cuda), h)
    assert torch.all(h == 0)


@pytest.mark.parametrize("fmt,n,k", [(I8, 1, 64), (I8, 100, 2048), (I8, 151936, 2048),
                                     (I4, 5000, 2560), (I8, 32003, 1056)])
def test_head_argmax(cuda, fmt, n, k):
    _, W = _weight(fmt, n, k, 41, cuda)
    x = wl.act_fp16(k, 42, cuda)
    idx = torch.full((1,), -1, dtype=torch.int32, device=cuda)
    ws = qg.head_workspace(n, cuda)
    logits = torch.empty(n, dtype=torch.float32, device=cuda)
    qg.qg_head_argmax(W, x, idx, ws, logits)
    qg.qg_stream_check()
    yr, mag = oracle_gemv(W, x)
    assert_within_bound(logits.cpu().numpy(), yr, mag)
    assert oracle.argmax_ok(int(idx.item()), yr)
    assert int(ws.sum().item()) == 0, "workspace must be left zeroed"
    # the device index is the argmax of its own logits, lowest index on ties
    ld = logits.cpu().numpy()
    assert int(idx.item()) == int(np.flatnonzero(ld == ld.max())[0])
    # no logits requested: same index
    idx2 = torch.full((1,), -1, dtype=torch.int32, device=cuda)
    qg.qg_head_argmax(W, x, idx2, ws)
    assert int(idx2.item()) == int(idx.item())


def test_head_argmax_boosted_row_and_ties(cuda):
    n, k = 40000, 512
    w = wl.weight_fp32(n, k, 51, cuda)
    x = torch.ones(k, dtype=torch.float16, device=cuda)
    ws = qg.head_workspace(n, cuda)
    idx = torch.zeros(1, dtype=torch.int32, device=cuda)
    for v in (0, 12345, n - 1):
        w2 = w.clone()
        w2[v] += 1.0                                     # row v dominates
        qg.qg_head_argmax(qg.quantize(w2, I8), x, idx, ws)
        assert int(idx.item()) == v
    # exact ties: identical rows -> the lowest index wins
    w3 = w.clone()
    w3[777] = 0.05
    w3[30001] = 0.05
    w3[20] = 0.05
    qg.qg_head_argmax(qg.quantize(w3, I8), x, idx, ws)
    assert int(idx.item()) == 20
    assert int(ws.sum().item()) == 0


def test_head_argmax_tied_embedding(cuda):
    """A tied head is the embedding table E [V, H] quantized as the head:
    logits = E_dq x (oracle fp64 on the quantized table)."""
    V, H = 8192, 2048
    E = wl.weight_fp32(V, H, wl.QWEN3VL_2B.weight_seed(-1, "head"), cuda)
    W = qg.quantize(E, I8)
    assert_codes_equal(W, E)
    x = wl.act_fp16(H, 7, cuda)
    logits = torch.empty(V, dtype=torch.float32, device=cuda)
    idx = torch.zeros(1, dtype=torch.int32, device=cuda)
    qg.qg_head_argmax(W, x, idx, qg.head_workspace(V, cuda), logits)
    c, s, _ = host_weight(W)
    Edq = c.astype(np.float64) * np.repeat(s.view(np.float16).astype(np.float64), 32, axis=1)
    ref = Edq @ x.cpu().numpy().astype(np.float64)
    yr, mag = oracle_gemv(W, x)
    np.testing.assert_allclose(yr, ref, rtol=1e-12, atol=1e-12)
    assert_within_bound(logits.cpu().numpy(), yr, mag)


# ------------------------------------------------ plain fp16 weights -------
@pytest.mark.parametrize("n,k", [(1, 8), (37, 264), (300, 2048), (4103, 2560), (151936, 2048),
                                 (20011, 4096)])
def test_fp16_weight_gemv_and_head(cuda, n, k):
    """The int8lin bundle's tied fp16 head: GEMV and head argmax straight over
    fp16 weights, vs the oracle's exact fp64 matvec of the same values."""
    w = wl.weight_fp32(n, k, 700 + n % 31, cuda).half()
    W = qg.QWeight.fp16(w)
    x = wl.act_fp16(k, 701, cuda)
    y = torch.full((n,), float("nan"), dtype=torch.float32, device=cuda)
    y16 = torch.empty(n, dtype=torch.float16, device=cuda)
    qg.qg_gemv_s1(W, x, y, y16)
    idx = torch.full((1,), -1, dtype=torch.int32, device=cuda)
    logits = torch.empty(n, dtype=torch.float32, device=cuda)
    ws = qg.head_workspace(n, cuda)
    qg.qg_head_argmax(W, x, idx, ws, logits)
    qg.qg_stream_check()
    rows = None if n <= 20011 else wl.sample_rows(n, 256, 3).tolist()
    yr, mag = oracle_gemv(W, x, rows)
    yd, ld = y.cpu().numpy(), logits.cpu().numpy()
    assert_within_bound(yd if rows is None else yd[rows], yr, mag)
    assert_within_bound(ld if rows is None else ld[rows], yr, mag)
    assert np.array_equal(bits(y16), oracle.f32_to_f16_bits(yd))
    full, _ = oracle_gemv(W, x) if rows is not None else (yr, mag)
    assert oracle.argmax_ok(int(idx.item()), full)
    assert int(ws.sum().item()) == 0


def test_fp16_weights_rejected_where_unsupported(cuda):
    W = qg.QWeight.fp16(wl.weight_fp32(64, 512, 1, cuda).half())
    X = wl.act_fp16((4, 512), 2, cuda)
    with pytest.raises(qg.QgError, match="QG_ERR_FORMAT"):
        qg.qg_gemm_s16(W, X, torch.empty((4, 64), dtype=torch.float32, device=cuda))
    with pytest.raises(qg.QgError, match="QG_ERR_FORMAT"):
        qg.qg_gate_up_swiglu(W, W, X[0], torch.empty(64, dtype=torch.float16, device=cuda))
