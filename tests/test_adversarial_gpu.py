"""S=1 (and S=16) parity on inputs built to break careless arithmetic, at the
unchanged bound |y - y_ref| <= 2e-3 sum_k |w_dq x|:

  * outlier blocks: each int8 block-32 has one +-1 entry and 31 entries of
    N(0, 1e-3), so its codes are one +-127 and mostly 0 or +-1 (an absmax
    block dominated by one weight, "Qwen3.8-27B ... -- Core AI", Verified:
    the absmax rule keeps the outlier exact and crushes the rest);
  * quiet columns: a quarter of the columns carry weight exactly 0 in every
    row while x there is +-30000, so sum |w_dq x| ignores the largest
    activations entirely -- a kernel that accumulates an offset code (such
    as 1152 + q) and subtracts it later fails here;
  * int4 groups that straddle 0 with an exact zero level (min -1, max 0.875:
    scale 0.125 and bias -1 exact in fp16, code 8 dequantizes to 0), quiet
    columns on that level -- a kernel that forms s sum q x + b sum x cancels
    catastrophically here;
  * short rows (k = 32, 64, 96 for int8; 64, 128, 192 for int4), and rows
    spanning many tiles.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_codes_equal, assert_within_bound, bits, oracle_gemv
from int4_quantized_decode_b200 import qgemv as qg
from int4_quantized_decode_b200 import workloads as wl

pytestmark = pytest.mark.gpu
I8, I4 = qg.FMT_I8_B32, qg.FMT_I4_G64


def _case(fmt, n, k, seed, dev):
    group = 32 if fmt == I8 else 64
    quiet = wl.quiet_columns(k, seed, 64 if k % 64 == 0 else group)
    if fmt == I8:
        w = wl.outlier_weight_fp32(n, k, seed + 1, quiet, dev)
    else:
        w = wl.affine_zero_weight_fp32(n, k, seed + 1, quiet, dev)
    x = wl.spiky_act_fp16(k, seed + 2, quiet, device=dev)
    return w, qg.quantize(w, fmt), x, quiet


SHAPES = ([(I8, n, k) for n, k in [(5, 32), (77, 64), (130, 96), (300, 2048), (2050, 6144),
                                    (64, 17408)]] +
          [(I4, n, k) for n, k in [(5, 64), (77, 128), (130, 192), (300, 2560), (1000, 9728),
                                    (6001, 2560)]])


@pytest.mark.parametrize("fmt,n,k", SHAPES)
def test_gemv_adversarial(cuda, fmt, n, k):
    w, W, x, quiet = _case(fmt, n, k, 1000 + n, cuda)
    assert_codes_equal(W, w)
    if fmt == I4:  # the construction really gives the exact zero level
        assert np.all(bits(W.scales) == 0x3000) and np.all(bits(W.biases) == 0xBC00)
        assert np.all(W.codes.cpu().numpy()[:, quiet.numpy()[0::2]] & 0x0F == 8)
    y = torch.full((n,), float("nan"), dtype=torch.float32, device=cuda)
    qg.qg_gemv_s1(W, x, y)
    qg.qg_stream_check()
    yr, mag = oracle_gemv(W, x)
    assert_within_bound(y.cpu().numpy(), yr, mag)


@pytest.mark.parametrize("fmt,n,k", [(I8, 300, 2048), (I8, 41, 96), (I4, 300, 2560),
                                     (I4, 41, 192)])
def test_swiglu_adversarial(cuda, fmt, n, k):
    _, Wg, x, _ = _case(fmt, n, k, 2000 + n, cuda)
    quiet = wl.quiet_columns(k, 2000 + n, 64 if k % 64 == 0 else 32)
    wu = (wl.outlier_weight_fp32 if fmt == I8 else wl.affine_zero_weight_fp32)(
        n, k, 3000 + n, quiet, cuda)
    Wu = qg.quantize(wu, fmt)
    h = torch.empty(n, dtype=torch.float16, device=cuda)
    qg.qg_gate_up_swiglu(Wg, Wu, x, h)
    qg.qg_stream_check()
    gr, mg = oracle_gemv(Wg, x)
    ur, mu = oracle_gemv(Wu, x)
    hr, hb = oracle.swiglu(gr, ur, mg, mu, oracle.GEMV_TOL)
    err = np.abs(h.cpu().numpy().astype(np.float64) - hr)
    assert np.all(err <= hb), f"worst {np.max(err - hb)}"


@pytest.mark.parametrize("fmt,n,k", [(I8, 5000, 2048), (I8, 333, 64), (I4, 5000, 2560)])
def test_head_adversarial(cuda, fmt, n, k):
    _, W, x, _ = _case(fmt, n, k, 4000 + n, cuda)
    idx = torch.zeros(1, dtype=torch.int32, device=cuda)
    logits = torch.empty(n, dtype=torch.float32, device=cuda)
    qg.qg_head_argmax(W, x, idx, qg.head_workspace(n, cuda), logits)
    qg.qg_stream_check()
    yr, mag = oracle_gemv(W, x)
    assert_within_bound(logits.cpu().numpy(), yr, mag)
    assert oracle.argmax_ok(int(idx.item()), yr)


@pytest.mark.parametrize("n,k,S", [(300, 2048, 16), (130, 512, 5)])
def test_gemm_s16_adversarial(cuda, n, k, S):
    quiet = wl.quiet_columns(k, 5000 + n, 64)
    W = qg.quantize(wl.outlier_weight_fp32(n, k, 5001 + n, quiet, cuda), I8)
    X = torch.stack([wl.spiky_act_fp16(k, 5100 + s, quiet, device=cuda) for s in range(S)])
    Y = torch.empty((S, n), dtype=torch.float32, device=cuda)
    qg.qg_gemm_s16(W, X, Y)
    qg.qg_stream_check()
    for s in range(S):
        yr, mag = oracle_gemv(W, X[s])
        assert_within_bound(Y[s].cpu().numpy(), yr, mag)


@pytest.mark.parametrize("n,k,S", [(300, 2560, 16), (77, 512, 3)])
def test_gemm_s16_adversarial_int4(cuda, n, k, S):
    """int4 at S <= 16 on the tensor cores: groups straddling 0 with an exact
    zero level under quiet columns of +-30000 activations."""
    quiet = wl.quiet_columns(k, 6000 + n, 64)
    W = qg.quantize(wl.affine_zero_weight_fp32(n, k, 6001 + n, quiet, cuda), I4)
    X = torch.stack([wl.spiky_act_fp16(k, 6100 + s, quiet, device=cuda) for s in range(S)])
    Y = torch.empty((S, n), dtype=torch.float32, device=cuda)
    qg.qg_gemm_s16(W, X, Y)
    qg.qg_stream_check()
    for s in range(S):
        yr, mag = oracle_gemv(W, X[s])
        assert_within_bound(Y[s].cpu().numpy(), yr, mag)


@pytest.mark.parametrize("fmt,n,k,S", [(I8, 300, 2048, 16), (I8, 41, 512, 4), (I4, 300, 2560, 16),
                                       (I4, 41, 512, 4)])
def test_swiglu_s16_adversarial(cuda, fmt, n, k, S):
    """The S <= 16 gate/up (pair tiles) on the same constructions."""
    quiet = wl.quiet_columns(k, 7000 + n, 64)
    make = wl.outlier_weight_fp32 if fmt == I8 else wl.affine_zero_weight_fp32
    Wg = qg.quantize(make(n, k, 7001 + n, quiet, cuda), fmt)
    Wu = qg.quantize(make(n, k, 7002 + n, quiet, cuda), fmt)
    X = torch.stack([wl.spiky_act_fp16(k, 7100 + s, quiet, device=cuda) for s in range(S)])
    H = torch.empty((S, n), dtype=torch.float16, device=cuda)
    qg.qg_gate_up_swiglu(Wg, Wu, X, H)
    qg.qg_stream_check()
    Hd = H.cpu().numpy().astype(np.float64)
    for s in range(S):
        gr, mg = oracle_gemv(Wg, X[s])
        ur, mu = oracle_gemv(Wu, X[s])
        hr, hb = oracle.swiglu(gr, ur, mg, mu, oracle.GEMV_TOL)
        err = np.abs(Hd[s] - hr)
        assert np.all(err <= hb), f"token {s}: worst {np.max(err - hb)}"
