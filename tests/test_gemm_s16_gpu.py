"""S <= 16 chunked-prefill GEMM (tcgen05 tensor cores), int8 block-32 and int4
group-64 weights, vs the fp64 oracle, and the
chunk-consistency invariant: every row of the chunk agrees with the S=1 GEMV
within the same bound, and the head argmax of the last row is the same
("Qwen3.8-27B ... -- Core AI", The vision path: chunked vs S=1 prefill must
give the same greedy tokens)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_codes_equal, assert_within_bound, oracle_gemv
from int4_quantized_decode_b200 import qgemv as qg
from int4_quantized_decode_b200 import workloads as wl

pytestmark = pytest.mark.gpu
I8, I4 = qg.FMT_I8_B32, qg.FMT_I4_G64


S16_SHAPES = [(1, 512, 16), (64, 512, 16), (100, 512, 3), (1000, 2048, 16), (4096, 4096, 16),
              (6144, 4096, 7), (4096, 12288, 16), (333, 1536, 2), (2050, 1024, 16),
              (130, 2560, 16)]


@pytest.mark.parametrize("fmt,n,k,S", [(I8, n, k, S) for n, k, S in S16_SHAPES] +
                         [(I4, n, k, S) for n, k, S in S16_SHAPES])
def test_gemm_s16_parity(cuda, fmt, n, k, S):
    w = wl.weight_fp32(n, k, 300 + S, cuda)
    W = qg.quantize(w, fmt)
    X = wl.act_fp16((S, k), 400 + n % 13, cuda)
    Y = torch.full((S, n), float("nan"), dtype=torch.float32, device=cuda)
    qg.qg_gemm_s16(W, X, Y)
    qg.qg_stream_check()
    if n * k <= 16 * 2**20:
        assert_codes_equal(W, w)
    Yd = Y.cpu().numpy()
    y1 = torch.empty(n, dtype=torch.float32, device=cuda)
    for s in range(S):
        yr, mag = oracle_gemv(W, X[s])
        assert_within_bound(Yd[s], yr, mag)
        # chunk consistency: the S=1 path on the same row is within the bound too
        qg.qg_gemv_s1(W, X[s], y1)
        assert_within_bound(y1.cpu().numpy(), yr, mag)


@pytest.mark.parametrize("fmt", [I8, I4])
def test_gemm_s16_deterministic(cuda, fmt):
    n, k, S = 4096, 4096, 16
    W = qg.quantize(wl.weight_fp32(n, k, 5, cuda), fmt)
    X = wl.act_fp16((S, k), 6, cuda)
    Y1 = torch.empty((S, n), dtype=torch.float32, device=cuda)
    Y2 = torch.empty_like(Y1)
    qg.qg_gemm_s16(W, X, Y1)
    qg.qg_gemm_s16(W, X, Y2)
    qg.qg_stream_check()
    assert torch.equal(Y1, Y2)


# gate/up runs as pair tiles (64 gate + 64 up rows per tensor-core tile): the
# shapes run stream-K (three CTAs of a cluster over two pair tiles: 12288x4096,
# 12248x4096 with a ragged last tile, 9728x2560) or split K over clusters
# (77x512, 1000x2048, 6144x2048, 130x2560), with ragged pair tiles (77, 1000,
# 130, 12248 rows) and S below 16
@pytest.mark.parametrize("fmt,n,k,S", [(I8, 12288, 4096, 16), (I8, 77, 512, 5), (I8, 1000, 2048, 16),
                                       (I8, 6144, 2048, 16), (I8, 130, 2560, 11),
                                       (I8, 12248, 4096, 7), (I8, 9728, 2560, 16),
                                       (I4, 12288, 4096, 16), (I4, 77, 512, 5),
                                       (I4, 1000, 2048, 16), (I4, 9728, 2560, 9)])
def test_swiglu_s16(cuda, fmt, n, k, S):
    Wg = qg.quantize(wl.weight_fp32(n, k, 61, cuda), fmt)
    Wu = qg.quantize(wl.weight_fp32(n, k, 62, cuda), fmt)
    X = wl.act_fp16((S, k), 63, cuda)
    H = torch.empty((S, n), dtype=torch.float16, device=cuda)
    qg.qg_gate_up_swiglu(Wg, Wu, X, H)
    qg.qg_stream_check()
    Hd = H.cpu().numpy().astype(np.float64)
    h1 = torch.empty(n, dtype=torch.float16, device=cuda)
    for s in range(S):
        gr, mg = oracle_gemv(Wg, X[s])
        ur, mu = oracle_gemv(Wu, X[s])
        hr, hb = oracle.swiglu(gr, ur, mg, mu, oracle.GEMV_TOL)
        assert np.all(np.abs(Hd[s] - hr) <= hb)
        qg.qg_gate_up_swiglu(Wg, Wu, X[s], h1)               # S=1 path, same row
        assert np.all(np.abs(h1.cpu().numpy().astype(np.float64) - hr) <= hb)


def test_chunk_head_argmax_matches_s1(cuda):
    """The greedy token of a 16-token prefill chunk equals the one-token
    decode's: the head logits of the chunk's last row, computed by the S=16
    tensor-core path, are within the bound of the oracle, their argmax passes
    the margin rule, and so does the S=1 fused head argmax of the same row;
    when the oracle's top-2 gap exceeds both rows' bounds the two indices are
    the same."""
    V, H, S = 151936, 4096, 16
    Wh = qg.quantize(wl.weight_fp32(V, H, wl.QWEN3VL_8B.weight_seed(-1, "head"), cuda), I8)
    X = wl.act_fp16((S, H), 71, cuda)
    Y = torch.empty((S, V), dtype=torch.float32, device=cuda)
    qg.qg_gemm_s16(Wh, X, Y)                                # the chunk, S = 16
    i1 = torch.zeros(1, dtype=torch.int32, device=cuda)
    qg.qg_head_argmax(Wh, X[S - 1], i1, qg.head_workspace(V, cuda))  # the same token, S = 1
    qg.qg_stream_check()
    yr, mag = oracle_gemv(Wh, X[S - 1])
    last = Y[S - 1].cpu().numpy()
    assert_within_bound(last, yr, mag)
    i16 = int(np.argmax(last))
    assert oracle.argmax_ok(i16, yr)
    assert oracle.argmax_ok(int(i1.item()), yr)
    top = np.argsort(yr)[::-1][:2]
    if yr[top[0]] - yr[top[1]] > 2 * oracle.GEMV_TOL * (mag[top[0]] + mag[top[1]]):
        assert i16 == int(i1.item()) == int(top[0])
