"""Decode attention (qg_decode_attention) vs the fp64 oracle.

Shapes are the pages' Qwen3-VL heads (head_dim 128, 8 kv heads; 16 or 32
query heads, i.e. 2 or 4 query heads per kv head) plus one query head per kv
head, at positions that leave the split chunks ragged, with the first token
(one key), and with long caches.  The bound per output element is
    |o - o_ref| <= 1e-3 * sum_j p_j |V_j| + ulp_f16(o_ref)
(fp32 scores and softmax against fp64, then one fp16 rounding).  The rows the
call appends are checked bit for bit (the value row) or to one fp16 unit (the
rotated key, rounded from fp64 on both sides), and no other cache row may
change."""
import numpy as np
import pytest
import torch

import oracle
from int4_quantized_decode_b200 import qgemv as qg

pytestmark = pytest.mark.gpu
D = 128


def _inputs(hq, hkv, l_max, seed, dev):
    g = torch.Generator(device="cpu").manual_seed(seed)
    qkv = torch.randn((hq + 2 * hkv) * D, generator=g, dtype=torch.float32)
    kc = torch.randn((hkv, l_max, D), generator=g, dtype=torch.float32).half()
    vc = torch.randn((hkv, l_max, D), generator=g, dtype=torch.float32).half()
    return qkv.to(dev), kc.to(dev), vc.to(dev)


def _bits(t):
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _check(o, o_ref, mag):
    od = o.cpu().float().numpy().astype(np.float64)
    ulp = np.array([oracle.ulp_f16(v) for v in o_ref])
    err = np.abs(od - o_ref)
    bound = 1e-3 * mag + ulp
    assert np.all(err <= bound), f"worst {np.max(err / bound):.3f} of the bound"


def _run(hq, hkv, l_max, pos, seed, dev, theta=qg.ROPE_THETA):
    qkv, kc, vc = _inputs(hq, hkv, l_max, seed, dev)
    kc0, vc0 = kc.clone(), vc.clone()
    o = torch.full((hq * D,), float("nan"), dtype=torch.float16, device=dev)
    ws = qg.attention_workspace(hq, hkv, dev)
    p = torch.tensor([pos], dtype=torch.int32, device=dev)
    qg.qg_decode_attention(qkv, kc, vc, p, o, ws, theta)
    qg.qg_stream_check()
    o_ref, mag, k_new, v_new = oracle.decode_attention(
        qkv.cpu().numpy(), hq, hkv, D, _bits(kc0), _bits(vc0), pos, theta)
    _check(o, o_ref, mag)
    # the appended rows
    kd = _bits(kc)[:, pos, :].reshape(-1).astype(np.int32)
    assert np.all(np.abs(kd - k_new.astype(np.int32)) <= 1), "rotated key off by > 1 unit"
    assert np.array_equal(_bits(vc)[:, pos, :].reshape(-1), v_new)
    # no other row changed
    keep = torch.ones(l_max, dtype=torch.bool)
    keep[pos] = False
    assert torch.equal(kc[:, keep.to(dev)], kc0[:, keep.to(dev)])
    assert torch.equal(vc[:, keep.to(dev)], vc0[:, keep.to(dev)])
    assert int(ws[:256].sum().item()) == 0, "the per-kv-head counters must be left zeroed"
    return o


@pytest.mark.parametrize("hq,hkv,l_max,pos", [
    (16, 8, 8, 0),          # the first token: one key
    (16, 8, 64, 1),
    (16, 8, 64, 37),        # fewer positions than splits
    (32, 8, 1000, 999),     # 2B / 4B / 8B head groups, cache full
    (16, 8, 4096, 2047),
    (32, 8, 3000, 1234),    # ragged chunks
    (8, 8, 300, 150),       # one query head per kv head
    (4, 1, 700, 699),       # a single kv head: splits over one head only
])
def test_decode_attention_parity(cuda, hq, hkv, l_max, pos):
    _run(hq, hkv, l_max, pos, 1000 + pos, cuda)


def test_decode_attention_long_context(cuda):
    _run(32, 8, 32768, 32767, 7, cuda)


def test_decode_attention_steps_build_the_cache(cuda):
    """Eight decode steps from an empty cache: each step appends its row, and
    each step's output matches the oracle run on the rows the earlier steps
    wrote; the cache rows equal the oracle's appended rows (value rows bit for
    bit)."""
    hq, hkv, l_max, steps = 16, 8, 16, 8
    kc = torch.zeros((hkv, l_max, D), dtype=torch.float16, device=cuda)
    vc = torch.zeros_like(kc)
    ws = qg.attention_workspace(hq, hkv, cuda)
    o = torch.empty(hq * D, dtype=torch.float16, device=cuda)
    p = torch.zeros(1, dtype=torch.int32, device=cuda)
    g = torch.Generator(device="cpu").manual_seed(3)
    for t in range(steps):
        qkv = torch.randn((hq + 2 * hkv) * D, generator=g).to(cuda)
        kprev, vprev = _bits(kc), _bits(vc)
        p.fill_(t)
        qg.qg_decode_attention(qkv, kc, vc, p, o, ws)
        qg.qg_stream_check()
        o_ref, mag, k_new, v_new = oracle.decode_attention(
            qkv.cpu().numpy(), hq, hkv, D, kprev, vprev, t, qg.ROPE_THETA)
        _check(o, o_ref, mag)
        assert np.array_equal(_bits(vc)[:, t, :].reshape(-1), v_new)
        kd = _bits(kc)[:, t, :].reshape(-1).astype(np.int32)
        assert np.all(np.abs(kd - k_new.astype(np.int32)) <= 1)
    assert not torch.any(kc[:, steps:]) and not torch.any(vc[:, steps:])


def test_decode_attention_deterministic_and_in_graph(cuda):
    hq, hkv, l_max, pos = 32, 8, 2048, 1500
    qkv, kc, vc = _inputs(hq, hkv, l_max, 11, cuda)
    ws = qg.attention_workspace(hq, hkv, cuda)
    p = torch.tensor([pos], dtype=torch.int32, device=cuda)
    o1 = torch.empty(hq * D, dtype=torch.float16, device=cuda)
    o2 = torch.empty_like(o1)
    qg.qg_decode_attention(qkv, kc, vc, p, o1, ws)
    qg.qg_decode_attention(qkv, kc, vc, p, o2, ws)
    qg.qg_stream_check()
    assert torch.equal(o1, o2)
    s = torch.cuda.Stream(device=cuda)
    s.wait_stream(torch.cuda.current_stream(cuda))
    graph = torch.cuda.CUDAGraph()
    o3 = torch.empty_like(o1)
    with torch.cuda.graph(graph, stream=s):
        qg.qg_decode_attention(qkv, kc, vc, p, o3, ws, stream=s)
    graph.replay()
    qg.qg_stream_check()
    assert torch.equal(o3, o1)


def test_decode_attention_position_out_of_range(cuda):
    hq, hkv, l_max = 16, 8, 32
    qkv, kc, vc = _inputs(hq, hkv, l_max, 5, cuda)
    kc0, vc0 = kc.clone(), vc.clone()
    ws = qg.attention_workspace(hq, hkv, cuda)
    o = torch.zeros(hq * D, dtype=torch.float16, device=cuda)
    for bad in (l_max, -1):
        p = torch.tensor([bad], dtype=torch.int32, device=cuda)
        qg.qg_decode_attention(qkv, kc, vc, p, o, ws)
        with pytest.raises(qg.QgError, match="QG_ERR_SHAPE"):
            qg.qg_stream_check()
    assert torch.equal(kc, kc0) and torch.equal(vc, vc0) and not torch.any(o)
    assert int(ws.sum().item()) == 0  # nothing ran: not even scratch was written
    # the next call with a valid position works
    p = torch.tensor([l_max - 1], dtype=torch.int32, device=cuda)
    qg.qg_decode_attention(qkv, kc, vc, p, o, ws)
    qg.qg_stream_check()
