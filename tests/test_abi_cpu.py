"""The C-ABI library without a GPU: it loads, exports exactly what
include/qgemv.h declares, and rejects bad arguments synchronously with a status
code (validation runs on the host before any CUDA call, so these calls never
launch anything)."""
import ctypes
import os
import re
import subprocess

import pytest

from int4_quantized_decode_b200 import build as qbuild
from int4_quantized_decode_b200 import qgemv as qg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qgemv.h")


@pytest.fixture(scope="module")
def L():
    qbuild.build()
    return qg.lib()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"QG_API\s+[\w\s\*]+?\b(qg_\w+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert header_functions() == sorted(qg.ABI_SYMBOLS)


def test_library_exports_every_declared_symbol(L):
    for name in header_functions():
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", qg.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = sorted(set(m for m in re.findall(r" T (qg_\w+)", out)))
    assert exported == header_functions()


def test_status_strings_and_version(L):
    for code, name in qg.STATUS_NAMES.items():
        assert qg.status_string(code).startswith(name)
    assert qg.status_string(99) == "QG_ERR_UNKNOWN"
    assert L.qg_abi_version() == 103
    assert L.qg_head_argmax_workspace_bytes(151936) >= 16


def W(fmt=0, n=8, k=64, codes=0x1000, scales=0x2000, biases=0x3000):
    return qg.CWeight(fmt, 0, n, k, codes, scales, biases)


def gemv(L, w, x=0x4000, y=0x5000, y16=None):
    return L.qg_gemv_s1(ctypes.byref(w) if w is not None else None, x, y, y16, None)


def test_gemv_validation(L):
    assert gemv(L, None) == 1                                  # NULL weight
    assert gemv(L, W(fmt=7)) == 4                              # unknown format
    assert gemv(L, W(codes=0)) == 1
    assert gemv(L, W(scales=0)) == 1
    assert gemv(L, W(fmt=1, k=128, biases=0)) == 1             # int4 needs biases
    assert gemv(L, W(k=48)) == 2                               # k % 32
    assert gemv(L, W(fmt=1, k=96)) == 2                        # k % 64
    assert gemv(L, W(n=0)) == 2
    assert gemv(L, W(k=0)) == 2                                # empty rows
    assert gemv(L, W(n=-1)) == 2
    assert gemv(L, W(codes=0x1008)) == 3                       # 16-byte codes
    assert gemv(L, W(scales=0x2002)) == 3
    assert gemv(L, W(), x=0) == 1
    assert gemv(L, W(), y=0, y16=None) == 1                    # need an output
    assert gemv(L, W(), x=0x4008) == 3
    assert gemv(L, W(), y=0x5002) == 3


def test_gemm_s16_and_swiglu_validation(L):
    w = W()
    assert L.qg_gemm_s16(ctypes.byref(w), 0x4000, 0, 0x5000, None) == 2
    assert L.qg_gemm_s16(ctypes.byref(w), 0x4000, 17, 0x5000, None) == 2
    assert L.qg_gemm_s16(ctypes.byref(w), None, 4, 0x5000, None) == 1
    wf = W(fmt=2, k=512)                                       # fp16 weights: S == 1 only
    assert L.qg_gemm_s16(ctypes.byref(wf), 0x4000, 4, 0x5000, None) == 4
    w256 = W(k=256)                                            # S > 1 needs k % 512 == 0
    assert L.qg_gemm_s16(ctypes.byref(w256), 0x4000, 4, 0x5000, None) == 2
    w4 = W(fmt=1, k=256)                                       # int4 too (S > 1)
    assert L.qg_gemm_s16(ctypes.byref(w4), 0x4000, 4, 0x5000, None) == 2
    assert L.qg_gate_up_swiglu(ctypes.byref(w4), ctypes.byref(w4), 0x4000, 4, 0x6000, None) == 2
    wg, wu = W(), W(fmt=1, k=64)
    assert L.qg_gate_up_swiglu(ctypes.byref(wg), ctypes.byref(wu), 0x4000, 1, 0x6000, None) == 4
    wu2 = W(n=16)
    assert L.qg_gate_up_swiglu(ctypes.byref(wg), ctypes.byref(wu2), 0x4000, 1, 0x6000, None) == 2
    assert L.qg_gate_up_swiglu(ctypes.byref(wg), ctypes.byref(wg), 0x4000, 1, None, None) == 1


def test_head_and_quantize_validation(L):
    w = W()
    assert L.qg_head_argmax(ctypes.byref(w), 0x4000, None, 0x5000, None, 256, None) == 5
    assert L.qg_head_argmax(ctypes.byref(w), 0x4000, None, 0x5000, 0x7000, 8, None) == 5
    assert L.qg_head_argmax(ctypes.byref(w), 0x4000, None, None, 0x7000, 256, None) == 1
    assert L.qg_head_argmax(ctypes.byref(w), 0x4000, None, 0x5000, 0x7008, 256, None) == 3
    assert L.qg_quantize_block32(None, 4, 64, 0x1000, 0x2000, None) == 1
    assert L.qg_quantize_block32(0x1000, 4, 40, 0x1000, 0x2000, None) == 2
    assert L.qg_quantize_block32(0x1000, 0, 64, 0x1000, 0x2000, None) == 2   # no rows
    assert L.qg_quantize_int4_g64(0x1000, 0, 64, 0x1000, 0x2000, 0x3000, None) == 2
    assert L.qg_quantize_block32(0x1004, 4, 64, 0x1000, 0x2000, None) == 3
    assert L.qg_quantize_int4_g64(0x1000, 4, 64, 0x1000, 0x2000, None, None) == 1
    assert L.qg_quantize_int4_g64(0x1000, 4, 96, 0x1000, 0x2000, 0x3000, None) == 2


def stage(op=0, w=None, w_up=None, x=0x4000, y=0x5000, y16=None, h=None, logits=None, idx=None):
    return qg.CStage(op, 0, w if w is not None else W(), w_up if w_up is not None else qg.CWeight(),
                     x, y, y16, h, logits, idx)


def plan(L, stages, ws=0x10000, nbytes=None, sweep=True):
    arr = (qg.CStage * max(1, len(stages)))(*stages)
    n = len(stages)
    if nbytes is None:
        nbytes = L.qg_sweep_workspace_bytes(max(n, 1))
    out = qg.CSweep()
    return L.qg_sweep_plan(arr if stages else None, n, ws, nbytes,
                           ctypes.byref(out) if sweep else None)


def test_sweep_validation(L):
    assert L.qg_sweep_workspace_bytes(0) == 0
    assert L.qg_sweep_workspace_bytes(1) > 0
    assert L.qg_sweep_workspace_bytes(113) > L.qg_sweep_workspace_bytes(1)
    assert plan(L, []) == 1                                    # NULL stages
    assert plan(L, [stage()], sweep=False) == 1                # NULL descriptor
    arr = (qg.CStage * 1)(stage())
    out = qg.CSweep()
    assert L.qg_sweep_plan(arr, 0, 0x10000, 1 << 20, ctypes.byref(out)) == 2
    assert plan(L, [stage()], nbytes=64) == 5                  # workspace too small
    assert plan(L, [stage()], ws=None) == 5
    assert plan(L, [stage()], ws=0x10010) == 3                 # 256-byte alignment
    assert plan(L, [stage(op=9)]) == 4                         # unknown op
    assert plan(L, [stage(w=W(fmt=7))]) == 4
    assert plan(L, [stage(x=None)]) == 1
    assert plan(L, [stage(x=0x4008)]) == 3
    assert plan(L, [stage(y=None)]) == 1                       # GEMV needs an output
    assert plan(L, [stage(op=1, y=None)]) == 1                 # SwiGLU: no w_up
    assert plan(L, [stage(op=1, w_up=W(fmt=1, k=128), y=None, h=0x6000)]) == 4
    assert plan(L, [stage(op=1, w_up=W(n=16), y=None, h=0x6000)]) == 2
    assert plan(L, [stage(op=1, w_up=W(), y=None)]) == 1       # SwiGLU needs h
    assert plan(L, [stage(op=2, y=None)]) == 1                 # head needs idx
    assert plan(L, [stage(op=2, y=None, idx=0x7002)]) == 3
    # a bad stage anywhere fails the whole plan
    assert plan(L, [stage(), stage(), stage(x=None)]) == 1
    sw = qg.CSweep(1, 0)
    assert L.qg_sweep_run(ctypes.byref(sw), None, None) == 1
    assert L.qg_sweep_run(None, 0x10000, None) == 1
    assert L.qg_sweep_run(ctypes.byref(qg.CSweep(0, 0)), 0x10000, None) == 2
    assert L.qg_sweep_run(ctypes.byref(sw), 0x10010, None) == 3


def test_fp16_weight_validation(L):
    assert gemv(L, W(fmt=2, k=12, scales=0)) == 2              # rows of whole 16-byte vectors
    assert gemv(L, W(fmt=2, codes=0x1008, scales=0)) == 3
    assert gemv(L, W(fmt=2, codes=0, scales=0)) == 1
    w = W(fmt=2, k=64, scales=0)
    assert L.qg_gate_up_swiglu(ctypes.byref(w), ctypes.byref(w), 0x4000, 1, 0x6000, None) == 4
    assert L.qg_gemm_s16(ctypes.byref(w), 0x4000, 4, 0x5000, None) == 4


def test_decode_step_validation(L):
    w = W()
    h, g = 0x8000, 0x9000
    assert L.qg_embedding_gather(None, 10, 64, 0x4000, h, None) == 1
    assert L.qg_embedding_gather(0x1000, 0, 64, 0x4000, h, None) == 2
    assert L.qg_embedding_gather(0x1001, 10, 64, 0x4000, h, None) == 3
    assert L.qg_rmsnorm_gemv_s1(ctypes.byref(w), None, g, 1e-6, 0x5000, None, None) == 1
    assert L.qg_rmsnorm_gemv_s1(ctypes.byref(w), h, g, -1.0, 0x5000, None, None) == 2
    assert L.qg_rmsnorm_gemv_s1(ctypes.byref(w), h + 4, g, 1e-6, 0x5000, None, None) == 3
    assert L.qg_rmsnorm_gemv_s1(ctypes.byref(w), h, g, 1e-6, None, None, None) == 1
    assert L.qg_gemv_s1_residual(ctypes.byref(w), 0x4000, None, None) == 1
    assert L.qg_gemv_s1_residual(ctypes.byref(w), 0x4008, h, None) == 3
    wf = W(fmt=2, k=64, scales=0)
    assert L.qg_rmsnorm_gate_up_swiglu(ctypes.byref(wf), ctypes.byref(wf), h, g, 1e-6, 0x6000,
                                       None) == 4
    assert L.qg_rmsnorm_head_argmax(ctypes.byref(w), h, g, 1e-6, None, 0x7000, 0x7100, 8,
                                    None) == 5


def test_decode_attention_validation(L):
    ws_n = L.qg_decode_attention_workspace_bytes(16, 8)
    assert ws_n >= 8 * 4 + 8 * 2 * 130 * 4
    assert L.qg_decode_attention_workspace_bytes(16, 5) == 0          # hq % hkv != 0
    qkv, kc, vc, pos, o, ws = 0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 0x60000

    def call(**kw):
        a = dict(qkv=qkv, hq=16, hkv=8, d=128, kc=kc, vc=vc, l_max=64, pos=pos, theta=5e6,
                 o=o, ws=ws, ws_n=ws_n)
        a.update(kw)
        return L.qg_decode_attention(a["qkv"], a["hq"], a["hkv"], a["d"], a["kc"], a["vc"],
                                     a["l_max"], a["pos"], a["theta"], a["o"], a["ws"],
                                     a["ws_n"], None)
    assert call(qkv=None) == 1
    assert call(pos=None) == 1
    assert call(ws=None) == 1
    assert call(d=64) == 2                                 # head_dim 128 only
    assert call(hq=24) == 2                                # hq / hkv = 3
    assert call(hq=64) == 2                                # hq / hkv = 8
    assert call(l_max=0) == 2
    assert call(theta=0.0) == 2
    assert call(kc=kc + 8) == 3
    assert call(o=o + 2) == 3
    assert call(ws=ws + 16) == 3
    assert call(ws_n=ws_n - 1) == 5
