"""CPU oracle for weight-only quantized decode -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it, and the
two share no code: this wrapper loads ``liboracle.so`` built from
``oracle/oracle.c`` (plain C, fp64 where the method is exact) and hands it
numpy arrays.

Every function restates the plain definition from the pages (citations in
``oracle.h``); ``tests/test_oracle_pins.py`` pins each one against something
other than itself.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

GCC_FLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
             "-ffp-contract=off", "-fno-fast-math"]

FMT_I8_B32 = 0
FMT_I4_G64 = 1
FMT_F16 = 2  # plain fp16 weights (the tied fp16 head of the int8lin bundle)


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc) unless it is up to date."""
    fresh = (os.path.exists(_LIB)
             and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)
             and os.path.getmtime(_LIB) >= os.path.getmtime(
                 os.path.join(_HERE, "oracle.h")))
    if force or not fresh:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        D = ctypes.c_double
        L.orc_f32_to_f16.argtypes = [ctypes.c_float]
        L.orc_f32_to_f16.restype = ctypes.c_uint16
        L.orc_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.orc_f16_to_f64.restype = D
        L.orc_rint_half_even.argtypes = [ctypes.c_float]
        L.orc_rint_half_even.restype = D
        L.orc_quantize_block32.argtypes = [P, I64, I64, P, P]
        L.orc_quantize_block32.restype = None
        L.orc_quantize_int4_g64.argtypes = [P, I64, I64, P, P, P]
        L.orc_quantize_int4_g64.restype = None
        L.orc_dequant_row_i8.argtypes = [P, P, I64, I64, P]
        L.orc_dequant_row_i8.restype = None
        L.orc_dequant_row_i4.argtypes = [P, P, P, I64, I64, P]
        L.orc_dequant_row_i4.restype = None
        L.orc_matvec.argtypes = [ctypes.c_int, P, P, P, I64, I64, P, P, P]
        L.orc_matvec.restype = None
        L.orc_silu.argtypes = [D]
        L.orc_silu.restype = D
        L.orc_silu_grad.argtypes = [D]
        L.orc_silu_grad.restype = D
        L.orc_ulp_f16.argtypes = [D]
        L.orc_ulp_f16.restype = D
        L.orc_swiglu.argtypes = [P, P, P, P, I64, D, P, P]
        L.orc_swiglu.restype = None
        L.orc_argmax.argtypes = [P, I64]
        L.orc_argmax.restype = I64
        L.orc_num_threads.argtypes = []
        L.orc_set_num_threads.argtypes = [ctypes.c_int]
        L.orc_set_num_threads.restype = None
        L.orc_f64_to_f16.argtypes = [D]
        L.orc_f64_to_f16.restype = ctypes.c_uint16
        L.orc_rmsnorm.argtypes = [P, P, I64, D, P, P]
        L.orc_rmsnorm.restype = None
        L.orc_rope.argtypes = [P, I64, I64, D, P]
        L.orc_rope.restype = None
        L.orc_decode_attention.argtypes = [P, I64, I64, I64, P, P, I64, I64, D, P, P, P, P]
        L.orc_decode_attention.restype = None
        L.orc_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


# ----------------------------------------------------------------- fp16 ----

def f32_to_f16_bits(x) -> np.ndarray:
    """IEEE binary32 -> binary16 bits, RNE (oracle's own conversion)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    f = lib().orc_f32_to_f16
    out = np.empty(x.shape, dtype=np.uint16)
    flat, oflat = x.reshape(-1), out.reshape(-1)
    for i in range(flat.size):
        oflat[i] = f(float(flat[i]))
    return out


def f16_bits_to_f64(h) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    f = lib().orc_f16_to_f64
    out = np.empty(h.shape, dtype=np.float64)
    flat, oflat = h.reshape(-1), out.reshape(-1)
    for i in range(flat.size):
        oflat[i] = f(int(flat[i]))
    return out


def rint_half_even(r: float) -> float:
    return lib().orc_rint_half_even(float(np.float32(r)))


# ------------------------------------------------------------ quantizers ---

def quantize_block32(w: np.ndarray):
    """int8 per-block-32 symmetric absmax -> (codes int8 [n,k], scales u16 [n,k/32])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, k = w.shape
    assert k % 32 == 0
    codes = np.empty((n, k), dtype=np.int8)
    scales = np.empty((n, k // 32), dtype=np.uint16)
    lib().orc_quantize_block32(_p(w), n, k, _p(codes), _p(scales))
    return codes, scales


def quantize_int4_g64(w: np.ndarray):
    """int4 group-64 affine -> (codes u8 [n,k/2], scales u16 [n,k/64], biases u16 [n,k/64])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, k = w.shape
    assert k % 64 == 0
    codes = np.empty((n, k // 2), dtype=np.uint8)
    scales = np.empty((n, k // 64), dtype=np.uint16)
    biases = np.empty((n, k // 64), dtype=np.uint16)
    lib().orc_quantize_int4_g64(_p(w), n, k, _p(codes), _p(scales), _p(biases))
    return codes, scales, biases


def dequant_i8(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    n, k = codes.shape
    out = np.empty((n, k), dtype=np.float64)
    for r in range(n):
        lib().orc_dequant_row_i8(_p(codes), _p(scales), k, r,
                                 out[r].ctypes.data_as(ctypes.c_void_p))
    return out


def dequant_i4(codes: np.ndarray, scales: np.ndarray, biases: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    biases = np.ascontiguousarray(biases, dtype=np.uint16)
    n, k2 = codes.shape
    k = 2 * k2
    out = np.empty((n, k), dtype=np.float64)
    for r in range(n):
        lib().orc_dequant_row_i4(_p(codes), _p(scales), _p(biases), k, r,
                                 out[r].ctypes.data_as(ctypes.c_void_p))
    return out


# ---------------------------------------------------------------- matvec ---

def matvec(fmt: int, codes, scales, biases, x_bits):
    """fp64 dequantize-then-matvec: returns (y [n], mag [n]) with
    y[r] = sum_k w_dq[r,k] x[k] and mag[r] = sum_k |w_dq[r,k] x[k]|."""
    codes = np.ascontiguousarray(codes)
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    n = codes.shape[0]
    if fmt == FMT_F16:  # plain fp16 weights: codes are the fp16 bits [n, k]
        assert codes.dtype == np.uint16
        k = codes.shape[1]
        assert x_bits.shape == (k,)
        y = np.empty(n, dtype=np.float64)
        mag = np.empty(n, dtype=np.float64)
        lib().orc_matvec(fmt, _p(codes), None, None, n, k, _p(x_bits), _p(y), _p(mag))
        return y, mag
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    if fmt == FMT_I8_B32:
        assert codes.dtype == np.int8
        k = codes.shape[1]
        bp = None
    else:
        assert codes.dtype == np.uint8
        k = 2 * codes.shape[1]
        biases = np.ascontiguousarray(biases, dtype=np.uint16)
        bp = _p(biases)
    assert x_bits.shape == (k,)
    y = np.empty(n, dtype=np.float64)
    mag = np.empty(n, dtype=np.float64)
    lib().orc_matvec(fmt, _p(codes), _p(scales), bp, n, k, _p(x_bits), _p(y), _p(mag))
    return y, mag


# ------------------------------------------------------- SwiGLU / argmax ---

def silu(g: float) -> float:
    return lib().orc_silu(float(g))


def silu_grad(g: float) -> float:
    return lib().orc_silu_grad(float(g))


def ulp_f16(v: float) -> float:
    return lib().orc_ulp_f16(float(v))


def swiglu(g, u, mag_g, mag_u, tol: float):
    """h = silu(g) * u (fp64) and the per-element bound (see oracle.h)."""
    g = np.ascontiguousarray(g, dtype=np.float64)
    u = np.ascontiguousarray(u, dtype=np.float64)
    mag_g = np.ascontiguousarray(mag_g, dtype=np.float64)
    mag_u = np.ascontiguousarray(mag_u, dtype=np.float64)
    n = g.shape[0]
    h = np.empty(n, dtype=np.float64)
    bound = np.empty(n, dtype=np.float64)
    lib().orc_swiglu(_p(g), _p(u), _p(mag_g), _p(mag_u), n, float(tol), _p(h), _p(bound))
    return h, bound


def num_threads() -> int:
    return int(lib().orc_num_threads())


def set_num_threads(n: int) -> None:
    """Threads the oracle's parallel loops use from now on."""
    lib().orc_set_num_threads(int(n))


def argmax(v) -> int:
    v = np.ascontiguousarray(v, dtype=np.float64)
    return int(lib().orc_argmax(_p(v), v.shape[0]))


# ----------------------------------------------------------- the gates ----

# Float outputs: |y - y_ref| <= GEMV_TOL * sum_k |w_dq x| per row.
GEMV_TOL = 2e-3
# Greedy argmax: a device index within this logit margin of the max passes.
ARGMAX_MARGIN = 1e-3


def argmax_ok(idx: int, logits_ref: np.ndarray, margin: float = ARGMAX_MARGIN) -> bool:
    """The device's greedy token passes if it is the oracle's (smallest index of
    the max) or if its oracle logit is within ``margin`` of the max: the
    analogue of the pages' teacher-forced margin rule for knife-edge ties."""
    ref = argmax(logits_ref)
    if idx == ref:
        return True
    if not (0 <= idx < logits_ref.shape[0]):
        return False
    return bool(logits_ref[idx] >= logits_ref[ref] - margin)


# ------------------------------------------------- RMSNorm / fp64 -> fp16 ---

def f64_to_f16_bits(x) -> np.ndarray:
    """fp64 -> fp16 bit patterns, one IEEE round-to-nearest-even."""
    a = np.asarray(x, dtype=np.float64)
    f = lib().orc_f64_to_f16
    return np.array([f(float(v)) for v in a.ravel()], dtype=np.uint16).reshape(a.shape)


def rmsnorm(h, gamma_bits, eps: float):
    """The decoder's pre-norm RMSNorm: (x fp16 bits [k], x before rounding fp64 [k])
    for an fp32 hidden state h and fp16 gains."""
    h = np.ascontiguousarray(h, dtype=np.float32)
    g = np.ascontiguousarray(gamma_bits, dtype=np.uint16)
    k = h.shape[0]
    assert g.shape == (k,)
    x = np.empty(k, dtype=np.uint16)
    xe = np.empty(k, dtype=np.float64)
    lib().orc_rmsnorm(_p(h), _p(g), k, float(eps), _p(x), _p(xe))
    return x, xe


def rope(x, pos: int, theta: float):
    """RoPE (rotate-half pairing) of one head vector at position pos, fp64."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty_like(x)
    lib().orc_rope(_p(x), x.shape[0], int(pos), float(theta), _p(out))
    return out


def decode_attention(qkv, hq: int, hkv: int, d: int, kcache, vcache, pos: int, theta: float):
    """One decode step's attention (see orc_decode_attention): returns
    (o fp64 [hq*d], mag fp64 [hq*d], k_new fp16 bits [hkv*d], v_new fp16 bits [hkv*d]).
    kcache / vcache: fp16 bits [hkv, l_max, d]; rows 0..pos-1 are read."""
    qkv = np.ascontiguousarray(qkv, dtype=np.float32)
    kc = np.ascontiguousarray(kcache, dtype=np.uint16)
    vc = np.ascontiguousarray(vcache, dtype=np.uint16)
    assert qkv.shape == ((hq + 2 * hkv) * d,) and hq % hkv == 0
    assert kc.shape == vc.shape and kc.shape[0] == hkv and kc.shape[2] == d
    l_max = kc.shape[1]
    assert 0 <= pos < l_max
    o = np.empty(hq * d, dtype=np.float64)
    mag = np.empty(hq * d, dtype=np.float64)
    k_new = np.empty(hkv * d, dtype=np.uint16)
    v_new = np.empty(hkv * d, dtype=np.uint16)
    lib().orc_decode_attention(_p(qkv), hq, hkv, d, _p(kc), _p(vc), l_max, int(pos),
                               float(theta), _p(k_new), _p(v_new), _p(o), _p(mag))
    return o, mag, k_new, v_new
