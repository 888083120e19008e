"""Python binding of libqgemv's C ABI (include/qgemv.h).

Argument marshalling only: every function takes torch CUDA tensors, checks
dtypes and shapes, and calls the C entry point of the same name on the current
torch stream.  All arithmetic runs in the library's kernels; there is no CPU
or PyTorch fallback, and importing a function without the built library
raises at once.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqgemv.so")

QG_OK = 0
STATUS_NAMES = {0: "QG_OK", 1: "QG_ERR_NULL", 2: "QG_ERR_SHAPE", 3: "QG_ERR_ALIGN",
                4: "QG_ERR_FORMAT", 5: "QG_ERR_WORKSPACE", 6: "QG_ERR_CUDA",
                7: "QG_ERR_TIMEOUT", 8: "QG_ERR_PLAN"}
FMT_I8_B32 = 0
FMT_I4_G64 = 1
FMT_F16 = 2  # plain fp16 weights (the tied fp16 head of the int8lin bundle)

# every symbol include/qgemv.h declares
ABI_SYMBOLS = ("qg_quantize_block32", "qg_quantize_int4_g64", "qg_gemv_s1",
               "qg_gemm_s16", "qg_gate_up_swiglu", "qg_head_argmax_workspace_bytes",
               "qg_head_argmax", "qg_stream_check", "qg_status_string", "qg_abi_version",
               "qg_last_cuda_error", "qg_head_argmax_noalloc", "qg_sweep_workspace_bytes",
               "qg_sweep_plan", "qg_sweep_run", "qg_embedding_gather", "qg_rmsnorm_gemv_s1",
               "qg_rmsnorm_gate_up_swiglu", "qg_rmsnorm_head_argmax", "qg_gemv_s1_residual",
               "qg_rmsnorm_f16",
               "qg_decode_attention_workspace_bytes", "qg_decode_attention")
ROPE_THETA = 5e6  # rope theta of the pages' Qwen3-VL decoders
STAGE_GEMV, STAGE_SWIGLU, STAGE_HEAD_ARGMAX = 0, 1, 2


class QgError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = f"{fn} failed: {status_string(status)}"
        if status == 6:
            msg += f" ({lib().qg_last_cuda_error().decode()})"
        super().__init__(msg)


class CWeight(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("n", ctypes.c_int64), ("k", ctypes.c_int64),
                ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("biases", ctypes.c_void_p)]


class CStage(ctypes.Structure):
    _fields_ = [("op", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("w", CWeight), ("w_up", CWeight), ("x", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("y16", ctypes.c_void_p), ("h", ctypes.c_void_p),
                ("logits", ctypes.c_void_p), ("idx", ctypes.c_void_p)]


class CSweep(ctypes.Structure):
    _fields_ = [("n_stages", ctypes.c_int32), ("kernel", ctypes.c_int32),
                ("reserved", ctypes.c_int64 * 3)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libqgemv.so (built by int4_quantized_decode_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libqgemv.so is not built ({LIB_PATH}); run "
                "`python -m int4_quantized_decode_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        W = ctypes.POINTER(CWeight)
        L.qg_quantize_block32.argtypes = [P, I64, I64, P, P, P]
        L.qg_quantize_int4_g64.argtypes = [P, I64, I64, P, P, P, P]
        L.qg_gemv_s1.argtypes = [W, P, P, P, P]
        L.qg_gemm_s16.argtypes = [W, P, I, P, P]
        L.qg_gate_up_swiglu.argtypes = [W, W, P, I, P, P]
        L.qg_head_argmax_workspace_bytes.argtypes = [I64]
        L.qg_head_argmax_workspace_bytes.restype = ctypes.c_size_t
        L.qg_head_argmax.argtypes = [W, P, P, P, P, ctypes.c_size_t, P]
        L.qg_head_argmax_noalloc.argtypes = [W, P, P, P, P]
        L.qg_sweep_workspace_bytes.argtypes = [I]
        L.qg_sweep_workspace_bytes.restype = ctypes.c_size_t
        L.qg_sweep_plan.argtypes = [ctypes.POINTER(CStage), I, P, ctypes.c_size_t,
                                    ctypes.POINTER(CSweep)]
        L.qg_sweep_run.argtypes = [ctypes.POINTER(CSweep), P, P]
        F = ctypes.c_float
        L.qg_embedding_gather.argtypes = [P, I64, I64, P, P, P]
        L.qg_rmsnorm_gemv_s1.argtypes = [W, P, P, F, P, P, P]
        L.qg_rmsnorm_gate_up_swiglu.argtypes = [W, W, P, P, F, P, P]
        L.qg_rmsnorm_head_argmax.argtypes = [W, P, P, F, P, P, P, ctypes.c_size_t, P]
        L.qg_gemv_s1_residual.argtypes = [W, P, P, P]
        L.qg_rmsnorm_f16.argtypes = [P, P, I64, F, P, P]
        L.qg_decode_attention_workspace_bytes.argtypes = [I, I]
        L.qg_decode_attention_workspace_bytes.restype = ctypes.c_size_t
        L.qg_decode_attention.argtypes = [P, I, I, I, P, P, I64, P, ctypes.c_double, P, P,
                                          ctypes.c_size_t, P]
        L.qg_stream_check.argtypes = [P]
        L.qg_status_string.argtypes = [I]
        L.qg_status_string.restype = ctypes.c_char_p
        L.qg_abi_version.argtypes = []
        L.qg_last_cuda_error.argtypes = []
        L.qg_last_cuda_error.restype = ctypes.c_char_p
        for name in ABI_SYMBOLS:
            if name not in ("qg_head_argmax_workspace_bytes", "qg_status_string",
                            "qg_last_cuda_error", "qg_sweep_workspace_bytes",
                            "qg_decode_attention_workspace_bytes"):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().qg_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != QG_OK:
        raise QgError(fn, status)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _cuda(t: torch.Tensor, dtype, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


@dataclass
class QWeight:
    """A quantized weight [n, k] held in torch CUDA tensors."""
    fmt: int
    n: int
    k: int
    codes: torch.Tensor            # int8 [n, k], uint8 [n, k/2] or fp16 [n, k]
    scales: Optional[torch.Tensor]  # int16 (fp16 bits) [n, k/block]; None for fp16 weights
    biases: Optional[torch.Tensor] = None

    @staticmethod
    def fp16(w: torch.Tensor) -> "QWeight":
        """Plain fp16 weights [n, k] (no quantization), e.g. a tied fp16 head."""
        _cuda(w, torch.float16, "w")
        return QWeight(FMT_F16, w.shape[0], w.shape[1], w, None)

    @staticmethod
    def empty(fmt: int, n: int, k: int, device="cuda") -> "QWeight":
        if fmt == FMT_I8_B32:
            return QWeight(fmt, n, k, torch.empty((n, k), dtype=torch.int8, device=device),
                           torch.empty((n, k // 32), dtype=torch.int16, device=device))
        return QWeight(fmt, n, k, torch.empty((n, k // 2), dtype=torch.uint8, device=device),
                       torch.empty((n, k // 64), dtype=torch.int16, device=device),
                       torch.empty((n, k // 64), dtype=torch.int16, device=device))

    def rows(self, r0: int, r1: int) -> "QWeight":
        """View of rows [r0, r1) (row ranges are valid weights on their own)."""
        return QWeight(self.fmt, r1 - r0, self.k, self.codes[r0:r1],
                       None if self.scales is None else self.scales[r0:r1],
                       None if self.biases is None else self.biases[r0:r1])

    @property
    def nbytes(self) -> int:
        b = self.codes.numel() * self.codes.element_size()
        if self.scales is not None:
            b += self.scales.numel() * 2
        if self.biases is not None:
            b += self.biases.numel() * 2
        return b

    def c(self) -> CWeight:
        return CWeight(self.fmt, 0, self.n, self.k, self.codes.data_ptr(),
                       self.scales.data_ptr() if self.scales is not None else None,
                       self.biases.data_ptr() if self.biases is not None else None)


# ------------------------------------------------------------ entry points --

def qg_quantize_block32(w: torch.Tensor, out: QWeight, stream=None) -> QWeight:
    _cuda(w, torch.float32, "w")
    n, k = w.shape
    assert out.fmt == FMT_I8_B32 and out.n == n and out.k == k
    _check("qg_quantize_block32",
           lib().qg_quantize_block32(_ptr(w), n, k, _ptr(out.codes), _ptr(out.scales),
                                     _stream(stream)))
    return out


def qg_quantize_int4_g64(w: torch.Tensor, out: QWeight, stream=None) -> QWeight:
    _cuda(w, torch.float32, "w")
    n, k = w.shape
    assert out.fmt == FMT_I4_G64 and out.n == n and out.k == k
    _check("qg_quantize_int4_g64",
           lib().qg_quantize_int4_g64(_ptr(w), n, k, _ptr(out.codes), _ptr(out.scales),
                                      _ptr(out.biases), _stream(stream)))
    return out


def quantize(w: torch.Tensor, fmt: int, out: Optional[QWeight] = None, stream=None) -> QWeight:
    n, k = w.shape
    out = out if out is not None else QWeight.empty(fmt, n, k, device=w.device)
    if fmt == FMT_I8_B32:
        return qg_quantize_block32(w, out, stream)
    return qg_quantize_int4_g64(w, out, stream)


def qg_gemv_s1(W: QWeight, x: torch.Tensor, y: Optional[torch.Tensor] = None,
               y16: Optional[torch.Tensor] = None, stream=None) -> None:
    _cuda(x, torch.float16, "x")
    if y is not None:
        _cuda(y, torch.float32, "y")
    if y16 is not None:
        _cuda(y16, torch.float16, "y16")
    cw = W.c()
    _check("qg_gemv_s1", lib().qg_gemv_s1(ctypes.byref(cw), _ptr(x), _ptr(y), _ptr(y16),
                                          _stream(stream)))


def qg_gemm_s16(W: QWeight, X: torch.Tensor, Y: torch.Tensor, stream=None) -> None:
    _cuda(X, torch.float16, "X")
    _cuda(Y, torch.float32, "Y")
    S = X.shape[0]
    cw = W.c()
    _check("qg_gemm_s16", lib().qg_gemm_s16(ctypes.byref(cw), _ptr(X), S, _ptr(Y),
                                            _stream(stream)))


def qg_gate_up_swiglu(Wg: QWeight, Wu: QWeight, X: torch.Tensor, H: torch.Tensor,
                      stream=None) -> None:
    _cuda(X, torch.float16, "X")
    _cuda(H, torch.float16, "H")
    S = X.shape[0] if X.dim() == 2 else 1
    cg, cu = Wg.c(), Wu.c()
    _check("qg_gate_up_swiglu",
           lib().qg_gate_up_swiglu(ctypes.byref(cg), ctypes.byref(cu), _ptr(X), S, _ptr(H),
                                   _stream(stream)))


def qg_head_argmax_workspace_bytes(n: int) -> int:
    return int(lib().qg_head_argmax_workspace_bytes(int(n)))


def head_workspace(n: int, device="cuda") -> torch.Tensor:
    """A zeroed workspace for qg_head_argmax (it stays zeroed between calls)."""
    return torch.zeros(qg_head_argmax_workspace_bytes(n), dtype=torch.uint8, device=device)


def qg_head_argmax(W: QWeight, x: torch.Tensor, idx: torch.Tensor, workspace: torch.Tensor,
                   logits: Optional[torch.Tensor] = None, stream=None) -> None:
    _cuda(x, torch.float16, "x")
    _cuda(idx, torch.int32, "idx")
    _cuda(workspace, torch.uint8, "workspace")
    if logits is not None:
        _cuda(logits, torch.float32, "logits")
    cw = W.c()
    _check("qg_head_argmax",
           lib().qg_head_argmax(ctypes.byref(cw), _ptr(x), _ptr(logits), _ptr(idx),
                                _ptr(workspace), workspace.numel(), _stream(stream)))


def qg_head_argmax_noalloc(W: QWeight, x: torch.Tensor, idx: torch.Tensor,
                           logits: Optional[torch.Tensor] = None, stream=None) -> None:
    """qg_head_argmax without a caller workspace (the library's built-in
    scratch; calls must not overlap on the GPU)."""
    _cuda(x, torch.float16, "x")
    _cuda(idx, torch.int32, "idx")
    if logits is not None:
        _cuda(logits, torch.float32, "logits")
    cw = W.c()
    _check("qg_head_argmax_noalloc",
           lib().qg_head_argmax_noalloc(ctypes.byref(cw), _ptr(x), _ptr(logits), _ptr(idx),
                                        _stream(stream)))


def qg_stream_check(stream=None) -> None:
    _check("qg_stream_check", lib().qg_stream_check(_stream(stream)))


# ----------------------------------------------------------------- sweeps --
def stage_gemv(W: QWeight, x: torch.Tensor, y: Optional[torch.Tensor] = None,
               y16: Optional[torch.Tensor] = None) -> CStage:
    """A sweep stage equal to qg_gemv_s1(W, x, y, y16)."""
    _cuda(x, torch.float16, "x")
    if y is not None:
        _cuda(y, torch.float32, "y")
    if y16 is not None:
        _cuda(y16, torch.float16, "y16")
    return CStage(STAGE_GEMV, 0, W.c(), CWeight(), _ptr(x), _ptr(y), _ptr(y16), None, None,
                  None)


def stage_swiglu(Wg: QWeight, Wu: QWeight, x: torch.Tensor, h: torch.Tensor) -> CStage:
    """A sweep stage equal to qg_gate_up_swiglu(Wg, Wu, x, h) with S = 1."""
    _cuda(x, torch.float16, "x")
    _cuda(h, torch.float16, "h")
    return CStage(STAGE_SWIGLU, 0, Wg.c(), Wu.c(), _ptr(x), None, None, _ptr(h), None, None)


def stage_head(W: QWeight, x: torch.Tensor, idx: torch.Tensor,
               logits: Optional[torch.Tensor] = None) -> CStage:
    """A sweep stage equal to qg_head_argmax(W, x, idx, ..., logits)."""
    _cuda(x, torch.float16, "x")
    _cuda(idx, torch.int32, "idx")
    if logits is not None:
        _cuda(logits, torch.float32, "logits")
    return CStage(STAGE_HEAD_ARGMAX, 0, W.c(), CWeight(), _ptr(x), None, None, None,
                  _ptr(logits), _ptr(idx))


def qg_sweep_workspace_bytes(n_stages: int) -> int:
    return int(lib().qg_sweep_workspace_bytes(int(n_stages)))


def qg_sweep_plan(stages, workspace: torch.Tensor) -> CSweep:
    """Plan `stages` (a list of CStage) into `workspace` (a uint8 CUDA tensor,
    256-byte aligned, of at least qg_sweep_workspace_bytes(len(stages))
    bytes).  Synchronous."""
    _cuda(workspace, torch.uint8, "workspace")
    arr = (CStage * len(stages))(*stages)
    sw = CSweep()
    _check("qg_sweep_plan", lib().qg_sweep_plan(arr, len(stages), _ptr(workspace),
                                                workspace.numel(), ctypes.byref(sw)))
    return sw


def qg_sweep_run(sweep: CSweep, workspace: torch.Tensor, stream=None) -> None:
    _check("qg_sweep_run", lib().qg_sweep_run(ctypes.byref(sweep), _ptr(workspace),
                                              _stream(stream)))


class SweepPlan:
    """A planned sweep: its workspace, its host descriptor, and the tensors
    its stages point to (kept alive as long as the plan)."""

    def __init__(self, stages, tensors, device="cuda"):
        n = len(stages)
        nbytes = qg_sweep_workspace_bytes(n)
        self._buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        off = (-self._buf.data_ptr()) % 256                # a 256-byte aligned view
        self.workspace = self._buf[off:off + nbytes]
        self.n_stages = n
        self.tensors = list(tensors)
        self.sweep = qg_sweep_plan(stages, self.workspace)

    def run(self, stream=None) -> None:
        qg_sweep_run(self.sweep, self.workspace, stream)


# ------------------------------------------------------ decode-step fusions --
def qg_embedding_gather(table: torch.Tensor, token: torch.Tensor, h: torch.Tensor,
                        stream=None) -> None:
    """h = fp32(table[token]) for the device-side token id (int32 [1])."""
    _cuda(table, torch.float16, "table")
    _cuda(token, torch.int32, "token")
    _cuda(h, torch.float32, "h")
    V, H = table.shape
    _check("qg_embedding_gather", lib().qg_embedding_gather(_ptr(table), V, H, _ptr(token),
                                                            _ptr(h), _stream(stream)))


def _norm_args(h, gamma):
    _cuda(h, torch.float32, "h")
    _cuda(gamma, torch.float16, "gamma")


def qg_rmsnorm_gemv_s1(W: QWeight, h: torch.Tensor, gamma: torch.Tensor, eps: float,
                       y: Optional[torch.Tensor] = None, y16: Optional[torch.Tensor] = None,
                       stream=None) -> None:
    _norm_args(h, gamma)
    if y is not None:
        _cuda(y, torch.float32, "y")
    if y16 is not None:
        _cuda(y16, torch.float16, "y16")
    cw = W.c()
    _check("qg_rmsnorm_gemv_s1",
           lib().qg_rmsnorm_gemv_s1(ctypes.byref(cw), _ptr(h), _ptr(gamma), float(eps), _ptr(y),
                                    _ptr(y16), _stream(stream)))


def qg_rmsnorm_f16(h: torch.Tensor, gamma: torch.Tensor, eps: float, x16: torch.Tensor,
                   stream=None) -> None:
    """x16 = fp16(RMSNorm(h; gamma, eps)) as the RMSNorm-input calls stage it."""
    _norm_args(h, gamma)
    _cuda(x16, torch.float16, "x16")
    _check("qg_rmsnorm_f16", lib().qg_rmsnorm_f16(_ptr(h), _ptr(gamma), h.numel(), float(eps),
                                                  _ptr(x16), _stream(stream)))


def qg_gemv_s1_residual(W: QWeight, x: torch.Tensor, h: torch.Tensor, stream=None) -> None:
    """h += W x (the residual stream)."""
    _cuda(x, torch.float16, "x")
    _cuda(h, torch.float32, "h")
    cw = W.c()
    _check("qg_gemv_s1_residual",
           lib().qg_gemv_s1_residual(ctypes.byref(cw), _ptr(x), _ptr(h), _stream(stream)))


def qg_rmsnorm_gate_up_swiglu(Wg: QWeight, Wu: QWeight, h: torch.Tensor, gamma: torch.Tensor,
                              eps: float, H: torch.Tensor, stream=None) -> None:
    _norm_args(h, gamma)
    _cuda(H, torch.float16, "H")
    cg, cu = Wg.c(), Wu.c()
    _check("qg_rmsnorm_gate_up_swiglu",
           lib().qg_rmsnorm_gate_up_swiglu(ctypes.byref(cg), ctypes.byref(cu), _ptr(h),
                                           _ptr(gamma), float(eps), _ptr(H), _stream(stream)))


def qg_rmsnorm_head_argmax(W: QWeight, h: torch.Tensor, gamma: torch.Tensor, eps: float,
                           idx: torch.Tensor, workspace: torch.Tensor,
                           logits: Optional[torch.Tensor] = None, stream=None) -> None:
    _norm_args(h, gamma)
    _cuda(idx, torch.int32, "idx")
    _cuda(workspace, torch.uint8, "workspace")
    if logits is not None:
        _cuda(logits, torch.float32, "logits")
    cw = W.c()
    _check("qg_rmsnorm_head_argmax",
           lib().qg_rmsnorm_head_argmax(ctypes.byref(cw), _ptr(h), _ptr(gamma), float(eps),
                                        _ptr(logits), _ptr(idx), _ptr(workspace),
                                        workspace.numel(), _stream(stream)))


# ------------------------------------------------------- decode attention --
def attention_workspace(hq: int, hkv: int, device="cuda") -> torch.Tensor:
    """A zeroed workspace for qg_decode_attention (its counters stay zeroed
    between calls; the rest is scratch)."""
    n = lib().qg_decode_attention_workspace_bytes(hq, hkv)
    if n == 0:
        raise QgError("qg_decode_attention_workspace_bytes", 2)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def qg_decode_attention(qkv: torch.Tensor, kcache: torch.Tensor, vcache: torch.Tensor,
                        pos: torch.Tensor, o: torch.Tensor, workspace: torch.Tensor,
                        theta: float = ROPE_THETA, stream=None) -> None:
    """One decode step's attention: appends the token's rotated key and value
    at row *pos of the fp16 caches [hkv, l_max, d] and writes o (fp16 [hq*d])
    from the fp32 q|k|v projection output."""
    _cuda(qkv, torch.float32, "qkv")
    _cuda(kcache, torch.float16, "kcache")
    _cuda(vcache, torch.float16, "vcache")
    _cuda(pos, torch.int32, "pos")
    _cuda(o, torch.float16, "o")
    if kcache.dim() != 3 or kcache.shape != vcache.shape:
        raise ValueError("kcache and vcache must both be [hkv, l_max, d]")
    hkv, l_max, d = kcache.shape
    hq = o.numel() // d
    if o.numel() != hq * d or qkv.numel() != (hq + 2 * hkv) * d:
        raise ValueError("qkv must be [(hq + 2 hkv) d] and o [hq d]")
    _check("qg_decode_attention",
           lib().qg_decode_attention(_ptr(qkv), hq, hkv, d, _ptr(kcache), _ptr(vcache), l_max,
                                     _ptr(pos), float(theta), _ptr(o), _ptr(workspace),
                                     workspace.numel(), _stream(stream)))

