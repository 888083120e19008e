"""Shared helpers for the GPU parity tests: host copies of device tensors in
the oracle's dtypes, and the bound checks the tests assert."""
import numpy as np
import torch

import oracle


def bits(t: torch.Tensor) -> np.ndarray:
    """fp16/int16 tensor -> numpy uint16 bit patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def host_weight(W, rows=None):
    """(codes, scales, biases) of a QWeight on the host, optionally a row subset."""
    c, s = W.codes, W.scales
    b = W.biases
    if rows is not None:
        r = torch.as_tensor(rows, device=c.device)
        c = c.index_select(0, r)
        s = s.index_select(0, r) if s is not None else None
        b = b.index_select(0, r) if b is not None else None
    if W.fmt == 2:  # plain fp16 weights: the oracle takes their bit patterns
        return bits(c), None, None
    c = c.cpu().numpy()
    return c, bits(s), (bits(b) if b is not None else None)


def oracle_quantize(fmt, w_rows: np.ndarray):
    if fmt == 0:
        c, s = oracle.quantize_block32(w_rows)
        return c, s, None
    return oracle.quantize_int4_g64(w_rows)


def assert_codes_equal(W, w_fp32: torch.Tensor, rows=None):
    """Device codes/scales(/biases) equal the oracle's quantization of the same
    fp32 rows, bit for bit."""
    if rows is None:
        w_rows = w_fp32.cpu().numpy()
    else:
        w_rows = w_fp32.index_select(0, torch.as_tensor(rows, device=w_fp32.device)).cpu().numpy()
    dc, ds, db = host_weight(W, rows)
    oc, os_, ob = oracle_quantize(W.fmt, w_rows)
    assert np.array_equal(dc, oc), f"codes differ at {np.argwhere(dc != oc)[:5]}"
    assert np.array_equal(ds, os_), f"scales differ at {np.argwhere(ds != os_)[:5]}"
    if ob is not None:
        assert np.array_equal(db, ob), "biases differ"


def oracle_gemv(W, x16: torch.Tensor, rows=None):
    """fp64 y_ref and mag = sum |w_dq x| for (a subset of) W's rows, from the
    device codes (whose equality with the oracle's is checked separately)."""
    c, s, b = host_weight(W, rows)
    return oracle.matvec(W.fmt, c, s, b, bits(x16))


def assert_within_bound(y_dev: np.ndarray, y_ref: np.ndarray, mag: np.ndarray,
                        tol: float = oracle.GEMV_TOL):
    err = np.abs(y_dev.astype(np.float64) - y_ref)
    bad = np.nonzero(~(err <= tol * mag))[0]
    assert bad.size == 0, (f"{bad.size} rows out of bound; worst row {bad[0]}: "
                           f"dev {y_dev[bad[0]]} ref {y_ref[bad[0]]} bound {tol * mag[bad[0]]}")
    return float((err / np.maximum(mag, 1e-300)).max())
