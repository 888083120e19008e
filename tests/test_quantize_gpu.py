"""Device quantizers vs the CPU oracle: codes, scales and biases bit-exact."""
import numpy as np
import pytest
import torch

from helpers import assert_codes_equal, bits
from int4_quantized_decode_b200 import qgemv as qg
from int4_quantized_decode_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,k", [(1, 32), (3, 96), (37, 2048), (129, 2560), (64, 17408)])
@pytest.mark.parametrize("seed", [0, 7])
def test_block32_random(cuda, n, k, seed):
    w = wl.weight_fp32(n, k, seed, cuda)
    W = qg.quantize(w, qg.FMT_I8_B32)
    assert_codes_equal(W, w)


@pytest.mark.parametrize("n,k", [(1, 64), (5, 192), (33, 2560), (17, 9728)])
@pytest.mark.parametrize("seed", [1, 8])
def test_int4_random(cuda, n, k, seed):
    w = wl.weight_fp32(n, k, seed, cuda)
    W = qg.quantize(w, qg.FMT_I4_G64)
    assert_codes_equal(W, w)


def _special_rows(k, device):
    rng = np.random.default_rng(3)
    w = np.zeros((8, k), dtype=np.float32)
    w[1] = 0.37                                       # constant
    w[2] = -1.25
    w[3] = 1e-4 * np.linspace(-1, 1, k)               # subnormal fp16 scales
    w[4] = rng.normal(0, 50.0, k)                     # large values
    w[5] = rng.normal(0, 0.02, k)
    w[5, ::7] = 0.0                                   # exact zeros inside blocks
    w[6, ::2] = -0.0                                  # signed zeros
    w[7] = np.round(rng.normal(0, 4, k)) * 0.5        # many exact half-integers of s
    return torch.from_numpy(w).to(device)


@pytest.mark.parametrize("fmt", [qg.FMT_I8_B32, qg.FMT_I4_G64])
def test_special_blocks(cuda, fmt):
    w = _special_rows(256, cuda)
    W = qg.quantize(w, fmt)
    assert_codes_equal(W, w)


def test_single_gemv_weight_full(cuda):
    """The single 2048 x 2048 GEMV weight (W seed 0) matches in full."""
    cfg = wl.GEMV_2048
    w = wl.weight_fp32(cfg["n"], cfg["k"], cfg["w_seed"], cuda)
    W = qg.quantize(w, qg.FMT_I8_B32)
    assert_codes_equal(W, w)
    qg.qg_stream_check()


def test_quantize_into_row_slices(cuda):
    """Quantizing into row ranges of a fused buffer equals quantizing alone."""
    a = wl.weight_fp32(128, 512, 21, cuda)
    b = wl.weight_fp32(64, 512, 22, cuda)
    fused = qg.QWeight.empty(qg.FMT_I8_B32, 192, 512, cuda)
    qg.quantize(a, qg.FMT_I8_B32, fused.rows(0, 128))
    qg.quantize(b, qg.FMT_I8_B32, fused.rows(128, 192))
    Wa = qg.quantize(a, qg.FMT_I8_B32)
    Wb = qg.quantize(b, qg.FMT_I8_B32)
    assert torch.equal(fused.codes[:128], Wa.codes) and torch.equal(fused.codes[128:], Wb.codes)
    assert np.array_equal(bits(fused.scales[128:]), bits(Wb.scales))
