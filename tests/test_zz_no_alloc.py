"""qg_head_argmax_noalloc: the head argmax for callers that cannot allocate
device memory (for example a plugin whose host framework owns every device
allocation).  Called straight through the C ABI, it must give what
qg_head_argmax gives with a caller-provided workspace, on two calls in a row
with different inputs: repeated calls that share the one built-in scratch
array agree with the workspace call each time.  (A completed head call
leaves its key and ticket at zero, so these calls find the array clean; the
call's own clearing of it is there for a call that follows one that did not
complete.)  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from int4_quantized_decode_b200 import qgemv as qg
from int4_quantized_decode_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _noalloc(W, x, idx, logits, stream):
    cw = W.c()
    return qg.lib().qg_head_argmax_noalloc(ctypes.byref(cw), ctypes.c_void_p(x.data_ptr()),
                                           ctypes.c_void_p(logits.data_ptr()),
                                           ctypes.c_void_p(idx.data_ptr()),
                                           ctypes.c_void_p(stream.cuda_stream))


@pytest.mark.parametrize("fmt,n,k", [(qg.FMT_I8_B32, 151936, 2048), (qg.FMT_I4_G64, 30011, 2560)])
def test_noalloc_matches_workspace_call_twice(cuda, fmt, n, k):
    W = qg.quantize(wl.weight_fp32(n, k, 81, cuda), fmt)
    stream = torch.cuda.current_stream()
    ws = qg.head_workspace(n, cuda)
    for call, seed in enumerate((82, 83)):
        x = wl.act_fp16(k, seed, cuda)
        ref_idx = torch.full((1,), -1, dtype=torch.int32, device=cuda)
        ref_logits = torch.empty(n, dtype=torch.float32, device=cuda)
        qg.qg_head_argmax(W, x, ref_idx, ws, ref_logits)
        idx = torch.full((1,), -2, dtype=torch.int32, device=cuda)
        logits = torch.empty(n, dtype=torch.float32, device=cuda)
        assert _noalloc(W, x, idx, logits, stream) == qg.QG_OK
        qg.qg_stream_check()
        assert int(idx.item()) == int(ref_idx.item()), f"call {call}"
        np.testing.assert_allclose(logits.cpu().numpy(), ref_logits.cpu().numpy(),
                                   rtol=1e-6, atol=1e-6)


def test_noalloc_rejects_bad_arguments(cuda):
    W = qg.quantize(wl.weight_fp32(64, 64, 84, cuda), qg.FMT_I8_B32)
    x = wl.act_fp16(64, 85, cuda)
    stream = torch.cuda.current_stream()
    cw = W.c()
    L = qg.lib()
    assert L.qg_head_argmax_noalloc(None, ctypes.c_void_p(x.data_ptr()), None,
                                    ctypes.c_void_p(x.data_ptr()), None) == 1
    assert L.qg_head_argmax_noalloc(ctypes.byref(cw), ctypes.c_void_p(x.data_ptr()), None,
                                    None, ctypes.c_void_p(stream.cuda_stream)) == 1
