"""bench.py host logic on CPU: the workload table, the configuration each
workload reports, the byte counts it measures against, and the lookup of the
committed DRAM-traffic figure (no GPU)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from int4_quantized_decode_b200 import workloads as wl  # noqa: E402


def test_every_workload_parses_and_names_a_decoder():
    for name, spec in bench.WORKLOADS.items():
        a = bench.parse_args(["--workload", name])
        assert a.workload == name and a.gpus == 1
        dec = getattr(wl, spec[0])
        assert spec[1] in bench.FMT_NAME and spec[2] in bench.FMT_NAME
        assert spec[3] in (1, 16)
        if len(spec) > 5:               # a K/V cache only inside the decode step
            assert spec[4] is True and spec[5] > 0 and dec.q_dim % dec.head_dim == 0
    assert bench.parse_args([]).workload == bench.DEFAULT_WORKLOAD == "qwen3vl-2b"
    assert bench.parse_args(["--workload", bench.SINGLE_GEMV]).workload == "gemv-2048"


def test_config_names_what_each_workload_runs():
    for name, spec in bench.WORKLOADS.items():
        a = bench.parse_args(["--workload", name])
        dec = getattr(wl, spec[0])
        cfg = bench._config(a, dec, spec[1], spec[2], spec[3], 1)
        text = cfg["workload"]
        assert dec.name in text and f"S={spec[3]}" in text
        if bench._context(name):
            assert f"{bench._context(name)}-row" in text and "attention" in text
        elif len(spec) > 4:
            assert "minus attention" in text
        assert cfg["layers"] == dec.layers and cfg["vocab"] == dec.vocab


def test_sweep_bytes_match_the_formats():
    d = wl.QWEN3VL_2B
    i8 = bench._sweep_bytes(d, 0, 0)
    assert i8 == int(d.weight_count(include_head=False) * 1.0625 + d.vocab * d.hidden * 1.0625)
    assert i8 == 1827979264  # the 2B sweep: codes + fp16 scales of every matrix and the head
    i4 = bench._sweep_bytes(wl.QWEN3VL_4B, 1, 0)
    assert i4 == int(wl.QWEN3VL_4B.weight_count(include_head=False) * 0.5625 +
                     wl.QWEN3VL_4B.vocab * wl.QWEN3VL_4B.hidden * 1.0625)


def test_traffic_lookup_is_keyed_by_kernel_workload_and_sources():
    digest = bench.csrc_digest()
    assert len(digest) == 16 and digest == bench.csrc_digest()
    line = None
    with open(bench.PROFILE_TRAFFIC) as f:
        for raw in f:
            if raw.startswith("kernel="):
                line = dict(p.split("=", 1) for p in raw.split())
    assert line is not None and int(line["bytes_per_launch"]) > 0
    kernel = line["kernel"].replace("_", " ")
    want = float(line["bytes_per_launch"]) if line["csrc"] == digest else None
    assert bench.profiled_traffic(kernel, line["workload"]) == want
    assert bench.profiled_traffic(kernel, "no-such-workload") is None
    assert bench.profiled_traffic("no such kernel", line["workload"]) is None
