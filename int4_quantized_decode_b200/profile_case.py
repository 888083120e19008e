"""Launch one libqgemv kernel case a few times, for profilers.

    python -m int4_quantized_decode_b200.profile_case --op swiglu --n 6144 --k 2048
    python -m int4_quantized_decode_b200.profile_case --op attention --n 16 --k 16384
    python -m int4_quantized_decode_b200.profile_case --op sweep --decoder qwen3vl-2b

For --op attention, n is the number of query heads (8 kv heads, head_dim 128)
and k the K/V cache rows; the token sits at the last row.  --op sweep runs
the int8 S=1 weight sweep of a decoder as one persistent launch per sweep
(qg_sweep_run), `--launches` times (n and k unused).

Builds one seeded weight (two for swiglu), quantizes it, and launches the op
`--launches` times on the current device, then synchronizes.  It prints
nothing but a one-line summary, so `ncu -k regex:... -c N` can capture the
launches of exactly that kernel.
"""
from __future__ import annotations

import argparse

import torch

from . import qgemv as qg
from . import workloads as wl

OPS = ("gemv", "swiglu", "head", "s16", "s16swiglu", "quantize", "attention", "sweep")
DECODERS = {"qwen3vl-2b": wl.QWEN3VL_2B, "qwen3vl-4b": wl.QWEN3VL_4B, "qwen3vl-8b": wl.QWEN3VL_8B}


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--op", choices=OPS, required=True)
    ap.add_argument("--n", type=int, default=0)
    ap.add_argument("--k", type=int, default=0)
    ap.add_argument("--decoder", choices=sorted(DECODERS), default="qwen3vl-2b")
    ap.add_argument("--fmt", type=int, default=qg.FMT_I8_B32, choices=(0, 1))
    ap.add_argument("--S", type=int, default=16)
    ap.add_argument("--launches", type=int, default=3)
    a = ap.parse_args(argv)
    dev = torch.device("cuda:0")
    if a.op == "sweep":
        from .sweep import DecodeSweep
        sw = DecodeSweep(DECODERS[a.decoder], qg.FMT_I8_B32, qg.FMT_I8_B32, S=1, device=dev)
        sw.make_plan()
        torch.cuda.synchronize()
        for _ in range(a.launches):
            sw.step(persistent=True)
        qg.qg_stream_check()
        print(f"sweep {a.decoder} persistent x{a.launches}")
        return 0
    if a.n < 1 or a.k < 1:
        ap.error("--n and --k are required for this op")
    if a.op == "attention":
        hkv, hd = 8, 128
        kc = wl.act_fp16((hkv, a.k, hd), 11, dev)
        vc = wl.act_fp16((hkv, a.k, hd), 12, dev)
        qkv = wl.act_fp16((a.n + 2 * hkv) * hd, 13, dev).float()
        o = torch.empty(a.n * hd, dtype=torch.float16, device=dev)
        ws = qg.attention_workspace(a.n, hkv, dev)
        pos = torch.full((1,), a.k - 1, dtype=torch.int32, device=dev)
        torch.cuda.synchronize()
        for _ in range(a.launches):
            qg.qg_decode_attention(qkv, kc, vc, pos, o, ws)
        qg.qg_stream_check()
        print(f"attention hq={a.n} hkv={hkv} rows={a.k} x{a.launches}")
        return 0
    w = wl.weight_fp32(a.n, a.k, 7, dev)
    if a.op == "quantize":
        out = qg.QWeight.empty(a.fmt, a.n, a.k, dev)
        for _ in range(a.launches):
            qg.quantize(w, a.fmt, out)
        torch.cuda.synchronize()
        print(f"quantize n={a.n} k={a.k} x{a.launches}")
        return 0
    W = qg.quantize(w, a.fmt)
    del w
    W2 = qg.quantize(wl.weight_fp32(a.n, a.k, 8, dev), a.fmt) if "swiglu" in a.op else None
    S = a.S if a.op.startswith("s16") else 1
    x = wl.act_fp16((S, a.k) if S > 1 else a.k, 9, dev)
    y = torch.empty((S, a.n), dtype=torch.float32, device=dev)
    h = torch.empty((S, a.n), dtype=torch.float16, device=dev)
    idx = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = qg.head_workspace(a.n, dev)
    torch.cuda.synchronize()
    for _ in range(a.launches):
        if a.op == "gemv":
            qg.qg_gemv_s1(W, x, y[0])
        elif a.op == "swiglu":
            qg.qg_gate_up_swiglu(W, W2, x, h[0])
        elif a.op == "head":
            qg.qg_head_argmax(W, x, idx, ws)
        elif a.op == "s16":
            qg.qg_gemm_s16(W, x, y)
        else:
            qg.qg_gate_up_swiglu(W, W2, x, h)
    qg.qg_stream_check()
    print(f"{a.op} fmt={a.fmt} n={a.n} k={a.k} S={S} x{a.launches}")
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
