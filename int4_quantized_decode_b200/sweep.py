"""One decode step's weight sweep through libqgemv, captured in a CUDA graph.

"Decode reads the whole model per token" ("Qwen3.8-27B ... -- Core AI", The
vision path / bandwidth note; "Qwen3-VL 4B -- Core AI (.aimodel)", Measured):
a sweep reads every decoder weight once.  Per layer it runs

    qkv(+output gate) GEMV  ->  o GEMV  ->  gate/up + SwiGLU  ->  down GEMV

and finishes with the LM head fused with the greedy argmax.  q|(gate)|k|v are
row-concatenated into one weight (rows are independent, so the fused matrix is
just the projections' rows one after another).  Attention and norms are not
part of the weight stream; as their stand-in, o reads fp16(q_out), each layer
takes a fresh seeded activation for qkv and gate/up, and down reads the SwiGLU
output.  With S = 16 (chunked prefill) every projection runs on the tensor-core
path with a [16, K] chunk, o reads a fresh seeded chunk, and the head reads the
chunk's last row.

With decode_step=True (S = 1) the sweep is a whole decode step minus
attention instead, carrying a real fp32 hidden state h from token to token:

    h = E[token]                                     (embedding gather)
    per layer:  qkv = W_qkv RMSNorm(h)               (y16 = fp16 q|k|v)
                h  += W_o  fp16(q)                   (attention stand-in)
                hh  = SwiGLU(W_g, W_u; RMSNorm(h))
                h  += W_down hh
    token = argmax( W_head RMSNorm(h) )               (the next step's token)

so a graph of several sweeps is an autoregressive chain.

At S = 1 the sweep runs either as 4 launches per layer + 1 (one per call, with
programmatic dependent launch between them) or as ONE persistent launch that
runs the same stages in the same order (qg_sweep_plan / qg_sweep_run); the two
give bit-identical results.

All work is enqueued through the C ABI on the current stream; this module only
allocates buffers, draws the seeded weights, and replays the graph.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List, Optional, Tuple

import torch

from . import qgemv as qg
from . import workloads as wl


@dataclass
class LayerWeights:
    qkv: qg.QWeight
    o: qg.QWeight
    gate: qg.QWeight
    up: qg.QWeight
    down: qg.QWeight


class DecodeSweep:
    """Quantized weights of a decoder plus the buffers of one sweep."""

    def __init__(self, dec: wl.Decoder, body_fmt: int = qg.FMT_I8_B32,
                 head_fmt: int = qg.FMT_I8_B32, S: int = 1, device="cuda",
                 keep_logits: bool = False, decode_step: bool = False, eps: float = 1e-6,
                 context: int = 0):
        assert 1 <= S <= 16
        self.dec, self.S, self.device = dec, S, torch.device(device)
        self.body_fmt, self.head_fmt = body_fmt, head_fmt
        if S > 1:
            assert body_fmt == qg.FMT_I8_B32 and head_fmt == qg.FMT_I8_B32
        assert body_fmt != qg.FMT_F16, "fp16 weights serve the head only"
        assert not decode_step or S == 1, "the decode step runs S = 1"
        assert context == 0 or decode_step, "attention runs inside the decode step"
        self.decode_step, self.eps, self.context = decode_step, eps, context
        self.layers: List[LayerWeights] = []
        for l in range(dec.layers):
            self.layers.append(self._make_layer(l))
        self.head = self._quantized("head", -1, dec.vocab, dec.hidden, head_fmt)
        self._make_buffers(keep_logits)
        if decode_step:
            self._make_decode_state()
        self.graph: Optional[torch.cuda.CUDAGraph] = None
        self.plan: Optional[qg.SweepPlan] = None

    # ------------------------------------------------------------ weights --
    def _quantized(self, proj: str, layer: int, n: int, k: int, fmt: int,
                   out: Optional[qg.QWeight] = None) -> qg.QWeight:
        w = wl.weight_fp32(n, k, self.dec.weight_seed(layer, proj), self.device)
        if fmt == qg.FMT_F16:  # plain fp16 weights (the int8lin bundle's tied fp16 head)
            return qg.QWeight.fp16(w.half())
        q = qg.quantize(w, fmt, out)
        del w
        return q

    def _make_layer(self, l: int) -> LayerWeights:
        d, f = self.dec, self.body_fmt
        qkv = qg.QWeight.empty(f, d.qkv_rows, d.hidden, self.device)
        r = 0
        for name, rows in d.qkv_parts():
            self._quantized(name, l, rows, d.hidden, f, qkv.rows(r, r + rows))
            r += rows
        return LayerWeights(
            qkv=qkv,
            o=self._quantized("o", l, d.hidden, d.q_dim, f),
            gate=self._quantized("gate", l, d.inter, d.hidden, f),
            up=self._quantized("up", l, d.inter, d.hidden, f),
            down=self._quantized("down", l, d.hidden, d.inter, f))

    # ------------------------------------------------------------ buffers --
    def _make_buffers(self, keep_logits: bool) -> None:
        d, S, dev = self.dec, self.S, self.device
        # every activation of a sweep lives in one or two contiguous tensors so
        # a host caller can refresh them with one copy each
        if S == 1:
            self.x_all = torch.empty((d.layers + 1, d.hidden), dtype=torch.float16, device=dev)
            for l in range(d.layers):
                self.x_all[l] = wl.act_fp16(d.hidden, d.x_seed(l), dev)
            self.x_all[d.layers] = wl.act_fp16(d.hidden, d.x_seed(-1), dev)
            self.x_o_all = None
        else:
            self.x_all = torch.empty((d.layers + 1, S, d.hidden), dtype=torch.float16, device=dev)
            for l in range(d.layers):
                self.x_all[l] = wl.act_fp16((S, d.hidden), d.chunk_seed(l), dev)
            self.x_all[d.layers] = wl.act_fp16((S, d.hidden), d.chunk_seed(-1), dev)
            self.x_o_all = torch.empty((d.layers, S, d.q_dim), dtype=torch.float16, device=dev)
            for l in range(d.layers):
                self.x_o_all[l] = wl.act_fp16((S, d.q_dim), d.chunk_seed(l) + 100000, dev)
        self.x = [self.x_all[l] for l in range(d.layers)]
        self.x_head = self.x_all[d.layers]
        self.x_o = None if self.x_o_all is None else [self.x_o_all[l] for l in range(d.layers)]
        self.y_qkv = torch.empty((S, d.qkv_rows), dtype=torch.float32, device=dev)
        self.y16_qkv = torch.empty((d.qkv_rows,), dtype=torch.float16, device=dev)
        self.y_o = torch.empty((S, d.hidden), dtype=torch.float32, device=dev)
        self.h = torch.empty((S, d.inter), dtype=torch.float16, device=dev)
        self.y_down = torch.empty((S, d.hidden), dtype=torch.float32, device=dev)
        self.logits = (torch.empty(d.vocab, dtype=torch.float32, device=dev)
                       if keep_logits else None)
        self.idx = torch.zeros(1, dtype=torch.int32, device=dev)
        self.ws = qg.head_workspace(d.vocab, dev)

    def _make_decode_state(self) -> None:
        d, dev = self.dec, self.device
        # the fp16 embedding table (for a tied head the same draw the head
        # was quantized from), the RMSNorm gains, the hidden state and token
        self.embed = wl.weight_fp32(d.vocab, d.hidden, d.weight_seed(-1, "embed"), dev).half()
        self.gamma_attn = [wl.gamma_fp16(d.hidden, d.gamma_seed(l, 0), dev) for l in range(d.layers)]
        self.gamma_mlp = [wl.gamma_fp16(d.hidden, d.gamma_seed(l, 1), dev) for l in range(d.layers)]
        self.gamma_final = wl.gamma_fp16(d.hidden, d.gamma_seed(-1, 0), dev)
        self.hstate = torch.zeros(d.hidden, dtype=torch.float32, device=dev)
        self.idx.fill_(1)  # the first step's token
        if self.context:
            # Attention over a K/V cache of `context` rows per layer: the step
            # decodes the token at the last row; rows before it are seeded
            # history (rotated keys and values ~ N(0, 1) in fp16).
            hd = d.head_dim
            assert not d.out_gate and d.q_dim % hd == 0 and d.kv_dim % hd == 0
            hkv = d.kv_dim // hd
            self.kcache, self.vcache = [], []
            for l in range(d.layers):
                self.kcache.append(wl.act_fp16((hkv, self.context, hd), d.kv_seed(l, 0), dev))
                self.vcache.append(wl.act_fp16((hkv, self.context, hd), d.kv_seed(l, 1), dev))
            self.pos = torch.full((1,), self.context - 1, dtype=torch.int32, device=dev)
            self.attn_out = torch.empty(d.q_dim, dtype=torch.float16, device=dev)
            self.attn_ws = qg.attention_workspace(d.q_dim // hd, hkv, dev)

    @property
    def kv_bytes(self) -> int:
        """K/V cache bytes one decode step's attention reads (every row up to
        and including the current position, both caches, every layer)."""
        if not self.context:
            return 0
        return self.dec.layers * 2 * self.dec.kv_dim * self.context * 2

    # ------------------------------------------------------------- sweep --
    @property
    def weight_bytes(self) -> int:
        """Algorithmic bytes one sweep streams: codes + scales (+ biases)."""
        b = sum(L.qkv.nbytes + L.o.nbytes + L.gate.nbytes + L.up.nbytes + L.down.nbytes
                for L in self.layers)
        return b + self.head.nbytes

    def launches_per_sweep(self, persistent: bool = False) -> int:
        if persistent:
            return 1
        per_layer = 5 if self.context else 4
        return per_layer * self.dec.layers + (2 if self.decode_step else 1)

    def inputs(self) -> List[torch.Tensor]:
        """The per-step input tensors (contiguous), in a fixed order: the
        activations, or for the decode step the token it starts from."""
        if self.decode_step:
            return [self.idx]
        return [self.x_all] if self.x_o_all is None else [self.x_all, self.x_o_all]

    def head_input(self) -> torch.Tensor:
        return self.x_head if self.S == 1 else self.x_head[self.S - 1]

    def layer_calls(self, l: int, stream=None) -> List[Tuple[str, int, Callable[[], None]]]:
        """Layer l's launches in run order as (kind, bytes, enqueue): kind is
        one of qkv, attention, o, gate_up, down; bytes are the algorithmic
        bytes the launch streams (weights; K/V rows for attention)."""
        d, L = self.dec, self.layers[l]
        calls: List[Tuple[str, int, Callable[[], None]]] = []
        if self.decode_step:
            h = self.hstate
            calls.append(("qkv", L.qkv.nbytes, lambda: qg.qg_rmsnorm_gemv_s1(
                L.qkv, h, self.gamma_attn[l], self.eps, self.y_qkv[0], self.y16_qkv, stream)))
            if self.context:
                calls.append(("attention", 2 * d.kv_dim * self.context * 2,
                              lambda: qg.qg_decode_attention(
                                  self.y_qkv[0], self.kcache[l], self.vcache[l], self.pos,
                                  self.attn_out, self.attn_ws, stream=stream)))
                calls.append(("o", L.o.nbytes,
                              lambda: qg.qg_gemv_s1_residual(L.o, self.attn_out, h, stream)))
            else:
                calls.append(("o", L.o.nbytes, lambda: qg.qg_gemv_s1_residual(
                    L.o, self.y16_qkv[: d.q_dim], h, stream)))
            calls.append(("gate_up", L.gate.nbytes + L.up.nbytes,
                          lambda: qg.qg_rmsnorm_gate_up_swiglu(
                              L.gate, L.up, h, self.gamma_mlp[l], self.eps, self.h[0], stream)))
            calls.append(("down", L.down.nbytes,
                          lambda: qg.qg_gemv_s1_residual(L.down, self.h[0], h, stream)))
        elif self.S == 1:
            calls.append(("qkv", L.qkv.nbytes, lambda: qg.qg_gemv_s1(
                L.qkv, self.x[l], self.y_qkv[0], self.y16_qkv, stream)))
            calls.append(("o", L.o.nbytes, lambda: qg.qg_gemv_s1(
                L.o, self.y16_qkv[: d.q_dim], self.y_o[0], None, stream)))
            calls.append(("gate_up", L.gate.nbytes + L.up.nbytes, lambda: qg.qg_gate_up_swiglu(
                L.gate, L.up, self.x[l], self.h[0], stream)))
            calls.append(("down", L.down.nbytes, lambda: qg.qg_gemv_s1(
                L.down, self.h[0], self.y_down[0], None, stream)))
        else:
            calls.append(("qkv", L.qkv.nbytes,
                          lambda: qg.qg_gemm_s16(L.qkv, self.x[l], self.y_qkv, stream)))
            calls.append(("o", L.o.nbytes,
                          lambda: qg.qg_gemm_s16(L.o, self.x_o[l], self.y_o, stream)))
            calls.append(("gate_up", L.gate.nbytes + L.up.nbytes, lambda: qg.qg_gate_up_swiglu(
                L.gate, L.up, self.x[l], self.h, stream)))
            calls.append(("down", L.down.nbytes,
                          lambda: qg.qg_gemm_s16(L.down, self.h, self.y_down, stream)))
        return calls

    def run_layer(self, l: int, stream=None) -> None:
        """Enqueue layer l's launches on `stream` (default: current): four, five with
        the attention of a decode step over a K/V cache."""
        for _, _, enqueue in self.layer_calls(l, stream):
            enqueue()

    def run_head(self, stream=None) -> None:
        if self.decode_step:
            qg.qg_rmsnorm_head_argmax(self.head, self.hstate, self.gamma_final, self.eps, self.idx,
                                      self.ws, self.logits, stream)
            return
        qg.qg_head_argmax(self.head, self.head_input(), self.idx, self.ws, self.logits, stream)

    def run_embed(self, stream=None) -> None:
        """h = E[token], the token the previous step chose."""
        qg.qg_embedding_gather(self.embed, self.idx, self.hstate, stream)

    def stages(self) -> List[qg.CStage]:
        """The S = 1 sweep as persistent-launch stages, in run_layer's order."""
        assert self.S == 1, "the persistent sweep runs S = 1 stages"
        assert not self.decode_step, "the persistent sweep has no RMSNorm or residual stages"
        d, st = self.dec, []
        for l, L in enumerate(self.layers):
            st.append(qg.stage_gemv(L.qkv, self.x[l], self.y_qkv[0], self.y16_qkv))
            st.append(qg.stage_gemv(L.o, self.y16_qkv[: d.q_dim], self.y_o[0]))
            st.append(qg.stage_swiglu(L.gate, L.up, self.x[l], self.h[0]))
            st.append(qg.stage_gemv(L.down, self.h[0], self.y_down[0]))
        st.append(qg.stage_head(self.head, self.head_input(), self.idx, self.logits))
        return st

    def make_plan(self) -> qg.SweepPlan:
        """Plan the persistent sweep (synchronous; outside stream capture)."""
        if self.plan is None:
            self.plan = qg.SweepPlan(self.stages(), [], self.device)
        return self.plan

    def step(self, stream=None, persistent: bool = False) -> None:
        """Enqueue one sweep on `stream` (default: the current stream)."""
        if persistent:
            self.make_plan().run(stream)
            return
        if self.decode_step:
            self.run_embed(stream)
        for l in range(self.dec.layers):
            self.run_layer(l, stream)
        self.run_head(stream)

    def capture(self, sweeps_per_graph: int = 1,
                persistent: bool = False) -> torch.cuda.CUDAGraph:
        """Capture `sweeps_per_graph` back-to-back sweeps into one CUDA graph."""
        if persistent:
            self.make_plan()
        s = torch.cuda.Stream(device=self.device)
        s.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(s):
            self.step(persistent=persistent)  # warm the launch paths outside capture
        torch.cuda.current_stream(self.device).wait_stream(s)
        torch.cuda.synchronize(self.device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for _ in range(sweeps_per_graph):
                self.step(persistent=persistent)
        self.graph = g
        self.sweeps_per_graph = sweeps_per_graph
        return g
