"""Workload shapes and seeded synthetic inputs.

This module holds no arithmetic of the method: only the decoder shapes the
pages describe and seeded random draws.  Both the CUDA path and the CPU oracle
are fed from here (the oracle through host copies of the same tensors), and
nothing here quantizes, dequantizes or multiplies.

Shapes:
  * "Qwen3-VL (2B / 4B / 8B, vision-language) -- Core AI", architecture
    paragraph and size table: vocab 151 936, head_dim 128, 8 KV heads,
    SwiGLU; 2B = 28 layers, hidden 2048, 16 q-heads, SwiGLU 6144; 4B = 36
    layers, hidden 2560, 32 q-heads, SwiGLU 9728; 8B = 36 layers, hidden 4096,
    32 q-heads, SwiGLU 12288.  2B/4B tie the LM head to the embedding, 8B is
    untied ("Qwen3-VL 4B & 8B -- Core ML stateful", Gotchas).
  * "Qwen3.8-27B (VLM: text decoder + vision path) -- Core AI", intro: 64
    layers, 24 q / 4 KV heads of head_dim 256, a swish output gate (a q-sized
    projection), dense MLP 17408, untied 248 320-vocab head.  The page gives no
    hidden size; 5120 is taken, and every layer gets full-attention shapes.

Synthetic data: weights are fp32 N(0, 0.02), activations fp16 = RNE(fp32
N(0, 1)), drawn with torch.Generator on the requested device.  The pages use
real checkpoints and prompts; these seeded tensors stand in for them.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import torch

W_STD = 0.02

# proj ids used in weight seeds
PROJ_ID = {"q": 0, "k": 1, "v": 2, "o": 3, "gate": 4, "up": 5, "down": 6,
           "outgate": 7, "embed": 14, "head": 15}


@dataclass(frozen=True)
class Decoder:
    """Decoder shape: the weight matrices one decode token reads."""
    name: str
    seed_id: int
    layers: int
    hidden: int
    q_dim: int
    kv_dim: int
    inter: int
    vocab: int
    tied_head: bool
    out_gate: bool = False  # extra q-sized projection fused with q

    # --- fused row-concatenations used by the sweep -----------------------
    def qkv_parts(self) -> List[Tuple[str, int]]:
        """Row blocks of the fused q|(outgate)|k|v projection, in order."""
        parts = [("q", self.q_dim)]
        if self.out_gate:
            parts.append(("outgate", self.q_dim))
        parts += [("k", self.kv_dim), ("v", self.kv_dim)]
        return parts

    @property
    def qkv_rows(self) -> int:
        return sum(n for _, n in self.qkv_parts())

    def layer_matrices(self) -> List[Tuple[str, int, int]]:
        """(name, rows N, cols K) of every weight matrix of one layer."""
        mats = [(p, n, self.hidden) for p, n in self.qkv_parts()]
        mats += [("o", self.hidden, self.q_dim),
                 ("gate", self.inter, self.hidden),
                 ("up", self.inter, self.hidden),
                 ("down", self.hidden, self.inter)]
        return mats

    def all_matrices(self) -> List[Tuple[int, str, int, int]]:
        """(layer or -1 for the head, name, N, K) for the whole sweep."""
        out = []
        for l in range(self.layers):
            out += [(l, n, r, c) for n, r, c in self.layer_matrices()]
        out.append((-1, "head", self.vocab, self.hidden))
        return out

    def weight_count(self, include_head: bool = True) -> int:
        body = self.layers * sum(r * c for _, r, c in self.layer_matrices())
        return body + (self.vocab * self.hidden if include_head else 0)

    # --- seeds ------------------------------------------------------------
    def weight_seed(self, layer: int, proj: str) -> int:
        if proj == "head" or (proj == "embed" and self.tied_head):
            return 1000 * self.seed_id + PROJ_ID["head"]  # a tied head is the embedding
        if proj == "embed":
            return 1000 * self.seed_id + PROJ_ID["embed"]
        return 1000 * self.seed_id + 16 * layer + PROJ_ID[proj]

    def gamma_seed(self, layer: int, which: int) -> int:
        """Seed of an RMSNorm gain vector: which 0 = before attention, 1 =
        before the MLP; layer -1 = the final norm before the head."""
        return 700000 + 1000 * self.seed_id + 2 * (layer if layer >= 0 else 499) + which

    def x_seed(self, layer: int) -> int:
        """Seed of the fresh fp16 activation of layer ``layer`` (-1: head)."""
        return 500000 + 1000 * self.seed_id + (layer if layer >= 0 else 999)

    def kv_seed(self, layer: int, which: int) -> int:
        """Seed of layer ``layer``'s synthetic K (which 0) or V (which 1)
        cache history: the rows earlier decode steps would have written."""
        return 800000 + 1000 * self.seed_id + 2 * layer + which

    @property
    def head_dim(self) -> int:
        return 128  # the pages' Qwen3-VL decoders

    def chunk_seed(self, layer: int) -> int:
        """Seed of the S=16 activation chunk of layer ``layer`` (-1: head)."""
        return 600000 + 1000 * self.seed_id + (layer if layer >= 0 else 999)


QWEN3VL_2B = Decoder("qwen3vl-2b", 2, layers=28, hidden=2048, q_dim=2048,
                     kv_dim=1024, inter=6144, vocab=151936, tied_head=True)
QWEN3VL_4B = Decoder("qwen3vl-4b", 3, layers=36, hidden=2560, q_dim=4096,
                     kv_dim=1024, inter=9728, vocab=151936, tied_head=True)
QWEN3VL_8B = Decoder("qwen3vl-8b", 4, layers=36, hidden=4096, q_dim=4096,
                     kv_dim=1024, inter=12288, vocab=151936, tied_head=False)
DENSE_27B = Decoder("dense-27b", 5, layers=64, hidden=5120, q_dim=6144,
                    kv_dim=1024, inter=17408, vocab=248320, tied_head=False,
                    out_gate=True)

DECODERS = {d.name: d for d in (QWEN3VL_2B, QWEN3VL_4B, QWEN3VL_8B, DENSE_27B)}

# Single 2048 x 2048 int8 block-32 GEMV: W seed 0, x seed 1.
GEMV_2048 = dict(name="gemv-2048", n=2048, k=2048, w_seed=0, x_seed=1)


# ----------------------------------------------------------- generators ----

def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weight_fp32(n: int, k: int, seed: int, device="cpu") -> torch.Tensor:
    """fp32 N(0, 0.02) weight [n, k] (row-major, Linear.weight order)."""
    w = torch.randn((n, k), generator=_gen(seed, device), device=device,
                    dtype=torch.float32)
    return w.mul_(W_STD)


def act_fp16(shape, seed: int, device="cpu", std: float = 1.0) -> torch.Tensor:
    """fp16 activation: fp32 N(0, std) rounded to fp16 (torch's RNE cast)."""
    if isinstance(shape, int):
        shape = (shape,)
    x = torch.randn(shape, generator=_gen(seed, device), device=device,
                    dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.float16)


def sample_rows(n: int, count: int, seed: int) -> torch.Tensor:
    """Sorted distinct row indices for sampled full-size checks, always
    including the first and last row (int64, CPU)."""
    g = _gen(seed, "cpu")
    if count >= n:
        return torch.arange(n, dtype=torch.int64)
    idx = torch.randperm(n, generator=g)[: max(count - 2, 0)]
    idx = torch.cat([idx, torch.tensor([0, n - 1])])
    return torch.unique(idx).sort().values


def gamma_fp16(k: int, seed: int, device="cuda") -> torch.Tensor:
    """RMSNorm gains: fp16 = RNE(1 + 0.1 N(0, 1)) drawn like the activations."""
    return (1.0 + 0.1 * act_fp16(k, seed, device).float()).half()


# ------------------------------------------------ adversarial structure ----
# Inputs shaped to stress the S=1 arithmetic rather than to look like a
# trained model: quantization blocks dominated by one outlier (their other
# codes round to 0 or +-1), columns whose weights are exactly 0 in every row
# while the activation there is huge, and affine int4 groups that straddle 0
# with an exact zero level.  They are plain seeded draws with a fixed layout;
# no quantization arithmetic happens here.

def quiet_columns(k: int, seed: int, group: int, frac: float = 0.25) -> torch.Tensor:
    """A bool mask [k] (CPU) of columns that carry an exact-zero weight in
    every row: about `frac` of each group of `group` columns, never the
    group's first two columns (the int4 layout below keeps its extremes
    there)."""
    g = _gen(seed, "cpu")
    m = torch.rand(k, generator=g) < frac
    m.view(-1, group)[:, :2] = False
    return m


def outlier_weight_fp32(n: int, k: int, seed: int, quiet: torch.Tensor,
                        device="cpu") -> torch.Tensor:
    """fp32 [n, k]: every block of 32 along k holds one entry of magnitude 1
    (random sign, at a random position outside the quiet columns when it can)
    and entries N(0, 1e-3) elsewhere, so int8 block-32 absmax codes are one
    +-127 and mostly 0 or +-1; quiet columns are exactly 0 in every row."""
    g = _gen(seed, "cpu")
    w = torch.randn((n, k), generator=g, dtype=torch.float32).mul_(1e-3)
    blocks = k // 32
    qb = quiet.view(blocks, 32)
    pos = torch.randint(0, 32, (n, blocks), generator=g)
    # move an outlier that landed on a quiet column to the block's first column
    pos = torch.where(qb[torch.arange(blocks), pos], torch.zeros_like(pos), pos)
    sign = torch.randint(0, 2, (n, blocks), generator=g).float().mul_(2).sub_(1)
    w.scatter_(1, torch.arange(blocks) * 32 + pos, sign)
    w[:, quiet] = 0.0
    return w.to(device)


def affine_zero_weight_fp32(n: int, k: int, seed: int, quiet: torch.Tensor,
                            device="cpu") -> torch.Tensor:
    """fp32 [n, k] for int4 group-64: every group holds -1 at its first column
    and 0.875 at its second (so its affine scale is 1.875/15 = 0.125 and its
    bias -1, both exact in fp16, and the level q = 8 dequantizes to exactly
    0), quiet columns exactly 0 (code 8), and U(-1, 0.875) elsewhere."""
    g = _gen(seed, "cpu")
    w = torch.rand((n, k), generator=g, dtype=torch.float32).mul_(1.875).sub_(1.0)
    wg = w.view(n, k // 64, 64)
    wg[:, :, 0] = -1.0
    wg[:, :, 1] = 0.875
    w[:, quiet] = 0.0
    return w.to(device)


def spiky_act_fp16(k: int, seed: int, quiet: torch.Tensor, big: float = 30000.0,
                   device="cpu") -> torch.Tensor:
    """fp16 [k]: N(0, 1) with +-`big` (random sign) at the quiet columns."""
    g = _gen(seed, "cpu")
    x = torch.randn(k, generator=g, dtype=torch.float32)
    sign = torch.randint(0, 2, (k,), generator=g).float().mul_(2).sub_(1)
    x = torch.where(quiet, sign * big, x)
    return x.to(torch.float16).to(device)
