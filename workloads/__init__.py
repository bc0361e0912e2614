"""Seeded synthetic workloads for the hybrid linear/softmax token mixer.

This module is shared by the test oracle and by the CUDA path. It holds the
workload table and the random draws, and nothing of the method's arithmetic:
no projection, feature map, attention, gate or router lives here.

Shapes follow the video-token counts the pages describe: a 480x832 clip of 81
frames maps to 21 latent frames of 15x26 patches (N = 8,190) [ai-papers.net
summary, section "実験結果と高速化"], and 720p maps to 21 x 23 x 40 = 19,320
tokens, the "about 19,000 tokens" of the 720p setting [ai-papers.net summary,
section "ハイブリッド線形アテンション"]. No public suite is used: the pages'
VBench needs trained weights, so these synthetic tensors stand in for it.

Random numbers: one PCG64 stream per named tensor, seeded from
SeedSequence([seed, tag]) so every tensor is reproducible on its own. Values are
drawn in fp32, then rounded to the run dtype (bf16 round-to-nearest-even); the
same bytes go to the GPU and, upcast to fp64, to the oracle.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence

import numpy as np

# ---------------------------------------------------------------------------
# workload table
# ---------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class StackWorkload:
    """One hybrid-stack workload: x [B, N, D] through L mixer layers."""

    name: str
    index: int          # position in the table; seed = 1234 + index
    B: int
    N: int
    H: int
    d: int
    L: int
    dtype: str          # "f32" or "bf16"
    softmax_period: int = 4   # anchor every 4th layer
    attnres_block: int = 8    # 0 = AttnRes off
    w_std: Optional[float] = None  # default 1/sqrt(D)

    @property
    def D(self) -> int:
        return self.H * self.d

    @property
    def seed(self) -> int:
        return 1234 + self.index

    @property
    def weight_std(self) -> float:
        return self.w_std if self.w_std is not None else 1.0 / math.sqrt(self.D)


@dataclasses.dataclass(frozen=True)
class CoreWorkload:
    """An isolated attention-core workload: Q, K, V, G ~ N(0, 1) of [B, N, H*d]."""

    name: str
    index: int
    B: int
    Ns: Sequence[int]
    H: int
    d: int
    dtype: str

    @property
    def D(self) -> int:
        return self.H * self.d

    @property
    def seed(self) -> int:
        return 1234 + self.index


HYBRID4_F32 = StackWorkload("hybrid4_f32_n1024", 0, B=1, N=1024, H=4, d=64, L=4,
                            dtype="f32", attnres_block=0)
STACK480P = StackWorkload("stack480p_n8190", 1, B=1, N=8190, H=16, d=128, L=8, dtype="bf16")
STACK720P = StackWorkload("stack720p_n19320", 2, B=1, N=19320, H=24, d=128, L=24, dtype="bf16")
LONG4 = StackWorkload("long4_n37720", 3, B=1, N=37720, H=24, d=128, L=4, dtype="bf16")
LINSWEEP = CoreWorkload("linsweep_b2", 4, B=2, Ns=(4096, 19320, 75440, 150880), H=24, d=128,
                        dtype="bf16")

STACKS: Dict[str, StackWorkload] = {w.name: w for w in (HYBRID4_F32, STACK480P, STACK720P, LONG4)}

# tags of the per-tensor streams
TAG_X, TAG_Q, TAG_K, TAG_V, TAG_G, TAG_WR = 0, 10, 11, 12, 13, 300
TAG_WQKVG, TAG_WO = 100, 200
TAG_WGATE = 14        # write-gate logits [B, N, H] of an isolated linear layer
TAG_WWG = 400         # write-gate projection weights W_wg[l] [H, D] (tag 400 + l)


# ---------------------------------------------------------------------------
# rounding to the run dtype
# ---------------------------------------------------------------------------


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def round_to(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp32 values to the run dtype and return them as fp32."""
    if dtype == "f32":
        return np.ascontiguousarray(a, dtype=np.float32)
    if dtype == "bf16":
        return bf16_bits_to_f32(bf16_bits(a))
    raise ValueError(f"unknown dtype {dtype!r}")


# ---------------------------------------------------------------------------
# draws
# ---------------------------------------------------------------------------


def rng(seed: int, tag: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tag])))


def normal(shape, std: float, seed: int, tag: int, dtype: str) -> np.ndarray:
    """N(0, std^2) in fp32, rounded to `dtype`, returned as fp32."""
    a = rng(seed, tag).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return round_to(a, dtype)


def normal_par(shape, std: float, seed: int, tag: int, dtype: str, rows_per_chunk: int = 4096,
               threads: int = 0) -> np.ndarray:
    """N(0, std^2) like `normal`, for large tensors: the leading-axis-flattened
    rows are drawn in chunks of `rows_per_chunk`, chunk i from its own stream
    SeedSequence([seed, tag, i]), on a thread pool. The values depend only on
    (shape, seed, tag, rows_per_chunk), not on the number of threads."""
    import concurrent.futures as cf
    import os
    shape = tuple(shape)
    rows = int(np.prod(shape[:-1])) if len(shape) > 1 else 1
    width = shape[-1]
    out = np.empty((rows, width), dtype=np.float32)

    def fill(i):
        r0, r1 = i * rows_per_chunk, min(rows, (i + 1) * rows_per_chunk)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tag, i])))
        a = g.standard_normal(size=(r1 - r0, width), dtype=np.float32)
        if std != 1.0:
            a *= np.float32(std)
        out[r0:r1] = round_to(a, dtype)

    n = (rows + rows_per_chunk - 1) // rows_per_chunk
    with cf.ThreadPoolExecutor(threads or min(32, os.cpu_count() or 1)) as ex:
        list(ex.map(fill, range(n)))
    return out.reshape(shape)


def core_inputs_par(B: int, N: int, H: int, d: int, dtype: str, seed: int) -> Dict[str, np.ndarray]:
    """Q, K, V, G ~ N(0, 1) of [B, N, H*d] drawn with `normal_par`."""
    return {name: normal_par((B, N, H * d), 1.0, seed, tag, dtype)
            for name, tag in (("q", TAG_Q), ("k", TAG_K), ("v", TAG_V), ("g", TAG_G))}


def core_inputs(B: int, N: int, H: int, d: int, dtype: str, seed: int,
                q_scale: float = 1.0) -> Dict[str, np.ndarray]:
    """Q, K, V, gate logits G ~ N(0, 1), each [B, N, H*d]. `q_scale` scales Q
    before rounding (a peaky-softmax case)."""
    D = H * d
    out = {}
    for name, tag in (("q", TAG_Q), ("k", TAG_K), ("v", TAG_V), ("g", TAG_G)):
        std = q_scale if name == "q" else 1.0
        out[name] = normal((B, N, D), std, seed, tag, dtype)
    return out


def stack_weights(w: StackWorkload, layers: Optional[Sequence[int]] = None,
                  zero_wo: bool = False) -> Dict[str, object]:
    """W_qkvg[l] [4D, D], W_o[l] [D, D] (nn.Linear [out, in]) and W_r [D, D].

    `layers` selects which 1-based layers to draw (all by default); the others
    are None, so a sampled check can skip the cost of drawing them."""
    D, std = w.D, w.weight_std
    sel = set(range(1, w.L + 1)) if layers is None else set(layers)
    wq: List[Optional[np.ndarray]] = []
    wo: List[Optional[np.ndarray]] = []
    for l in range(1, w.L + 1):
        if l in sel:
            wq.append(normal((4 * D, D), std, w.seed, TAG_WQKVG + l, w.dtype))
            if zero_wo:
                wo.append(np.zeros((D, D), np.float32))
            else:
                wo.append(normal((D, D), std, w.seed, TAG_WO + l, w.dtype))
        else:
            wq.append(None)
            wo.append(None)
    wr = normal((D, D), std, w.seed, TAG_WR, w.dtype)
    return {"w_qkvg": wq, "w_o": wo, "w_r": wr}


def stack_x(w: StackWorkload) -> np.ndarray:
    return normal((w.B, w.N, w.D), 1.0, w.seed, TAG_X, w.dtype)


# ---------------------------------------------------------------------------
# device-side draws for bench-size tensors
# ---------------------------------------------------------------------------


def normal_torch(shape, std: float, seed: int, tag: int, dtype: str, device="cuda"):
    """N(0, std^2) drawn by torch's seeded Philox generator on `device`, rounded
    to `dtype` (torch's round-to-nearest-even). Used where numpy would take
    minutes (the 720p stack's 1.1e9 weights, the long-video activations); the
    tests copy such tensors to the host to give the oracle their exact values."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1000003 + tag) & 0x7FFFFFFFFFFFFFFF)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16) if dtype == "bf16" else t
