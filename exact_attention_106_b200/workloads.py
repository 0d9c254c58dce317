"""Seeded synthetic workloads for exact attention.

This module only draws random inputs and names the problem shapes; it holds
none of the attention arithmetic.  Both the CUDA path and the fp64 oracle are
fed from here, so that they see the very same bf16 values.

Recipe (shared by tests and the benchmark):
  * every tensor is drawn as float32 i.i.d. N(0, 1) with a CPU
    ``torch.Generator`` seeded per tensor, then rounded to bfloat16
    (round-to-nearest-even, torch's cast);
  * seeds: Q = base + 0, K = base + 1, V = base + 2, dO = base + 3, where
    ``base`` is 1000 x (workload number) plus 100 x (sweep point number);
  * layout is contiguous ``[B, H, N, d]``, the (batch, heads, seq_len,
    head_dim) order of the PyTorch example in "11.11 Flash Attention",
    §Using Flash Attention, and of the (B, N_h, T, D_h) shapes in
    "Flash Attention: From Theory to Implementation", introduction;
  * the "stability" workload multiplies Q by 8 on heads [H/2, H) of every
    batch, in float32 before the bf16 cast (x8 is exact in bf16).
  * a problem too large to draw whole on the host (the 64-bit offsets case)
    is drawn one head at a time for the heads that are checked
    (``make_head``: seed = base + 10 x (b x H + h) + tensor index); the
    other heads are filler of the same distribution, which cannot reach a
    checked head (every head is an independent problem).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    seed_base: int
    scale: Optional[float] = None      # None -> 1/sqrt(d)
    q_boost_heads_from: Optional[int] = None  # heads h >= this get Q*8
    q_boost: float = 8.0

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.d)

    @property
    def shape(self):
        return (self.B, self.H, self.N, self.d)

    def pairs(self) -> int:
        """Unmasked (query, key) pairs: the algorithmic work unit."""
        per_head = self.N * (self.N + 1) // 2 if self.causal else self.N * self.N
        return self.B * self.H * per_head

    def fwd_flops(self) -> int:
        """Two matmuls (QK^T and PV) of 2*d flops per unmasked pair."""
        return 4 * self.d * self.pairs()

    def bwd_flops(self) -> int:
        """Five matmuls: the recomputed QK^T plus dV, dP, dQ and dK."""
        return 10 * self.d * self.pairs()


def _seeded_normal(shape, seed: int) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float32)


def make_inputs(w: Workload, with_grad_out: bool = True, dtype: torch.dtype = torch.bfloat16):
    """Return (q, k, v, do) as contiguous CPU tensors [B,H,N,d] of ``dtype``
    (bfloat16 by default; float16 for the fp16 path), each rounded to
    nearest-even from the same float32 draw."""
    q = _seeded_normal(w.shape, w.seed_base + 0)
    if w.q_boost_heads_from is not None:
        q[:, w.q_boost_heads_from:] *= w.q_boost
    k = _seeded_normal(w.shape, w.seed_base + 1)
    v = _seeded_normal(w.shape, w.seed_base + 2)
    out = [q.to(dtype), k.to(dtype), v.to(dtype)]
    if with_grad_out:
        out.append(_seeded_normal(w.shape, w.seed_base + 3).to(dtype))
    else:
        out.append(None)
    return tuple(out)


def make_head(w: Workload, b: int, h: int, dtype: torch.dtype = torch.bfloat16):
    """(q, k, v, do) of head (b, h) alone, each [N, d], on the host."""
    base = w.seed_base + 10 * (b * w.H + h)
    return tuple(_seeded_normal((w.N, w.d), base + t).to(dtype) for t in range(4))


# ---------------------------------------------------------------------------
# The named workloads.  Sizes follow the shapes the pages use: head_dim 64/128,
# 32 heads, sequence lengths from 512 to 32768.
# ---------------------------------------------------------------------------
TINY = Workload("tiny_1x1x128x64", 1, 1, 128, 64, False, 1000, scale=1.0 / 8.0)
SMALL_CAUSAL_STABILITY = Workload("stability_2x8x1024x64_causal_q8", 2, 8, 1024, 64, True,
                                  2000, q_boost_heads_from=4)
LLAMA_BLOCK = Workload("llama_block_4x16x4096x128_causal", 4, 16, 4096, 128, True, 3000)
LONG_CONTEXT = Workload("long_context_1x32x16384x128_causal", 1, 32, 16384, 128, True, 4000)

NAMED = [TINY, SMALL_CAUSAL_STABILITY, LLAMA_BLOCK, LONG_CONTEXT]

# A second small case, past the short-row (N <= 1024) forward configuration:
# the two-sub-tile forward and the head_dim-128 backward, ragged last tile.
SMOKE_D128 = Workload("smoke_1x2x1280x128_causal", 1, 2, 1280, 128, True, 6000)

# Element offsets past 2^31: the last head of each [B, H, N, d] tensor starts
# at element (H - 1) * N * d = 2.19e9, and its rows of the padded backward
# accumulator past 2^31 elements too; N is ragged (64 full tiles + 37 rows).
# 4.4 GB per bf16 tensor, about 45 GB on the device for forward + backward.
LARGE_OFFSETS = Workload("offsets64_1x2080x8229x128_causal", 1, 2080, 8229, 128, True, 5000)

SWEEP_TOKENS = 16384
SWEEP_N = [512, 1024, 2048, 4096, 8192, 16384]


def sweep() -> List[Workload]:
    """Fixed 16384 tokens per batch: B = 16384 / N, H = 32."""
    out = []
    idx = 0
    for d in (64, 128):
        for causal in (False, True):
            for n in SWEEP_N:
                idx += 1
                out.append(Workload(
                    f"sweep_{SWEEP_TOKENS // n}x32x{n}x{d}_{'causal' if causal else 'full'}",
                    SWEEP_TOKENS // n, 32, n, d, causal, 5000 + 100 * idx))
    return out


# head_dim 256, the largest the pages mention (PyTorch SDPA's limit, "11.11
# Flash Attention", section "Using Flash Attention"); forward only.
HDIM256 = [Workload("hdim256_2x16x8192x256_causal", 2, 16, 8192, 256, True, 8000),
           Workload("hdim256_1x16x16384x256_full", 1, 16, 16384, 256, False, 8100)]

SINGLE_HEAD_32K = Workload("single_head_1x1x32768x128_full", 1, 1, 32768, 128, False, 6000)
SINGLE_HEAD_32K_CAUSAL = Workload("single_head_1x1x32768x128_causal", 1, 1, 32768, 128, True, 6100)


# ---------------------------------------------------------------------------
# Decode: Nq new queries per head against Nk cached keys and values (the
# serving use named on the pages: vLLM, TensorRT-LLM).  Q is [B, H, Nq, d],
# K and V [B, H, Nk, d]; under the causal mask the queries are the last Nq
# positions.  Same recipe: float32 N(0, 1) draws per tensor rounded to bf16.
# ---------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    H: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    seed_base: int

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def pairs(self) -> int:
        if self.causal:  # query i sees Nk - Nq + i + 1 keys
            per = self.Nq * (self.Nk - self.Nq) + self.Nq * (self.Nq + 1) // 2
        else:
            per = self.Nq * self.Nk
        return self.B * self.H * per

    def fwd_flops(self) -> int:
        return 4 * self.d * self.pairs()

    def bytes_moved(self) -> int:
        """Algorithmic HBM bytes: read Q, K, V (bf16), write O (bf16) and LSE (fp32)."""
        bh = self.B * self.H
        return bh * (2 * self.Nq * self.d * 2 + 2 * self.Nk * self.d * 2 + self.Nq * 4)


def make_decode_inputs(w: DecodeWorkload):
    """(q, k, v) as contiguous CPU bfloat16 tensors."""
    q = _seeded_normal((w.B, w.H, w.Nq, w.d), w.seed_base + 0)
    k = _seeded_normal((w.B, w.H, w.Nk, w.d), w.seed_base + 1)
    v = _seeded_normal((w.B, w.H, w.Nk, w.d), w.seed_base + 2)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


DECODE_1Q = DecodeWorkload("decode_8x32_q1_k32768x128_causal", 8, 32, 1, 32768, 128, True, 7000)
DECODE_16Q = DecodeWorkload("decode_8x32_q16_k32768x128_causal", 8, 32, 16, 32768, 128, True, 7100)
DECODES = [DECODE_1Q, DECODE_16Q]


def by_name(name: str):
    for w in NAMED + sweep() + [SINGLE_HEAD_32K, SINGLE_HEAD_32K_CAUSAL] + DECODES + HDIM256:
        if w.name == name:
            return w
    raise KeyError(name)
