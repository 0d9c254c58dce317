"""GPU parity on seeded random shapes: lengths 1..3000, head_dim 64/128, 1..12
(batch, head) pairs, causal or not, scales 0.05..0.3.  Between them they reach
every launch form (lean and two-sub-tile forward; persistent and one-CTA-per-
tile backward, with even and odd key-tile counts and fewer units than SMs)
with ragged tails.  Same tolerances as the other parity tests."""
import math
import random

import pytest
import torch

from parity_util import check_all, oracle_ref, run_cuda

pytestmark = pytest.mark.gpu


def _cases(n=24, seed=2026):
    rng = random.Random(seed)
    out = []
    for i in range(n):
        N = rng.choice([rng.randint(1, 300), rng.randint(300, 1100), rng.randint(1100, 3000)])
        d = rng.choice([64, 128])
        B = rng.randint(1, 3)
        H = rng.randint(1, 4)
        causal = rng.random() < 0.5
        scale = round(rng.uniform(0.05, 0.3), 4)
        out.append((i, B, H, N, d, causal, scale))
    return out


@pytest.mark.parametrize("case", _cases(), ids=lambda c: f"{c[0]}-{c[1]}x{c[2]}x{c[3]}x{c[4]}-{'c' if c[5] else 'f'}")
def test_random_shape(cuda_device, case):
    i, B, H, N, d, causal, scale = case
    g = torch.Generator().manual_seed(7000 + i)
    q, k, v, do = (torch.randn((B, H, N, d), generator=g).bfloat16() for _ in range(4))
    got = run_cuda(q, k, v, do, causal, scale)
    check_all(got, oracle_ref(q, k, v, do, causal, scale), what=f"B={B} H={H} N={N} d={d} causal={causal}")
