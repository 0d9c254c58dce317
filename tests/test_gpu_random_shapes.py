"""GPU parity on seeded random shapes: lengths 1..3000, head_dim 64/128, 1..12
(batch, head) pairs, causal or not, scales 0.05..0.3.  Between them they reach
every launch form (lean and two-sub-tile forward; persistent and one-CTA-per-
tile backward, with even and odd key-tile counts and fewer units than SMs)
with ragged tails.  Also the split-key forward on random query and key counts
(1..300 and 1..6000), bf16 and fp16, with automatic and forced key ranges.
Same tolerances as the other parity tests."""
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


def _kv_cases(n=16, seed=2027):
    rng = random.Random(seed)
    out = []
    for i in range(n):
        nk = rng.randint(1, 6000)
        nq = rng.choice([1, rng.randint(1, 16), rng.randint(1, 300)])
        causal = rng.random() < 0.5 and nq <= nk
        out.append((i, rng.randint(1, 3), rng.randint(1, 4), nq, nk, rng.choice([64, 128]), causal,
                    rng.choice([0, 0, 1, 2, 5]), rng.choice(["bf16", "fp16"])))
    return out


@pytest.mark.parametrize("case", _kv_cases(), ids=lambda c: f"{c[0]}-{c[3]}q{c[4]}k{c[5]}-{'c' if c[6] else 'f'}-s{c[7]}-{c[8]}")
def test_random_split_key_shape(cuda_device, case):
    """The split-key forward (automatic or forced ranges) on random query and
    key counts, against the oracle's decode (bottom-right causal alignment)."""
    import exact_attention_106_b200 as ex
    import oracle
    from parity_util import check_lse, check_o, to_np
    i, B, H, nq, nk, d, causal, splits, dt = case
    dtype = torch.bfloat16 if dt == "bf16" else torch.float16
    g = torch.Generator().manual_seed(8000 + i)
    q = torch.randn((B, H, nq, d), generator=g).to(dtype)
    k, v = (torch.randn((B, H, nk, d), generator=g).to(dtype) for _ in range(2))
    scale = 1 / math.sqrt(d)
    o, lse = ex.forward_kvsplit(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), causal=causal,
                                scale=scale, splits=splits)
    torch.cuda.synchronize()
    assert ex.device_status() == 0
    o_ref, lse_ref = oracle.decode(q, k, v, scale, causal)
    what = f"{dt} B={B} H={H} nq={nq} nk={nk} d={d} causal={causal} splits={splits}"
    check_o(to_np(o), o_ref, what)
    check_lse(to_np(lse), lse_ref, what)
