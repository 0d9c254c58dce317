"""GPU parity at the largest offsets: a [1, 2080, 8229, 128] causal problem
whose last head starts past element 2^31 of every tensor (and of the padded
fp32 dQ accumulator), so a 32-bit element offset anywhere in the forward,
the three backward stages or their TMA maps would land in the wrong head.

The tensors are 4.4 GB each and are drawn on the device; the first and the
last head are overwritten with host-seeded values (workloads.make_head) and
checked against the fp64 oracle; every head is checked for finite outputs
and for the gradient identity sum_j dV_j = sum_i dO_i.
"""
import numpy as np
import pytest
import torch

import exact_attention_106_b200 as ex
import oracle
from exact_attention_106_b200 import workloads as W
from parity_util import check_grad, check_lse, check_o, to_np

pytestmark = pytest.mark.gpu


def _run_and_check(w, dev):
    B, H, N, d = w.shape
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed_base)
    q, k, v, do = (torch.randn(w.shape, generator=g, device=dev, dtype=torch.bfloat16) for _ in range(4))
    heads = [(0, 0), (0, H - 1)]
    host = {}
    for b, h in heads:
        host[(b, h)] = W.make_head(w, b, h)
        for dst, src in zip((q, k, v, do), host[(b, h)]):
            dst[b, h].copy_(src)
    o, lse = ex.forward(q, k, v, causal=w.causal, scale=w.softmax_scale)
    dq, dk, dv = ex.backward(q, k, v, o, lse, do, causal=w.causal, scale=w.softmax_scale)
    torch.cuda.synchronize()
    assert ex.device_status() == 0
    for t, name in ((o, "o"), (lse, "lse"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        assert bool(torch.isfinite(t).all()), name
    # chain rule: the keys' dV rows sum to the queries' dO rows, per head
    dv_sum = torch.sum(dv, dim=2, dtype=torch.float32)
    do_sum = torch.sum(do, dim=2, dtype=torch.float32)
    err = float((dv_sum - do_sum).abs().max())
    assert err <= 2e-2 * float(do_sum.abs().max()) + 2.0, err
    for b, h in heads:
        hq, hk, hv, hdo = host[(b, h)]
        ref = oracle.backward_head(hq, hk, hv, hdo, w.softmax_scale, w.causal)
        what = f"{w.name} head ({b}, {h})"
        check_o(to_np(o[b, h]), ref["o"], what + " O")
        check_lse(to_np(lse[b, h]), ref["lse"], what + " LSE")
        for key, t in (("dq", dq), ("dk", dk), ("dv", dv)):
            check_grad(to_np(t[b, h]), ref[key], f"{what} {key}")


def test_element_offsets_past_2_31(cuda_device):
    w = W.LARGE_OFFSETS
    B, H, N, d = w.shape
    assert (H - 1) * N * d > 2**31
    assert (H - 1) * ((N + 127) // 128 * 128) * d > 2**31
    torch.cuda.empty_cache()
    try:
        _run_and_check(w, cuda_device)
    finally:
        torch.cuda.empty_cache()  # hand the ~45 GB back before the next test
