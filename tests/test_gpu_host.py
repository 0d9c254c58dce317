"""attn_fwd_bwd_host: forward and backward over page-locked host tensors,
copies pipelined over chunks of (batch, head) pairs.

The chunks run the same kernels on the same rows as the device-resident
calls, so O, LSE, dK and dV must agree with them bit for bit; dQ is summed by
reduce-adds in an order that is not fixed, so it is held to two bf16 units in
the last place.  One case is also checked against the fp64 oracle.
"""
import math

import pytest
import torch

import exact_attention_106_b200 as ex
from exact_attention_106_b200 import workloads as W
from parity_util import check_all, oracle_ref, to_np

pytestmark = pytest.mark.gpu


def _inputs(B, H, N, d, seed):
    w = W.Workload(name=f"host_{B}x{H}x{N}x{d}", B=B, H=H, N=N, d=d, causal=False, seed_base=seed)
    return W.make_inputs(w)


def _host_run(q, k, v, do, causal, scale, heads_per_chunk, device):
    B, H, N, d = q.shape
    hq, hk, hv, hdo = (x.contiguous().pin_memory() for x in (q, k, v, do))
    out = tuple(torch.empty((B, H, N, d), dtype=torch.bfloat16).pin_memory() for _ in range(4))
    ho, hdq, hdk, hdv = out
    hlse = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
    # guard the host outputs against stale values from an earlier use of the memory
    for t in (ho, hdq, hdk, hdv):
        t.fill_(float("nan"))
    hlse.fill_(float("nan"))
    ex.forward_backward_host(hq, hk, hv, hdo, (ho, hlse, hdq, hdk, hdv), causal=causal, scale=scale,
                             device=device, heads_per_chunk=heads_per_chunk)
    torch.cuda.synchronize(device)
    assert ex.device_status(device) == 0
    return ho, hlse, hdq, hdk, hdv


def _device_run(q, k, v, do, causal, scale, device):
    qd, kd, vd, dod = (x.to(device) for x in (q, k, v, do))
    o, lse = ex.forward(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = ex.backward(qd, kd, vd, o, lse, dod, causal=causal, scale=scale)
    torch.cuda.synchronize(device)
    assert ex.device_status(device) == 0
    return tuple(t.cpu() for t in (o, lse, dq, dk, dv))


@pytest.mark.parametrize("B,H,N,d,causal,hpc", [
    (2, 3, 300, 64, True, 0),      # 6 pairs, automatic chunks of 1
    (1, 5, 1000, 128, False, 2),   # chunks 2, 2, 1 (ragged last chunk, both buffer sets reused)
    (1, 4, 129, 128, True, 3),     # chunks 3, 1
    (1, 2, 513, 128, True, 8),     # one chunk larger than the problem
])
def test_host_call_matches_device_calls(cuda_device, B, H, N, d, causal, hpc):
    q, k, v, do = _inputs(B, H, N, d, seed=7000 + N)
    scale = 1.0 / math.sqrt(d)
    ho, hlse, hdq, hdk, hdv = _host_run(q, k, v, do, causal, scale, hpc, cuda_device)
    o, lse, dq, dk, dv = _device_run(q, k, v, do, causal, scale, cuda_device)
    for name, a, b in (("O", ho, o), ("LSE", hlse, lse), ("dK", hdk, dk), ("dV", hdv, dv)):
        assert torch.equal(a, b), f"{name} differs between the host-pipelined and device calls"
    ulp = 2.0 ** -7  # bf16: 8 significant bits
    torch.testing.assert_close(hdq.float(), dq.float(), rtol=2 * ulp, atol=1e-6)


def test_host_call_against_oracle(cuda_device):
    B, H, N, d, causal = 1, 3, 640, 128, True
    q, k, v, do = _inputs(B, H, N, d, seed=7100)
    scale = 1.0 / math.sqrt(d)
    ho, hlse, hdq, hdk, hdv = _host_run(q, k, v, do, causal, scale, 2, cuda_device)
    got = {"o": to_np(ho), "lse": to_np(hlse), "dq": to_np(hdq), "dk": to_np(hdk), "dv": to_np(hdv)}
    ref = oracle_ref(q, k, v, do, causal, scale)
    check_all(got, ref, what="host pipeline 1x3x640x128 causal")


def test_host_call_with_pageable_buffers(cuda_device):
    # not page-locked: slower, same results
    B, H, N, d = 1, 2, 256, 64
    q, k, v, do = _inputs(B, H, N, d, seed=7200)
    out = tuple(torch.empty((B, H, N, d), dtype=torch.bfloat16) for _ in range(4))
    lse = torch.empty((B, H, N), dtype=torch.float32)
    ho, hdq, hdk, hdv = out
    ex.forward_backward_host(q, k, v, do, (ho, lse, hdq, hdk, hdv), causal=False, device=cuda_device,
                             heads_per_chunk=1)
    torch.cuda.synchronize(cuda_device)
    o, lse_d, dq, dk, dv = _device_run(q, k, v, do, False, 1.0 / math.sqrt(d), cuda_device)
    assert torch.equal(ho, o) and torch.equal(lse, lse_d) and torch.equal(hdk, dk) and torch.equal(hdv, dv)
