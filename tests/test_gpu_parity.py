"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded bf16 inputs, plus edge cases and invariants that need no oracle."""
import math

import numpy as np
import pytest
import torch

import exact_attention_106_b200 as ex
from exact_attention_106_b200 import workloads as W
from parity_util import check_all, check_grad, check_o, oracle_ref, run_cuda, to_np

pytestmark = pytest.mark.gpu


def _inputs(B, H, N, d, seed, q_mult=1.0):
    g = torch.Generator().manual_seed(seed)
    q, k, v, do = (torch.randn((B, H, N, d), generator=g) for _ in range(4))
    return (q * q_mult).bfloat16(), k.bfloat16(), v.bfloat16(), do.bfloat16()


def test_tiny_exactness_config(cuda_device):
    w = W.TINY
    q, k, v, do = W.make_inputs(w)
    got = run_cuda(q, k, v, do, w.causal, w.softmax_scale)
    ref = oracle_ref(q, k, v, do, w.causal, w.softmax_scale)
    check_all(got, ref, what=w.name)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 127, 128, 129, 255, 256, 257, 383, 1000])
def test_ragged_lengths(cuda_device, N, d, causal):
    q, k, v, do = _inputs(1, 2, N, d, seed=N * 7 + d + int(causal))
    scale = 1 / math.sqrt(d)
    got = run_cuda(q, k, v, do, causal, scale)
    ref = oracle_ref(q, k, v, do, causal, scale)
    check_all(got, ref, what=f"N={N} d={d} causal={causal}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1025, 1500, 2049, 3001, 4095])
def test_mid_lengths(cuda_device, N, d, causal):
    """Lengths past the short-row forward configuration (the backward runs
    persistent CTAs up to 2048): ragged tails, odd and even numbers of query
    blocks and key tiles, several heads."""
    q, k, v, do = _inputs(2, 3, N, d, seed=N * 7 + d + int(causal))
    scale = 1 / math.sqrt(d)
    got = run_cuda(q, k, v, do, causal, scale)
    check_all(got, oracle_ref(q, k, v, do, causal, scale), what=f"N={N} d={d} causal={causal}")


def test_small_causal_stability_config(cuda_device):
    w = W.SMALL_CAUSAL_STABILITY
    q, k, v, do = W.make_inputs(w)
    got = run_cuda(q, k, v, do, w.causal, w.softmax_scale)
    ref = oracle_ref(q, k, v, do, w.causal, w.softmax_scale)
    check_all(got, ref, what=w.name)


@pytest.mark.parametrize("scale", [0.01, 0.3, 2.0])
def test_other_scales_and_batch_heads(cuda_device, scale):
    q, k, v, do = _inputs(3, 5, 300, 64, seed=11)
    for causal in (False, True):
        got = run_cuda(q, k, v, do, causal, scale)
        ref = oracle_ref(q, k, v, do, causal, scale)
        check_all(got, ref, what=f"scale={scale} causal={causal}")


@pytest.mark.parametrize("d", [64, 128])
def test_all_equal_scores(cuda_device, d):
    """Q = 0: every visible key gets the same weight; O = mean of visible V."""
    N = 300
    q = torch.zeros((1, 1, N, d), dtype=torch.bfloat16)
    _, k, v, do = _inputs(1, 1, N, d, seed=3)
    for causal in (False, True):
        got = run_cuda(q, k, v, do, causal, 1 / math.sqrt(d))
        vv = v[0, 0].double().numpy()
        want = np.cumsum(vv, 0) / np.arange(1, N + 1)[:, None] if causal else np.broadcast_to(vv.mean(0), vv.shape)
        check_o(got["o"][0, 0], want, "all-equal")
        want_lse = np.log(np.arange(1, N + 1)) if causal else np.full(N, math.log(N))
        np.testing.assert_allclose(got["lse"][0, 0], want_lse, rtol=1e-3, atol=1e-3)


@pytest.mark.parametrize("d", [64, 128])
def test_invariants_without_oracle(cuda_device, d):
    B, H, N = 2, 3, 700
    q, k, v, do = _inputs(B, H, N, d, seed=21)
    scale = 1 / math.sqrt(d)
    dev = cuda_device
    # V = ones -> O = ones
    o, _ = ex.forward(q.to(dev), k.to(dev), torch.ones_like(v).to(dev), causal=True, scale=scale)
    assert float((o.float() - 1).abs().max()) <= 1e-2
    # N = 1 -> O = V
    o1, lse1 = ex.forward(q[:, :, :1].contiguous().to(dev), k[:, :, :1].contiguous().to(dev),
                          v[:, :, :1].contiguous().to(dev), causal=False, scale=scale)
    assert torch.equal(o1.cpu(), v[:, :, :1])
    # causal row 0 -> O_0 = V_0
    r = run_cuda(q, k, v, do, True, scale)
    np.testing.assert_allclose(r["o"][:, :, 0], to_np(v[:, :, 0]), rtol=0, atol=1e-2)
    # sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i (per head)
    for causal in (False, True):
        r = run_cuda(q, k, v, do, causal, scale)
        dk_sum = r["dk"].sum(axis=2)
        assert float(np.max(np.abs(dk_sum))) <= 5e-2 * float(np.max(np.abs(r["dk"]))) * math.sqrt(N)
        dv_sum, do_sum = r["dv"].sum(axis=2), to_np(do).sum(axis=2)
        assert float(np.max(np.abs(dv_sum - do_sum))) <= 2e-2 * float(np.max(np.abs(do_sum))) + 0.5


def test_forward_is_deterministic_and_status_clean(cuda_device):
    q, k, v, _ = (x.to(cuda_device) for x in _inputs(2, 4, 1000, 128, seed=5))
    o1, l1 = ex.forward(q, k, v, causal=True)
    o2, l2 = ex.forward(q, k, v, causal=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert ex.device_status() == 0


def test_outputs_stay_inside_their_buffers(cuda_device):
    """Guard bytes around every output and NaN-prefilled outputs: nothing is
    written outside, everything inside is written."""
    B, H, N, d = 2, 3, 333, 128
    q, k, v, do = (x.to(cuda_device) for x in _inputs(B, H, N, d, seed=9))
    n = B * H * N * d
    G = 4096

    def guarded(numel, dtype):
        buf = torch.full((numel + 2 * G,), float("nan"), dtype=dtype, device=cuda_device)
        return buf, buf[G:G + numel]

    ob, o = guarded(n, torch.bfloat16)
    lb, lse = guarded(B * H * N, torch.float32)
    ex.forward(q, k, v, causal=True, out=o.view(B, H, N, d), lse=lse.view(B, H, N))
    grads = [guarded(n, torch.bfloat16) for _ in range(3)]
    ex.backward(q, k, v, o.view(B, H, N, d), lse.view(B, H, N), do, causal=True,
                out=[g[1].view(B, H, N, d) for g in grads])
    torch.cuda.synchronize()
    for buf, inner in [(ob, o), (lb, lse)] + grads:
        assert torch.isnan(buf[:G].float()).all() and torch.isnan(buf[-G:].float()).all()
        assert torch.isfinite(inner.float()).all()
    assert ex.device_status() == 0


def test_backward_stages_equal_composite(cuda_device):
    B, H, N, d = 1, 2, 517, 64
    q, k, v, do = (x.to(cuda_device) for x in _inputs(B, H, N, d, seed=13))
    o, lse = ex.forward(q, k, v, causal=True)
    dq1, dk1, dv1 = ex.backward(q, k, v, o, lse, do, causal=True)
    ws = ex.alloc_workspace(B, H, N, d, cuda_device)
    dq2, dk2, dv2 = (torch.empty_like(q) for _ in range(3))
    stages = list(ex.bwd_stages(q, k, v, o, lse, do, dq2, dk2, dv2, ws, causal=True))
    assert stages == ["preprocess", "dkdv", "dq_convert"]
    torch.cuda.synchronize()
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    check_grad(to_np(dq2), to_np(dq1), "staged dq")  # dQ reduction order may differ
