"""GPU parity of the e4m3 forward (attn_fwd_fp8) against the fp64 oracle.

Inputs: float32 N(0, 1) draws quantized per tensor to e4m3 with the factor
s = max|x| / 448; the oracle gets the exact real values (e4m3 value * s).

Tolerance, from the arithmetic.  The kernel's scores come from exact e4m3
products accumulated in fp32, its softmax sums and LSE are fp32, so the LSE
keeps the forward's bound (1e-3 relative, floored at 1).  Each probability is
rounded to e4m3 before the P V product: a relative error of at most 2^-4.
So, per element, |O - O_ref| <= 2^-4 * (sum_j P_ij |V_j|) / l_i (all errors
of one sign), plus the bf16 rounding of the output (2^-8 |O|) and 1e-3 for
the fp32 accumulation and the exp2 approximations.  sum_j P_ij |V_j| / l_i is
the oracle's output for |V|.
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_106_b200 as ex
import oracle
from exact_attention_106_b200 import workloads as W
from parity_util import check_lse, to_np

pytestmark = pytest.mark.gpu
E4M3_MAX = 448.0


def _quantize(x):
    s = float(x.abs().max()) / E4M3_MAX
    x8 = (x / s).to(torch.float8_e4m3fn)
    return x8, s, x8.to(torch.float64) * s


def _check_fp8(q32, k32, v32, causal, scale, dev, what):
    (q8, qs, qr), (k8, ks, kr), (v8, vs, vr) = (_quantize(t) for t in (q32, k32, v32))
    o, lse = ex.forward_fp8(q8.to(dev), k8.to(dev), v8.to(dev), qs, ks, vs, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert ex.device_status() == 0
    o, lse = to_np(o), to_np(lse)
    o_ref, lse_ref = oracle.forward(qr, kr, vr, scale, causal)
    o_abs, _ = oracle.forward(qr, kr, vr.abs(), scale, causal)
    assert np.isfinite(o).all(), what
    bound = 2.0 ** -4 * o_abs + 2.0 ** -8 * np.abs(o_ref) + 1e-3
    excess = float(np.max(np.abs(o - o_ref) - bound))
    assert excess <= 0, f"{what}: O error exceeds its bound by {excess:.3e}"
    check_lse(lse, lse_ref, what)
    return float(np.max(np.abs(o - o_ref)))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 127, 128, 129, 300, 1000])
def test_fp8_ragged_lengths(cuda_device, N, causal):
    g = torch.Generator().manual_seed(N + int(causal))
    q, k, v = (torch.randn((2, 3, N, 128), generator=g) for _ in range(3))
    _check_fp8(q, k, v, causal, 1 / math.sqrt(128), cuda_device, f"fp8 N={N} causal={causal}")


def test_fp8_llama_block_shape_sampled_heads(cuda_device):
    """4x16x4096x128 causal (the LLaMA-block shape): the full launch; six heads against the oracle."""
    w = W.LLAMA_BLOCK
    g = torch.Generator().manual_seed(11)
    x = [torch.randn(w.shape, generator=g) for _ in range(3)]
    (q8, qs, qr), (k8, ks, kr), (v8, vs, vr) = (_quantize(t) for t in x)
    o, lse = ex.forward_fp8(q8.to(cuda_device), k8.to(cuda_device), v8.to(cuda_device), qs, ks, vs, causal=True)
    torch.cuda.synchronize()
    o, lse = to_np(o), to_np(lse)
    heads = [(0, 0), (1, 5), (2, 9), (3, 15)]
    o_ref, lse_ref = oracle.forward(qr, kr, vr, w.softmax_scale, True, heads=heads)
    o_abs, _ = oracle.forward(qr, kr, vr.abs(), w.softmax_scale, True, heads=heads)
    for b, h in heads:
        bound = 2.0 ** -4 * o_abs[b, h] + 2.0 ** -8 * np.abs(o_ref[b, h]) + 1e-3
        assert (np.abs(o[b, h] - o_ref[b, h]) <= bound).all(), (b, h)
        check_lse(lse[b, h], lse_ref[b, h], f"fp8 head {b},{h}")


def test_fp8_long_context_sampled_heads(cuda_device):
    """1x32x16384x128 causal, the shape and inputs of the e4m3 bench point (the
    long-context draws, quantized per tensor): the full launch, the first and
    last heads against the oracle."""
    w = W.LONG_CONTEXT
    x = W.make_inputs(w, with_grad_out=False, dtype=torch.float32)[:3]
    (q8, qs, qr), (k8, ks, kr), (v8, vs, vr) = (_quantize(t) for t in x)
    o, lse = ex.forward_fp8(q8.to(cuda_device), k8.to(cuda_device), v8.to(cuda_device), qs, ks, vs, causal=True)
    torch.cuda.synchronize()
    assert ex.device_status() == 0
    heads = [(0, 0), (0, 31)]
    o = np.stack([to_np(o[b, h]) for b, h in heads])
    lse = np.stack([to_np(lse[b, h]) for b, h in heads])
    o_ref, lse_ref = oracle.forward(qr, kr, vr, w.softmax_scale, True, heads=heads)
    o_abs, _ = oracle.forward(qr, kr, vr.abs(), w.softmax_scale, True, heads=heads)
    for i, (b, h) in enumerate(heads):
        bound = 2.0 ** -4 * o_abs[b, h] + 2.0 ** -8 * np.abs(o_ref[b, h]) + 1e-3
        excess = float(np.max(np.abs(o[i] - o_ref[b, h]) - bound))
        assert excess <= 0, f"fp8 long context head {b},{h}: O error exceeds its bound by {excess:.3e}"
        check_lse(lse[i], lse_ref[b, h], f"fp8 long context head {b},{h}")


def test_fp8_large_scores_stability(cuda_device):
    """Q x 8: near one-hot rows, where the reference maximum moves often."""
    g = torch.Generator().manual_seed(5)
    q, k, v = (torch.randn((1, 2, 700, 128), generator=g) for _ in range(3))
    _check_fp8(q * 8, k, v, True, 1 / math.sqrt(128), cuda_device, "fp8 Qx8")


def test_fp8_error_is_small_in_practice(cuda_device):
    """Beyond the worst-case bound: on N(0,1) data the e4m3 path stays close
    to the oracle (typical error far below the bound)."""
    g = torch.Generator().manual_seed(8)
    q, k, v = (torch.randn((1, 4, 2048, 128), generator=g) for _ in range(3))
    err = _check_fp8(q, k, v, False, 1 / math.sqrt(128), cuda_device, "fp8 typical")
    assert err < 0.05, err


def test_fp8_rejects_other_head_dims_and_bad_descales(cuda_device):
    from exact_attention_106_b200 import _lib
    lib = _lib.load()
    d = torch.empty(1 << 16, dtype=torch.uint8, device=cuda_device).data_ptr()
    assert lib.attn_fwd_fp8(d, d, d, d, d, 1, 1, 8, 64, 0.1, 0, 1.0, 1.0, 1.0, None) == _lib.ATTN_ERR_INVALID
    assert lib.attn_fwd_fp8(d, d, d, d, d, 1, 1, 8, 128, 0.1, 0, 0.0, 1.0, 1.0, None) == _lib.ATTN_ERR_INVALID
    assert lib.attn_fwd_fp8(d, d, d, d, d, 1, 1, 8, 128, 0.1, 0, 1.0, float("nan"), 1.0, None) == \
        _lib.ATTN_ERR_INVALID
