"""GPU parity of the fp16 entry points (attn_fwd_fp16, attn_bwd_fp16).

The same seeded float32 draws as the bf16 tests, rounded to fp16 instead;
the fp64 oracle takes those fp16 values upcast exactly.  fp16 keeps 3 more
mantissa bits than bf16, so the bf16 tolerances (O max-abs 2e-2, LSE 1e-3
relative, gradients 5e-2 relative to max) hold with room to spare.
"""
import math

import pytest
import torch

from exact_attention_106_b200 import workloads as W
from parity_util import check_all, oracle_ref, run_cuda

pytestmark = pytest.mark.gpu

F16 = torch.float16


def _inputs(B, H, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    return tuple(torch.randn((B, H, N, d), generator=g).to(F16) for _ in range(4))


def test_fp16_tiny_exactness_config(cuda_device):
    w = W.TINY
    q, k, v, do = W.make_inputs(w, dtype=F16)
    got = run_cuda(q, k, v, do, w.causal, w.softmax_scale)
    check_all(got, oracle_ref(q, k, v, do, w.causal, w.softmax_scale), what="fp16 " + w.name)


def test_fp16_small_causal_stability_config(cuda_device):
    """Q x 8 on heads 4..7: near one-hot rows stress the rescale."""
    w = W.SMALL_CAUSAL_STABILITY
    q, k, v, do = W.make_inputs(w, dtype=F16)
    got = run_cuda(q, k, v, do, w.causal, w.softmax_scale)
    check_all(got, oracle_ref(q, k, v, do, w.causal, w.softmax_scale), what="fp16 " + w.name)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 127, 128, 129, 255, 257, 383, 1000])
def test_fp16_ragged_lengths(cuda_device, N, d, causal):
    q, k, v, do = _inputs(1, 2, N, d, seed=N * 13 + d + int(causal))
    scale = 1 / math.sqrt(d)
    got = run_cuda(q, k, v, do, causal, scale)
    check_all(got, oracle_ref(q, k, v, do, causal, scale), what=f"fp16 N={N} d={d} causal={causal}")


def test_fp16_llama_block_sampled_heads(cuda_device):
    """4x16x4096x128 causal in fp16: the full launch, six heads against the oracle."""
    w = W.LLAMA_BLOCK
    q, k, v, do = W.make_inputs(w, dtype=F16)
    got = run_cuda(q, k, v, do, w.causal, w.softmax_scale)
    heads = [(0, 0), (0, 15), (1, 3), (2, 8), (3, 0), (3, 15)]
    ref = oracle_ref(q, k, v, do, w.causal, w.softmax_scale, heads=heads)
    check_all(got, ref, heads=heads, what="fp16 " + w.name)


def test_fp16_and_bf16_paths_are_different_kernels(cuda_device):
    """The same fp32 draw through both element types: both match the oracle
    on their own rounded inputs, and the fp16 result is the closer one."""
    import numpy as np
    g = torch.Generator().manual_seed(3)
    x = [torch.randn((1, 2, 300, 128), generator=g) for _ in range(4)]
    errs = {}
    for dt in (torch.bfloat16, F16):
        q, k, v, do = (t.to(dt) for t in x)
        got = run_cuda(q, k, v, do, True, 0.1)
        ref = oracle_ref(*(t.double() for t in x), True, 0.1)  # exact fp32 inputs
        errs[dt] = float(np.max(np.abs(got["o"] - ref["o"])))
    assert errs[F16] < errs[torch.bfloat16], errs


def test_fp16_long_context_sampled_heads(cuda_device):
    """1x32x16384x128 causal in fp16, the shape of the fp16 bench point: the
    full launch, the first and last heads against the oracle."""
    w = W.LONG_CONTEXT
    q, k, v, do = W.make_inputs(w, dtype=F16)
    got = run_cuda(q, k, v, do, w.causal, w.softmax_scale)
    heads = [(0, 0), (0, 31)]
    ref = oracle_ref(q, k, v, do, w.causal, w.softmax_scale, heads=heads)
    check_all(got, ref, heads=heads, what="fp16 " + w.name)
