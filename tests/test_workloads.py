"""The seeded input generators: deterministic, shaped and scaled as stated."""
import math

import torch

from exact_attention_106_b200 import workloads as W


def test_named_shapes_and_flop_counts():
    assert W.TINY.shape == (1, 1, 128, 64) and not W.TINY.causal and W.TINY.softmax_scale == 0.125
    assert W.SMALL_CAUSAL_STABILITY.shape == (2, 8, 1024, 64) and W.SMALL_CAUSAL_STABILITY.causal
    assert W.LLAMA_BLOCK.shape == (4, 16, 4096, 128)
    assert abs(W.LLAMA_BLOCK.softmax_scale - 1 / math.sqrt(128)) < 1e-15
    assert W.LONG_CONTEXT.shape == (1, 32, 16384, 128)
    w = W.LONG_CONTEXT
    assert w.pairs() == 32 * 16384 * 16385 // 2
    assert w.fwd_flops() == 4 * 128 * w.pairs() and w.bwd_flops() == 10 * 128 * w.pairs()
    sw = W.sweep()
    assert len(sw) == 24 and all(x.B * x.N == 16384 and x.H == 32 for x in sw)
    assert len({x.seed_base for x in sw}) == 24


def test_inputs_are_deterministic_bf16():
    a = W.make_inputs(W.TINY)
    b = W.make_inputs(W.TINY)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and x.is_contiguous() and x.shape == W.TINY.shape
        assert torch.equal(x, y)
    assert not torch.equal(a[0], a[1])


def test_stability_boost_on_upper_heads_only():
    w = W.SMALL_CAUSAL_STABILITY
    q = W.make_inputs(w)[0].float()
    lo, hi = q[:, :4].std().item(), q[:, 4:].std().item()
    assert 0.9 < lo < 1.1 and 7.5 < hi < 8.5
