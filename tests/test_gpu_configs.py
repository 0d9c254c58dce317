"""GPU parity at the workloads' full sizes.

  * LLaMA-block 4x16x4096x128 causal: every head against the oracle.
  * long context 1x32x16384x128 causal: heads {0, 7, 16, 31} against the
    oracle (each is a complete 16384-token problem), the rest by invariants;
    peak device memory stays linear in N.
  * sweep at 16384 tokens per batch (N 512..16384, d 64/128, causal and not):
    heads {0, 31} of the first and last batch against the oracle.
  * single head 1x1x32768x128 forward, causal and not: every row.
The launches are the same kernels and launch shapes that bench.py times.
"""
import numpy as np
import pytest
import torch

import exact_attention_106_b200 as ex
from exact_attention_106_b200 import workloads as W
from parity_util import check_all, check_grad, oracle_ref, run_cuda, to_np

pytestmark = pytest.mark.gpu


def test_llama_block_all_heads(cuda_device):
    w = W.LLAMA_BLOCK
    q, k, v, do = W.make_inputs(w)
    got = run_cuda(q, k, v, do, w.causal, w.softmax_scale)
    ref = oracle_ref(q, k, v, do, w.causal, w.softmax_scale)
    check_all(got, ref, what=w.name)


def test_long_context_sampled_heads_and_footprint(cuda_device):
    w = W.LONG_CONTEXT
    B, H, N, d = w.shape
    q, k, v, do = W.make_inputs(w)
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    got = run_cuda(q, k, v, do, w.causal, w.softmax_scale)
    peak = torch.cuda.max_memory_allocated() - base
    heads = [(0, 0), (0, 7), (0, 16), (0, 31)]
    ref = oracle_ref(q, k, v, do, w.causal, w.softmax_scale, heads=heads)
    check_all(got, ref, heads=heads, what=w.name)
    # every head: finite outputs, and the gradient identities of the chain rule
    for key in ("o", "lse", "dq", "dk", "dv"):
        assert np.isfinite(got[key]).all(), key
    dv_sum, do_sum = got["dv"].sum(axis=2), to_np(do).sum(axis=2)
    assert float(np.max(np.abs(dv_sum - do_sum))) <= 2e-2 * float(np.max(np.abs(do_sum))) + 2.0
    # linear footprint: 4 inputs + 5 outputs + workspace, no N x N buffer
    linear = 9 * B * H * N * d * 2 + B * H * N * 4 + ex.bwd_workspace_bytes(B, H, N, d)
    one_score_matrix = B * H * N * N * 2
    assert peak <= 2 * linear, (peak, linear)
    assert peak < one_score_matrix / 10, (peak, one_score_matrix)


@pytest.mark.parametrize("w", W.sweep(), ids=lambda w: w.name)
def test_sweep_sampled_heads(cuda_device, w):
    q, k, v, do = W.make_inputs(w)
    got = run_cuda(q, k, v, do, w.causal, w.softmax_scale)
    heads = sorted({(0, 0), (0, 31), (w.B - 1, 0), (w.B - 1, 31)})
    ref = oracle_ref(q, k, v, do, w.causal, w.softmax_scale, heads=heads)
    check_all(got, ref, heads=heads, what=w.name)
    for key in ("o", "lse", "dq", "dk", "dv"):
        assert np.isfinite(got[key]).all(), key


@pytest.mark.parametrize("w", [W.SINGLE_HEAD_32K, W.SINGLE_HEAD_32K_CAUSAL], ids=lambda w: w.name)
def test_single_head_32k_forward(cuda_device, w):
    q, k, v, _ = W.make_inputs(w, with_grad_out=False)
    got = run_cuda(q, k, v, None, w.causal, w.softmax_scale, with_bwd=False)
    ref = oracle_ref(q, k, v, None, w.causal, w.softmax_scale, with_bwd=False)
    check_all(got, ref, what=w.name, with_bwd=False)
