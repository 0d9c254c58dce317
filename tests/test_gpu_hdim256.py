"""GPU parity of the forward at head_dim 256 (one 128-row query sub-tile per
CTA), bf16 and fp16, whole and split over key ranges, against the fp64
oracle with the forward's tolerances (O max-abs 2e-2, LSE 1e-3 relative).
The backward does not take head_dim 256: its dK and dV accumulators alone
would fill the tensor memory; it must refuse the size."""
import math

import pytest
import torch

import exact_attention_106_b200 as ex
import oracle
from exact_attention_106_b200 import _lib
from exact_attention_106_b200 import workloads as W
from parity_util import check_lse, check_o, oracle_ref, run_cuda, to_np

pytestmark = pytest.mark.gpu


def _inputs(B, H, N, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    return tuple(torch.randn((B, H, N, 256), generator=g).to(dtype) for _ in range(3))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 127, 128, 129, 255, 256, 257, 700])
def test_hdim256_ragged_lengths(cuda_device, N, causal):
    q, k, v = _inputs(2, 2, N, N + int(causal))
    got = run_cuda(q, k, v, None, causal, 1 / 16, with_bwd=False)
    ref = oracle_ref(q, k, v, None, causal, 1 / 16, with_bwd=False)
    check_o(got["o"], ref["o"], f"d=256 N={N} causal={causal}")
    check_lse(got["lse"], ref["lse"], f"d=256 N={N} causal={causal}")


def test_hdim256_fp16(cuda_device):
    q, k, v = _inputs(1, 3, 600, 5, torch.float16)
    for causal in (False, True):
        got = run_cuda(q, k, v, None, causal, 1 / 16, with_bwd=False)
        ref = oracle_ref(q, k, v, None, causal, 1 / 16, with_bwd=False)
        check_o(got["o"], ref["o"], f"fp16 d=256 causal={causal}")
        check_lse(got["lse"], ref["lse"], f"fp16 d=256 causal={causal}")


def test_hdim256_bench_workload_sampled_heads(cuda_device):
    """2x16x8192x256 causal: the full launch bench.py times, four heads against the oracle."""
    w = W.HDIM256[0]
    q, k, v, _ = W.make_inputs(w, with_grad_out=False)
    got = run_cuda(q, k, v, None, w.causal, w.softmax_scale, with_bwd=False)
    heads = [(0, 0), (0, 15), (1, 7), (1, 15)]
    ref = oracle_ref(q, k, v, None, w.causal, w.softmax_scale, heads=heads, with_bwd=False)
    import numpy as np
    sel = lambda a: np.stack([a[b, h] for b, h in heads])  # noqa: E731
    check_o(sel(got["o"]), sel(ref["o"]), w.name)
    check_lse(sel(got["lse"]), sel(ref["lse"]), w.name)


@pytest.mark.parametrize("nq,nk,splits", [(1, 5000, 0), (16, 3000, 3), (1000, 1000, 4)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16], ids=["bf16", "fp16"])
def test_hdim256_kvsplit(cuda_device, nq, nk, splits, dtype):
    g = torch.Generator().manual_seed(nq + nk)
    q = torch.randn((1, 2, nq, 256), generator=g).to(dtype)
    k, v = (torch.randn((1, 2, nk, 256), generator=g).to(dtype) for _ in range(2))
    for causal in (False, True):
        o, lse = ex.forward_kvsplit(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), causal=causal,
                                    splits=splits)
        torch.cuda.synchronize()
        o_ref, lse_ref = oracle.decode(q, k, v, 1 / 16, causal)
        check_o(to_np(o), o_ref, f"d=256 kvsplit nq={nq} causal={causal}")
        check_lse(to_np(lse), lse_ref, f"d=256 kvsplit nq={nq} causal={causal}")


def test_backward_refuses_hdim256(cuda_device):
    lib = _lib.load()
    assert lib.attn_bwd_workspace_bytes(1, 1, 128, 256) == 0
    q = torch.zeros((1, 1, 128, 256), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.zeros((1, 1, 128), dtype=torch.float32, device=cuda_device)
    with pytest.raises(ex.ExattnError) as e:
        ex.backward(q, q, q, q, lse, q, workspace=torch.empty(16, dtype=torch.uint8, device=cuda_device))
    assert e.value.status == _lib.ATTN_ERR_INVALID
