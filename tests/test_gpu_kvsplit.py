"""GPU parity of the split-key forward (attn_fwd_kvsplit) against the fp64
oracle: decode shapes (few queries, long key history, causal mask aligned
bottom-right), square problems with forced splits, and the single-head 32K
causal problem it exists for.  Tolerances as for the forward: O max-abs
2e-2, LSE 1e-3 relative (floored at 1)."""
import math

import numpy as np
import pytest
import torch

import exact_attention_106_b200 as ex
import oracle
from exact_attention_106_b200 import _lib
from exact_attention_106_b200 import workloads as W
from parity_util import check_lse, check_o, to_np

pytestmark = pytest.mark.gpu


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).bfloat16()


def _run(q, k, v, causal, scale, splits, dev):
    o, lse = ex.forward_kvsplit(q.to(dev), k.to(dev), v.to(dev), causal=causal, scale=scale, splits=splits)
    torch.cuda.synchronize()
    assert ex.device_status() == 0
    return to_np(o), to_np(lse)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk", [(1, 1), (1, 300), (7, 300), (16, 4097), (1, 4097), (130, 1000)])
@pytest.mark.parametrize("splits", [0, 1, 3])
def test_decode_shapes(cuda_device, nq, nk, d, causal, splits):
    B, H = 2, 3
    q, k, v = _rand((B, H, nq, d), nq * 31 + nk), _rand((B, H, nk, d), nk + 7), _rand((B, H, nk, d), nk + 9)
    scale = 1 / math.sqrt(d)
    o, lse = _run(q, k, v, causal, scale, splits, cuda_device)
    o_ref, lse_ref = oracle.decode(q, k, v, scale, causal)
    what = f"nq={nq} nk={nk} d={d} causal={causal} splits={splits}"
    check_o(o, o_ref, what)
    check_lse(lse, lse_ref, what)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk,d,splits", [(1, 4097, 128, 0), (16, 4097, 64, 3), (130, 1000, 128, 0),
                                            (7, 300, 64, 1), (1, 20000, 128, 0)])
def test_decode_shapes_fp16(cuda_device, nq, nk, d, causal, splits):
    """attn_fwd_kvsplit_fp16: the same shapes on fp16 inputs (the oracle takes
    the fp16 values upcast exactly)."""
    B, H = 2, 3
    g = torch.Generator().manual_seed(nq * 17 + nk + d)
    q, k, v = (torch.randn(shape, generator=g).half() for shape in ((B, H, nq, d), (B, H, nk, d), (B, H, nk, d)))
    scale = 1 / math.sqrt(d)
    o, lse = _run(q, k, v, causal, scale, splits, cuda_device)
    o_ref, lse_ref = oracle.decode(q, k, v, scale, causal)
    what = f"fp16 nq={nq} nk={nk} d={d} causal={causal} splits={splits}"
    check_o(o, o_ref, what)
    check_lse(lse, lse_ref, what)


def test_kvsplit_rejects_mixed_dtypes(cuda_device):
    q = torch.zeros((1, 1, 1, 64), dtype=torch.float16, device=cuda_device)
    k = torch.zeros((1, 1, 8, 64), dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(ValueError):
        ex.forward_kvsplit(q, k, k)
    with pytest.raises(ValueError):
        ex.forward_kvsplit(q.float(), k.float(), k.float())


@pytest.mark.parametrize("N,splits", [(1000, 3), (257, 2), (2048, 16), (640, 64)])
def test_square_problem_with_forced_splits(cuda_device, N, splits):
    """Nq = Nk: the causal mask is the square one of attn_fwd; splitting the
    keys must not change the result beyond rounding."""
    q, k, v = (_rand((1, 2, N, 128), N + i) for i in range(3))
    for causal in (False, True):
        o, lse = _run(q, k, v, causal, 0.09, splits, cuda_device)
        o_ref, lse_ref = oracle.forward(q, k, v, 0.09, causal)
        check_o(o, o_ref, f"N={N} splits={splits} causal={causal}")
        check_lse(lse, lse_ref, f"N={N} splits={splits} causal={causal}")


def test_split_count_follows_the_request(cuda_device):
    lib = _lib.load()
    assert lib.attn_fwd_kvsplit_count(1, 1, 1000, 1000, 128, 1, 3) == 3
    assert lib.attn_fwd_kvsplit_count(1, 1, 1000, 1000, 128, 1, 500) == 8  # capped at the 8 key tiles
    assert lib.attn_fwd_kvsplit_count(1, 1, 1000, 1000, 128, 1, 1) == 1
    assert lib.attn_fwd_kvsplit_workspace_bytes(1, 1, 1000, 1000, 128, 1, 1) == 0
    # enough (batch, head, block) CTAs for four waves: no split
    assert lib.attn_fwd_kvsplit_count(4, 32, 4096, 4096, 128, 1, 0) == 1


def test_single_head_32k_causal_every_row(cuda_device):
    """The single-head N = 32768 causal problem through the split forward
    (automatic ranges), every row against the oracle."""
    w = W.SINGLE_HEAD_32K_CAUSAL
    q, k, v, _ = W.make_inputs(w, with_grad_out=False)
    S, _ = ex.kvsplit_plan(*w.shape[:3], w.N, w.d, True, 0)
    assert S > 1
    o, lse = _run(q, k, v, True, w.softmax_scale, 0, cuda_device)
    o_ref, lse_ref = oracle.forward(q, k, v, w.softmax_scale, True)
    check_o(o, o_ref, w.name + " kvsplit")
    check_lse(lse, lse_ref, w.name + " kvsplit")


def test_decode_workload_sampled_heads(cuda_device):
    """The decode bench workload, 8x32 heads of 1 query against 32768 keys,
    causal: the full launch, four heads against the oracle."""
    w = W.DECODE_1Q
    q, k, v = W.make_decode_inputs(w)
    o, lse = _run(q, k, v, w.causal, w.softmax_scale, 0, cuda_device)
    heads = [(0, 0), (3, 17), (7, 31), (5, 2)]
    o_ref, lse_ref = oracle.decode(q, k, v, w.softmax_scale, w.causal, heads=heads)
    sel = lambda a: np.stack([a[b, h] for b, h in heads])  # noqa: E731
    check_o(sel(o), sel(o_ref), w.name)
    check_lse(sel(lse), sel(lse_ref), w.name)


def test_kvsplit_rejects_bad_arguments(cuda_device):
    lib = _lib.load()
    d = torch.empty(1 << 20, dtype=torch.uint8, device=cuda_device)
    pp = d.data_ptr()
    # causal with more queries than keys; no keys; workspace too small
    assert lib.attn_fwd_kvsplit(pp, pp, pp, pp, pp, 1, 1, 200, 100, 64, 0.1, 1, 0, pp, 1 << 20, None) == \
        _lib.ATTN_ERR_INVALID
    assert lib.attn_fwd_kvsplit(pp, pp, pp, pp, pp, 1, 1, 10, 0, 64, 0.1, 0, 0, pp, 1 << 20, None) == \
        _lib.ATTN_ERR_INVALID
    assert lib.attn_fwd_kvsplit(pp, pp, pp, pp, pp, 1, 1, 1000, 1000, 64, 0.1, 0, 4, pp, 16, None) == \
        _lib.ATTN_ERR_INVALID
