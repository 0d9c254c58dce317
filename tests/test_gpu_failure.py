"""Failure detection without a GPU fault.

Every wait of the kernels on their internal barriers is limited in time.  Here
the kernels are told to skip their first K/V load, so one role waits on a
barrier that nothing completes, with the limit set to 20 ms: the kernels must
record ATTN_ERR_TIMEOUT, leave their loops, let in-flight copies and MMAs
finish and return, and the CUDA context must stay usable (a correct run right
after, with injection off and the limit restored, matches the oracle).
Nothing here faults, traps or hangs the GPU.
"""
import math

import pytest
import torch

import exact_attention_106_b200 as ex
from exact_attention_106_b200 import _lib
from parity_util import check_all, oracle_ref, run_cuda

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128])
def test_wait_limit_runs_out_and_context_survives(cuda_device, d):
    lib = _lib.load()
    g = torch.Generator().manual_seed(d)
    q, k, v, do = (torch.randn((1, 2, 700, d), generator=g).bfloat16() for _ in range(4))
    qd, kd, vd, dod = (x.to(cuda_device) for x in (q, k, v, do))
    assert ex.device_status() == 0
    lib.attn_set_wait_timeout_ns(20_000_000)
    lib.attn_debug_inject_stall(1)
    try:
        o, lse = ex.forward(qd, kd, vd, causal=True)
        st_fwd = ex.device_status()
        ex.backward(qd, kd, vd, o, lse, dod, causal=True)
        st_bwd = ex.device_status()
    finally:
        lib.attn_debug_inject_stall(0)
        lib.attn_set_wait_timeout_ns(0)
    assert st_fwd == _lib.ATTN_ERR_TIMEOUT
    assert st_bwd == _lib.ATTN_ERR_TIMEOUT
    assert ex.device_status() == 0  # the status word was cleared by the read
    scale = 1 / math.sqrt(d)
    got = run_cuda(q, k, v, do, True, scale)
    ref = oracle_ref(q, k, v, do, True, scale)
    check_all(got, ref, what=f"after timeout d={d}")


def test_check_flag_raises_on_timeout(cuda_device):
    """forward(check=True) / backward(check=True) turn a recorded wait timeout
    into ExattnError instead of returning undefined outputs silently."""
    lib = _lib.load()
    g = torch.Generator().manual_seed(5)
    q, k, v, do = (torch.randn((1, 2, 300, 128), generator=g).bfloat16().to(cuda_device) for _ in range(4))
    o, lse = ex.forward(q, k, v, causal=True, check=True)  # clean run: no raise
    lib.attn_set_wait_timeout_ns(20_000_000)
    lib.attn_debug_inject_stall(1)
    try:
        with pytest.raises(ex.ExattnError) as e1:
            ex.forward(q, k, v, causal=True, check=True)
        with pytest.raises(ex.ExattnError) as e2:
            ex.backward(q, k, v, o, lse, do, causal=True, check=True)
    finally:
        lib.attn_debug_inject_stall(0)
        lib.attn_set_wait_timeout_ns(0)
    assert e1.value.status == _lib.ATTN_ERR_TIMEOUT and e2.value.status == _lib.ATTN_ERR_TIMEOUT
    assert ex.device_status() == 0


def test_check_flag_raises_on_timeout_in_the_split_and_e4m3_forwards(cuda_device):
    """The split-key and e4m3 forwards run the same kernel with the same
    bounded waits: an injected stall surfaces as ATTN_ERR_TIMEOUT through
    check=True, and the context stays usable."""
    lib = _lib.load()
    g = torch.Generator().manual_seed(9)
    q = torch.randn((1, 2, 16, 128), generator=g).bfloat16().to(cuda_device)
    kv = torch.randn((1, 2, 3000, 128), generator=g).bfloat16().to(cuda_device)
    x8 = torch.randn((1, 2, 300, 128), generator=g).to(torch.float8_e4m3fn).to(cuda_device)
    lib.attn_set_wait_timeout_ns(20_000_000)
    lib.attn_debug_inject_stall(1)
    try:
        with pytest.raises(ex.ExattnError) as e1:
            ex.forward_kvsplit(q, kv, kv, causal=True, splits=3, check=True)
        with pytest.raises(ex.ExattnError) as e2:
            ex.forward_fp8(x8, x8, x8, 1.0, 1.0, 1.0, causal=True, check=True)
    finally:
        lib.attn_debug_inject_stall(0)
        lib.attn_set_wait_timeout_ns(0)
    assert e1.value.status == _lib.ATTN_ERR_TIMEOUT and e2.value.status == _lib.ATTN_ERR_TIMEOUT
    assert ex.device_status() == 0
    o, _ = ex.forward_kvsplit(q, kv, kv, causal=True, splits=3, check=True)  # clean run afterwards
    assert torch.isfinite(o.float()).all()
