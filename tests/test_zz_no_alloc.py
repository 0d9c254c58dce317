"""attn_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc: code held to a device-memory budget fixed
at start-up, plugins whose host program owns the device allocator, and code
where an allocation (which can synchronise the whole device) is not allowed.
For them the library keeps the backward's scratch in its own fixed device
array of EXATTN_NOALLOC_SCRATCH_BYTES.  This file checks, through the C ABI,
that the variant gives the same results as attn_bwd with a caller-provided
workspace, twice in a row on the shared array, that it allocates nothing, and
that it refuses problems too big for the array.

It is collected last on purpose (file name), so a run that stops at its first
failure has already run every other test.
"""
import math

import pytest
import torch

import exact_attention_106_b200 as ex
from exact_attention_106_b200 import _lib
from parity_util import check_grad, to_np

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 64 * 1024 * 1024


def _noalloc(lib, q, k, v, o, lse, do, dq, dk, dv, causal, scale):
    B, H, N, d = q.shape
    return lib.attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, scale,
                                int(causal), torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("shape,causal", [((2, 3, 517, 64), True), ((1, 4, 1000, 128), False),
                                          ((2, 8, 1024, 64), True)])
def test_noalloc_matches_workspace_backward_twice(cuda_device, shape, causal):
    lib = _lib.load()
    B, H, N, d = shape
    scale = 1.0 / math.sqrt(d)
    g = torch.Generator().manual_seed(N + d)
    q, k, v, do = (torch.randn(shape, generator=g).bfloat16().to(cuda_device) for _ in range(4))
    o, lse = ex.forward(q, k, v, causal=causal, scale=scale)
    ref = ex.backward(q, k, v, o, lse, do, causal=causal, scale=scale)
    outs = [tuple(torch.full_like(q, float("nan")) for _ in range(3)) for _ in range(2)]
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for dq, dk, dv in outs:  # two calls in a row on the shared scratch array
        st = _noalloc(lib, q, k, v, o, lse, do, dq, dk, dv, causal, scale)
        assert st == _lib.ATTN_OK, _lib.status_string(st)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] >= free_before - (1 << 20), "device memory was allocated"
    assert ex.device_status() == 0
    for dq, dk, dv in outs:
        for got, want, name in zip((dq, dk, dv), ref, ("dq", "dk", "dv")):
            check_grad(to_np(got), to_np(want), f"noalloc {name}")


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_device):
    lib = _lib.load()
    # d = 128: 1008 padded 128-row tiles fit in 64 MiB, 1009 do not.
    assert lib.attn_bwd_workspace_bytes(1, 1008, 128, 128) <= SCRATCH_BYTES
    assert lib.attn_bwd_workspace_bytes(1, 1009, 128, 128) > SCRATCH_BYTES
    p = 1 << 20  # never dereferenced: the size check comes first
    args = [p] * 9
    assert lib.attn_bwd_noalloc(*args, 1, 1009, 128, 128, 0.1, 0, None) == _lib.ATTN_ERR_INVALID
    assert lib.attn_bwd_noalloc(*args, 1, 32, 16384, 128, 0.1, 1, None) == _lib.ATTN_ERR_INVALID
    assert lib.attn_bwd_noalloc(*args, 1, 1, 8, 96, 0.1, 0, None) == _lib.ATTN_ERR_INVALID


def test_noalloc_follows_a_device_reset(cuda_device, tmp_path):
    """After cudaDeviceReset the context, and with it the scratch array, is
    created anew, possibly at another address; the next attn_bwd_noalloc call
    must use the new one.  Run in a child process that holds a single CUDA
    runtime (a build of the library linked against the shared libcudart, no
    torch), so the reset re-creates the context the library's kernels use."""
    import json
    import os
    import subprocess
    import sys

    from exact_attention_106_b200 import build as b

    cudart = "/usr/local/cuda/lib64/libcudart.so.12"
    if not os.path.exists(cudart):
        pytest.fail(f"{cudart} missing: cannot build the shared-runtime variant")
    so = str(tmp_path / "libexattn_cudart_shared.so")
    proc = subprocess.run(b.build_command(so, cudart="shared"), capture_output=True, text=True)
    assert proc.returncode == 0, proc.stderr[-2000:]
    child = os.path.join(os.path.dirname(os.path.abspath(__file__)), "noalloc_reset_child.py")
    env = dict(os.environ, CUDA_VISIBLE_DEVICES=os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0])
    run = subprocess.run([sys.executable, child, cudart, so], capture_output=True, text=True, timeout=300, env=env)
    assert run.returncode == 0, run.stdout[-2000:] + run.stderr[-2000:]
    res = json.loads(run.stdout.strip().splitlines()[-1])
    for phase in ("before", "after"):
        # dK and dV have a fixed summation order; dQ's reduce-adds do not
        assert res[phase]["dk"] == 0.0 and res[phase]["dv"] == 0.0, res
        assert res[phase]["dq"] <= 5e-2, res
