"""The C-ABI library: loads without a GPU, exports every declared symbol, and
rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

from exact_attention_106_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "exattn.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(_lib.SIGNATURES)


def test_every_declared_symbol_is_exported(lib):
    raw = ctypes.CDLL(_lib.LIB_PATH)
    for name in declared_functions():
        assert hasattr(raw, name), name


def test_status_strings(lib):
    assert _lib.status_string(0) == "ATTN_OK"
    assert _lib.status_string(4) == "ATTN_ERR_TIMEOUT"
    assert _lib.status_string(99) == "ATTN_ERR_UNKNOWN"


P = 1 << 20  # a fake, 16-byte aligned "device" address; never dereferenced


def fwd(lib, **kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B=1, H=1, N=8, d=64, scale=0.125, causal=0, stream=None)
    a.update(kw)
    return lib.attn_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["N"], a["d"],
                        a["scale"], a["causal"], a["stream"])


@pytest.mark.parametrize("kw", [
    dict(d=96), dict(d=32), dict(d=512), dict(B=-1), dict(N=-5), dict(scale=0.0), dict(scale=-1.0),
    dict(scale=float("inf")), dict(scale=float("nan")), dict(q=None), dict(lse=None),
    dict(k=P + 8), dict(o=P + 2),
    # padded rows of the [B*H, N] view past 2^31 - 1 (the kernels' 32-bit row coordinates)
    dict(H=1 << 16, N=1 << 16), dict(H=1 << 14, N=1 << 17), dict(B=1 << 15, H=1 << 16, N=1),
    dict(H=1 << 16, N=1 << 16, d=256), dict(H=1 << 14, N=(1 << 17) - 127, d=128),
])
def test_fwd_rejects_bad_arguments_on_host(lib, kw):
    assert fwd(lib, **kw) == _lib.ATTN_ERR_INVALID


@pytest.mark.parametrize("kw", [dict(B=0), dict(H=0), dict(N=0), dict(N=0, q=None, o=None)])
def test_empty_problem_is_a_no_op(lib, kw):
    assert fwd(lib, **kw) == _lib.ATTN_OK


def test_workspace_size(lib):
    assert lib.attn_bwd_workspace_bytes(1, 1, 1, 64) == (128 * 64 + 2 * 128) * 4
    assert lib.attn_bwd_workspace_bytes(2, 3, 129, 128) == 6 * (256 * 128 + 2 * 256) * 4
    assert lib.attn_bwd_workspace_bytes(1, 1, 8, 80) == 0
    assert lib.attn_bwd_workspace_bytes(1, 1, 8, 256) == 0  # the backward takes d = 64, 128 only
    assert lib.attn_bwd_workspace_bytes(0, 1, 8, 64) == 0


def test_bwd_rejects_small_workspace_and_misalignment(lib):
    need = lib.attn_bwd_workspace_bytes(1, 2, 300, 128)
    args = [P] * 9 + [1, 2, 300, 128, 0.1, 1]
    assert lib.attn_bwd(*args, P, need - 1, None) == _lib.ATTN_ERR_INVALID
    assert lib.attn_bwd(*args, P + 16, need, None) == _lib.ATTN_ERR_INVALID  # workspace not 256-aligned
    assert lib.attn_bwd_preprocess(P, P, P, 1, 2, 300, 128, P, need - 4, None) == _lib.ATTN_ERR_INVALID
    assert lib.attn_bwd_dkdv(P, P, P, P, P, P, 1, 2, 300, 128, 0.1, 1, P, 0, None) == _lib.ATTN_ERR_INVALID
    assert lib.attn_bwd_dq_convert(P, 1, 2, 300, 64, 0.0, P, need, None) == _lib.ATTN_ERR_INVALID
    assert lib.attn_bwd(*([P] * 9), 0, 2, 300, 128, 0.1, 1, None, 0, None) == _lib.ATTN_OK
    assert lib.attn_bwd(*([P] * 9), 1, 2, 300, 256, 0.1, 1, P, 1 << 30, None) == _lib.ATTN_ERR_INVALID


def _stage_bytes(G, N, d):
    r = lambda x: (x + 255) // 256 * 256  # noqa: E731
    np_ = (N + 127) // 128 * 128
    return 8 * r(G * N * d * 2) + r(G * N * 4) + r(G * np_ * d * 4 + 2 * G * np_ * 4)


def test_host_buffer_size(lib):
    # 32 pairs, automatic chunks of 4 pairs, three buffer sets
    assert lib.attn_fwd_bwd_host_buffer_bytes(1, 32, 16384, 128, 0) == 3 * _stage_bytes(4, 16384, 128)
    # fewer chunks than buffer sets: one set per chunk
    assert lib.attn_fwd_bwd_host_buffer_bytes(1, 3, 300, 64, 8) == _stage_bytes(3, 300, 64)
    assert lib.attn_fwd_bwd_host_buffer_bytes(2, 3, 300, 64, 4) == 2 * _stage_bytes(4, 300, 64)
    assert lib.attn_fwd_bwd_host_buffer_bytes(2, 3, 300, 64, 1) == 3 * _stage_bytes(1, 300, 64)
    assert lib.attn_fwd_bwd_host_buffer_bytes(1, 1, 8, 80, 0) == 0
    assert lib.attn_fwd_bwd_host_buffer_bytes(1, 2, 8, 64, -1) == 0


def test_host_call_rejects_bad_arguments(lib):
    need = lib.attn_fwd_bwd_host_buffer_bytes(1, 2, 300, 128, 1)
    host = [P] * 9
    good = [1, 2, 300, 128, 0.1, 1]
    assert lib.attn_fwd_bwd_host(*host, *good, P, need - 1, 1, None) == _lib.ATTN_ERR_INVALID  # buffer too small
    assert lib.attn_fwd_bwd_host(*host, *good, P + 16, need, 1, None) == _lib.ATTN_ERR_INVALID  # misaligned
    assert lib.attn_fwd_bwd_host(*host, *good, None, need, 1, None) == _lib.ATTN_ERR_INVALID
    assert lib.attn_fwd_bwd_host(*host, *good, P, need, -1, None) == _lib.ATTN_ERR_INVALID
    assert lib.attn_fwd_bwd_host(None, *host[1:], *good, P, need, 1, None) == _lib.ATTN_ERR_INVALID
    assert lib.attn_fwd_bwd_host(*host, 1, 2, 300, 96, 0.1, 1, P, need, 1, None) == _lib.ATTN_ERR_INVALID
    assert lib.attn_fwd_bwd_host(*host, 1, 2, 300, 128, 0.0, 1, P, need, 1, None) == _lib.ATTN_ERR_INVALID
    assert lib.attn_fwd_bwd_host(*host, 1, 0, 300, 128, 0.1, 1, None, 0, 0, None) == _lib.ATTN_OK  # empty


def test_kvsplit_and_fp8_reject_bad_arguments_on_host(lib):
    v = _lib.ATTN_ERR_INVALID
    # causal with more queries than keys; no keys; negative split count; d = 96
    for fn in (lib.attn_fwd_kvsplit, lib.attn_fwd_kvsplit_fp16):
        assert fn(P, P, P, P, P, 1, 1, 20, 10, 64, 0.1, 1, 0, P, 1 << 20, None) == v
        assert fn(P, P, P, P, P, 1, 1, 20, 0, 64, 0.1, 0, 0, P, 1 << 20, None) == v
        assert fn(P, P, P, P, P, 1, 1, 20, 20, 64, 0.1, 0, -1, P, 1 << 20, None) == v
        assert fn(P, P, P, P, P, 1, 1, 20, 20, 96, 0.1, 0, 0, P, 1 << 20, None) == v
        assert fn(None, None, None, None, None, 1, 1, 0, 10, 64, 0.1, 0, 0, None, 0, None) == 0
    assert lib.attn_fwd_kvsplit_count(1, 1, 20, 10, 64, 1, 0) == 0
    # e4m3: d must be 128, descale factors finite and > 0
    assert lib.attn_fwd_fp8(P, P, P, P, P, 1, 1, 8, 64, 0.1, 0, 1.0, 1.0, 1.0, None) == v
    assert lib.attn_fwd_fp8(P, P, P, P, P, 1, 1, 8, 128, 0.1, 0, 1.0, -1.0, 1.0, None) == v
    # empty problems are a no-op
    assert lib.attn_fwd_kvsplit(None, None, None, None, None, 1, 1, 0, 10, 64, 0.1, 0, 0, None, 0, None) == 0


def test_kvsplit_plan_on_host(lib):
    """The split count and workspace size need no GPU: one range (no
    workspace) when (batch, head, block) CTAs fill four waves, and the
    workspace holds (d + 1) fp32 per row and range, each part 256-aligned."""
    assert lib.attn_fwd_kvsplit_count(4, 32, 8192, 8192, 128, 1, 0) == 1
    assert lib.attn_fwd_kvsplit_workspace_bytes(4, 32, 8192, 8192, 128, 1, 0) == 0
    S = lib.attn_fwd_kvsplit_count(1, 1, 32768, 32768, 128, 1, 0)
    assert 2 <= S <= 64
    rows = S * 32768
    assert lib.attn_fwd_kvsplit_workspace_bytes(1, 1, 32768, 32768, 128, 1, 0) == \
        (rows * 128 * 4 + 255) // 256 * 256 + (rows * 4 + 255) // 256 * 256
    assert lib.attn_fwd_kvsplit_count(1, 1, 1000, 1000, 64, 0, 4) == 4
    # 5 asked over 8 key tiles: ranges of ceil(8 / 5) = 2 tiles, so 4 of them
    assert lib.attn_fwd_kvsplit_count(1, 1, 1000, 1000, 64, 0, 5) == 4


def test_kvsplit_plan_is_per_whole_tile(lib):
    """A decode loop's key count grows by one per step: the automatic plan is
    made on whole key tiles, so the counts within one 128-key tile share it
    (and the planner's cache holds one entry per tile, not per step)."""
    for B, H, Nq in ((8, 32, 1), (8, 32, 16), (1, 8, 16)):
        for t0 in (256, 781):
            plans = {lib.attn_fwd_kvsplit_count(B, H, Nq, nk, 128, 1, 0) for nk in range(128 * t0 + 1, 128 * (t0 + 1) + 1)}
            assert len(plans) == 1, (B, H, Nq, t0, plans)
            assert 1 <= plans.pop() <= 64


def test_wait_limit_from_the_environment():
    """EXATTN_WAIT_TIMEOUT_NS sets the device-side wait limit when the library
    loads; a malformed or negative value is refused rather than ignored."""
    import subprocess
    import sys
    code = "import exact_attention_106_b200._lib as L; L.load()"
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for val, ok in (("5000000", True), ("0", True), ("abc", False), ("-1", False)):
        r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True,
                           env=dict(os.environ, EXATTN_WAIT_TIMEOUT_NS=val))
        assert (r.returncode == 0) == ok, (val, r.stderr[-300:])
