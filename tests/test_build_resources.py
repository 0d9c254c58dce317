"""Compiled register counts that the kernels' launch configurations rely on,
read from ptxas's resource report of the in-tree build (no GPU needed).

* A CTA's warps are spread over the SM's four sub-partitions, each with a
  16K-register file: warps_per_sub_partition * 32 * registers <= 16384, or the
  launch fails.
* The backward moves registers between warpgroups with setmaxnreg: the drain
  warpgroup's increase must not exceed what the producer/MMA warpgroup frees,
  or setmaxnreg.inc waits forever (the host refuses such a build at run time;
  this catches it at build time).
"""
import math
import os
import re

import pytest

from exact_attention_106_b200 import build

CSRC = os.path.join(build.PKG_DIR, "csrc")


@pytest.fixture(scope="module")
def registers():
    build.build()
    regs, cur = {}, None
    for line in open(build.RESOURCES_PATH).read().splitlines():
        m = re.search(r"Compiling entry function '(\w+)'", line)
        if m:
            cur = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and cur:
            regs[cur] = int(m.group(1))
            cur = None
    return regs


def _const(path, name):
    m = re.search(r"static constexpr int %s = (\d+);" % name, open(os.path.join(CSRC, path)).read())
    assert m, name
    return int(m.group(1))


ELEMS = ["13__nv_bfloat16", "6__half"]  # mangled element types the kernels are instantiated for


def _kernel(regs, stem, d, params, elem, flag=None):
    """Register count of exattn::stem<d, elem[, flag]>(params); flag is a bool template argument."""
    extra = "" if flag is None else f"Lb{int(flag)}E"
    name = f"_ZN6exattn{len(stem)}{stem}ILi{d}E{elem}{extra}EEvNS_{len(params)}{params}E"
    assert name in regs, sorted(regs)
    return regs[name]


@pytest.mark.parametrize("persist", [False, True])
@pytest.mark.parametrize("elem", ELEMS)
@pytest.mark.parametrize("d", [64, 128])
def test_backward_register_split_fits(registers, d, elem, persist):
    r = _kernel(registers, "attn_bwd_kernel", d, "BwdParams", elem, flag=persist)
    threads = _const("bwd.cuh", "kThreads")
    drain, side = _const("bwd.cuh", "kRegsDrain"), _const("bwd.cuh", "kRegsSide")
    # warpgroup 2 (drain) rises from r to `drain`, warpgroup 3 falls from r to `side`
    assert drain - r <= r - side, (r, drain, side)
    per_sub = math.ceil(threads // 32 / 4)
    assert per_sub * 32 * r <= 16384, (r, per_sub)
    # after the split, one warp of each warpgroup per sub-partition
    assert 32 * (2 * r + drain + side) <= 16384


@pytest.mark.parametrize("elem,d", [(e, d) for e in ELEMS for d in (64, 128, 256)] + [("13__nv_fp8_e4m3", 128)])
def test_forward_fits_the_sub_partitions(registers, d, elem):
    r = _kernel(registers, "attn_fwd_kernel", d, "FwdParams", elem, flag=False)
    src = open(os.path.join(CSRC, "fwd.cuh")).read()
    assert "static constexpr int kSub = (D == 256 || kLean) ? 1 : 2;" in src
    assert "static constexpr int kThreads = 128 * kSub + 64;" in src
    threads = 128 * (1 if d == 256 else 2) + 64  # softmax warps per sub-tile, producer and MMA warps
    per_sub = math.ceil(threads // 32 / 4)
    assert per_sub * 32 * r <= 16384, (r, per_sub)


@pytest.mark.parametrize("elem", ELEMS)
@pytest.mark.parametrize("d", [64, 128])
def test_lean_forward_fits_two_per_sm(registers, d, elem):
    """Lean CTAs (one 128-row sub-tile, 192 threads) run two per SM: both CTAs' warps share the
    sub-partitions' register files, and both CTAs' shared memory and TMEM columns share the SM's."""
    r = _kernel(registers, "attn_fwd_kernel", d, "FwdParams", elem, flag=True)
    src = open(os.path.join(CSRC, "fwd.cuh")).read()
    assert "static constexpr int kCtasPerSm = kLean ? 2 : 1;" in src
    assert "static constexpr uint32_t kTmemCols = kLean ? 256u : 512u;" in src
    assert "static constexpr int kSlots = kLean ? 2 :" in src
    warps = 2 * (128 + 64) // 32  # two CTAs of 4 softmax warps, a producer and an MMA warp
    assert math.ceil(warps / 4) * 32 * r <= 16384, r
    es = 1 if elem == "13__nv_fp8_e4m3" else 2
    smem = (1 + 2) * 128 * d * es + 256  # Q sub-tile, two K/V slots, barriers
    assert 2 * (smem + 1024) <= 228 * 1024, smem  # 1 KB per CTA is reserved by the system
    assert 2 * 256 <= 512  # TMEM columns of the two resident CTAs
