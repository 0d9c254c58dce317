"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and compare with the fp64 oracle under the stated tolerances.

Tolerances (on the same seeded bf16 inputs):
  O      max |O - O_ref| <= 2e-2 over the whole tensor
  LSE    |LSE - LSE_ref| <= 1e-3 * max(1, |LSE_ref|) per row
  dQ/dK/dV  max |g - g_ref| / max(max |g_ref|, 1e-3) <= 5e-2 per tensor
"""
import numpy as np
import torch

import exact_attention_106_b200 as ex
import oracle

O_ATOL = 2e-2
LSE_RTOL = 1e-3
GRAD_RTOL = 5e-2


def to_np(t):
    return t.detach().to("cpu", torch.float64).numpy()


def run_cuda(q, k, v, do, causal, scale, with_bwd=True, device="cuda:0"):
    """CPU bf16 inputs -> CUDA path -> CPU outputs (dict of float64 arrays)."""
    qd, kd, vd = (x.to(device) for x in (q, k, v))
    o, lse = ex.forward(qd, kd, vd, causal=causal, scale=scale)
    out = {"o": o, "lse": lse}
    if with_bwd:
        dod = do.to(device)
        dq, dk, dv = ex.backward(qd, kd, vd, o, lse, dod, causal=causal, scale=scale)
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert ex.device_status() == 0
    return {key: to_np(val) for key, val in out.items()}


def check_o(o, o_ref, what=""):
    err = float(np.max(np.abs(o - o_ref)))
    assert np.isfinite(o).all(), f"{what}: non-finite O"
    assert err <= O_ATOL, f"{what}: max|dO| = {err:.3e} > {O_ATOL}"
    return err


def check_lse(lse, lse_ref, what=""):
    assert np.isfinite(lse).all(), f"{what}: non-finite LSE"
    rel = np.abs(lse - lse_ref) / np.maximum(1.0, np.abs(lse_ref))
    err = float(np.max(rel))
    assert err <= LSE_RTOL, f"{what}: LSE rel err {err:.3e} > {LSE_RTOL}"
    return err


# Floor of the relative-to-max denominator: where the exact gradient is all
# zeros (N = 1 gives dQ = dK = 0), fp32 rounding leaves ~1e-8; the check then
# reads |g| <= 5e-2 * 1e-3.
GRAD_FLOOR = 1e-3


def check_grad(g, g_ref, what=""):
    assert np.isfinite(g).all(), f"{what}: non-finite gradient"
    den = max(float(np.max(np.abs(g_ref))), GRAD_FLOOR)
    err = float(np.max(np.abs(g - g_ref))) / den
    assert err <= GRAD_RTOL, f"{what}: rel-to-max err {err:.3e} > {GRAD_RTOL}"
    return err


def check_all(got, ref, heads=None, what="", with_bwd=True):
    """Compare (optionally only the listed (b, h) heads)."""
    sel = (lambda a: a) if heads is None else (lambda a: np.stack([a[b, h] for b, h in heads]))
    errs = {"o": check_o(sel(got["o"]), sel(ref["o"]), what + " O"),
            "lse": check_lse(sel(got["lse"]), sel(ref["lse"]), what + " LSE")}
    if with_bwd:
        for key in ("dq", "dk", "dv"):
            errs[key] = check_grad(sel(got[key]), sel(ref[key]), f"{what} {key}")
    return errs


def oracle_ref(q, k, v, do, causal, scale, heads=None, with_bwd=True):
    if with_bwd:
        return oracle.backward(q, k, v, do, scale, causal, heads=heads)
    o, lse = oracle.forward(q, k, v, scale, causal, heads=heads)
    return {"o": o, "lse": lse}
