"""The tiled online-softmax algorithm, restated in fp64, equals the oracle.

"11.11 Flash Attention", §The Tiling Algorithm describes the forward as a
walk over K/V blocks (outer) and Q blocks (inner) that keeps, per query row,
a running maximum m and a running sum l of exponentials, rescales the
earlier partial output by exp(m_old - m_new) whenever the maximum grows, and
re-normalises O after every step.  §Flash Attention 2 swaps the two loops
(Q outer) and trims the non-matmul work; the CUDA forward uses that order,
divides by l once at the end, and only moves its reference maximum when the
new block maximum exceeds it by more than a threshold (exact: O and l are
always scaled against the same reference).

These tests restate both orders in plain numpy float64 (written here from the
description, not from the page's listing) and check that they reproduce the
two-pass oracle to ~1e-12: the algebra the kernels rely on is exact.
"""
import math

import numpy as np
import pytest

import oracle


def _mask_block(s, r0, c0, causal, n):
    rows = np.arange(r0, r0 + s.shape[0])[:, None]
    cols = np.arange(c0, c0 + s.shape[1])[None, :]
    bad = cols >= n
    if causal:
        bad = bad | (cols > rows)
    return np.where(bad, -np.inf, s)


def tiled_kv_outer(q, k, v, scale, causal, br, bc):
    """K/V blocks outside, Q blocks inside, O normalised at every step."""
    n, d = q.shape
    out = np.zeros((n, d))
    run_sum = np.zeros(n)
    run_max = np.full(n, -np.inf)
    for c0 in range(0, n, bc):
        kb, vb = k[c0:c0 + bc], v[c0:c0 + bc]
        for r0 in range(0, n, br):
            rs = slice(r0, min(n, r0 + br))
            s = _mask_block(scale * q[rs] @ kb.T, r0, c0, causal, n)
            blk_max = s.max(axis=1)
            new_max = np.maximum(run_max[rs], blk_max)
            safe = np.where(np.isfinite(new_max), new_max, 0.0)
            keep = np.exp(run_max[rs] - safe)          # weight of what was there
            e = np.exp(s - safe[:, None])
            new_sum = keep * run_sum[rs] + e.sum(axis=1)
            with np.errstate(invalid="ignore", divide="ignore"):
                upd = ((keep * run_sum[rs])[:, None] * out[rs] + e @ vb) / new_sum[:, None]
            out[rs] = np.where(new_sum[:, None] > 0, upd, 0.0)
            run_sum[rs], run_max[rs] = new_sum, new_max
    return out, run_max + np.log(run_sum)


def tiled_q_outer(q, k, v, scale, causal, br, bc, threshold=0.0):
    """Q blocks outside, K/V blocks inside, one division at the end.

    The reference maximum ``ref`` only moves when a block maximum exceeds it by
    more than ``threshold`` (natural-log units); exponentials are taken against
    ``ref`` so they stay below exp(threshold).
    """
    n, d = q.shape
    out = np.zeros((n, d))
    lse = np.zeros(n)
    for r0 in range(0, n, br):
        rs = slice(r0, min(n, r0 + br))
        rows = rs.stop - rs.start
        acc = np.zeros((rows, d))
        l = np.zeros(rows)
        ref = np.full(rows, -np.inf)
        last = rs.stop if causal else n
        for c0 in range(0, last, bc):
            s = _mask_block(scale * q[rs] @ k[c0:c0 + bc].T, r0, c0, causal, n)
            blk_max = s.max(axis=1)
            move = blk_max > ref + threshold
            new_ref = np.where(move, np.maximum(ref, blk_max), ref)
            safe_new = np.where(np.isfinite(new_ref), new_ref, 0.0)
            alpha = np.where(np.isfinite(ref), np.exp(ref - safe_new), 0.0)
            acc *= alpha[:, None]
            l *= alpha
            ref = new_ref
            p = np.exp(s - safe_new[:, None])
            l += p.sum(axis=1)
            acc += p @ v[c0:c0 + bc]
        out[rs] = acc / l[:, None]
        lse[rs] = ref + np.log(l)
    return out, lse


CASES = [
    (64, 8, False, 16, 16), (64, 8, True, 16, 16), (100, 8, True, 32, 16),
    (100, 16, False, 16, 32), (129, 8, True, 64, 64), (7, 4, True, 4, 4),
]


@pytest.mark.parametrize("n,d,causal,br,bc", CASES)
def test_pages_order_matches_oracle(n, d, causal, br, bc):
    rng = np.random.default_rng(n * 31 + d)
    q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
    o_ref, lse_ref = oracle.forward_head(q, k, v, 1 / math.sqrt(d), causal)
    o, lse = tiled_kv_outer(q, k, v, 1 / math.sqrt(d), causal, br, bc)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("threshold", [0.0, math.log(256.0), 30.0])
@pytest.mark.parametrize("n,d,causal,br,bc", CASES)
def test_swapped_order_deferred_division_matches_oracle(n, d, causal, br, bc, threshold):
    rng = np.random.default_rng(n * 17 + d)
    q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
    q[: n // 2] *= 8.0                      # large scores stress the rescale
    o_ref, lse_ref = oracle.forward_head(q, k, v, 1 / math.sqrt(d), causal)
    o, lse = tiled_q_outer(q, k, v, 1 / math.sqrt(d), causal, br, bc, threshold)
    np.testing.assert_allclose(o, o_ref, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-11, atol=1e-11)
