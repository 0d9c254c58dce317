"""fp64 CPU oracle for exact scaled-dot-product attention, forward and backward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call
this module: only the test suite, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use it.  It shares no code with the CUDA path.

What it computes
----------------
The method computes exactly the plain attention definition (it "does not
approximate attention or change the math": "11.11 Flash Attention",
§Flash Attention: The Key Insight; likewise the red-flag note of
"Walk through the FlashAttention algorithm ..." that calls treating it as an
approximation a mistake).  So this oracle is that definition written out:

    S = scale * Q K^T                      ("11.11 Flash Attention",
    P = softmax(S) row-wise                 §Standard Attention: Step by Step,
    O = P V                                 Steps 1-3 and the formula
                                            softmax(Q K^T / sqrt(d_k)) V)

with, per row, the logsumexp LSE = m + ln(sum_j exp(S_j - m)), m = max_j S_j,
which is the "per-row m and l" the forward keeps for the backward
("Walk through the FlashAttention algorithm ...", answer to "How does the
backward pass avoid storing the n x n attention matrix?") folded into one
number.

The pages give no backward formulas; the backward here is the chain rule of
the forward definition above (dP = dO V^T, dS = P o (dP - rowsum(dO o O)),
dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO).

Rows are processed in blocks so that memory is O(block x N) per head; inside
a block the softmax is the exact two-pass form (max first, then exp and sum),
not the online form.  Causal masking (query i sees key j iff j <= i, a
square top-left mask) is not on the pages; it is the reading used here.

All arithmetic is float64 on inputs that are the bf16 values upcast exactly.
"""
from __future__ import annotations

import numpy as np

_ROW_BLOCK = 256


def _as_f64(x) -> np.ndarray:
    """Accept numpy arrays or CPU torch tensors (any float dtype)."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch  # local: the oracle itself needs only numpy
        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _scores(qb: np.ndarray, k: np.ndarray, scale: float, row0: int, causal: bool) -> np.ndarray:
    """S rows [row0, row0+len(qb)) = scale * Q_rows K^T, with the causal mask."""
    s = scale * (qb @ k.T)
    if causal:
        rows = np.arange(row0, row0 + qb.shape[0])[:, None]
        cols = np.arange(k.shape[0])[None, :]
        s = np.where(cols > rows, -np.inf, s)
    return s


def _softmax_rows(s: np.ndarray):
    """Two-pass exact softmax of each row; returns (P, LSE)."""
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    l = np.sum(e, axis=1, keepdims=True)
    return e / l, (m + np.log(l))[:, 0]


def forward_head(q, k, v, scale: float, causal: bool):
    """One (batch, head): q,k,v [N,d] -> (O [N,d], LSE [N]) in float64."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    n = q.shape[0]
    o = np.empty_like(q)
    lse = np.empty(n)
    for r0 in range(0, n, _ROW_BLOCK):
        r1 = min(n, r0 + _ROW_BLOCK)
        p, lse[r0:r1] = _softmax_rows(_scores(q[r0:r1], k, scale, r0, causal))
        o[r0:r1] = p @ v
    return o, lse


def backward_head(q, k, v, do, scale: float, causal: bool):
    """One (batch, head), fwd + bwd from scratch.

    Returns a dict with O, LSE, D (= rowsum(dO o O)), dQ, dK, dV, all float64.
    """
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    n = q.shape[0]
    o = np.empty_like(q)
    lse = np.empty(n)
    dd = np.empty(n)
    dq = np.empty_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for r0 in range(0, n, _ROW_BLOCK):
        r1 = min(n, r0 + _ROW_BLOCK)
        p, lse[r0:r1] = _softmax_rows(_scores(q[r0:r1], k, scale, r0, causal))
        o_blk = p @ v
        o[r0:r1] = o_blk
        do_blk = do[r0:r1]
        dp = do_blk @ v.T                                  # dP = dO V^T
        d_blk = np.sum(do_blk * o_blk, axis=1)             # D = rowsum(dO o O)
        dd[r0:r1] = d_blk
        ds = p * (dp - d_blk[:, None])                     # dS = P o (dP - D)
        dq[r0:r1] = scale * (ds @ k)                       # dQ = scale dS K
        dk += scale * (ds.T @ q[r0:r1])                    # dK = scale dS^T Q
        dv += p.T @ do_blk                                 # dV = P^T dO
    return {"o": o, "lse": lse, "D": dd, "dq": dq, "dk": dk, "dv": dv}


def forward(q, k, v, scale: float, causal: bool, heads=None):
    """Whole [B,H,N,d] tensors, or only the listed (b, h) pairs.

    Returns (O, LSE) as float64 arrays [B,H,N,d] and [B,H,N]; entries of heads
    that were not requested are NaN.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, H, N, d = q.shape
    o = np.full((B, H, N, d), np.nan)
    lse = np.full((B, H, N), np.nan)
    for b, h in (heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]):
        o[b, h], lse[b, h] = forward_head(q[b, h], k[b, h], v[b, h], scale, causal)
    return o, lse


def backward(q, k, v, do, scale: float, causal: bool, heads=None):
    """Whole [B,H,N,d] tensors, or only the listed (b, h) pairs.

    Returns a dict of float64 arrays (o, lse, D, dq, dk, dv); heads that were
    not requested are NaN.
    """
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    B, H, N, d = q.shape
    out = {
        "o": np.full((B, H, N, d), np.nan), "lse": np.full((B, H, N), np.nan),
        "D": np.full((B, H, N), np.nan), "dq": np.full((B, H, N, d), np.nan),
        "dk": np.full((B, H, N, d), np.nan), "dv": np.full((B, H, N, d), np.nan),
    }
    for b, h in (heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]):
        r = backward_head(q[b, h], k[b, h], v[b, h], do[b, h], scale, causal)
        for key, val in r.items():
            out[key][b, h] = val
    return out


# ---------------------------------------------------------------------------
# Decode: a few new queries against a long key/value history.
#
# The serving use the pages name ("Walk through the FlashAttention algorithm
# ...", the paragraph on products: vLLM / TensorRT-LLM; "11.11 Flash
# Attention", §Using Flash Attention, "vLLM") runs attention for the last Nq
# positions of a sequence of Nk tokens.  It is the same definition with a
# rectangular score matrix; under the causal mask the Nq queries are the LAST
# Nq positions, so query i (0-based among the Nq) sees key j iff
# j <= Nk - Nq + i (bottom-right alignment; for Nq = Nk it is the square mask
# used above).  The pages do not state the alignment; this is the reading.
# ---------------------------------------------------------------------------
def decode_head(q, k, v, scale: float, causal: bool):
    """One (batch, head): q [Nq,d], k,v [Nk,d] -> (O [Nq,d], LSE [Nq]) in float64."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    nq, nk = q.shape[0], k.shape[0]
    # the queries sit at absolute positions nk - nq .. nk - 1
    p, lse = _softmax_rows(_scores(q, k, scale, nk - nq, causal))
    return p @ v, lse


def decode(q, k, v, scale: float, causal: bool, heads=None):
    """Whole tensors q [B,H,Nq,d], k/v [B,H,Nk,d], or only the listed (b, h)
    pairs; returns (O [B,H,Nq,d], LSE [B,H,Nq]) as float64, NaN elsewhere."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, H, nq, d = q.shape
    o = np.full((B, H, nq, d), np.nan)
    lse = np.full((B, H, nq), np.nan)
    for b, h in (heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]):
        o[b, h], lse[b, h] = decode_head(q[b, h], k[b, h], v[b, h], scale, causal)
    return o, lse
