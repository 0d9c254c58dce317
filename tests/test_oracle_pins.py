"""Pins for the fp64 oracle: checks against things other than itself.

Each ``check_*`` helper takes the oracle's two per-head entry points, so the
same checks also run against deliberately broken copies of the oracle (at the
bottom of this file) to show that a plausible mistake fails at least one pin.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")
_EXPR_ENV = {"__builtins__": {}, "log": math.log, "exp": math.exp}


def _ev(x):
    if isinstance(x, list):
        return [_ev(y) for y in x]
    return float(eval(x, _EXPR_ENV))  # expressions from the golden file only


def _rand(n, d, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return [scale * rng.standard_normal((n, d)) for _ in range(4)]


# ---------------------------------------------------------------------------
# pin helpers
# ---------------------------------------------------------------------------
def check_golden(fwd, bwd):
    cases = json.load(open(GOLDEN))["cases"]
    for c in cases:
        q, k, v, do = (np.array(_ev(c[x])) for x in ("q", "k", "v", "do"))
        scale = _ev(c["scale"])
        o, lse = fwd(q, k, v, scale, c["causal"])
        np.testing.assert_allclose(o, np.array(_ev(c["o"])), rtol=0, atol=1e-13, err_msg=c["name"])
        np.testing.assert_allclose(lse, np.array(_ev(c["lse"])), rtol=0, atol=1e-13, err_msg=c["name"])
        r = bwd(q, k, v, do, scale, c["causal"])
        for key in ("dq", "dk", "dv"):
            np.testing.assert_allclose(r[key], np.array(_ev(c[key])), rtol=0, atol=1e-13,
                                       err_msg=f"{c['name']}:{key}")


def check_identical_keys(fwd, bwd):
    """All keys equal -> every visible key gets the same weight."""
    n, d, scale = 9, 4, 0.7
    q, k, v, _ = _rand(n, d, 1)
    k[:] = k[0]
    for causal in (False, True):
        o, lse = fwd(q, k, v, scale, causal)
        for i in range(n):
            vis = i + 1 if causal else n
            np.testing.assert_allclose(o[i], v[:vis].mean(axis=0), rtol=1e-12, atol=1e-12)
            s_i = scale * float(q[i] @ k[0])
            assert abs(lse[i] - (s_i + math.log(vis))) < 1e-12


def check_single_key(fwd, bwd):
    """N = 1: O = V, LSE = scale q.k, dQ = dK = 0, dV = dO."""
    q, k, v, do = _rand(1, 5, 2)
    for causal in (False, True):
        o, lse = fwd(q, k, v, 0.3, causal)
        np.testing.assert_allclose(o, v, rtol=0, atol=1e-14)
        assert abs(lse[0] - 0.3 * float(q[0] @ k[0])) < 1e-14
        r = bwd(q, k, v, do, 0.3, causal)
        np.testing.assert_allclose(r["dq"], 0, atol=1e-14)
        np.testing.assert_allclose(r["dk"], 0, atol=1e-14)
        np.testing.assert_allclose(r["dv"], do, atol=1e-14)


def check_row_shift(fwd, bwd):
    """K' = K + 1 u^T adds scale*q_i.u to row i: O, dQ, dK, dV unchanged; LSE shifts."""
    n, d, scale = 11, 6, 0.4
    q, k, v, do = _rand(n, d, 3)
    u = np.random.default_rng(33).standard_normal(d)
    for causal in (False, True):
        o, lse = fwd(q, k, v, scale, causal)
        o2, lse2 = fwd(q, k + u[None, :], v, scale, causal)
        np.testing.assert_allclose(o2, o, rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(lse2 - lse, scale * (q @ u), rtol=1e-11, atol=1e-11)
        r, r2 = bwd(q, k, v, do, scale, causal), bwd(q, k + u[None, :], v, do, scale, causal)
        for key in ("dq", "dk", "dv"):
            np.testing.assert_allclose(r2[key], r[key], rtol=1e-10, atol=1e-10)


def check_normalisation(fwd, bwd):
    """V = ones gives O = ones (rows of P sum to 1)."""
    n, d = 13, 3
    q, k, _, _ = _rand(n, d, 4, scale=3.0)
    for causal in (False, True):
        o, _ = fwd(q, k, np.ones((n, d)), 0.9, causal)
        np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-14)


def check_finite_differences(fwd, bwd):
    """Central differences of L = sum(O * dO) against dQ, dK, dV."""
    n, d, scale, h = 6, 3, 0.8, 1e-6
    q, k, v, do = _rand(n, d, 5)
    for causal in (False, True):
        r = bwd(q, k, v, do, scale, causal)

        def loss(qq, kk, vv):
            return float(np.sum(fwd(qq, kk, vv, scale, causal)[0] * do))

        for name, idx in (("dq", 0), ("dk", 1), ("dv", 2)):
            num = np.zeros((n, d))
            for i in range(n):
                for j in range(d):
                    args_p = [q.copy(), k.copy(), v.copy()]
                    args_m = [q.copy(), k.copy(), v.copy()]
                    args_p[idx][i, j] += h
                    args_m[idx][i, j] -= h
                    num[i, j] = (loss(*args_p) - loss(*args_m)) / (2 * h)
            err = np.max(np.abs(num - r[name])) / max(1e-12, np.max(np.abs(num)))
            assert err < 1e-6, (name, causal, err)


def check_gradient_identities(fwd, bwd):
    """sum_j dK_j = 0 (rows of dS sum to 0); sum_j dV_j = sum_i dO_i; D = sum_j P dP."""
    n, d, scale = 17, 4, 0.5
    q, k, v, do = _rand(n, d, 6)
    for causal in (False, True):
        r = bwd(q, k, v, do, scale, causal)
        np.testing.assert_allclose(r["dk"].sum(axis=0), 0, atol=1e-12)
        np.testing.assert_allclose(r["dv"].sum(axis=0), do.sum(axis=0), rtol=1e-12, atol=1e-12)
        # D_i = sum_j P_ij dP_ij, with P and dP built independently in torch fp64.
        qt, kt, vt, dot = (torch.from_numpy(x) for x in (q, k, v, do))
        s = scale * qt @ kt.T
        if causal:
            s = s.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), float("-inf"))
        p = torch.softmax(s, dim=-1)
        dp = dot @ vt.T
        np.testing.assert_allclose(r["D"], (p * dp).sum(-1).numpy(), rtol=1e-12, atol=1e-12)


def check_permutation(fwd, bwd):
    """Non-causal: permuting K,V rows together leaves O unchanged; permuting Q permutes O."""
    n, d, scale = 10, 4, 0.6
    q, k, v, _ = _rand(n, d, 7)
    perm = np.random.default_rng(77).permutation(n)
    o, lse = fwd(q, k, v, scale, False)
    o2, lse2 = fwd(q, k[perm], v[perm], scale, False)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-12)
    o3, lse3 = fwd(q[perm], k, v, scale, False)
    np.testing.assert_allclose(o3, o[perm], rtol=0, atol=0)
    np.testing.assert_allclose(lse3, lse[perm], rtol=0, atol=0)


def check_torch_sdpa(fwd, bwd):
    """Library special case: PyTorch's CPU fp64 SDPA and autograd."""
    for n, d, causal, scale, boost in ((37, 8, False, 0.35, 1.0), (37, 8, True, 0.35, 1.0),
                                       (64, 16, True, 0.25, 8.0)):
        q, k, v, do = _rand(n, d, 8 + n + d)
        q = q * boost
        qt, kt, vt = (torch.from_numpy(x).requires_grad_(True) for x in (q, k, v))
        ot = torch.nn.functional.scaled_dot_product_attention(
            qt[None, None], kt[None, None], vt[None, None], is_causal=causal, scale=scale)[0, 0]
        ot.backward(torch.from_numpy(do))
        s = scale * (qt @ kt.T)
        if causal:
            s = s.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), float("-inf"))
        lse_t = torch.logsumexp(s, dim=-1)
        o, lse = fwd(q, k, v, scale, causal)
        np.testing.assert_allclose(o, ot.detach().numpy(), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse, lse_t.detach().numpy(), rtol=1e-12, atol=1e-12)
        r = bwd(q, k, v, do, scale, causal)
        np.testing.assert_allclose(r["dq"], qt.grad.numpy(), rtol=1e-10, atol=1e-10)
        np.testing.assert_allclose(r["dk"], kt.grad.numpy(), rtol=1e-10, atol=1e-10)
        np.testing.assert_allclose(r["dv"], vt.grad.numpy(), rtol=1e-10, atol=1e-10)


ALL_CHECKS = [check_golden, check_identical_keys, check_single_key, check_row_shift,
              check_normalisation, check_finite_differences, check_gradient_identities,
              check_permutation, check_torch_sdpa]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check(oracle.forward_head, oracle.backward_head)


def test_row_blocking_is_invisible():
    """More rows than one oracle row block: results match torch fp64 too."""
    n, d = 600, 8
    q, k, v, do = _rand(n, d, 9)
    o, lse = oracle.forward_head(q, k, v, 0.3, True)
    ot = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(x)[None, None] for x in (q, k, v)), is_causal=True, scale=0.3)[0, 0]
    np.testing.assert_allclose(o, ot.numpy(), rtol=1e-12, atol=1e-12)


def test_batched_wrappers_and_head_sampling():
    rng = np.random.default_rng(10)
    q, k, v, do = (rng.standard_normal((2, 3, 20, 4)) for _ in range(4))
    o, lse = oracle.forward(q, k, v, 0.5, True)
    o1, lse1 = oracle.forward_head(q[1, 2], k[1, 2], v[1, 2], 0.5, True)
    np.testing.assert_array_equal(o[1, 2], o1)
    r = oracle.backward(q, k, v, do, 0.5, True, heads=[(0, 1)])
    assert np.isnan(r["dq"][1, 2]).all() and not np.isnan(r["dq"][0, 1]).any()
    np.testing.assert_allclose(r["o"][0, 1], o[0, 1], rtol=1e-14, atol=1e-14)


# ---------------------------------------------------------------------------
# Planted mistakes: broken copies of the oracle must fail at least one pin.
# ---------------------------------------------------------------------------
def _mutant(kind):
    base_fwd, base_bwd = oracle.forward_head, oracle.backward_head

    def fwd(q, k, v, scale, causal):
        if kind == "no_scale":
            return base_fwd(q, k, v, 1.0, causal)
        if kind == "transposed_scores":
            # uses K Q^T instead of Q K^T
            return base_fwd(k, q, v, scale, causal)
        if kind == "causal_flipped":
            o, lse = base_fwd(q[::-1], k[::-1], v[::-1], scale, causal)
            return o[::-1], lse[::-1]
        if kind == "lse_log2":
            o, lse = base_fwd(q, k, v, scale, causal)
            return o, lse / math.log(2.0)
        return base_fwd(q, k, v, scale, causal)

    def bwd(q, k, v, do, scale, causal):
        r = dict(base_bwd(q, k, v, do, scale, causal))
        if kind == "dq_missing_scale":
            r["dq"] = r["dq"] / scale
        elif kind == "dk_sign":
            r["dk"] = -r["dk"]
        elif kind == "dv_transposed":
            r["dv"] = r["dv"][::-1].copy()
        elif kind == "no_D":
            # dS = P * dP (forgets the rowsum term): dQ = scale * P*dP K
            rr = {}
            n = q.shape[0]
            s = scale * q @ k.T
            if causal:
                s = np.where(np.arange(n)[None] > np.arange(n)[:, None], -np.inf, s)
            p = np.exp(s - s.max(1, keepdims=True))
            p /= p.sum(1, keepdims=True)
            ds = p * (do @ v.T)
            rr["dq"], rr["dk"] = scale * ds @ k, scale * ds.T @ q
            r.update(rr)
        return r

    return fwd, bwd


@pytest.mark.parametrize("kind", ["no_scale", "transposed_scores", "causal_flipped", "lse_log2",
                                  "dq_missing_scale", "dk_sign", "dv_transposed", "no_D"])
def test_pins_catch_planted_mistake(kind):
    fwd, bwd = _mutant(kind)
    failures = 0
    for check in ALL_CHECKS:
        try:
            check(fwd, bwd)
        except AssertionError:
            failures += 1
    assert failures >= 1, f"no pin caught the planted mistake {kind}"
