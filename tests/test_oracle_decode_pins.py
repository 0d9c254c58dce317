"""Pins for the oracle's decode function (few queries, long key history,
bottom-right causal alignment): closed forms, a library special case and
invariants, plus planted mistakes that each fail one of them."""
import math

import numpy as np
import pytest
import torch

import oracle


def _rand(nq, nk, d, seed):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((nq, d)), rng.standard_normal((nk, d)), rng.standard_normal((nk, d))


def check_identical_keys(dec):
    """All keys equal: query i averages the V rows it sees; with the causal
    mask that is the first nk - nq + i + 1 of them."""
    nq, nk, d, scale = 5, 13, 4, 0.6
    q, k, v = _rand(nq, nk, d, 1)
    k[:] = k[0]
    for causal in (False, True):
        o, lse = dec(q, k, v, scale, causal)
        for i in range(nq):
            vis = nk - nq + i + 1 if causal else nk
            np.testing.assert_allclose(o[i], v[:vis].mean(axis=0), rtol=1e-12, atol=1e-12)
            assert abs(lse[i] - (scale * float(q[i] @ k[0]) + math.log(vis))) < 1e-12


def check_single_query_single_key(dec):
    q, k, v = _rand(1, 1, 6, 2)
    for causal in (False, True):
        o, lse = dec(q, k, v, 0.25, causal)
        np.testing.assert_allclose(o, v, atol=1e-14)
        assert abs(lse[0] - 0.25 * float(q[0] @ k[0])) < 1e-14


def check_last_query_sees_everything(dec):
    """Under the causal mask the last query is the newest position: it sees
    every key, exactly as without the mask; the first sees all but nq - 1."""
    q, k, v = _rand(4, 9, 3, 3)
    o_c, lse_c = dec(q, k, v, 0.5, True)
    o_f, lse_f = dec(q, k, v, 0.5, False)
    np.testing.assert_allclose(o_c[-1], o_f[-1], atol=1e-13)
    assert abs(lse_c[-1] - lse_f[-1]) < 1e-13
    o_0, _ = dec(q[:1], k[:6], v[:6], 0.5, False)  # query 0 sees keys 0..5
    np.testing.assert_allclose(o_c[0], o_0[0], atol=1e-13)


def check_sdpa(dec):
    """PyTorch CPU fp64 scaled_dot_product_attention with an explicit boolean
    mask (True = may attend) built for the bottom-right alignment."""
    nq, nk, d, scale = 7, 40, 8, 0.3
    q, k, v = _rand(nq, nk, d, 4)
    for causal in (False, True):
        o, lse = dec(q, k, v, scale, causal)
        i = np.arange(nq)[:, None]
        j = np.arange(nk)[None, :]
        mask = torch.from_numpy(j <= nk - nq + i) if causal else None
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None],
            attn_mask=None if mask is None else mask[None], scale=scale)[0].numpy()
        np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)
        s = scale * q @ k.T
        if causal:
            s = np.where(mask.numpy(), s, -np.inf)
        np.testing.assert_allclose(lse, np.log(np.exp(s).sum(axis=1)), rtol=1e-12, atol=1e-12)


def check_key_permutation(dec):
    """Without the mask, permuting K and V rows together changes nothing."""
    q, k, v = _rand(3, 17, 5, 5)
    perm = np.random.default_rng(55).permutation(17)
    o1, l1 = dec(q, k, v, 0.7, False)
    o2, l2 = dec(q, k[perm], v[perm], 0.7, False)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


def check_split_merge(dec):
    """Splitting the keys in two and merging the partial results by their
    logsumexps (O = sum_s exp(LSE_s - LSE) O_s, LSE = log sum_s exp(LSE_s))
    gives the whole: the algebra the split-KV kernel relies on, checked on
    the oracle's own partials (non-causal, so every part is a plain
    sub-problem)."""
    q, k, v = _rand(3, 30, 4, 6)
    o, lse = dec(q, k, v, 0.5, False)
    oa, la = dec(q, k[:11], v[:11], 0.5, False)
    ob, lb = dec(q, k[11:], v[11:], 0.5, False)
    m = np.maximum(la, lb)
    wa, wb = np.exp(la - m), np.exp(lb - m)
    np.testing.assert_allclose((wa[:, None] * oa + wb[:, None] * ob) / (wa + wb)[:, None], o, atol=1e-13)
    np.testing.assert_allclose(m + np.log(wa + wb), lse, atol=1e-13)


CHECKS = [check_identical_keys, check_single_query_single_key, check_last_query_sees_everything, check_sdpa,
          check_key_permutation, check_split_merge]


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_decode_oracle_pins(check):
    check(oracle.decode_head)


def test_decode_wrapper_matches_heads():
    rng = np.random.default_rng(9)
    q = rng.standard_normal((2, 3, 4, 8))
    k = rng.standard_normal((2, 3, 20, 8))
    v = rng.standard_normal((2, 3, 20, 8))
    o, lse = oracle.decode(q, k, v, 0.35, True, heads=[(1, 2)])
    oh, lh = oracle.decode_head(q[1, 2], k[1, 2], v[1, 2], 0.35, True)
    np.testing.assert_array_equal(o[1, 2], oh)
    assert np.isnan(o[0, 0]).all()


# --------------------------------------------------------------- planted bugs
def _dec_top_left(q, k, v, scale, causal):
    """Wrong alignment: the square top-left mask applied to a rectangular problem."""
    from oracle.attention import _scores, _softmax_rows, _as_f64
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    p, lse = _softmax_rows(_scores(q, k, scale, 0, causal))
    return p @ v, lse


def _dec_off_by_one(q, k, v, scale, causal):
    """Query i sees keys j < nk - nq + i (its own position excluded)."""
    from oracle.attention import _scores, _softmax_rows, _as_f64
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    p, lse = _softmax_rows(_scores(q, k, scale, k.shape[0] - q.shape[0] - 1, causal))
    return p @ v, lse


def _dec_no_scale(q, k, v, scale, causal):
    return oracle.decode_head(q, k, v, 1.0, causal)


@pytest.mark.filterwarnings("ignore::RuntimeWarning")  # a planted mask can hide every key of a row
@pytest.mark.parametrize("bad", [_dec_top_left, _dec_off_by_one, _dec_no_scale], ids=lambda f: f.__name__)
def test_planted_decode_mistakes_fail_a_pin(bad):
    failed = 0
    for check in CHECKS:
        try:
            check(bad)
        except AssertionError:
            failed += 1
    assert failed >= 1
