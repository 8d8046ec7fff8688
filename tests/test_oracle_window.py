"""Pins of the sliding-window oracle (CPU, no GPU).

The window reading (causal, key j visible to query i iff i - w <= j <= i)
is pinned by: scalar loops over range(max(0, i - w), i + 1) (a brute force
written without masks), w >= N - 1 reducing to plain causal attention,
w = 0 giving O = V and L = scale q_i . k_i, independence of a query's output
from keys left of its window, and central finite differences of the forward
for the backward (so the gradient formula is not checked against itself).
A planted off-by-one window (i - w < j) fails the brute force.
"""
import math

import numpy as np
import pytest

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def brute(q, k, v, scale, w):
    N = q.shape[0]
    o = np.zeros_like(v)
    lse = np.zeros(N)
    for i in range(N):
        js = list(range(max(0, i - w), i + 1))
        s = [scale * sum(q[i, t] * k[j, t] for t in range(q.shape[1])) for j in js]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        z = sum(e)
        for t in range(v.shape[1]):
            o[i, t] = sum(e[n] * v[j, t] for n, j in enumerate(js)) / z
        lse[i] = m + math.log(z)
    return o, lse


@pytest.mark.parametrize("w", [0, 1, 3, 7, 20])
def test_window_matches_brute_force(w):
    N, d = 11, 3
    q, k, v = _rand((1, 1, N, d), 1), _rand((1, 1, N, d), 2), _rand((1, 1, N, d), 3)
    o, lse = oracle.attn_fwd_gqa_ref(q, k, v, 0.7, True, window=w)
    ob, lb = brute(q[0, 0], k[0, 0], v[0, 0], 0.7, w)
    np.testing.assert_allclose(o[0, 0], ob, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], lb, atol=1e-12)
    rows = [0, 4, 10]
    orow, lrow = oracle.attn_fwd_rows_ref(q[0, 0], k[0, 0], v[0, 0], 0.7, True, rows, window=w)
    np.testing.assert_allclose(orow, ob[rows], atol=1e-12)
    np.testing.assert_allclose(lrow, lb[rows], atol=1e-12)


def test_wide_window_is_causal_and_zero_window_is_identity():
    N, d = 9, 4
    q, k, v = _rand((2, 2, N, d), 4), _rand((2, 2, N, d), 5), _rand((2, 2, N, d), 6)
    o, lse = oracle.attn_fwd_gqa_ref(q, k, v, 0.5, True, window=N - 1)
    o2, lse2 = oracle.attn_fwd_ref(q, k, v, 0.5, True)
    np.testing.assert_allclose(o, o2, atol=1e-14)
    np.testing.assert_allclose(lse, lse2, atol=1e-14)
    o0, lse0 = oracle.attn_fwd_gqa_ref(q, k, v, 0.5, True, window=0)
    np.testing.assert_allclose(o0, v, atol=1e-14)
    np.testing.assert_allclose(lse0, 0.5 * np.sum(q * k, axis=-1), atol=1e-14)


def test_keys_left_of_the_window_do_not_matter():
    N, d, w = 16, 4, 5
    q, k, v = _rand((1, 1, N, d), 7), _rand((1, 1, N, d), 8), _rand((1, 1, N, d), 9)
    o, _ = oracle.attn_fwd_gqa_ref(q, k, v, 0.6, True, window=w)
    k2, v2 = k.copy(), v.copy()
    k2[..., :4, :] += 3.0
    v2[..., :4, :] -= 2.0
    o2, _ = oracle.attn_fwd_gqa_ref(q, k2, v2, 0.6, True, window=w)
    # rows i >= 4 + w see no key below 4
    np.testing.assert_allclose(o[..., 4 + w:, :], o2[..., 4 + w:, :], atol=1e-14)
    assert not np.allclose(o[..., :4 + w, :], o2[..., :4 + w, :])


def test_window_backward_matches_finite_differences():
    B, H, H_kv, N, d, w = 1, 2, 1, 7, 3, 2
    q, k, v, do = _rand((B, H, N, d), 10), _rand((B, H_kv, N, d), 11), _rand((B, H_kv, N, d), 12), _rand((B, H, N, d), 13)
    dq, dk, dv = oracle.attn_bwd_gqa_ref(q, k, v, do, 0.8, True, window=w)

    def loss(q_, k_, v_):
        o, _ = oracle.attn_fwd_gqa_ref(q_, k_, v_, 0.8, True, window=w)
        return float(np.sum(o * do))
    eps = 1e-6
    for x, g, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[which], args_m[which] = xp, xm
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=1e-5, atol=1e-7)


def test_planted_off_by_one_window_fails_brute_force():
    N, d, w = 10, 3, 3
    q, k, v = _rand((N, d), 14), _rand((N, d), 15), _rand((N, d), 16)
    ob, _ = brute(q, k, v, 0.5, w)
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    s = 0.5 * q @ k.T
    s = np.where((j <= i) & (j > i - w), s, -np.inf)          # wrong: one key short
    p = np.exp(s - s.max(axis=1, keepdims=True))
    o_wrong = (p / p.sum(axis=1, keepdims=True)) @ v
    assert not np.allclose(o_wrong, ob, atol=1e-6)
