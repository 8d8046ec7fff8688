"""Pins of the ALiBi oracle (CPU, no GPU).

Reading: scores scale q.k - slope_h |i - j|, one slope per query head.
Pins that do not retype that formula:
  * slope 0 is plain attention;
  * causal ALiBi equals plain causal attention on inputs augmented by one
    dimension (q' = [q, 1], k' = [k, slope j / scale]): on a causal row the
    bias differs from +slope j by the row constant -slope i, which softmax
    ignores, and L shifts by exactly -slope i;
  * a very large slope leaves only the diagonal (causal): O = V;
  * a scalar brute force over (i, j) loops;
  * the backward against central finite differences of the forward.
A planted sign error (+slope |i - j|) fails the augmentation pin.
"""
import math

import numpy as np
import pytest

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_zero_slope_is_plain():
    q, k, v = (_rand((1, 2, 9, 4), s) for s in range(3))
    for causal in (False, True):
        o, l = oracle.attn_fwd_gqa_ref(q, k, v, 0.5, causal, alibi=[0.0, 0.0])
        o2, l2 = oracle.attn_fwd_ref(q, k, v, 0.5, causal)
        np.testing.assert_allclose(o, o2, atol=1e-14)
        np.testing.assert_allclose(l, l2, atol=1e-14)


@pytest.mark.parametrize("slope", [0.05, 0.5, 2.0])
def test_causal_alibi_equals_augmented_plain_attention(slope):
    N, d, scale = 13, 4, 0.6
    q, k, v = _rand((N, d), 4), _rand((N, d), 5), _rand((N, d), 6)
    o, l = oracle.attn_fwd_gqa_ref(q[None, None], k[None, None], v[None, None], scale, True, alibi=[slope])
    qa = np.concatenate([q, np.ones((N, 1))], axis=1)
    ka = np.concatenate([k, (slope * np.arange(N) / scale)[:, None]], axis=1)
    o2, l2 = oracle.attn_fwd_ref(qa[None, None], ka[None, None], v[None, None], scale, True)
    np.testing.assert_allclose(o[0, 0], o2[0, 0], atol=1e-12)
    np.testing.assert_allclose(l[0, 0], l2[0, 0] - slope * np.arange(N), atol=1e-12)


def test_large_slope_leaves_the_diagonal():
    q, k, v = (_rand((1, 1, 8, 4), s) for s in (7, 8, 9))
    o, _ = oracle.attn_fwd_gqa_ref(q, k, v, 0.5, True, alibi=[200.0])
    np.testing.assert_allclose(o, v, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_alibi_brute_force(causal):
    N, d, scale, slope = 7, 3, 0.9, 0.3
    q, k, v = _rand((N, d), 10), _rand((N, d), 11), _rand((N, d), 12)
    o, l = oracle.attn_fwd_gqa_ref(q[None, None], k[None, None], v[None, None], scale, causal, alibi=[slope])
    for i in range(N):
        js = range(i + 1) if causal else range(N)
        s = {j: scale * sum(q[i, t] * k[j, t] for t in range(d)) - slope * abs(i - j) for j in js}
        m = max(s.values())
        z = sum(math.exp(x - m) for x in s.values())
        for t in range(d):
            ref = sum(math.exp(s[j] - m) * v[j, t] for j in js) / z
            assert abs(o[0, 0, i, t] - ref) < 1e-12
        assert abs(l[0, 0, i] - (m + math.log(z))) < 1e-12


def test_alibi_backward_matches_finite_differences():
    B, H, H_kv, N, d = 1, 2, 1, 6, 3
    slopes = [0.25, 0.7]
    q, k, v, do = _rand((B, H, N, d), 13), _rand((B, H_kv, N, d), 14), _rand((B, H_kv, N, d), 15), _rand((B, H, N, d), 16)
    grads = oracle.attn_bwd_gqa_ref(q, k, v, do, 0.8, True, window=3, alibi=slopes)

    def loss(xs):
        o, _ = oracle.attn_fwd_gqa_ref(xs[0], xs[1], xs[2], 0.8, True, window=3, alibi=slopes)
        return float(np.sum(o * do))
    eps = 1e-6
    for which, g in enumerate(grads):
        x = (q, k, v)[which]
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xs_p, xs_m = [q, k, v], [q, k, v]
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            xs_p[which], xs_m[which] = xp, xm
            num[idx] = (loss(xs_p) - loss(xs_m)) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=1e-5, atol=1e-7)


def test_planted_sign_error_fails_augmentation_pin():
    N, d, scale, slope = 10, 4, 0.6, 0.4
    q, k, v = _rand((N, d), 17), _rand((N, d), 18), _rand((N, d), 19)
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    s = scale * q @ k.T + slope * np.abs(i - j)              # wrong sign
    s = np.where(j <= i, s, -np.inf)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    o_wrong = (p / p.sum(axis=1, keepdims=True)) @ v
    qa = np.concatenate([q, np.ones((N, 1))], axis=1)
    ka = np.concatenate([k, (slope * np.arange(N) / scale)[:, None]], axis=1)
    o_aug, _ = oracle.attn_fwd_ref(qa[None, None], ka[None, None], v[None, None], scale, True)
    assert not np.allclose(o_wrong, o_aug[0, 0], atol=1e-6)
