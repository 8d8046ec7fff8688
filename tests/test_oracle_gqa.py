"""Pins of the grouped-K/V-head oracle (CPU, no GPU).

The reading (query head h uses K/V head h // G) is pinned to torch's own
grouped scaled-dot-product attention (``enable_gqa=True``, fp64 on the CPU),
whose gradients come from autograd, so neither the head mapping nor the
summation of dK, dV over a group is checked against the oracle's own
formula.  Further pins: G = 1 is the plain oracle exactly; explicitly
repeating the K/V heads gives the same O and L through the plain oracle, and
the plain oracle's per-head dK, dV summed over each group; a planted mistake
(the head mapping h % H_kv instead of h // G) fails the torch pin.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import attention_ref as ar


def _rand(shape, seed):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape)


def _torch_gqa(q, k, v, do, scale, causal):
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    o = F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale, enable_gqa=True)
    (o * torch.tensor(do)).sum().backward()
    return o.detach().numpy(), tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


@pytest.mark.parametrize("H,H_kv", [(4, 2), (6, 3), (8, 1), (4, 4)])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_oracle_matches_torch_grouped_sdpa(H, H_kv, causal):
    B, N, d = 2, 19, 8
    q, k, v, do = _rand((B, H, N, d), 1), _rand((B, H_kv, N, d), 2), _rand((B, H_kv, N, d), 3), _rand((B, H, N, d), 4)
    scale = 0.37
    o_t, dq_t, dk_t, dv_t = _torch_gqa(q, k, v, do, scale, causal)
    o, lse = oracle.attn_fwd_gqa_ref(q, k, v, scale, causal)
    np.testing.assert_allclose(o, o_t, rtol=1e-12, atol=1e-12)
    dq, dk, dv = oracle.attn_bwd_gqa_ref(q, k, v, do, scale, causal)
    np.testing.assert_allclose(dq, dq_t, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(dk, dk_t, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(dv, dv_t, rtol=1e-10, atol=1e-11)


def test_gqa_group_one_is_plain_oracle():
    q, k, v, do = (_rand((1, 3, 11, 4), s) for s in range(4))
    o, lse = oracle.attn_fwd_gqa_ref(q, k, v, 0.5, True)
    o2, lse2 = oracle.attn_fwd_ref(q, k, v, 0.5, True)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-15)
    dq, dk, dv = oracle.attn_bwd_gqa_ref(q, k, v, do, 0.5, True)
    r = oracle.attn_bwd_ref(q, k, v, do, 0.5, True)
    for a, b in ((dq, r.dq), (dk, r.dk), (dv, r.dv)):
        np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-14)


def test_gqa_equals_plain_oracle_on_repeated_heads():
    B, H, H_kv, N, d = 1, 6, 2, 13, 4
    g = H // H_kv
    q, do = _rand((B, H, N, d), 5), _rand((B, H, N, d), 6)
    k, v = _rand((B, H_kv, N, d), 7), _rand((B, H_kv, N, d), 8)
    k_rep, v_rep = np.repeat(k, g, axis=1), np.repeat(v, g, axis=1)
    o, lse = oracle.attn_fwd_gqa_ref(q, k, v, 0.4, False)
    o2, lse2 = oracle.attn_fwd_ref(q, k_rep, v_rep, 0.4, False)
    np.testing.assert_allclose(o, o2, atol=1e-14)
    np.testing.assert_allclose(lse, lse2, atol=1e-14)
    dq, dk, dv = oracle.attn_bwd_gqa_ref(q, k, v, do, 0.4, False)
    r = oracle.attn_bwd_ref(q, k_rep, v_rep, do, 0.4, False)
    np.testing.assert_allclose(dq, r.dq, atol=1e-13)
    np.testing.assert_allclose(dk, r.dk.reshape(B, H_kv, g, N, d).sum(axis=2), atol=1e-13)
    np.testing.assert_allclose(dv, r.dv.reshape(B, H_kv, g, N, d).sum(axis=2), atol=1e-13)


def test_planted_head_mapping_mistake_fails_torch_pin():
    """h % H_kv is a plausible wrong mapping; the torch pin must reject it."""
    B, H, H_kv, N, d = 1, 4, 2, 9, 4
    q, k, v = _rand((B, H, N, d), 9), _rand((B, H_kv, N, d), 10), _rand((B, H_kv, N, d), 11)
    o_t, *_ = _torch_gqa(q, k, v, np.zeros((B, H, N, d)), 0.5, False)

    def wrong(q, k, v, scale, causal):
        out = np.zeros_like(q)
        for h in range(H):
            o, _ = ar.attn_fwd_ref(q[:, h:h + 1], k[:, h % H_kv:h % H_kv + 1], v[:, h % H_kv:h % H_kv + 1],
                                   scale, causal)
            out[:, h] = o[:, 0]
        return out, None

    o_w, _ = wrong(q, k, v, 0.5, False)
    assert not np.allclose(o_w, o_t, atol=1e-6)
    o_r, _ = oracle.attn_fwd_gqa_ref(q, k, v, 0.5, False)
    assert np.allclose(o_r, o_t, atol=1e-12)
