"""GPU parity of the bf16 forward (fa_fwd through the C ABI) against the fp64 oracle.

Sizes span several 128-row tiles and ragged tails; the full-size workload is
checked on sampled heads against the oracle and on every head against closed
forms that hold at any size.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_42_b200 import inputs
from tests.helpers import (assert_fwd_close, f64, LSE_MAX_ABS, max_abs, max_scaled_err, O_MAX_ABS,
                           O_REL_RMS, rel_rms)

pytestmark = pytest.mark.gpu


def _fa():
    import exact_io_aware_42_b200 as fa
    return fa


def run_fwd(q, k, v, causal, scale=None, window=None):
    fa = _fa()
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale, window=window)
    torch.cuda.synchronize()
    assert fa.get_status() == 0
    return o.cpu(), lse.cpu()


def test_fwd_tiny_workload():
    w = inputs.TINY
    q, k, v = inputs.make_workload(w)
    o, lse = run_fwd(q, k, v, False)
    o_ref, l_ref = oracle.attn_fwd_ref(q, k, v, 1 / math.sqrt(w.d), False)
    assert_fwd_close(o, lse, o_ref, l_ref, w.name)


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_small_workload(causal):
    w = inputs.SMALL
    q, k, v = inputs.make_workload(w)
    o, lse = run_fwd(q, k, v, causal)
    o_ref, l_ref = oracle.attn_fwd_ref(q, k, v, 1 / math.sqrt(w.d), causal)
    assert_fwd_close(o, lse, o_ref, l_ref, f"{w.name} causal={causal}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 7, 127, 128, 129, 200, 255, 256, 257, 383, 513])
def test_fwd_ragged(N, d, causal):
    q, k, v = inputs.make_qkv(1, 2, N, d, seed=100 + N + d)
    o, lse = run_fwd(q, k, v, causal)
    o_ref, l_ref = oracle.attn_fwd_ref(q, k, v, 1 / math.sqrt(d), causal)
    assert_fwd_close(o, lse, o_ref, l_ref, f"N={N} d={d} causal={causal}")


def test_fwd_long_workload_sampled_heads():
    w = inputs.LONG
    q, k, v, _ = inputs.make_workload(w)
    o, lse = run_fwd(q, k, v, True)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    for b, h in ((0, 0), (1, 7), (3, 15)):
        o_ref, l_ref = oracle.attn_fwd_ref(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1],
                                           v[b:b + 1, h:h + 1], 1 / math.sqrt(w.d), True)
        assert_fwd_close(o[b:b + 1, h:h + 1], lse[b:b + 1, h:h + 1], o_ref, l_ref, f"b={b} h={h}")


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_scale_zero_closed_form_full_size(causal):
    """scale = 0: every visible score is 0, so O is the (prefix) mean of V and
    L = ln(number of visible keys), at the full 4096-token size."""
    w = inputs.LONG
    q, k, v, _ = inputs.make_workload(w)
    o, lse = run_fwd(q, k, v, causal, scale=0.0)
    vv = f64(v)
    n = w.N
    if causal:
        cnt = np.arange(1, n + 1, dtype=np.float64)
        o_ref = np.cumsum(vv, axis=2) / cnt[None, None, :, None]
        l_ref = np.broadcast_to(np.log(cnt), lse.shape)
    else:
        o_ref = np.broadcast_to(vv.mean(axis=2, keepdims=True), vv.shape)
        l_ref = np.full(lse.shape, math.log(n))
    assert np.max(np.abs(f64(lse) - l_ref)) <= LSE_MAX_ABS
    assert np.max(np.abs(f64(o) - o_ref)) <= O_MAX_ABS


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_one_hot_values_recover_p(causal):
    """V = identity: O equals the probability matrix P itself."""
    N, d = 128, 128
    q, k, _ = inputs.make_qkv(1, 1, N, d, seed=7)
    v = torch.eye(N, d, dtype=torch.bfloat16)[None, None].contiguous()
    o, lse = run_fwd(q, k, v, causal)
    o_ref, l_ref = oracle.attn_fwd_ref(q, k, v, 1 / math.sqrt(d), causal)
    assert_fwd_close(o, lse, o_ref, l_ref, "one-hot V")


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_fwd_large_magnitude_exercises_rescale(causal, d):
    """Q x 8 with a growing ramp: the running max moves by more than the
    rescale threshold across tiles, so the O correction path runs (at
    d = 256 each of the two softmax warpgroups rescales its own O columns
    after the pair has agreed on the row maximum)."""
    N = 1024
    q, k, v = inputs.make_qkv(1, 2, N, d, seed=9)
    ramp = torch.linspace(0.2, 3.0, N)[None, None, :, None]
    q = (q.float() * 8.0).to(torch.bfloat16)
    k = (k.float() * ramp).to(torch.bfloat16)
    o, lse = run_fwd(q, k, v, causal)
    o_ref, l_ref = oracle.attn_fwd_ref(q, k, v, 1 / math.sqrt(d), causal)
    # Outside the benchmark workloads the softmax is nearly one-hot and |O|
    # reaches ~4, where one bf16 half-ulp of the output alone is 1.6e-2.  The
    # bound used here is derived from the arithmetic instead: bf16 rounding of
    # P (2^-8 relative) plus bf16 rounding of O (2^-8 relative), i.e. 1e-2
    # relative to max(1, |O|).
    err = np.abs(f64(o) - o_ref) / np.maximum(1.0, np.abs(o_ref))
    assert np.max(err) <= 1e-2, np.max(err)
    assert np.max(np.abs(f64(lse) - l_ref)) <= LSE_MAX_ABS


def test_fwd_identical_keys_give_mean():
    N, d = 300, 128
    q, k, v = inputs.make_qkv(2, 1, N, d, seed=11)
    k = k[:, :, :1].expand(-1, -1, N, -1).contiguous()
    o, lse = run_fwd(q, k, v, False)
    o_ref = np.broadcast_to(f64(v).mean(axis=2, keepdims=True), o.shape)
    assert np.max(np.abs(f64(o) - o_ref)) <= O_MAX_ABS


def test_fwd_empty_and_errors():
    fa = _fa()
    z = torch.empty((1, 1, 0, 64), dtype=torch.bfloat16, device="cuda")
    o, lse = fa.fwd(z, z, z)
    assert o.shape == (1, 1, 0, 64) and lse.shape == (1, 1, 0)
    x = torch.zeros((1, 1, 16, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.fwd(x, x, x)
    assert e.value.code == 2
    torch.cuda.synchronize()
    assert fa.get_status() == 0


@pytest.fixture
def restore_tuning():
    yield
    fa = _fa()
    for knob in fa.api.TUNING_KNOBS:
        fa.set_tuning(knob, -1)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("pairs,deg", [(0, 3), (2, 3), (4, 3), (2, 4), (4, 4)])
@pytest.mark.parametrize("causal", [False, True])
def test_fwd_exp2_split_variants(d, pairs, deg, causal, restore_tuning):
    """Every exp2 split the forward can run (0, 2 or 4 of 8 score pairs on the
    FMA-pipe polynomial, degree 3 or 4) meets the same tolerances, with
    several tiles and a ragged tail."""
    fa = _fa()
    fa.set_tuning("fwd_poly_pairs", pairs)
    fa.set_tuning("fwd_poly_degree", deg)
    assert fa.get_tuning("fwd_poly_pairs", d) == pairs and fa.get_tuning("fwd_poly_degree", d) == deg
    q, k, v = inputs.make_qkv(2, 2, 1000, d, seed=300 + d + pairs)
    o, lse = run_fwd(q, k, v, causal)
    o_ref, l_ref = oracle.attn_fwd_ref(q, k, v, 1 / math.sqrt(d), causal)
    assert_fwd_close(o, lse, o_ref, l_ref, f"d={d} pairs={pairs} deg={deg} causal={causal}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("persistent,group,q1", [(0, 1, 0), (0, 0, 0), (1, 0, 0), (1, 1, 0), (0, 0, 1)])
def test_fwd_kernel_variants_every_head(d, persistent, group, q1, restore_tuning):
    """The forward kernels (two query tiles per item: one CTA per work item,
    with the grouped and the global causal order, or the persistent grid; one
    query tile per item) on a problem with more work items than SMs and, at
    d = 128, two head groups (32 and 8 heads of N = 2048): every head matches
    the oracle on sampled rows, causal and not, plus one whole head."""
    fa = _fa()
    fa.set_tuning("fwd_persistent", persistent)
    fa.set_tuning("fwd_causal_group", group)
    fa.set_tuning("fwd_q1", q1)
    assert fa.get_tuning("fwd_persistent", d) == persistent and fa.get_tuning("fwd_q1", d) == q1
    N, H = 2048, 40
    q, k, v = inputs.make_qkv(1, H, N, d, seed=700 + d + 8 * q1 + 4 * group + 2 * persistent)
    # causal rows 0 and 1 average one or two keys, so |O| reaches a few units
    # and one bf16 half-ulp of O alone approaches 1e-2: O's elementwise bound
    # is taken relative to max(1, |O|) here (the masks tests' reading)
    rows = np.array([0, 1, 127, 128, 255, 256, 1023, 1500, 2046, 2047])
    for causal in (False, True):
        o, lse = run_fwd(q, k, v, causal)
        for h in list(range(H)) + [None]:
            if h is None:    # one whole head
                sl = (slice(0, 1), slice(33, 34))
                o_r, l_r = oracle.attn_fwd_ref(q[sl], k[sl], v[sl], 1 / math.sqrt(d), causal)
                o_k, l_k = o[sl], lse[sl]
            else:
                o_r, l_r = oracle.attn_fwd_rows_ref(q[0, h], k[0, h], v[0, h], 1 / math.sqrt(d), causal, rows)
                o_k, l_k = o[0, h, rows], lse[0, h, rows]
            tag = f"h={h} causal={causal}"
            assert max_scaled_err(o_k, o_r) <= O_MAX_ABS, tag
            assert rel_rms(o_k, o_r) <= O_REL_RMS, tag
            assert max_abs(l_k, l_r) <= LSE_MAX_ABS, tag


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("B,H,G,N,causal,window", [(2, 3, 1, 300, True, None), (2, 3, 1, 777, False, None),
                                                   (1, 4, 1, 1000, True, 200), (2, 8, 4, 1536, True, None),
                                                   (1, 2, 2, 2049, False, None), (3, 5, 1, 4100, True, None)])
def test_fwd_persistent_grid_matches_one_cta_per_item(d, B, H, G, N, causal, window, restore_tuning):
    """The two-tile forward's persistent grid runs the same arithmetic as one
    CTA per work item, item by item: O and L agree bit for bit, over ragged
    tails, GQA, a sliding window, and more work items than SMs."""
    fa = _fa()
    fa.set_tuning("fwd_q1", 0)
    q, k, v = inputs.make_gqa(B, H, H // G, N, d, seed=900 + N + d)
    out = {}
    for mode in (0, 1):
        fa.set_tuning("fwd_persistent", mode)
        o, lse = run_fwd(q, k, v, causal, window=window)
        out[mode] = (o.clone(), lse.clone())
    assert torch.equal(out[0][0], out[1][0]) and torch.equal(out[0][1], out[1][1])
    assert fa.get_status() == 0


def test_fwd_persistent_causal_beyond_the_deal_table(restore_tuning):
    """A causal problem with more work items than the host-made deal holds
    (9216 > 8192): the persistent grid falls back to rounds in snake order and
    still matches one CTA per work item bit for bit."""
    fa = _fa()
    fa.set_tuning("fwd_q1", 0)
    g = torch.Generator(device="cuda").manual_seed(77)
    q, k, v = (torch.randn(9, 32, 8192, 64, device="cuda", generator=g).to(torch.bfloat16) for _ in range(3))
    out = {}
    for mode in (0, 1):
        fa.set_tuning("fwd_persistent", mode)
        o, lse = fa.fwd(q, k, v, causal=True)
        torch.cuda.synchronize()
        out[mode] = (o, lse)
    assert torch.equal(out[0][0], out[1][0]) and torch.equal(out[0][1], out[1][1])
    assert fa.get_status() == 0


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 7, 127, 128, 129, 255, 257, 383, 513, 1000])
def test_fwd_d256_ragged(N, causal):
    """Head dim 256 (its own kernel: one query tile per work item, K/V in
    64-column panels) over several tiles and ragged tails."""
    q, k, v = inputs.make_qkv(1, 2, N, 256, seed=500 + N)
    o, lse = run_fwd(q, k, v, causal)
    o_ref, l_ref = oracle.attn_fwd_ref(q, k, v, 1 / math.sqrt(256), causal)
    assert_fwd_close(o, lse, o_ref, l_ref, f"d=256 N={N} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_d256_many_items_sampled_heads(causal):
    """More work items than SMs (several rounds of the persistent grid)."""
    q, k, v = inputs.make_qkv(4, 16, 2048, 256, seed=521)
    o, lse = run_fwd(q, k, v, causal)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    for b, h in ((0, 0), (2, 9), (3, 15)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        o_ref, l_ref = oracle.attn_fwd_ref(q[sl], k[sl], v[sl], 1 / math.sqrt(256), causal)
        assert_fwd_close(o[sl], lse[sl], o_ref, l_ref, f"d=256 b={b} h={h}")


@pytest.mark.parametrize("pairs,deg", [(2, 3), (4, 4)])
def test_fwd_d256_exp2_split(pairs, deg, restore_tuning):
    fa = _fa()
    fa.set_tuning("fwd_poly_pairs", pairs)
    fa.set_tuning("fwd_poly_degree", deg)
    q, k, v = inputs.make_qkv(1, 3, 700, 256, seed=530 + pairs)
    for causal in (False, True):
        o, lse = run_fwd(q, k, v, causal)
        o_ref, l_ref = oracle.attn_fwd_ref(q, k, v, 1 / math.sqrt(256), causal)
        assert_fwd_close(o, lse, o_ref, l_ref, f"d=256 pairs={pairs} deg={deg} causal={causal}")




@pytest.mark.parametrize("q1", [0, 1])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 7, 127, 129, 255, 300, 513])
def test_fwd_kernels_ragged_masks_groups(N, d, q1, restore_tuning):
    """Both bf16 forward kernels for d <= 128 (two query tiles per CTA; one
    query tile with two score buffers and P in its own TMEM columns, which
    the library picks by itself for problems this small) on ragged N, causal
    and not, with grouped K/V heads, a sliding window and ALiBi: the same
    tolerances as every other forward variant (O elementwise relative to
    max(1, |O|) where masks leave few keys)."""
    fa = _fa()
    fa.set_tuning("fwd_q1", q1)
    assert fa.get_tuning("fwd_q1", d) == q1
    q, k, v = inputs.make_gqa(2, 4, 2, N, d, seed=900 + N + d + q1)
    scale = 1 / math.sqrt(d)
    slopes = torch.tensor([2.0 ** (-8 * (h + 1) / 4) for h in range(4)], dtype=torch.float32)
    for causal, window, alibi in ((False, None, None), (True, None, None), (True, 100, None), (True, None, slopes)):
        o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, window=window,
                        alibi=None if alibi is None else alibi.cuda())
        torch.cuda.synchronize()
        assert fa.get_status() == 0
        o_ref, l_ref = oracle.attn_fwd_gqa_ref(q, k, v, scale, causal, window=window,
                                              alibi=None if alibi is None else alibi.numpy())
        tag = f"N={N} d={d} causal={causal} window={window} alibi={alibi is not None}"
        assert max_scaled_err(o.cpu(), o_ref) <= O_MAX_ABS, tag
        assert rel_rms(o.cpu(), o_ref) <= O_REL_RMS, tag
        assert max_abs(lse.cpu(), l_ref) <= LSE_MAX_ABS, tag
