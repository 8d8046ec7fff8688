"""GPU parity of the CTA-pair (cta_group::2) dK, dV kernel: the deterministic
backward at d = 128 with fa_set_tuning(FA_TUNE_BWD_PAIR, 1), through the C
ABI, against the fp64 oracle, and against the single-CTA deterministic
backward on the same inputs.

A pair owns 256 keys, so the cases include key counts that leave the second
CTA of the last pair partly or wholly past N (N = 129, 300, 513), causal
pairs whose first query block is hidden from the second CTA's keys, grouped
K/V heads (including the split of few K/V heads over several pairs, whose
fp32 partials are reduced afterwards), the sliding window and ALiBi.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_42_b200 import inputs
from tests.helpers import GRAD_REL_RMS, GRAD_RMS_FLOOR, f64, rel_rms

pytestmark = pytest.mark.gpu


def _fa():
    import exact_io_aware_42_b200 as fa
    return fa


@pytest.fixture
def pair_on():
    fa = _fa()
    fa.set_tuning("bwd_pair", 1)
    assert fa.get_tuning("bwd_pair", 128) == 1
    yield fa
    fa.set_tuning("bwd_pair", -1)


def grads(fa, q, k, v, do, causal, window=None, alibi=None):
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    al = None if alibi is None else alibi.cuda()
    o, lse = fa.fwd(qd, kd, vd, causal=causal, window=window, alibi=al)
    out = fa.bwd(qd, kd, vd, o, dod, lse, causal=causal, deterministic=True, window=window, alibi=al)
    torch.cuda.synchronize()
    assert fa.get_status() == 0
    return tuple(t.cpu() for t in out)


def check(got, ref, tag):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        g = f64(g)
        assert np.all(np.isfinite(g)), f"{tag} {name}: non-finite"
        e = rel_rms(g, r, GRAD_RMS_FLOOR)
        assert e <= GRAD_REL_RMS, f"{tag} {name}: relative RMS {e:.3e}"


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 7, 128, 129, 200, 256, 300, 513, 1000])
def test_pair_bwd_ragged(N, causal, pair_on):
    q, k, v, do = inputs.make_qkv(1, 2, N, 128, seed=1700 + N, with_do=True)
    got = grads(pair_on, q, k, v, do, causal)
    ref = oracle.attn_bwd_ref(q, k, v, do, 1 / math.sqrt(128), causal)
    check(got, (ref.dq, ref.dk, ref.dv), f"N={N} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_pair_matches_single_cta_kernel(causal):
    """Same inputs through both dK, dV kernels: dQ comes from the same dQ
    kernel (bit-identical); dK, dV agree to fp32 summation order."""
    fa = _fa()
    q, k, v, do = inputs.make_qkv(2, 4, 1000, 128, seed=1718, with_do=True)
    single = grads(fa, q, k, v, do, causal)
    fa.set_tuning("bwd_pair", 1)
    try:
        pair = grads(fa, q, k, v, do, causal)
        again = grads(fa, q, k, v, do, causal)
    finally:
        fa.set_tuning("bwd_pair", -1)
    assert torch.equal(pair[0], single[0])
    for a, b in zip(pair, again):            # reproducible
        assert torch.equal(a, b)
    for name, a, b in zip(("dk", "dv"), pair[1:], single[1:]):
        assert rel_rms(a, b, GRAD_RMS_FLOOR) <= 2e-3, name


@pytest.mark.parametrize("H,H_kv,N,causal,window,alibi", [
    (8, 2, 700, True, None, False),     # grouped heads
    (16, 1, 513, True, None, False),    # MQA: the group is split over several pairs
    (4, 4, 1000, True, 300, False),     # sliding window
    (4, 2, 600, False, None, True),     # ALiBi, non-causal
    (4, 4, 777, True, 200, True),       # window and ALiBi
])
def test_pair_bwd_masks_and_groups(H, H_kv, N, causal, window, alibi, pair_on):
    q, k, v, do = inputs.make_gqa(1, H, H_kv, N, 128, seed=1750 + N, with_do=True)
    sl = torch.tensor([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)], dtype=torch.float32) if alibi else None
    got = grads(pair_on, q, k, v, do, causal, window=window, alibi=sl)
    ref = oracle.attn_bwd_gqa_ref(q, k, v, do, 1 / math.sqrt(128), causal, window=window,
                                  alibi=None if sl is None else sl.numpy())
    check(got, ref, f"H={H} H_kv={H_kv} N={N} causal={causal} w={window} alibi={alibi}")


def test_pair_bwd_long_workload_sampled_heads(pair_on):
    w = inputs.LONG
    q, k, v, do = inputs.make_workload(w)
    dq, dk, dv = grads(pair_on, q, k, v, do, True)
    sum_dv = f64(dv).sum(axis=2)
    sum_do = f64(do).sum(axis=2)
    assert np.max(np.abs(sum_dv - sum_do)) <= 2e-2 * max(1.0, np.max(np.abs(sum_do)))
    for b, h in ((0, 0), (3, 15)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        ref = oracle.attn_bwd_ref(q[sl], k[sl], v[sl], do[sl], 1 / math.sqrt(w.d), True)
        check((dq[sl], dk[sl], dv[sl]), (ref.dq, ref.dk, ref.dv), f"b={b} h={h}")
