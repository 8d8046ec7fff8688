"""GPU parity of the head-dim-256 backward (fa_bwd / fa_bwd_ex at d = 256,
through the C ABI) against the fp64 oracle.

At d = 256 the backward runs as a dK, dV kernel per (key block, head-dim
half) and a dQ kernel per query block; its 64-row query and key blocks make
ragged ends fall at other places than at d = 128, so the cases include
N = 63, 64, 65, 191 besides the usual ones.  Every path sums in a fixed
order, so the results are bitwise reproducible.
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


def grads(q, k, v, do, causal, deterministic=False, window=None, alibi=None):
    fa = _fa()
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    al = None if alibi is None else alibi.cuda()
    o, lse = fa.fwd(qd, kd, vd, causal=causal, window=window, alibi=al)
    out = fa.bwd(qd, kd, vd, o, dod, lse, causal=causal, deterministic=deterministic, window=window, alibi=al)
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
@pytest.mark.parametrize("N", [1, 7, 63, 64, 65, 128, 129, 191, 300, 513])
def test_bwd_d256_ragged(N, causal):
    q, k, v, do = inputs.make_qkv(1, 2, N, 256, seed=2100 + N, with_do=True)
    got = grads(q, k, v, do, causal)
    ref = oracle.attn_bwd_ref(q, k, v, do, 1 / math.sqrt(256), causal)
    check(got, (ref.dq, ref.dk, ref.dv), f"d=256 N={N} causal={causal}")


@pytest.mark.parametrize("H,H_kv,N,causal,window,alibi", [
    (4, 2, 300, True, None, False),
    (8, 1, 257, True, None, False),     # MQA: the group is split over several CTAs
    (2, 2, 700, True, 150, False),
    (4, 2, 400, False, None, True),
    (2, 2, 513, True, 100, True),
])
def test_bwd_d256_masks_and_groups(H, H_kv, N, causal, window, alibi):
    q, k, v, do = inputs.make_gqa(1, H, H_kv, N, 256, seed=2150 + N, with_do=True)
    sl = torch.tensor([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)], dtype=torch.float32) if alibi else None
    got = grads(q, k, v, do, causal, window=window, alibi=sl)
    ref = oracle.attn_bwd_gqa_ref(q, k, v, do, 1 / math.sqrt(256), causal, window=window,
                                  alibi=None if sl is None else sl.numpy())
    check(got, ref, f"H={H} H_kv={H_kv} N={N} causal={causal} w={window} alibi={alibi}")


def test_bwd_d256_reproducible_and_both_entry_points_agree():
    q, k, v, do = inputs.make_qkv(2, 4, 700, 256, seed=2190, with_do=True)
    a = grads(q, k, v, do, True)
    b = grads(q, k, v, do, True, deterministic=True)
    c = grads(q, k, v, do, True)
    for x, y in ((a, b), (a, c)):
        for g, h in zip(x, y):
            assert torch.equal(g, h)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_d256_larger_sampled_heads(causal):
    q, k, v, do = inputs.make_qkv(2, 8, 2048, 256, seed=2199, with_do=True)
    dq, dk, dv = grads(q, k, v, do, causal)
    for b, h in ((0, 0), (1, 7)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        ref = oracle.attn_bwd_ref(q[sl], k[sl], v[sl], do[sl], 1 / math.sqrt(256), causal)
        check((dq[sl], dk[sl], dv[sl]), (ref.dq, ref.dk, ref.dv), f"b={b} h={h}")
