"""GPU parity of the deterministic backward (fa_bwd_deterministic through the
C ABI) against the fp64 oracle, and its reproducibility.

Same cases as the atomic backward's tests (ragged N, both head sizes, causal
or not, the small and the long workload), plus:
  * three runs give bitwise identical dQ, dK, dV (with an atomic-path run in
    between, so the device state differs);
  * dK and dV equal the atomic path's bit for bit: both come from the same
    main kernel arithmetic, only dQ is produced differently;
  * dQ from the two paths agrees to within a few bf16 roundings (both round
    dS to bf16 before the dS K product; the atomic path forms dS from P
    already rounded to bf16 for the dV product, this one from fp32 P, and
    each rounds its own dQ sum to bf16 at the end).
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


def run(q, k, v, do, causal, deterministic=True, scale=None):
    fa = _fa()
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.fwd(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, dod, lse, causal=causal, scale=scale, deterministic=deterministic)
    torch.cuda.synchronize()
    assert fa.get_status() == 0
    return dq.cpu(), dk.cpu(), dv.cpu()


def assert_grads_close(got, ref, tag):
    for name, g, r in zip(("dq", "dk", "dv"), got, (ref.dq, ref.dk, ref.dv)):
        g = f64(g)
        assert np.all(np.isfinite(g)), f"{tag} {name}: non-finite"
        e = rel_rms(g, r, GRAD_RMS_FLOOR)
        assert e <= GRAD_REL_RMS, f"{tag} {name}: relative RMS {e:.3e} > {GRAD_REL_RMS}"


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 7, 128, 129, 200, 256, 300, 513])
def test_det_bwd_ragged(N, d, causal):
    q, k, v, do = inputs.make_qkv(1, 2, N, d, seed=700 + N + d, with_do=True)
    got = run(q, k, v, do, causal)
    ref = oracle.attn_bwd_ref(q, k, v, do, 1 / math.sqrt(d), causal)
    assert_grads_close(got, ref, f"N={N} d={d} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_det_bwd_small_workload_shape(causal):
    w = inputs.SMALL
    q, k, v, do = inputs.make_qkv(w.B, w.H, w.N, w.d, w.seed, with_do=True)
    got = run(q, k, v, do, causal)
    ref = oracle.attn_bwd_ref(q, k, v, do, 1 / math.sqrt(w.d), causal)
    assert_grads_close(got, ref, f"{w.name} causal={causal}")


def test_det_bwd_scale_zero_and_custom():
    q, k, v, do = inputs.make_qkv(1, 2, 300, 128, seed=77, with_do=True)
    for scale in (0.0, 0.3):
        got = run(q, k, v, do, True, scale=scale)
        ref = oracle.attn_bwd_ref(q, k, v, do, scale, True)
        assert_grads_close(got, ref, f"scale={scale}")


def test_det_bwd_long_workload_sampled_heads_and_identities():
    w = inputs.LONG
    q, k, v, do = inputs.make_workload(w)
    dq, dk, dv = run(q, k, v, do, True)
    sum_dv = f64(dv).sum(axis=2)
    sum_do = f64(do).sum(axis=2)
    assert np.max(np.abs(sum_dv - sum_do)) <= 2e-2 * max(1.0, np.max(np.abs(sum_do)))
    for b, h in ((0, 0), (3, 15)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        ref = oracle.attn_bwd_ref(q[sl], k[sl], v[sl], do[sl], 1 / math.sqrt(w.d), True)
        assert_grads_close((dq[sl], dk[sl], dv[sl]), ref, f"b={b} h={h}")


@pytest.mark.parametrize("causal", [False, True])
def test_det_bwd_bitwise_reproducible_and_matches_atomic_dk_dv(causal):
    q, k, v, do = inputs.make_qkv(2, 4, 1000, 128, seed=18, with_do=True)
    a = run(q, k, v, do, causal)
    atomic = run(q, k, v, do, causal, deterministic=False)
    b = run(q, k, v, do, causal)
    c = run(q, k, v, do, causal)
    for x, y in ((a, b), (a, c)):
        for g, h in zip(x, y):
            assert torch.equal(g, h)
    assert torch.equal(a[1], atomic[1]) and torch.equal(a[2], atomic[2])
    assert rel_rms(a[0], atomic[0]) <= 5e-3


@pytest.mark.parametrize("d,H,H_kv,N,pair", [(128, 16, 16, 2048, 0), (64, 12, 4, 1300, 0), (128, 8, 8, 1536, 1),
                                              (256, 4, 2, 1000, 0), (128, 4, 1, 2048, 0)])
def test_det_bwd_causal_cta_order_does_not_change_results(d, H, H_kv, N, pair):
    """The causal CTA order (longest first within L2-sized head groups, or
    head by head) only changes which SM runs which block: the deterministic
    dQ, dK, dV agree bit for bit, for the single-CTA, CTA-pair (d = 128) and
    d = 256 kernels, grouped K/V heads and the split MQA path."""
    fa = _fa()
    q, k, v, do = (t.cuda() for t in inputs.make_gqa(2, H, H_kv, N, d, seed=4000 + N + d, with_do=True))
    o, lse = fa.fwd(q, k, v, causal=True)
    out = {}
    try:
        fa.set_tuning("bwd_pair", pair)
        for grouped in (0, 1):
            fa.set_tuning("bwd_causal_group", grouped)
            out[grouped] = fa.bwd(q, k, v, o, do, lse, causal=True, deterministic=True)
            torch.cuda.synchronize()
    finally:
        fa.set_tuning("bwd_causal_group", -1)
        fa.set_tuning("bwd_pair", -1)
    assert fa.get_status() == 0
    for a_, b_ in zip(out[0], out[1]):
        assert torch.equal(a_, b_)


def test_det_bwd_workspace_size_and_errors():
    fa = _fa()
    assert fa.bwd_workspace_size(2, 3, 100, 64, deterministic=True) == 2560
    x = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, 128), dtype=torch.float32, device="cuda")
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.bwd(x, x, x, x, x, lse, workspace=small, deterministic=True)
    assert e.value.code == 4
