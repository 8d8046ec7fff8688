"""GPU parity of grouped K/V heads (fa_fwd_ex, fa_bwd_ex, fa_fwd_fp8_ex with
H_kv < H, through the C ABI) against the fp64 grouped oracle.

Also exact identities of the implementation: with the K/V heads repeated
explicitly, the plain forward gives the same bits as the grouped one (same
kernel arithmetic, only the head index differs), and so does the
deterministic dQ; grouped dK, dV equal the per-head results summed over the
group up to bf16 rounding.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_42_b200 import inputs
from tests.helpers import (FP8_REL_RMS, GRAD_REL_RMS, GRAD_RMS_FLOOR, LSE_MAX_ABS, O_MAX_ABS,
                           O_REL_RMS, f64, rel_rms)

pytestmark = pytest.mark.gpu


def _fa():
    import exact_io_aware_42_b200 as fa
    return fa


def check_fwd(o, lse, o_ref, lse_ref, tag):
    o, lse = f64(o), f64(lse)
    assert np.max(np.abs(o - o_ref)) <= O_MAX_ABS, tag
    assert rel_rms(o, o_ref) <= O_REL_RMS, tag
    assert np.max(np.abs(lse - lse_ref)) <= LSE_MAX_ABS, tag


def check_grads(got, ref, tag):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        e = rel_rms(f64(g), r, GRAD_RMS_FLOOR)
        assert e <= GRAD_REL_RMS, f"{tag} {name}: {e:.3e}"


CASES = [(4, 2, 300, 128), (8, 1, 200, 64), (6, 3, 129, 128), (4, 1, 513, 64), (2, 2, 256, 128)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H,H_kv,N,d", CASES)
def test_gqa_fwd_bwd_parity(H, H_kv, N, d, causal):
    fa = _fa()
    q, k, v, do = inputs.make_gqa(2, H, H_kv, N, d, seed=900 + H + H_kv + N, with_do=True)
    scale = 1 / math.sqrt(d)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.fwd(qd, kd, vd, causal=causal)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_fwd_gqa_ref(q, k, v, scale, causal)
    check_fwd(o.cpu(), lse.cpu(), o_ref, lse_ref, f"fwd H={H} H_kv={H_kv} N={N}")
    ref = oracle.attn_bwd_gqa_ref(q, k, v, do, scale, causal)
    for det in (False, True):
        dq, dk, dv = fa.bwd(qd, kd, vd, o, dod, lse, causal=causal, deterministic=det)
        torch.cuda.synchronize()
        assert dk.shape == k.shape and dv.shape == v.shape
        check_grads((dq.cpu(), dk.cpu(), dv.cpu()), ref, f"bwd det={det} H={H} H_kv={H_kv} N={N}")
    assert fa.get_status() == 0


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_matches_repeated_heads_bitwise(causal):
    fa = _fa()
    B, H, H_kv, N, d = 2, 8, 2, 700, 128
    g = H // H_kv
    q, k, v, do = (t.cuda() for t in inputs.make_gqa(B, H, H_kv, N, d, seed=31, with_do=True))
    k_rep, v_rep = (t.repeat_interleave(g, dim=1).contiguous() for t in (k, v))
    o, lse = fa.fwd(q, k, v, causal=causal)
    o2, lse2 = fa.fwd(q, k_rep, v_rep, causal=causal)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    dq, dk, dv = fa.bwd(q, k, v, o, do, lse, causal=causal, deterministic=True)
    dq2, dk2, dv2 = fa.bwd(q, k_rep, v_rep, o, do, lse, causal=causal, deterministic=True)
    # B * H_kv * ceil(N / 128) = 24 thread blocks: the group is split over
    # several, whose fp32 partials are reduced in a fixed order
    dq3, dk3, dv3 = fa.bwd(q, k, v, o, do, lse, causal=causal, deterministic=True)
    torch.cuda.synchronize()
    assert torch.equal(dq, dq2)
    assert torch.equal(dq, dq3) and torch.equal(dk, dk3) and torch.equal(dv, dv3)
    for a, b in ((dk, dk2), (dv, dv2)):
        summed = b.float().reshape(B, H_kv, g, N, d).sum(dim=2)
        assert rel_rms(a.cpu(), summed.cpu()) <= 5e-3
    assert fa.get_status() == 0


def test_mqa_long_sampled_heads():
    """MQA at N = 4096: 16 query heads share one K/V head."""
    fa = _fa()
    B, H, N, d = 1, 16, 4096, 128
    q, k, v, do = inputs.make_gqa(B, H, 1, N, d, seed=37, with_do=True)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.fwd(qd, kd, vd, causal=True)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, dod, lse, causal=True)
    torch.cuda.synchronize()
    assert fa.get_status() == 0
    scale = 1 / math.sqrt(d)
    for h in (0, 15):
        o_ref, lse_ref = oracle.attn_fwd_ref(q[:, h:h + 1], k, v, scale, True)
        check_fwd(o.cpu()[:, h:h + 1], lse.cpu()[:, h:h + 1], o_ref, lse_ref, f"h={h}")
        r = oracle.attn_bwd_ref(q[:, h:h + 1], k, v, do[:, h:h + 1], scale, True)
        e = rel_rms(f64(dq.cpu()[:, h:h + 1]), r.dq, GRAD_RMS_FLOOR)
        assert e <= GRAD_REL_RMS, e
    # dV summed over the group: rows of P sum to one, so sum_keys dV = sum over heads and queries of dO
    sum_dv = f64(dv.cpu()).sum(axis=2)[:, 0]
    sum_do = f64(do).sum(axis=(1, 2))
    assert np.max(np.abs(sum_dv - sum_do)) <= 2e-2 * max(1.0, np.max(np.abs(sum_do)))


def test_gqa_fp8_forward():
    fa = _fa()
    B, H, H_kv, N, d = 1, 4, 2, 400, 128
    q, k, v = inputs.make_gqa(B, H, H_kv, N, d, seed=41, outliers=True)
    s = inputs.signs(d).cuda()
    q8, sq = fa.quant_fp8(q.cuda(), s)
    k8, sk = fa.quant_fp8(k.cuda(), s)
    v8, sv = fa.quant_fp8(v.cuda())
    o, lse = fa.fwd_fp8(q8, k8, v8, sq, sk, sv, causal=True)
    torch.cuda.synchronize()
    assert fa.get_status() == 0
    deq = [oracle.dequant_fp8_ref(c.cpu().numpy(), x.cpu().numpy()) for c, x in ((q8, sq), (k8, sk), (v8, sv))]
    # rotation: Q and K rotated by the same orthogonal map, so Q K^T is unchanged
    o_ref, _ = oracle.attn_fwd_gqa_ref(deq[0], deq[1], deq[2], 1 / math.sqrt(d), True)
    assert rel_rms(o.cpu(), o_ref) <= 3e-2


def test_gqa_bad_head_counts():
    fa = _fa()
    q = torch.zeros((1, 4, 128, 64), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 3, 128, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        fa.fwd(q, k, k)
    lse = torch.zeros((1, 4, 128), dtype=torch.float32, device="cuda")
    from exact_io_aware_42_b200._lib import lib
    code = lib().fa_fwd_ex(q.data_ptr(), k.data_ptr(), k.data_ptr(), q.data_ptr(), lse.data_ptr(),
                           1, 4, 3, 128, 64, 0.125, 0, -1, None, None)
    assert code == 1
    code = lib().fa_fwd_ex(q.data_ptr(), k.data_ptr(), k.data_ptr(), q.data_ptr(), lse.data_ptr(),
                           1, 4, 0, 128, 64, 0.125, 0, -1, None, None)
    assert code == 1
