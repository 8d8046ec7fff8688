"""GPU parity of ALiBi (alibi_slopes of fa_fwd_ex, fa_bwd_ex, fa_fwd_fp8_ex,
through the C ABI) against the fp64 oracle: causal and non-causal, ragged N,
both head sizes, with grouped heads and a sliding window, both backward
variants, the FP8 forward, and a full-size causal workload on sampled rows.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_42_b200 import inputs
from tests.helpers import (GRAD_REL_RMS, GRAD_RMS_FLOOR, LSE_MAX_ABS, O_MAX_ABS, O_REL_RMS, f64,
                           max_scaled_err, rel_rms)

pytestmark = pytest.mark.gpu


def _fa():
    import exact_io_aware_42_b200 as fa
    return fa


def slopes(H):
    """The geometric ALiBi slopes 2^(-8 (h + 1) / H)."""
    return torch.tensor([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)], dtype=torch.float32)


CASES = [(300, 128, True, None, 4, 4), (513, 64, True, None, 4, 2), (300, 128, False, None, 2, 2),
         (200, 64, False, None, 4, 1), (700, 128, True, 200, 4, 2), (129, 128, True, 0, 2, 2)]


@pytest.mark.parametrize("N,d,causal,w,H,H_kv", CASES)
def test_alibi_fwd_bwd_parity(N, d, causal, w, H, H_kv):
    fa = _fa()
    q, k, v, do = inputs.make_gqa(1, H, H_kv, N, d, seed=1300 + N + d, with_do=True)
    sl = slopes(H)
    scale = 1 / math.sqrt(d)
    qd, kd, vd, dod, sld = (t.cuda() for t in (q, k, v, do, sl))
    o, lse = fa.fwd(qd, kd, vd, causal=causal, window=w, alibi=sld)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_fwd_gqa_ref(q, k, v, scale, causal, window=w, alibi=sl.numpy())
    og, lg = f64(o.cpu()), f64(lse.cpu())
    assert max_scaled_err(og, o_ref) <= O_MAX_ABS
    assert rel_rms(og, o_ref) <= O_REL_RMS
    assert np.max(np.abs(lg - lse_ref)) <= LSE_MAX_ABS
    ref = oracle.attn_bwd_gqa_ref(q, k, v, do, scale, causal, window=w, alibi=sl.numpy())
    for det in (False, True):
        grads = fa.bwd(qd, kd, vd, o, dod, lse, causal=causal, deterministic=det, window=w, alibi=sld)
        torch.cuda.synchronize()
        for name, g, r in zip(("dq", "dk", "dv"), grads, ref):
            e = rel_rms(f64(g.cpu()), r, GRAD_RMS_FLOOR)
            assert e <= GRAD_REL_RMS, f"det={det} {name}: {e:.3e}"
    assert fa.get_status() == 0


def test_alibi_full_size_sampled_rows():
    fa = _fa()
    B, H, N, d = 1, 8, 4096, 128
    q, k, v = inputs.make_qkv(B, H, N, d, seed=59)
    sl = slopes(H)
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, alibi=sl.cuda())
    torch.cuda.synchronize()
    assert fa.get_status() == 0
    o, lse = o.cpu(), lse.cpu()
    rows = [0, 1, 127, 128, 2048, 4095]
    for h in (0, 7):
        o_ref, l_ref = oracle.attn_fwd_gqa_ref(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], 1 / math.sqrt(d),
                                               True, alibi=[float(sl[h])])
        assert max_scaled_err(o[0, h, rows], o_ref[0, 0, rows]) <= O_MAX_ABS
        assert np.max(np.abs(f64(lse[0, h, rows]) - l_ref[0, 0, rows])) <= LSE_MAX_ABS


def test_alibi_fp8_forward():
    fa = _fa()
    N, d, H = 600, 128, 2
    q, k, v = inputs.make_qkv(1, H, N, d, seed=61, outliers=True)
    s = inputs.signs(d).cuda()
    sl = slopes(H)
    q8, sq = fa.quant_fp8(q.cuda(), s)
    k8, sk = fa.quant_fp8(k.cuda(), s)
    v8, sv = fa.quant_fp8(v.cuda())
    o, _ = fa.fwd_fp8(q8, k8, v8, sq, sk, sv, causal=True, alibi=sl.cuda())
    torch.cuda.synchronize()
    assert fa.get_status() == 0
    deq = [oracle.dequant_fp8_ref(c.cpu().numpy(), x.cpu().numpy()) for c, x in ((q8, sq), (k8, sk), (v8, sv))]
    o_ref, _ = oracle.attn_fwd_gqa_ref(deq[0], deq[1], deq[2], 1 / math.sqrt(d), True, alibi=sl.numpy())
    assert rel_rms(o.cpu(), o_ref) <= 3e-2


@pytest.mark.parametrize("N,causal,w,H,H_kv,alibi", [(300, True, None, 4, 2, True), (513, False, None, 4, 1, True),
                                                     (700, True, 200, 4, 2, False), (700, True, 150, 2, 2, True)])
def test_masks_and_grouped_heads_forward_d256(N, causal, w, H, H_kv, alibi):
    """The head-dim-256 forward takes grouped K/V heads, the sliding window
    and ALiBi exactly like the d <= 128 kernel."""
    fa = _fa()
    q, k, v = inputs.make_gqa(1, H, H_kv, N, 256, seed=1400 + N)
    sl = slopes(H) if alibi else None
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, window=w,
                    alibi=sl.cuda() if alibi else None)
    torch.cuda.synchronize()
    assert fa.get_status() == 0
    o_ref, lse_ref = oracle.attn_fwd_gqa_ref(q, k, v, 1 / math.sqrt(256), causal, window=w,
                                             alibi=sl.numpy() if alibi else None)
    og, lg = f64(o.cpu()), f64(lse.cpu())
    assert max_scaled_err(og, o_ref) <= O_MAX_ABS
    assert rel_rms(og, o_ref) <= O_REL_RMS
    assert np.max(np.abs(lg - lse_ref)) <= LSE_MAX_ABS
