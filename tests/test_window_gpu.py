"""GPU parity of the causal sliding window (fa_fwd_ex, fa_bwd_ex, fa_fwd_fp8_ex
with window_left >= 0, through the C ABI) against the fp64 oracle.

Windows below, at and across the 128-key tile size, ragged N, both head
sizes, grouped heads combined with a window, both backward variants, the FP8
forward, a full-size workload checked on sampled rows, and the argument
errors (a window without causal, window_left < -1).
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


CASES = [(300, 128, 0), (300, 128, 1), (513, 64, 127), (513, 128, 128), (700, 128, 200),
         (1000, 64, 333), (129, 128, 64), (256, 64, 1000)]


@pytest.mark.parametrize("N,d,w", CASES)
def test_window_fwd_bwd_parity(N, d, w):
    fa = _fa()
    H, H_kv = (4, 2) if N % 2 else (2, 2)
    q, k, v, do = inputs.make_gqa(1, H, H_kv, N, d, seed=1100 + N + w, with_do=True)
    scale = 1 / math.sqrt(d)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.fwd(qd, kd, vd, causal=True, window=w)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_fwd_gqa_ref(q, k, v, scale, True, window=w)
    og, lg = f64(o.cpu()), f64(lse.cpu())
    assert max_scaled_err(og, o_ref) <= O_MAX_ABS
    assert rel_rms(og, o_ref) <= O_REL_RMS
    assert np.max(np.abs(lg - lse_ref)) <= LSE_MAX_ABS
    ref = oracle.attn_bwd_gqa_ref(q, k, v, do, scale, True, window=w)
    for det in (False, True):
        grads = fa.bwd(qd, kd, vd, o, dod, lse, causal=True, deterministic=det, window=w)
        torch.cuda.synchronize()
        for name, g, r in zip(("dq", "dk", "dv"), grads, ref):
            e = rel_rms(f64(g.cpu()), r, GRAD_RMS_FLOOR)
            assert e <= GRAD_REL_RMS, f"det={det} {name}: {e:.3e}"
    assert fa.get_status() == 0


def test_window_full_size_sampled_rows():
    fa = _fa()
    B, H, N, d, w = 2, 8, 4096, 128, 1024
    q, k, v = inputs.make_qkv(B, H, N, d, seed=47)
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, window=w)
    torch.cuda.synchronize()
    assert fa.get_status() == 0
    o, lse = o.cpu(), lse.cpu()
    rows = [0, 127, 128, 1023, 1024, 1025, 2047, 3000, 4095]
    for b, h in ((0, 0), (1, 7)):
        o_ref, l_ref = oracle.attn_fwd_rows_ref(q[b, h], k[b, h], v[b, h], 1 / math.sqrt(d), True, rows, window=w)
        assert max_scaled_err(o[b, h, rows], o_ref) <= O_MAX_ABS
        assert np.max(np.abs(f64(lse[b, h, rows]) - l_ref)) <= LSE_MAX_ABS


def test_window_fp8_forward():
    fa = _fa()
    N, d, w = 900, 128, 300
    q, k, v = inputs.make_qkv(1, 2, N, d, seed=53, outliers=True)
    s = inputs.signs(d).cuda()
    q8, sq = fa.quant_fp8(q.cuda(), s)
    k8, sk = fa.quant_fp8(k.cuda(), s)
    v8, sv = fa.quant_fp8(v.cuda())
    o, _ = fa.fwd_fp8(q8, k8, v8, sq, sk, sv, causal=True, window=w)
    torch.cuda.synchronize()
    assert fa.get_status() == 0
    deq = [oracle.dequant_fp8_ref(c.cpu().numpy(), x.cpu().numpy()) for c, x in ((q8, sq), (k8, sk), (v8, sv))]
    o_ref, _ = oracle.attn_fwd_gqa_ref(deq[0], deq[1], deq[2], 1 / math.sqrt(d), True, window=w)
    assert rel_rms(o.cpu(), o_ref) <= 3e-2


def test_window_argument_errors():
    fa = _fa()
    from exact_io_aware_42_b200._lib import lib
    q = torch.zeros((1, 2, 128, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 2, 128), dtype=torch.float32, device="cuda")
    args = (q.data_ptr(), q.data_ptr(), q.data_ptr(), q.data_ptr(), lse.data_ptr(), 1, 2, 2, 128, 64, 0.125)
    assert lib().fa_fwd_ex(*args, 0, 5, None, None) == 1       # window without causal
    assert lib().fa_fwd_ex(*args, 1, -2, None, None) == 1      # window_left < -1
    assert lib().fa_fwd_ex(*args, 1, -1, None, None) == 0      # no window
    torch.cuda.synchronize()
    with pytest.raises(ValueError):
        fa.fwd(q, q, q, causal=False, window=3)
