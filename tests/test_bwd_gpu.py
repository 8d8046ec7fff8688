"""GPU parity of the bf16 backward (fa_bwd through the C ABI) against the fp64 oracle.

The GPU forward's O and LSE feed the GPU backward, as a training step would
use them; the oracle differentiates the exact definition from the same bf16
inputs.  Full-size runs are checked on sampled heads and, on every head,
against identities that hold at any size:
  sum over keys of dV = sum over queries of dO   (rows of P sum to 1)
  sum over keys of dK = 0                         (rows of dS sum to 0)
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


def run_fwd_bwd(q, k, v, do, causal, scale=None):
    fa = _fa()
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.fwd(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, dod, lse, causal=causal, scale=scale)
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
def test_bwd_ragged(N, d, causal):
    q, k, v, do = inputs.make_qkv(1, 2, N, d, seed=300 + N + d, with_do=True)
    got = run_fwd_bwd(q, k, v, do, causal)
    ref = oracle.attn_bwd_ref(q, k, v, do, 1 / math.sqrt(d), causal)
    assert_grads_close(got, ref, f"N={N} d={d} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_small_workload_shape(causal):
    w = inputs.SMALL
    q, k, v, do = inputs.make_qkv(w.B, w.H, w.N, w.d, w.seed, with_do=True)
    got = run_fwd_bwd(q, k, v, do, causal)
    ref = oracle.attn_bwd_ref(q, k, v, do, 1 / math.sqrt(w.d), causal)
    assert_grads_close(got, ref, f"{w.name} causal={causal}")


def test_bwd_long_workload_sampled_heads_and_identities():
    w = inputs.LONG
    q, k, v, do = inputs.make_workload(w)
    dq, dk, dv = run_fwd_bwd(q, k, v, do, True)
    # identities on every head, at full size
    sum_dv = f64(dv).sum(axis=2)
    sum_do = f64(do).sum(axis=2)
    assert np.max(np.abs(sum_dv - sum_do)) <= 2e-2 * max(1.0, np.max(np.abs(sum_do)))
    sum_dk = f64(dk).sum(axis=2)
    scale_dk = np.sqrt(np.mean(f64(dk) ** 2)) * math.sqrt(w.N)
    assert np.max(np.abs(sum_dk)) <= 2e-2 * scale_dk
    for b, h in ((0, 0), (2, 9), (3, 15)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        ref = oracle.attn_bwd_ref(q[sl], k[sl], v[sl], do[sl], 1 / math.sqrt(w.d), True)
        assert_grads_close((dq[sl], dk[sl], dv[sl]), ref, f"b={b} h={h}")


def test_bwd_dk_dv_deterministic_dq_stable():
    q, k, v, do = inputs.make_qkv(2, 4, 1000, 128, seed=17, with_do=True)
    a = run_fwd_bwd(q, k, v, do, True)
    b = run_fwd_bwd(q, k, v, do, True)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert rel_rms(a[0], b[0]) <= 1e-3


def test_bwd_workspace_errors():
    fa = _fa()
    x = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, 128), dtype=torch.float32, device="cuda")
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.bwd(x, x, x, x, x, lse, workspace=small)
    assert e.value.code == 4
