"""fa_bwd_noalloc: the backward for callers that cannot allocate device
memory (a host framework that owns all device memory through its own pool,
or a latency-critical path that must not pay cudaMalloc's device
synchronisation).  It runs the regular backward on scratch built into the
library, so its gradients must match fa_bwd with a caller-provided workspace,
call after call.

Kept in a file pytest collects last, so a stop-at-first-failure run has
already run every other test before this one.
"""
import ctypes
import math

import pytest
import torch

from exact_io_aware_42_b200 import inputs
from tests.helpers import GRAD_RMS_FLOOR, rel_rms

pytestmark = pytest.mark.gpu


def _call_noalloc(L, q, k, v, o, do, lse, causal):
    B, H, N, d = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    code = L.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                            lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d,
                            ctypes.c_float(1 / math.sqrt(d)), int(causal),
                            torch.cuda.current_stream().cuda_stream)
    return code, (dq, dk, dv)


def _check_against_workspace_backward(got, ref, tag):
    """dK and dV come out in a fixed order on both paths: bit-identical.  dQ
    sums key blocks in an order that varies from run to run (fp32 reductions),
    so it may differ in rare last bf16 bits: relative RMS within 1e-4."""
    dq, dk, dv = got
    rdq, rdk, rdv = ref
    assert torch.equal(dk, rdk), f"{tag}: dk differs"
    assert torch.equal(dv, rdv), f"{tag}: dv differs"
    e = rel_rms(dq, rdq, GRAD_RMS_FLOOR)
    assert e <= 1e-4, f"{tag} dq: relative RMS {e:.3e}"


@pytest.mark.parametrize("causal", [True, False])
def test_noalloc_matches_workspace_backward_on_consecutive_calls(causal):
    import exact_io_aware_42_b200 as fa
    from exact_io_aware_42_b200._lib import lib
    L = lib()
    q, k, v, do = (t.cuda() for t in inputs.make_qkv(2, 4, 1000, 128, seed=23, with_do=True))
    o, lse = fa.fwd(q, k, v, causal=causal)
    ref = fa.bwd(q, k, v, o, do, lse, causal=causal)
    for call in range(2):
        code, got = _call_noalloc(L, q, k, v, o, do, lse, causal)
        assert code == 0, f"call {call}: status {code}"
        torch.cuda.synchronize()
        assert fa.get_status() == 0
        _check_against_workspace_backward(got, ref, f"call {call}")


def test_noalloc_after_a_larger_problem_left_the_scratch_dirty():
    """A first call on a larger problem (N = 3000) leaves different contents
    in the shared scratch, laid out for that shape; the next, smaller call
    must not see any of it."""
    import exact_io_aware_42_b200 as fa
    from exact_io_aware_42_b200._lib import lib
    L = lib()
    big = [t.cuda() for t in inputs.make_qkv(2, 4, 3000, 128, seed=29, with_do=True)]
    ob, lb = fa.fwd(*big[:3], causal=False)
    code, _ = _call_noalloc(L, *big[:3], ob, big[3], lb, False)
    assert code == 0
    q, k, v, do = (t.cuda() for t in inputs.make_qkv(2, 4, 1000, 128, seed=31, with_do=True))
    o, lse = fa.fwd(q, k, v, causal=True)
    ref = fa.bwd(q, k, v, o, do, lse, causal=True)
    code, got = _call_noalloc(L, q, k, v, o, do, lse, True)
    assert code == 0
    torch.cuda.synchronize()
    assert fa.get_status() == 0
    _check_against_workspace_backward(got, ref, "after N=3000")


def test_noalloc_binding_checks_every_tensor():
    import exact_io_aware_42_b200 as fa
    q, k, v, do = (t.cuda() for t in inputs.make_qkv(1, 2, 256, 64, seed=37, with_do=True))
    o, lse = fa.fwd(q, k, v)
    with pytest.raises(ValueError):
        fa.bwd_noalloc(q, k[:, :, :128].contiguous(), v, o, do, lse)
    with pytest.raises(ValueError):
        fa.bwd_noalloc(q, k, v, o, do[..., :32].contiguous(), lse)
    with pytest.raises(ValueError):
        fa.bwd_noalloc(q, k, v, o, do, lse[:, :1].contiguous())
    dq, dk, dv = fa.bwd_noalloc(q, k, v, o, do, lse)
    torch.cuda.synchronize()
    assert fa.get_status() == 0 and dq.shape == q.shape


def test_noalloc_rejects_problems_beyond_its_scratch():
    from exact_io_aware_42_b200._lib import lib
    L = lib()
    # 65,028 rows at d = 128 need more than the 32 MiB built in; nothing is launched
    x = torch.zeros((1, 1, 16, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, 16), dtype=torch.float32, device="cuda")
    p = x.data_ptr()
    code = L.fa_bwd_noalloc(p, p, p, p, p, lse.data_ptr(), p, p, p, 1, 1, 65028, 128,
                            ctypes.c_float(0.1), 0, None)
    assert code == 8
    assert L.fa_status_string(code) == b"FA_ERR_SCRATCH_LIMIT"
