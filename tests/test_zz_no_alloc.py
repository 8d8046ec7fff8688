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
from tests.helpers import GRAD_REL_RMS, GRAD_RMS_FLOOR, rel_rms

pytestmark = pytest.mark.gpu


def _call_noalloc(L, q, k, v, o, do, lse, causal):
    B, H, N, d = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    code = L.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                            lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d,
                            ctypes.c_float(1 / math.sqrt(d)), int(causal),
                            torch.cuda.current_stream().cuda_stream)
    return code, (dq, dk, dv)


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
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            e = rel_rms(g, r, GRAD_RMS_FLOOR)
            assert e <= GRAD_REL_RMS, f"call {call} {name}: relative RMS {e:.3e}"


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
