"""Failure detection on the GPU without a fault: a pipeline wait that can
never complete must end after its bound with FA_ERR_PIPELINE_TIMEOUT in the
device status word, and the context must stay usable afterwards."""
import math
import time

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    import numpy as np

    import exact_io_aware_42_b200 as fa
    import oracle
    from exact_io_aware_42_b200 import inputs
    from exact_io_aware_42_b200._lib import lib
    L = lib()
    torch.cuda.synchronize()
    fa.clear_status()
    t0 = time.time()
    assert L.fa_selftest_wait_timeout(torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    dt = time.time() - t0
    st = fa.get_status()
    assert st & 0xFF == 6 and (st >> 8) == 0x7F, hex(st)
    assert dt < 30, dt
    fa.clear_status()
    assert fa.get_status() == 0
    # the context still computes correctly
    q, k, v = inputs.make_qkv(1, 2, 256, 64, seed=5)
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    torch.cuda.synchronize()
    assert fa.get_status() == 0
    o_ref, l_ref = oracle.attn_fwd_ref(q, k, v, 1 / math.sqrt(64), True)
    assert np.max(np.abs(o.double().cpu().numpy() - o_ref)) <= 1e-2
    assert np.max(np.abs(lse.double().cpu().numpy() - l_ref)) <= 1e-4
