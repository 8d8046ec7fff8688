"""Host-side checks of the C ABI that need no GPU: the library builds and
loads, exports every entry point include/fa.h declares, and rejects bad
arguments with the documented status codes before touching the device."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


@pytest.fixture(scope="module")
def L():
    from exact_io_aware_42_b200 import build
    from exact_io_aware_42_b200._lib import lib
    build.build()
    return lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_documented_calls():
    names = declared_functions()
    for n in ("fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_quant_fp8", "fa_fwd_fp8",
              "fa_get_status", "fa_clear_status", "fa_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    from exact_io_aware_42_b200._lib import SIGNATURES
    for name in declared_functions():
        assert hasattr(L, name), name
        assert name in SIGNATURES, f"{name} has no ctypes signature"


def test_status_strings(L):
    assert L.fa_status_string(0) == b"FA_OK"
    assert L.fa_status_string(6) == b"FA_ERR_PIPELINE_TIMEOUT"
    assert L.fa_status_string(6 | (3 << 8)) == b"FA_ERR_PIPELINE_TIMEOUT"
    assert L.fa_status_string(99) == b"FA_ERR_UNKNOWN"


A = 4096  # a 16-byte aligned fake device address; never dereferenced on these paths


@pytest.mark.parametrize("args,code", [
    ((A, A, A, A, A, 1, 1, 128, 96, 0.1, 0), 2),         # d unsupported
    ((A, A, A, A, A, 1, 1, 128, 192, 0.1, 0), 2),
    ((A, A, A, A, A, 1, 1, 128, 512, 0.1, 0), 2),
    ((A, A, A, A, A, -1, 1, 128, 64, 0.1, 0), 1),        # negative size
    ((A, A, A, A, A, 1, 1, -5, 64, 0.1, 0), 1),
    ((A, A, A, A, A, 1, 1, 128, 64, -0.5, 0), 1),        # negative scale
    ((A, A, A, A, A, 1, 1, 128, 64, float("nan"), 0), 1),
    ((A, A, A, A, A, 1, 1, (1 << 20) + 1, 64, 0.1, 0), 2),  # N above the limit
    ((None, A, A, A, A, 1, 1, 128, 64, 0.1, 0), 1),      # null pointer
    ((A + 8, A, A, A, A, 1, 1, 128, 64, 0.1, 0), 3),     # misaligned
    ((A, A, A, A, A + 2, 1, 1, 128, 64, 0.1, 0), 3),     # lse not 4-byte aligned
    ((None, None, None, None, None, 1, 1, 0, 64, 0.1, 0), 0),   # empty problem
    ((None, None, None, None, None, 0, 8, 128, 128, 0.1, 1), 0),
])
def test_fwd_argument_errors(L, args, code):
    assert L.fa_fwd(*args, None) == code


def test_workspace_size(L):
    assert L.fa_bwd_workspace_size(1, 1, 128, 96) == 0
    assert L.fa_bwd_workspace_size(-1, 1, 128, 64) == 0
    got = L.fa_bwd_workspace_size(4, 16, 4096, 128)
    rows = 4 * 16 * 4096
    assert got == rows * 128 * 4 + rows * 4
    assert L.fa_bwd_workspace_size(1, 1, 1, 64) == 256 + 256


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_device_reports_no_device(L):
    assert L.fa_fwd(A, A, A, A, A, 1, 1, 128, 64, 0.1, 0, None) == 7


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import exact_io_aware_42_b200._lib as lb
    monkeypatch.setattr(lb, "_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(lb, "_LIB", None)
    with pytest.raises(RuntimeError, match="missing"):
        lb.lib()


@pytest.mark.parametrize("hkv,causal,window,alibi,code", [
    (3, 0, -1, None, 1),        # H = 4 not a multiple of H_kv = 3
    (0, 0, -1, None, 1),        # H_kv < 1
    (2, 0, 5, None, 1),         # window without causal
    (2, 1, -2, None, 1),        # window_left < -1
    (2, 1, 5, A + 2, 3),        # ALiBi slopes not 4-byte aligned
])
def test_fwd_ex_argument_errors(L, hkv, causal, window, alibi, code):
    assert L.fa_fwd_ex(A, A, A, A, A, 1, 4, hkv, 128, 64, 0.1, causal, window, alibi, None) == code


def test_bwd_ex_argument_errors(L):
    args = (A,) * 9 + (1, 4, 2, 128, 64, 0.1)
    assert L.fa_bwd_ex(*args, 0, 7, None, 0, A, 1 << 30, None) == 1      # window without causal
    assert L.fa_bwd_ex(*args, 1, -1, None, 0, A, 16, None) == 4          # workspace too small
    assert L.fa_bwd_ex(*(A,) * 9, 1, 4, 3, 128, 64, 0.1, 1, -1, None, 0, A, 1 << 30, None) == 1


def test_ex_workspace_sizes(L):
    # H_kv = H: the plain sizes
    assert L.fa_bwd_ex_workspace_size(4, 16, 16, 4096, 128, 0) == L.fa_bwd_workspace_size(4, 16, 4096, 128)
    assert L.fa_bwd_ex_workspace_size(4, 16, 16, 4096, 128, 1) == \
        L.fa_bwd_deterministic_workspace_size(4, 16, 4096, 128)
    # MQA B4 H16 N4096: 128 (K/V head, key block) pairs, split S = 4: fp32 partials 4 x 2 x 4 x 4096 x 128
    part = 4 * 2 * 4 * 4096 * 128 * 4
    assert L.fa_bwd_ex_workspace_size(4, 16, 1, 4096, 128, 1) == \
        L.fa_bwd_deterministic_workspace_size(4, 16, 4096, 128) + part
    # GQA 32:8 at B4 N4096 fills the GPU (1024 pairs): no partials
    assert L.fa_bwd_ex_workspace_size(4, 32, 8, 4096, 128, 0) == L.fa_bwd_workspace_size(4, 32, 4096, 128)
    assert L.fa_bwd_ex_workspace_size(1, 4, 3, 128, 64, 0) == 0
    assert L.fa_bwd_deterministic_workspace_size(2, 3, 100, 64) == 2560


def test_tuning_controls(L):
    """fa_set_tuning accepts only the documented values, -1 restores the
    default, and fa_get_tuning reports what a call would use (no device
    needed)."""
    from exact_io_aware_42_b200._lib import (TUNE_BWD_POLY_GROUPS, TUNE_DQ_POLY_PAIRS, TUNE_FWD_POLY_DEGREE,
                                             TUNE_FWD_POLY_PAIRS)
    d128 = L.fa_get_tuning(TUNE_FWD_POLY_PAIRS, 128)
    d64 = L.fa_get_tuning(TUNE_FWD_POLY_PAIRS, 64)
    assert d128 in (0, 2, 4) and d64 in (0, 2, 4)
    assert L.fa_set_tuning(TUNE_FWD_POLY_PAIRS, 2) == 0
    assert L.fa_get_tuning(TUNE_FWD_POLY_PAIRS, 128) == 2 and L.fa_get_tuning(TUNE_FWD_POLY_PAIRS, 64) == 2
    assert L.fa_set_tuning(TUNE_FWD_POLY_PAIRS, -1) == 0
    assert L.fa_get_tuning(TUNE_FWD_POLY_PAIRS, 128) == d128
    for knob, bad in ((TUNE_FWD_POLY_PAIRS, 3), (TUNE_FWD_POLY_DEGREE, 5), (TUNE_BWD_POLY_GROUPS, 4),
                      (TUNE_DQ_POLY_PAIRS, 1), (0, 0), (99, 0)):
        assert L.fa_set_tuning(knob, bad) == 1
    assert L.fa_get_tuning(TUNE_FWD_POLY_DEGREE, 64) in (3, 4)
    assert L.fa_get_tuning(TUNE_DQ_POLY_PAIRS, 128) == 0
    assert L.fa_get_tuning(99, 64) == -1
    from exact_io_aware_42_b200._lib import (TUNE_BWD_CAUSAL_GROUP, TUNE_FWD_CAUSAL_GROUP, TUNE_FWD_PERSISTENT,
                                             TUNE_FWD_Q1)
    assert L.fa_get_tuning(TUNE_FWD_Q1, 128) == -1      # chosen per call by default
    assert L.fa_get_tuning(TUNE_FWD_PERSISTENT, 128) == -1
    assert L.fa_get_tuning(TUNE_FWD_PERSISTENT, 256) == 1   # the d = 256 kernel is always persistent
    assert L.fa_set_tuning(7, 0) == 1                   # a retired knob number
    assert L.fa_get_tuning(TUNE_BWD_CAUSAL_GROUP, 128) == 1
    for knob in (TUNE_FWD_PERSISTENT, TUNE_FWD_CAUSAL_GROUP, TUNE_FWD_Q1, TUNE_BWD_CAUSAL_GROUP):
        default = L.fa_get_tuning(knob, 128)
        assert default in ((-1,) if knob in (TUNE_FWD_Q1, TUNE_FWD_PERSISTENT, TUNE_FWD_CAUSAL_GROUP) else (0, 1))
        for v in (0, 1):
            assert L.fa_set_tuning(knob, v) == 0 and L.fa_get_tuning(knob, 128) == v
        assert L.fa_set_tuning(knob, 2) == 1
        assert L.fa_set_tuning(knob, -1) == 0 and L.fa_get_tuning(knob, 128) == default


def test_exp2_selftest_argument_errors(L):
    assert L.fa_selftest_exp2(A, A, 3, 3, None) == 1          # odd count
    assert L.fa_selftest_exp2(A, A, 4, 6, None) == 1          # no such degree
    assert L.fa_selftest_exp2(None, A, 4, 3, None) == 1
    assert L.fa_selftest_exp2(A + 4, A, 4, 3, None) == 3      # not 8-byte aligned
    assert L.fa_selftest_exp2(None, None, 0, 3, None) == 0    # empty


def test_head_dim_256_limits(L):
    """d = 256: the forward and the backward take it (the backward is always
    the reproducible one, with the D-only workspace); the quantiser and the
    FP8 forward reject it before touching the device."""
    rows = 2 * 3 * 100
    ws = (rows * 4 + 255) // 256 * 256
    assert L.fa_bwd_workspace_size(2, 3, 100, 256) == ws
    assert L.fa_bwd_deterministic_workspace_size(2, 3, 100, 256) == ws
    assert L.fa_bwd_ex_workspace_size(2, 3, 3, 100, 256, 0) == ws
    assert L.fa_bwd(*(A,) * 9, 1, 1, 128, 256, 0.1, 0, A, 16, None) == 4      # workspace too small
    assert L.fa_quant_fp8(A, A, A, 1, 1, 128, 256, None, None) == 2
    assert L.fa_fwd_fp8(*(A,) * 8, 1, 1, 128, 256, 0.1, 0, None) == 2
    assert L.fa_fwd(A, A, A, A, A, 1, 1, 128, 320, 0.1, 0, None) == 2
