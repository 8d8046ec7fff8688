"""GPU parity of the FP8 path (fa_quant_fp8, fa_fwd_fp8 through the C ABI).

Quantisation: without rotation the E4M3 codes and block scales must equal the
oracle's bit for bit (same fp32 quotient, same round-to-nearest-even).  With
rotation the kernel rotates in fp32 (fast Walsh-Hadamard transform) while the
oracle rotates in fp64, so a code may differ by one step only where the
oracle's quotient lies within a tiny relative distance of a rounding tie;
everything else must match.

Attention: the kernel's own error is measured against the fp64 oracle on
the DEQUANTISED inputs.  Against the truth (the fp64 oracle on the
unquantised inputs) the error is dominated by the E4M3 format: on these
inputs (N(0, 1) with 0.1% of entries x20) the quantisation of Q and K alone,
simulated exactly by the oracle, already gives ~6.6e-2 relative RMS with the
rotation and ~1.1e-1 without, above the 5e-2 target.  The tests therefore
check that the kernel adds at most 1e-2 to the format's own error, that the
rotation lowers the error, and report both numbers.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_42_b200 import inputs
from tests.helpers import FP8_REL_RMS, LSE_MAX_ABS, f64, rel_rms

pytestmark = pytest.mark.gpu


def _fa():
    import exact_io_aware_42_b200 as fa
    return fa


def gpu_quant(x, signs=None):
    fa = _fa()
    codes, scales = fa.quant_fp8(x.cuda(), None if signs is None else signs.cuda())
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 100, 128, 300, 1024])
def test_quant_bit_exact_without_rotation(N, d):
    q, _, _ = inputs.make_qkv(2, 3, N, d, seed=40 + N, outliers=True)
    codes, scales = gpu_quant(q)
    rc, rs = oracle.quant_fp8_ref(f64(q), False)
    assert np.array_equal(scales, rs)
    assert np.array_equal(codes, rc)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [100, 1024])
def test_quant_rotated_matches_up_to_ties(N, d):
    q, _, _ = inputs.make_qkv(2, 3, N, d, seed=60 + N, outliers=True)
    s = inputs.signs(d)
    codes, scales = gpu_quant(q, s)
    rc, rs = oracle.quant_fp8_ref(f64(q), True, s.numpy())
    np.testing.assert_allclose(scales, rs, rtol=1e-5)
    diff = codes != rc
    frac = diff.mean()
    assert frac < 2e-3, frac
    if diff.any():
        # every differing code must be a neighbour, at a quotient next to a tie
        xr = oracle.rotation_ref(f64(q), s.numpy())
        sc = np.repeat(rs.astype(np.float64), 128, axis=2)[:, :, :N, None]
        quot = np.abs(xr / sc)[diff]
        gc, oc = codes[diff], rc[diff]
        zero = ((gc & 0x7F) == 0) & ((oc & 0x7F) == 0)          # +0 vs -0: both zero
        gc, oc, quot = gc[~zero], oc[~zero], quot[~zero]
        a = oracle.e4m3_decode_ref(gc & 0x7F)
        b = oracle.e4m3_decode_ref(oc & 0x7F)
        small = np.maximum(a, b) <= 2.0 ** -9                  # 0 vs smallest subnormal
        assert np.all(((gc & 0x80) == (oc & 0x80)) | small)
        assert np.all(np.abs((gc & 0x7F).astype(int) - (oc & 0x7F).astype(int)) == 1)
        mid = (a + b) / 2
        assert np.all(np.abs(quot - mid) <= 1e-5 * np.maximum(mid, 2.0 ** -9))


def test_quant_zero_block_scale_one():
    x = torch.zeros((1, 1, 200, 128), dtype=torch.bfloat16)
    x[0, 0, 150, 3] = 2.0
    codes, scales = gpu_quant(x)
    assert scales[0, 0, 0] == 1.0 and np.all(codes[0, 0, :128] == 0)
    assert scales[0, 0, 1] == np.float32(2.0) / np.float32(448.0)


def fp8_attention(q, k, v, causal, rotate, scale=None):
    fa = _fa()
    d = q.shape[-1]
    s = inputs.signs(d).cuda() if rotate else None
    q8, sq = fa.quant_fp8(q.cuda(), s)
    k8, sk = fa.quant_fp8(k.cuda(), s)
    v8, sv = fa.quant_fp8(v.cuda(), None)
    o, lse = fa.fwd_fp8(q8, k8, v8, sq, sk, sv, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.get_status() == 0
    return o.cpu(), lse.cpu()


def format_error(q, k, v, causal, rotate):
    """Relative RMS of exact attention on the dequantised inputs vs the truth:
    the error of the E4M3 block format itself (no kernel involved)."""
    d = q.shape[-1]
    s = inputs.signs(d).numpy()
    qf, kf, vf = f64(q), f64(k), f64(v)
    dq = oracle.dequant_fp8_ref(*oracle.quant_fp8_ref(qf, rotate, s))
    dk = oracle.dequant_fp8_ref(*oracle.quant_fp8_ref(kf, rotate, s))
    dv = oracle.dequant_fp8_ref(*oracle.quant_fp8_ref(vf, False))
    o_t, _ = oracle.attn_fwd_ref(qf, kf, vf, 1 / math.sqrt(d), causal)
    o_q, _ = oracle.attn_fwd_ref(dq, dk, dv, 1 / math.sqrt(d), causal)
    return rel_rms(o_q, o_t), o_t


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [7, 128, 300, 1000])
def test_fp8_fwd_small(N, causal):
    q, k, v = inputs.make_qkv(1, 2, N, 128, seed=80 + N, outliers=True)
    for rotate in (True, False):
        e_fmt, o_ref = format_error(q, k, v, causal, rotate)
        o, lse = fp8_attention(q, k, v, causal, rotate)
        assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
        e = rel_rms(o, o_ref)
        assert e <= max(FP8_REL_RMS, e_fmt + 1e-2), (rotate, e, e_fmt)


def test_fp8_fwd_workload_sampled_heads_rotated_vs_naive(record_property):
    w = inputs.FP8
    q, k, v = inputs.make_workload(w)
    res = {}
    for rotate in (True, False):
        o, lse = fp8_attention(q, k, v, False, rotate)
        assert torch.isfinite(o.float()).all()
        errs, fmts = [], []
        for b, h in ((0, 0), (1, 11)):
            sl = (slice(b, b + 1), slice(h, h + 1))
            e_fmt, o_ref = format_error(q[sl], k[sl], v[sl], False, rotate)
            errs.append(rel_rms(o[sl], o_ref))
            fmts.append(e_fmt)
        tag = "rotated" if rotate else "naive"
        res[tag], res[tag + "_format"] = max(errs), max(fmts)
        assert max(errs) <= max(fmts) + 1e-2, (tag, errs, fmts)
    record_property("fp8_rel_rms", res)
    print(f"FP8 relative RMS vs fp64 truth: rotated {res['rotated']:.4e} (format alone "
          f"{res['rotated_format']:.4e}), naive {res['naive']:.4e} (format alone {res['naive_format']:.4e})")
    assert res["rotated"] < res["naive"]


def test_fp8_kernel_error_isolated_from_quantisation():
    """Against the oracle on the dequantised inputs, only the kernel's own
    rounding (P in E4M3, O in bf16) remains."""
    q, k, v = inputs.make_qkv(1, 2, 1024, 128, seed=91, outliers=True)
    fa = _fa()
    q8, sq = fa.quant_fp8(q.cuda())
    k8, sk = fa.quant_fp8(k.cuda())
    v8, sv = fa.quant_fp8(v.cuda())
    o, _ = fa.fwd_fp8(q8, k8, v8, sq, sk, sv)
    deq = [oracle.dequant_fp8_ref(c.cpu().numpy(), s_.cpu().numpy()) for c, s_ in ((q8, sq), (k8, sk), (v8, sv))]
    o_ref, _ = oracle.attn_fwd_ref(deq[0], deq[1], deq[2], 1 / math.sqrt(128), False)
    assert rel_rms(o.cpu(), o_ref) <= 3e-2


def test_fp8_fwd_rejects_d64():
    fa = _fa()
    x = torch.zeros((1, 1, 128, 64), dtype=torch.uint8, device="cuda")
    s = torch.ones((1, 1, 1), dtype=torch.float32, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.fwd_fp8(x, x, x, s, s, s)
    assert e.value.code == 2


@pytest.mark.parametrize("d", [64, 128])
def test_quant_tiny_blocks_bit_exact(d):
    """Blocks whose amax / 448 is below the smallest normal fp32 take the
    scale 2^-126 on both sides; codes must match the oracle bit for bit (no
    NaN codes from an infinite reciprocal)."""
    g = torch.Generator().manual_seed(77)
    x = torch.randn(1, 2, 300, d, generator=g) * 1e-37
    x[0, 1, 128:256] = torch.randn(128, d, generator=g) * 2.0 ** -130    # bf16 subnormals
    x[0, 1, 256:] = torch.randn(44, d, generator=g)                      # an ordinary block
    x = x.to(torch.bfloat16)
    codes, scales = gpu_quant(x)
    rc, rs = oracle.quant_fp8_ref(f64(x), False)
    assert np.array_equal(scales, rs)
    bad = np.argwhere(codes != rc)
    detail = []
    for idx in bad[:12]:
        idx = tuple(idx)
        xv = float(f64(x)[idx])
        qv = np.float32(np.float32(xv) / rs[idx[0], idx[1], idx[2] // 128])
        detail.append(f"{idx}: x={xv:.6e} q={float(qv):.9e} gpu=0x{codes[idx]:02x} oracle=0x{rc[idx]:02x}")
    assert bad.size == 0, f"{len(bad)} codes differ:\n" + "\n".join(detail)
    assert scales[0, 0, 0] == oracle.MIN_SCALE and not np.any((codes & 0x7F) == 0x7F)


def test_fp8_fwd_rotated_block_vs_per_tensor_baseline(record_property):
    """The pages' comparison ("FA3": block quantisation plus the Hadamard
    rotation against baseline FP8 with one scale per tensor), both run through
    the FP8 kernel on the FP8 workload and measured against the fp64 truth on
    two heads (every 8th query row).  The per-tensor codes come from the
    oracle's quantiser and are passed to the kernel with constant block
    scales; the rotated codes come from the library's quantiser."""
    fa = _fa()
    w = inputs.FP8
    q, k, v = inputs.make_workload(w)
    d = w.d
    sc = 1 / math.sqrt(d)
    nb = fa.n_blocks(w.N)
    o_rot, _ = fp8_attention(q, k, v, False, True)
    dev = []
    for x in (q, k, v):
        c, s = oracle.quant_fp8_per_tensor_codes_ref(f64(x))
        dev.append((torch.from_numpy(c).cuda(), torch.full((w.B, x.shape[1], nb), float(s), device="cuda")))
    o_pt, _ = fa.fwd_fp8(dev[0][0], dev[1][0], dev[2][0], dev[0][1], dev[1][1], dev[2][1])
    torch.cuda.synchronize()
    assert fa.get_status() == 0
    o_pt = o_pt.cpu()
    rows = np.arange(0, w.N, 8)
    e_rot, e_pt = [], []
    for b, h in ((0, 0), (1, 11)):
        o_t, _ = oracle.attn_fwd_rows_ref(q[b, h], k[b, h], v[b, h], sc, False, rows)
        e_rot.append(rel_rms(o_rot[b, h][rows], o_t))
        e_pt.append(rel_rms(o_pt[b, h][rows], o_t))
    ratio = max(e_pt) / max(e_rot)
    record_property("fp8_rotated_block", max(e_rot))
    record_property("fp8_per_tensor_naive", max(e_pt))
    print(f"FP8 kernel vs fp64 truth: rotated block {max(e_rot):.4e}, per-tensor naive {max(e_pt):.4e}, "
          f"ratio {ratio:.2f} (the pages report 2.6x on their inputs)")
    assert max(e_rot) < max(e_pt)
    assert max(e_rot) <= 7.5e-2 + 1e-2


# The FP8 kernel's own error against the oracle on the dequantised inputs is
# that of P rounded to E4M3: a half-ulp of 2^-4 relative, 3.6e-2 RMS for a
# uniformly distributed rounding error; O averages it over the row's keys,
# so its relative RMS stays below that (measured ~3e-2).
FP8_KERNEL_REL_RMS = 2.0 ** -4 / math.sqrt(3.0)


@pytest.mark.parametrize("pairs", [2, 4])
def test_fp8_fwd_exp2_split_variants(pairs):
    """The FP8 forward with part of its exp2 on the FMA-pipe polynomial: within
    the E4M3 rounding bound of P against the oracle on the dequantised inputs,
    and within a few E4M3 code flips of the SFU-only kernel."""
    fa = _fa()
    q, k, v = inputs.make_qkv(1, 2, 1000, 128, seed=93 + pairs, outliers=True)
    q8, sq = fa.quant_fp8(q.cuda())
    k8, sk = fa.quant_fp8(k.cuda())
    v8, sv = fa.quant_fp8(v.cuda())
    deq = [oracle.dequant_fp8_ref(c.cpu().numpy(), s_.cpu().numpy()) for c, s_ in ((q8, sq), (k8, sk), (v8, sv))]
    for causal in (False, True):
        o_sfu, _ = fa.fwd_fp8(q8, k8, v8, sq, sk, sv, causal=causal)
        fa.set_tuning("fp8_poly_pairs", pairs)
        try:
            o, _ = fa.fwd_fp8(q8, k8, v8, sq, sk, sv, causal=causal)
        finally:
            fa.set_tuning("fp8_poly_pairs", -1)
        torch.cuda.synchronize()
        assert fa.get_status() == 0
        o_ref, _ = oracle.attn_fwd_ref(deq[0], deq[1], deq[2], 1 / math.sqrt(128), causal)
        assert rel_rms(o.cpu(), o_ref) <= FP8_KERNEL_REL_RMS
        assert rel_rms(o.cpu(), o_sfu.cpu()) <= 1e-2


@pytest.mark.parametrize("persistent", [0, 1])
def test_fp8_fwd_kernel_variants_and_lse(persistent):
    """Both FP8 forward kernels (one CTA per work item; the persistent grid):
    O within the E4M3 rounding bound of P against the oracle on the
    dequantised inputs, and L within the bf16 path's bound (the scores are
    exact products of the dequantised inputs, and the row sum is fp32), on
    more work items than SMs."""
    fa = _fa()
    q, k, v = inputs.make_qkv(1, 24, 1500, 128, seed=97 + persistent, outliers=True)
    q8, sq = fa.quant_fp8(q.cuda())
    k8, sk = fa.quant_fp8(k.cuda())
    v8, sv = fa.quant_fp8(v.cuda())
    deq = [oracle.dequant_fp8_ref(c.cpu().numpy(), s_.cpu().numpy()) for c, s_ in ((q8, sq), (k8, sk), (v8, sv))]
    fa.set_tuning("fwd_persistent", persistent)
    try:
        for causal in (False, True):
            o, lse = fa.fwd_fp8(q8, k8, v8, sq, sk, sv, causal=causal)
            torch.cuda.synchronize()
            assert fa.get_status() == 0
            for h in (0, 11, 23):
                sl = (slice(0, 1), slice(h, h + 1))
                o_ref, l_ref = oracle.attn_fwd_ref(deq[0][sl], deq[1][sl], deq[2][sl], 1 / math.sqrt(128), causal)
                assert rel_rms(o[sl].cpu(), o_ref) <= FP8_KERNEL_REL_RMS, (h, causal)
                assert np.max(np.abs(f64(lse[sl].cpu()) - l_ref)) <= LSE_MAX_ABS, (h, causal)
    finally:
        fa.set_tuning("fwd_persistent", -1)
