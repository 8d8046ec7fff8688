"""Pins for the FP8 (E4M3) quantisation oracle (CPU only).

The E4M3 table and encoder are checked against torch's own float8_e4m3fn
conversion (a library routine) and the format's known landmarks; the
Hadamard matrix against scipy's and against orthogonality; the block
quantiser against the E4M3 error bound and the amax-to-448 property.
"""
import math

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from oracle import fp8_ref


def test_decode_table_matches_torch_and_landmarks():
    tab = oracle.e4m3_decode_table()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    finite = ~np.isnan(ref)
    assert np.array_equal(np.isnan(tab), np.isnan(ref))
    assert np.array_equal(tab[finite], ref[finite])
    assert tab[0x7E] == 448.0 and tab[0xFE] == -448.0
    assert tab[0x01] == 2.0 ** -9            # smallest subnormal
    assert tab[0x08] == 2.0 ** -6            # smallest normal
    assert tab[0x38] == 1.0
    assert np.isnan(tab[0x7F]) and np.isnan(tab[0xFF])


def test_encoder_matches_torch_rne_on_dense_grid_and_ties():
    tab = oracle.e4m3_decode_table()
    pos = np.sort(tab[:0x7F])
    mids = (pos[1:] + pos[:-1]) / 2            # exact ties
    rng = np.random.default_rng(0)
    grid = np.concatenate([pos, mids, rng.uniform(0, 448, 20000),
                           np.exp(rng.uniform(np.log(1e-4), np.log(448), 20000)),
                           np.nextafter(mids, 0), np.nextafter(mids, 1000)])
    grid = np.concatenate([grid, -grid]).astype(np.float32).astype(np.float64)
    ours = oracle.e4m3_encode_ref(grid)
    theirs = torch.tensor(grid, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, theirs)


def test_encoder_saturates_and_nan():
    codes = oracle.e4m3_encode_ref(np.array([448.0, 449.0, 464.0, 479.0, 500.0, 1e30, -1e30, np.nan]))
    assert codes.tolist()[:7] == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE]
    assert codes[7] == 0x7F


def test_hadamard_orthogonality_and_scipy():
    for d in (1, 2, 4, 64, 128):
        h = oracle.hadamard_ref(d)
        assert np.array_equal(h, scipy.linalg.hadamard(d))
        assert np.array_equal(h @ h.T, d * np.eye(d))
    with pytest.raises(ValueError):
        oracle.hadamard_ref(96)


def test_rotation_preserves_scores_and_attention():
    rng = np.random.default_rng(1)
    d = 64
    s = np.where(rng.random(d) < 0.5, -1.0, 1.0)
    q, k, v = (rng.standard_normal((1, 2, 20, d)) for _ in range(3))
    qr, kr = oracle.rotation_ref(q, s), oracle.rotation_ref(k, s)
    np.testing.assert_allclose(qr @ np.swapaxes(kr, -1, -2), q @ np.swapaxes(k, -1, -2), rtol=1e-12, atol=1e-12)
    o1, l1 = oracle.attn_fwd_ref(q, k, v, 0.125, False)
    o2, l2 = oracle.attn_fwd_ref(qr, kr, v, 0.125, False)
    np.testing.assert_allclose(o2, o1, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(l2, l1, rtol=1e-12, atol=1e-12)
    # the rotation really mixes coordinates: a one-hot row spreads to +-1/sqrt(d)
    e0 = np.zeros((1, 1, 1, d)); e0[..., 3] = 1.0
    assert np.allclose(np.abs(oracle.rotation_ref(e0, s)), 1 / math.sqrt(d))


@pytest.mark.parametrize("rotate", [False, True])
def test_block_quant_error_bound_and_amax(rotate):
    g = torch.Generator().manual_seed(5)
    B, H, N, d = 1, 2, 300, 64             # 3 blocks, the last one ragged (44 rows)
    x = torch.randn(B, H, N, d, generator=g)
    x = torch.where(torch.rand(B, H, N, d, generator=g) < 1e-2, x * 20, x).to(torch.bfloat16)
    s = np.where(np.random.default_rng(2).random(d) < 0.5, -1.0, 1.0)
    codes, scales = oracle.quant_fp8_ref(x.double().numpy(), rotate, s)
    assert codes.shape == (B, H, N, d) and scales.shape == (B, H, 3)
    xr = oracle.rotation_ref(x.double().numpy(), s) if rotate else x.double().numpy()
    deq = oracle.dequant_fp8_ref(codes, scales)
    for b in range(B):
        for h in range(H):
            for j in range(3):
                blk = xr[b, h, j * 128:(j + 1) * 128]
                sc = float(scales[b, h, j])
                assert sc == pytest.approx(np.max(np.abs(blk)) / 448.0, rel=1e-6)
                err = np.abs(deq[b, h, j * 128:(j + 1) * 128] - blk)
                # E4M3: 3 mantissa bits -> half-ulp 2^-4 relative; subnormal half-step 2^-10
                bound = np.maximum(np.abs(blk) * 2.0 ** -4, sc * 2.0 ** -10) * (1 + 1e-6)
                assert np.all(err <= bound)
                # the block's largest magnitude lands on +-448
                c = codes[b, h, j * 128:(j + 1) * 128]
                assert np.any((c == 0x7E) | (c == 0xFE))


def test_zero_block_gets_unit_scale():
    x = np.zeros((1, 1, 130, 8))
    x[0, 0, 128:] = 1.0
    codes, scales = oracle.quant_fp8_ref(x, False)
    assert scales[0, 0, 0] == 1.0 and np.all(codes[0, 0, :128] == 0)
    assert scales[0, 0, 1] == np.float32(1.0) / np.float32(448.0)


def test_per_tensor_is_worse_than_per_block_with_outliers():
    """With outliers present, one scale per block loses less than one per tensor."""
    g = torch.Generator().manual_seed(6)
    x = torch.randn(1, 1, 1024, 128, generator=g)
    x = torch.where(torch.rand(1, 1, 1024, 128, generator=g) < 1e-3, x * 20, x)
    x[0, 0, 5, 7] = 300.0                    # one block holds a large outlier
    x = x.double().numpy()
    codes, scales = oracle.quant_fp8_ref(x, False)
    e_blk = np.sqrt(np.mean((oracle.dequant_fp8_ref(codes, scales) - x) ** 2))
    e_tns = np.sqrt(np.mean((oracle.quant_fp8_per_tensor_ref(x) - x) ** 2))
    assert e_blk < e_tns


def test_planted_mistake_ties_away_is_caught():
    """An encoder that rounds ties away from zero must disagree with torch."""
    tab = oracle.e4m3_decode_table()
    pos = np.sort(tab[:0x7F])
    mids = (pos[1:] + pos[:-1]) / 2
    ours = fp8_ref.e4m3_encode_ref(mids)
    away = np.searchsorted(pos, mids, side="left").astype(np.uint8)   # always round up
    theirs = torch.tensor(mids, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, theirs) and not np.array_equal(away, theirs)


def test_tiny_block_scale_is_floored_at_smallest_normal():
    """A block whose amax / 448 would be subnormal takes the scale 2^-126
    (the smallest normal fp32); its codes are finite, exact multiples and
    decode back within the E4M3 bound.  The per-tensor quantiser follows the
    same rule."""
    x = np.zeros((1, 1, 128, 8))
    x[0, 0, 0, :4] = [1e-37, -3e-38, 2.0 ** -130, 0.0]     # amax / 448 ~ 2.2e-40: subnormal
    codes, scales = oracle.quant_fp8_ref(x, False)
    assert scales[0, 0, 0] == np.float32(2.0 ** -126) == oracle.MIN_SCALE
    vals = oracle.e4m3_decode_ref(codes)
    assert np.all(np.isfinite(vals)) and np.all(np.abs(vals) <= 448.0)
    deq = oracle.dequant_fp8_ref(codes, scales)
    xf = x.astype(np.float32).astype(np.float64)
    bound = np.maximum(np.abs(xf) * 2.0 ** -4, 2.0 ** -126 * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(np.abs(deq - xf) <= bound)
    assert codes[0, 0, 0, 3] == 0 and np.all(codes[0, 0, 1:] == 0)
    c1, s1 = oracle.quant_fp8_per_tensor_codes_ref(x)
    assert s1 == oracle.MIN_SCALE and np.array_equal(c1, codes)
    # just above the floor the plain rule applies
    x2 = x.copy()
    x2[0, 0, 0, 0] = 448.0 * 2.0 ** -120
    _, s2 = oracle.quant_fp8_ref(x2, False)
    assert s2[0, 0, 0] == np.float32(2.0 ** -120)


def test_fp8_target_is_below_what_e4m3_can_reach_on_the_fp8_workload(record_property):
    """The FP8 forward's 5e-2 relative-RMS target against the unquantised
    truth is not reachable by any E4M3 kernel on the FP8 workload (N(0, 1)
    with 0.1 % of entries x20, B2 H16 N8192 d128, non-causal): exact fp64
    attention on the quantised values alone, with no kernel rounding at all,
    already exceeds it.  Computed with the oracle only, on two heads and
    every 8th query row (rows of a non-causal head are independent).

    * Q, K, V block-quantised with the rotation (the kernel's inputs);
    * only Q, K quantised, V exact (the reading that keeps P V in bf16);
    both are above 5e-2.  The baselines: block scales without the rotation,
    and one scale per tensor without the rotation (the FA3 pages' "baseline
    FP8"), both worse than the rotated block format."""
    from exact_io_aware_42_b200 import inputs
    q, k, v = inputs.make_workload(inputs.FP8)
    d = q.shape[-1]
    sc = 1 / math.sqrt(d)
    s = inputs.signs(d).numpy()
    rows = np.arange(0, q.shape[2], 8)
    out = {}
    for b, h in ((0, 0), (1, 11)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        qf, kf, vf = (t[sl].double().numpy() for t in (q, k, v))

        def deq(x, rot):
            return oracle.dequant_fp8_ref(*oracle.quant_fp8_ref(x, rot, s))[0, 0]

        def err(qq, kk, vv):
            o, _ = oracle.attn_fwd_rows_ref(qq, kk, vv, sc, False, rows)
            den = np.sqrt(np.mean(o_t ** 2))
            return float(np.sqrt(np.mean((o - o_t) ** 2)) / den)

        o_t, _ = oracle.attn_fwd_rows_ref(qf[0, 0], kf[0, 0], vf[0, 0], sc, False, rows)
        qr, kr, vb = deq(qf, True), deq(kf, True), deq(vf, False)
        pt = [oracle.quant_fp8_per_tensor_ref(x)[0, 0] for x in (qf, kf, vf)]
        e = {"qkv_rotated": err(qr, kr, vb), "qk_rotated_v_exact": err(qr, kr, vf[0, 0]),
             "qkv_block_naive": err(deq(qf, False), deq(kf, False), vb),
             "qkv_tensor_naive": err(*pt)}
        out[(b, h)] = e
        assert e["qkv_rotated"] > 5e-2 and e["qk_rotated_v_exact"] > 5e-2, e
        assert e["qkv_tensor_naive"] > e["qkv_rotated"] and e["qkv_block_naive"] > e["qkv_rotated"], e
        # the rotated block format itself stays within 1.5x of the target
        assert e["qkv_rotated"] < 7.5e-2, e
    record_property("fp8_format_errors", {f"{b},{h}": v_ for (b, h), v_ in out.items()})
    print({f"{b},{h}": {k_: round(x, 4) for k_, x in v_.items()} for (b, h), v_ in out.items()})
