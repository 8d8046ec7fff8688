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
