"""fp64/fp32 oracle for the FP8 (E4M3) block quantisation with optional
random-sign Hadamard rotation ("incoherent processing").

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Sources: [Librarian] "FA3 -- the Hopper moment", pillar 3 (per-tile scale
instead of a whole-tensor scale; pre-multiplication by a random orthogonal
Hadamard-based matrix before quantising), and [Lineage] "FA3 (2024)", idea 3
(E4M3 inputs, block quantisation, random rotation via Hadamard).

Readings where the pages are silent:

* Block: 128 consecutive rows of one (b, h) times all d columns, one fp32
  scale per block.  (The Librarian page says 64 x d tiles; the workload under
  test asks for 128-row blocks.)
* Scale: ``scale = fp32(amax) / 448`` in IEEE fp32, 448 being the largest
  finite E4M3 magnitude; a block whose amax is 0 gets scale 1.  The scale
  is floored at 2^-126, the smallest normal fp32: below that amax / 448 is
  subnormal and has no finite fp32 reciprocal, which a kernel that divides
  by multiplying with the reciprocal cannot use.  With the floor every
  quotient still lies within [-448, 448].
* Code: ``e4m3(fp32(x) / scale)`` -- the quotient is rounded to fp32 first
  (the kernel's precision), then to E4M3 with round-to-nearest-even and
  saturation to +-448 (OCP e4m3fn: no infinities, 0x7F/0xFF are NaN).
* Rotation: ``M = diag(s) H_d / sqrt(d)`` with H_d the Sylvester Hadamard
  matrix and s in {+1, -1}^d given by the caller; X <- X M along d.  M is
  orthogonal, so (Q M)(K M)^T = Q K^T and the attention scores are unchanged.
  V is never rotated.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
MIN_SCALE = np.float32(2.0 ** -126)   # smallest normal fp32
QBLOCK_ROWS = 128


def _e4m3_value(code: int) -> float:
    """Value of one E4M3 (e4m3fn) byte from the format's definition."""
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    mant = code & 0x7
    if e == 0xF and mant == 0x7:
        return float("nan")
    if e == 0:                       # subnormal: mant/8 * 2^(1-7)
        return sign * (mant / 8.0) * 2.0 ** (-6)
    return sign * (1.0 + mant / 8.0) * 2.0 ** (e - 7)


def e4m3_decode_table() -> np.ndarray:
    """All 256 E4M3 byte values as fp64 (NaN at 0x7F and 0xFF)."""
    return np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)


_TABLE = e4m3_decode_table()
_POS = _TABLE[:0x7F]        # codes 0x00..0x7E: non-negative finite, increasing


def e4m3_encode_ref(x) -> np.ndarray:
    """Round fp values to E4M3 bytes: nearest, ties to even code, saturating.

    Table-driven: the two neighbouring representable magnitudes are found in
    the sorted table of codes 0x00..0x7E and the nearer one is taken; on a tie
    the even code (mantissa LSB 0) wins.  Magnitudes above 448 saturate to 448.
    The sign bit follows the sign of x (so -0.0 and tiny negatives give 0x80).
    NaN maps to 0x7F.
    """
    x = np.asarray(x, dtype=np.float64)
    flat = x.ravel()
    out = np.empty(flat.shape, dtype=np.uint8)
    mag = np.abs(flat)
    nan = np.isnan(flat)
    mag_c = np.where(nan, 0.0, np.minimum(mag, E4M3_MAX))
    hi = np.searchsorted(_POS, mag_c, side="left")          # first table value >= mag
    hi = np.clip(hi, 0, _POS.size - 1)
    lo = np.clip(hi - 1, 0, _POS.size - 1)
    d_hi = _POS[hi] - mag_c
    d_lo = mag_c - _POS[lo]
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(_POS[hi] == mag_c, hi, code).astype(np.uint8)   # exact hit
    sign = np.signbit(flat).astype(np.uint8) << 7
    out[:] = code | sign
    out[nan] = 0x7F
    return out.reshape(x.shape)


def e4m3_decode_ref(codes) -> np.ndarray:
    """E4M3 bytes -> fp64 values."""
    return _TABLE[np.asarray(codes, dtype=np.uint8)]


def hadamard_ref(d: int) -> np.ndarray:
    """Sylvester Hadamard matrix H_d (entries +-1), d a power of two."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    h = np.ones((1, 1))
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


def rotation_ref(x, signs) -> np.ndarray:
    """X M along the last axis, M = diag(s) H_d / sqrt(d), in fp64."""
    x = np.asarray(x, dtype=np.float64)
    s = np.asarray(signs, dtype=np.float64)
    d = x.shape[-1]
    m = (s[:, None] * hadamard_ref(d)) / np.sqrt(d)
    return x @ m


def quant_fp8_ref(x, rotate: bool, signs=None, block_rows: int = QBLOCK_ROWS):
    """Per-block E4M3 quantisation of x [B, H, N, d].

    Returns (codes uint8 [B, H, N, d], scales fp32 [B, H, ceil(N / block_rows)]).
    With ``rotate`` the rows are first multiplied by M (``rotation_ref``), the
    rotated values being rounded to fp32 before the amax and the division,
    which is where the kernel holds them.
    """
    x = np.asarray(x, dtype=np.float64)
    if rotate:
        xr = rotation_ref(x, signs).astype(np.float32)
    else:
        xr = x.astype(np.float32)          # bf16 inputs: exact
    B, H, N, d = xr.shape
    nblk = -(-N // block_rows)
    scales = np.ones((B, H, nblk), dtype=np.float32)
    codes = np.zeros((B, H, N, d), dtype=np.uint8)
    for b in range(B):
        for h in range(H):
            for j in range(nblk):
                blk = xr[b, h, j * block_rows:(j + 1) * block_rows]
                amax = np.float32(np.max(np.abs(blk))) if blk.size else np.float32(0)
                sc = np.float32(1.0) if amax == 0 else max(np.float32(amax / np.float32(E4M3_MAX)), MIN_SCALE)
                scales[b, h, j] = sc
                q = (blk / sc).astype(np.float32)      # IEEE fp32 quotient
                codes[b, h, j * block_rows:(j + 1) * block_rows] = e4m3_encode_ref(q)
    return codes, scales


def dequant_fp8_ref(codes, scales, block_rows: int = QBLOCK_ROWS) -> np.ndarray:
    """codes [B, H, N, d] and per-block scales -> fp64 values code * scale."""
    vals = e4m3_decode_ref(codes)
    sc = np.repeat(np.asarray(scales, dtype=np.float64), block_rows, axis=2)
    return vals * sc[:, :, :vals.shape[2], None]


def quant_fp8_per_tensor_codes_ref(x):
    """Whole-tensor E4M3 quantisation without rotation (the baseline the FA3
    pillar improves on): one scale for the whole tensor, the same rules as a
    block otherwise.  Returns (codes uint8, scale fp32)."""
    x = np.asarray(x, dtype=np.float64).astype(np.float32)
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0)
    sc = np.float32(1.0) if amax == 0 else max(np.float32(amax / np.float32(E4M3_MAX)), MIN_SCALE)
    return e4m3_encode_ref((x / sc).astype(np.float32)), sc


def quant_fp8_per_tensor_ref(x):
    """Whole-tensor E4M3 quantisation, dequantised: fp64 values code * scale."""
    codes, sc = quant_fp8_per_tensor_codes_ref(x)
    return e4m3_decode_ref(codes) * np.float64(sc)
