"""FP8-E4M3 format and per-tensor absmax quantisation, written from the format.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The AMD ROCm summary page (xDiT on Radeon AI PRO R9700S, "what is new" and "tuning
guide") says xDiT runs attention through an FP8 backend (``--attention_backend
aiter_flydsl_fp8``), that the hardware executes FP8 natively, and that FP8 outputs
may differ from BF16 so they must be compared on fixed seeds.  The pages do not fix
the FP8 layout or the scaling; the readings used here:

* E4M3 with no infinities ("fn" variant): 1 sign bit, 4 exponent bits with bias 7,
  3 mantissa bits; exponent field 0 encodes subnormals m/8 * 2^-6; the codes
  S.1111.111 are NaN; the largest finite magnitude is 1.75 * 2^8 = 448.
* Encoding rounds to the nearest representable value, ties to the even code
  (mantissa LSB 0), and saturates magnitudes above 448 to 448 (``satfinite``).
  The sign of zero is kept.
* Per-tensor scale: amax = max |x|; descale = amax / 448 in float32 (descale = 1
  when amax = 0); codes = encode(float32(x) / descale) with an IEEE float32 division.
  The dequantised value is decode(code) * descale.
* Per-block scale (a finer variant of the same scheme, not described by the pages): a
  [B,H,S,D] tensor is cut, per (b, h), into blocks of 128 consecutive rows (tokens), the
  last one ragged; each block is quantised exactly as a tensor of its own, with its own
  descale.  Descales form a float32 [B,H,ceil(S/128)] array.  An all-zero block records
  descale 0 (its codes are those of x / 1, all zero): that tells it apart from a block whose
  maximum is 448, and its dequantised values are zero either way.
"""

from __future__ import annotations

from typing import Tuple

import numpy as np

E4M3_MAX = 448.0


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Value of each E4M3 code (uint8) as float64; NaN codes give NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    sub = (m / 8.0) * 2.0 ** -6
    val = np.where(e == 0, sub, normal)
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


def _positive_table() -> np.ndarray:
    """Values of the finite non-negative codes 0x00..0x7E, increasing with the code."""
    return e4m3_decode(np.arange(0x7F, dtype=np.uint8))


_TABLE = _positive_table()


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Saturating round-to-nearest-even encode of real values (any float dtype, taken
    exactly) to E4M3 codes (uint8)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    a_sat = np.minimum(a, E4M3_MAX)
    hi = np.searchsorted(_TABLE, a_sat, side="left")          # first table value >= a
    hi = np.minimum(hi, len(_TABLE) - 1)
    lo = np.maximum(hi - 1, 0)
    d_hi = _TABLE[hi] - a_sat
    d_lo = a_sat - _TABLE[lo]
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(np.signbit(x), code | np.uint8(0x80), code).astype(np.uint8)
    code = np.where(np.isnan(x), np.uint8(0x7F), code).astype(np.uint8)
    return code


def absmax_descale(x: np.ndarray) -> np.float32:
    """descale = amax / 448 in float32 (1 when the tensor is all zero)."""
    amax = np.float32(np.max(np.abs(np.asarray(x, dtype=np.float32)))) if x.size else np.float32(0)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(amax / np.float32(E4M3_MAX))


def quantize_per_tensor(x: np.ndarray) -> Tuple[np.ndarray, np.float32]:
    """(codes uint8, descale float32) for a tensor of bf16 (or float32) values."""
    x32 = np.asarray(x, dtype=np.float32)
    descale = absmax_descale(x32)
    scaled = (x32 / descale).astype(np.float32)               # IEEE float32 division
    return e4m3_encode(scaled), descale


def dequantize(codes: np.ndarray, descale: float) -> np.ndarray:
    """decode(code) * descale in float64."""
    return e4m3_decode(codes) * float(np.float32(descale))


BLOCK_ROWS = 128


def quantize_per_block(x: np.ndarray, block_rows: int = BLOCK_ROWS) -> Tuple[np.ndarray, np.ndarray]:
    """(codes uint8 [B,H,S,D], descales float32 [B,H,nblk]) for a [B,H,S,D] tensor: every
    run of block_rows rows of one (b, h) is quantised per tensor on its own."""
    x32 = np.asarray(x, dtype=np.float32)
    B, H, S, D = x32.shape
    nblk = (S + block_rows - 1) // block_rows
    codes = np.empty(x32.shape, dtype=np.uint8)
    descales = np.empty((B, H, nblk), dtype=np.float32)
    for b in range(B):
        for h in range(H):
            for i in range(nblk):
                rows = slice(i * block_rows, min(S, (i + 1) * block_rows))
                codes[b, h, rows], descales[b, h, i] = quantize_per_tensor(x32[b, h, rows])
                if not np.any(x32[b, h, rows]):
                    descales[b, h, i] = 0.0
    return codes, descales


def dequantize_per_block(codes: np.ndarray, descales: np.ndarray, block_rows: int = BLOCK_ROWS) -> np.ndarray:
    """decode(code) * descale of the code's block, in float64."""
    S = codes.shape[2]
    per_row = np.repeat(np.asarray(descales, dtype=np.float32).astype(np.float64), block_rows, axis=2)[:, :, :S]
    return e4m3_decode(codes) * per_row[..., None]
