"""Oracle: OCP FP8 E4M3 rounding and the scaled e4m3 GEMM.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

[TileShare] Tab. S2 and Fig. 4 run the decoder's linear layers in FP8.  The pages
do not state the scaling; the reading taken is one scale per output channel of a
weight (absmax / 448) and one per token of an activation (absmax / 448), values
rounded to nearest-even onto the E4M3 grid and saturated at +-448, the products
accumulated exactly (float64 here) and the result multiplied by both scales.

E4M3 ("E4M3FN" in the OCP 8-bit floating point specification): 1 sign bit, 4
exponent bits with bias 7, 3 mantissa bits; exponent field 0 is subnormal
(value m/8 * 2^-6); no infinities; S.1111.111 is NaN, so the largest finite
magnitude is 1.75 * 2^8 = 448.
"""

import math

import numpy as np

E4M3_MAX = 448.0


def decode_e4m3(code: int) -> float:
    """Value of an 8-bit E4M3 code (NaN for S.1111.111)."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    mnt = code & 0x7
    if e == 0xF and mnt == 0x7:
        return float("nan")
    if e == 0:
        return s * (mnt / 8.0) * 2.0 ** -6
    return s * (1.0 + mnt / 8.0) * 2.0 ** (e - 7)


def round_e4m3_scalar(x: float) -> float:
    """Nearest E4M3 value to x, ties to even, saturating at +-448."""
    if x != x:
        return x
    a = abs(x)
    if a >= E4M3_MAX:
        return math.copysign(E4M3_MAX, x)
    if a < 2.0 ** -6:
        quantum = 2.0 ** -9                      # subnormal spacing
    else:
        _, E = math.frexp(a)                     # a = f * 2^E, f in [0.5, 1)
        quantum = 2.0 ** (E - 1 - 3)             # 3 mantissa bits below the leading one
    q = a / quantum
    lo = math.floor(q)
    rem = q - lo
    if rem > 0.5 or (rem == 0.5 and lo % 2 == 1):
        lo += 1
    return math.copysign(lo * quantum, x)


def round_e4m3(x: np.ndarray) -> np.ndarray:
    """Array form of round_e4m3_scalar (same steps, elementwise, exact in float64)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, E = np.frexp(a)
    quantum = np.where(a < 2.0 ** -6, 2.0 ** -9, np.ldexp(1.0, E - 4))
    q = a / quantum
    lo = np.floor(q)
    rem = q - lo
    up = (rem > 0.5) | ((rem == 0.5) & (np.mod(lo, 2) == 1))
    r = (lo + up) * quantum
    r = np.where(a >= E4M3_MAX, E4M3_MAX, r)
    r = np.where(np.isnan(x), x, np.copysign(r, x))
    return r


def row_scales(x: np.ndarray) -> np.ndarray:
    """Per-row scale absmax / 448 (1 for an all-zero row)."""
    amax = np.abs(x).max(axis=-1)
    return np.where(amax > 0, amax / E4M3_MAX, 1.0)


def quantize_rows(x: np.ndarray):
    """(codes as float64 values on the E4M3 grid, per-row scales)."""
    s = row_scales(x)
    return round_e4m3(x / s[:, None]), s


def scaled_matmul(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """x [n, K] @ w [m, K].T in e4m3: per-token scales of x, per-channel scales of w."""
    qx, sx = quantize_rows(np.asarray(x, np.float64))
    qw, sw = quantize_rows(np.asarray(w, np.float64))
    return (qx @ qw.T) * sx[:, None] * sw[None, :]
