"""CPU oracle of the low-precision state rows -- TEST INFRASTRUCTURE.

The m.163.com article on SDM (section 八, the memory-efficiency paragraph) reports that the
state checkpoints of long-context fine-tuning can be stored as fp8 or int4 without loss.  This
module states, from the formats' definitions, what a checkpoint row holds:

    bf16  one 16-bit code per value: the fp32 value rounded to nearest, ties to even, to
          8 significand bits (no scale);
    e4m3  one 8-bit code per value and one fp32 scale per row, s = amax / 448: the code is
          the OCP FP8 E4M3 value nearest to q = x * (1 / s) (ties to even, saturating at
          +-448); a value that rounds to zero takes the code of +0;
    int4  one 4-bit two's-complement code per value (two per byte, the even element in the
          low nibble) and one fp32 scale per row, s = amax / 7: the code is q = x * (1 / s)
          rounded to nearest, ties to even, clamped to [-7, 7].

amax is the row's largest |x|.  The value coded is q = x * r with r = 1 / s; the scale s,
its reciprocal r, the product q and the decoded value code * s are each one fp32 operation
rounded to nearest.  A scale below the smallest normal fp32, 2^-126 (amax below about
5.3e-36 for E4M3 and 8.2e-38 for int4, or zero), is stored as 0 with all-zero codes, so that r
stays finite.  Those fp32
steps decide the codes, so the oracle takes them in fp32 as the kernels do; everything else
is exact.  Inputs are finite.

Only the test-suite, the smoke check and the benchmark's CPU-baseline leg may import this
module; the product path never does.
"""

from __future__ import annotations

import numpy as np

FORMATS = {"bf16": 1, "e4m3": 2, "int4": 3}
E4M3_MAX = 448.0
INT4_MAX = 7


# ----------------------------------------------------------------------------- E4M3
def e4m3_value(code: int) -> float:
    """The value of an E4M3 code (OCP 8-bit floating point, E4M3: sign, 4 exponent bits with
    bias 7, 3 mantissa bits; no infinities; S.1111.111 is NaN)."""
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * 2.0 ** -6 * (m / 8.0)
    return sign * 2.0 ** (e - 7) * (1.0 + m / 8.0)


# the 127 finite non-negative magnitudes, ascending with their codes 0..126
_E4M3_POS = np.array([e4m3_value(c) for c in range(127)], dtype=np.float64)


def e4m3_encode(x: float) -> int:
    """The E4M3 code nearest to x (ties to the even code), saturating at +-448; the sign of
    x goes to bit 7, except that a zero result is always the code of +0 (0x00)."""
    neg = np.signbit(x)
    a = abs(float(x))
    if a >= E4M3_MAX:
        code = 126
    else:
        i = int(np.searchsorted(_E4M3_POS, a, side="right")) - 1  # _E4M3_POS[i] <= a
        lo, hi = _E4M3_POS[i], _E4M3_POS[i + 1]
        dlo, dhi = a - lo, hi - a  # exact: a and the grid points are doubles on a fine grid
        if dlo < dhi:
            code = i
        elif dhi < dlo:
            code = i + 1
        else:
            code = i if i % 2 == 0 else i + 1
    return code | (0x80 if neg and code != 0 else 0)


# ----------------------------------------------------------------------------- bf16
def bf16_encode(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 codes, round to nearest, ties to even (finite inputs): the upper 16 bits
    of the fp32 pattern after adding half an ulp of the kept part, minus one when the kept
    part is even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    keep_odd = (u >> 16) & 1
    return ((u + 0x7FFF + keep_odd) >> 16).astype(np.uint16)


def bf16_decode(c: np.ndarray) -> np.ndarray:
    return (np.asarray(c, np.uint16).astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------- rows
FLT_MIN = np.float32(2.0 ** -126)


def row_scale(row: np.ndarray, fmt: str) -> np.float32:
    amax = np.float32(np.max(np.abs(row.astype(np.float32)))) if row.size else np.float32(0)
    top = np.float32(E4M3_MAX if fmt == "e4m3" else INT4_MAX)
    s = np.float32(amax / top)
    return s if s >= FLT_MIN else np.float32(0)


def pack(M: np.ndarray, fmt: str):
    """Rows of M [rows, d_v] (fp32) -> (codes, scales).  codes: uint16 [rows, d_v] for bf16,
    uint8 [rows, d_v] for e4m3, uint8 [rows, d_v / 2] for int4; scales: fp32 [rows] (None for
    bf16)."""
    M = np.ascontiguousarray(M, dtype=np.float32)
    rows, d_v = M.shape
    if fmt == "bf16":
        return bf16_encode(M), None
    scales = np.zeros(rows, np.float32)
    if fmt == "e4m3":
        codes = np.zeros((rows, d_v), np.uint8)
    elif fmt == "int4":
        assert d_v % 2 == 0
        codes = np.zeros((rows, d_v // 2), np.uint8)
    else:
        raise ValueError(fmt)
    for r in range(rows):
        s = row_scale(M[r], fmt)
        scales[r] = s
        if s == 0:
            continue
        q = M[r] * np.float32(np.float32(1) / s)  # fp32 reciprocal, fp32 product
        if fmt == "e4m3":
            codes[r] = [e4m3_encode(float(v)) for v in q]
        else:
            k = np.clip(np.rint(q), -INT4_MAX, INT4_MAX).astype(np.int64)  # rint: ties to even
            nib = (k & 0xF).astype(np.uint8)
            codes[r] = nib[0::2] | (nib[1::2] << 4)
    return codes, scales


def unpack(codes: np.ndarray, scales, fmt: str, d_v: int) -> np.ndarray:
    """(codes, scales) -> fp32 rows [rows, d_v]: code value times the row's scale (one fp32
    multiply)."""
    if fmt == "bf16":
        return bf16_decode(codes).reshape(-1, d_v)
    rows = codes.shape[0]
    out = np.zeros((rows, d_v), np.float32)
    for r in range(rows):
        s = np.float32(scales[r])
        if fmt == "e4m3":
            vals = np.array([e4m3_value(int(c)) for c in codes[r]], np.float32)
        else:
            lo = (codes[r] & 0xF).astype(np.int64)
            hi = (codes[r] >> 4).astype(np.int64)
            k = np.empty(d_v, np.int64)
            k[0::2], k[1::2] = lo, hi
            vals = np.where(k >= 8, k - 16, k).astype(np.float32)
        out[r] = vals * s
    return out
