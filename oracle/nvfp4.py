"""NVFP4 quantiser of the oracle (test infrastructure only; see the package docstring).

NVFP4 as used for the routed experts ([P2] "Variants": routed experts quantised to NVFP4,
run W4A4 on Blackwell): a value v is stored as an E2M1 code q, with one unsigned E4M3
scale S per 16 consecutive values along the contraction dimension and one FP32 tensor
scale alpha per tensor, so that v ~= e2m1(q) * e4m3(S) * alpha.

Quantisation rule Q(v, alpha) for one block of 16 FP32 values, every step an IEEE FP32
operation with round-to-nearest-even:
  1. amax = max |v_i|
  2. s = amax / (6 * alpha)                   (6 = largest E2M1 magnitude)
  3. S = E4M3(s), round-to-nearest-even, saturating to 448 (never NaN)
  4. if S == 0 (covers amax == 0): the scale code and all 16 codes are 0
  5. d = S * alpha
  6. q_i = E2M1(v_i / d), round-to-nearest-even, saturating to +-6, sign kept
Tensor scale of a weight tensor: alpha = amax(tensor) / 2688, 2688 = 6 * 448.

The E4M3 and E2M1 roundings below are written from the bit definitions of the formats
(E4M3: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormal step 2^-9,
largest finite 448; E2M1: 1 sign, 2 exponent bits with bias 1, 1 mantissa bit, values
{0, 0.5, 1, 1.5, 2, 3, 4, 6}).  Packing: element 2i in the low nibble, 2i+1 in the high.
"""

from __future__ import annotations

import numpy as np

E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
# Midpoints between consecutive E2M1 magnitudes; midpoint i lies between codes i and i+1.
_E2M1_MIDS = (E2M1_VALUES[:-1] + E2M1_VALUES[1:]) / 2.0
E4M3_MAX = 448.0


def _e4m3_value_table() -> np.ndarray:
    """Value of each of the 128 non-negative E4M3 codes, from the bit layout (0x7F = NaN)."""
    vals = np.empty(128, dtype=np.float64)
    for code in range(128):
        e, m = code >> 3, code & 7
        if e == 0:
            vals[code] = m * 2.0 ** -9
        else:
            vals[code] = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    vals[0x7F] = np.nan
    return vals


_E4M3_TABLE = _e4m3_value_table()


def e4m3_decode(codes) -> np.ndarray:
    """Unsigned E4M3 code (uint8, sign bit must be 0) -> exact value as float64."""
    c = np.asarray(codes, dtype=np.uint8)
    if np.any(c & 0x80):
        raise ValueError("scale codes are unsigned E4M3: sign bit must be clear")
    return _E4M3_TABLE[c]


def e4m3_encode(s) -> np.ndarray:
    """Non-negative finite FP32 -> E4M3 code, round-to-nearest-even, saturating to 448."""
    s = np.asarray(s, dtype=np.float32).astype(np.float64)
    if np.any(~np.isfinite(s)) or np.any(s < 0):
        raise ValueError("e4m3_encode expects finite non-negative input")
    _, ex = np.frexp(s)  # s = f * 2**ex with f in [0.5, 1), so s in [2**(ex-1), 2**ex)
    e = np.maximum(ex - 1, -6)  # exponent of the binade; below 2^-6 the step stays 2^-9
    quantum = np.ldexp(1.0, e - 3)  # 3 mantissa bits
    val = np.rint(s / quantum) * quantum  # np.rint rounds half to even; division is exact
    val = np.minimum(val, E4M3_MAX)  # satfinite: everything past 448 clamps to 448
    code = np.zeros(s.shape, dtype=np.int64)
    sub = val < 2.0 ** -6
    code[sub] = np.rint(val[sub] / 2.0 ** -9).astype(np.int64)
    nrm = ~sub
    if np.any(nrm):
        _, ex2 = np.frexp(val[nrm])
        e2 = ex2 - 1
        mant = val[nrm] / np.ldexp(1.0, e2) - 1.0  # in [0, 1), multiple of 1/8
        code[nrm] = ((e2 + 7) << 3) | np.rint(mant * 8.0).astype(np.int64)
    return code.astype(np.uint8)


def e2m1_encode(v) -> np.ndarray:
    """FP32 -> 4-bit E2M1 code (bit 3 = sign), round-to-nearest-even, saturating to 6.

    The sign bit copies the sign of the input, so -0.0 and small negatives that round to
    zero give code 0x8 (negative zero); +0 and -0 are equal values.
    """
    v = np.asarray(v, dtype=np.float32)
    if np.any(~np.isfinite(v)):
        raise ValueError("e2m1_encode expects finite input")
    a = np.abs(v).astype(np.float64)
    # code = number of midpoints strictly below |v|; at an exact midpoint this rounds
    # down, so move ties whose lower code is odd up to the even neighbour.
    code = np.zeros(a.shape, dtype=np.int64)
    for i, mid in enumerate(_E2M1_MIDS):
        code += a > mid
        if i % 2 == 1:
            code += a == mid
    sign = np.signbit(v).astype(np.int64)
    return (code | (sign << 3)).astype(np.uint8)


def e2m1_decode(codes) -> np.ndarray:
    """4-bit E2M1 code -> exact value as float64."""
    c = np.asarray(codes, dtype=np.uint8)
    mag = E2M1_VALUES[c & 7]
    return np.where(c & 8, -mag, mag)


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[..., 2n] 4-bit codes -> [..., n] bytes; element 2i low nibble, 2i+1 high nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    """Inverse of pack_nibbles."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def tensor_scale(w) -> np.float32:
    """FP32 tensor scale of a weight tensor: fl32(amax / 2688)."""
    amax = np.max(np.abs(np.asarray(w, dtype=np.float32)))
    return np.float32(np.float32(amax) / np.float32(6.0 * E4M3_MAX))


def quantize_nvfp4(v, alpha):
    """Q(v, alpha) along the last axis in blocks of 16.

    v: FP32 array [..., K], K a multiple of 16.  alpha: FP32 tensor scale (> 0).
    Returns (packed codes uint8 [..., K/2], scale codes uint8 [..., K/16]).
    """
    v = np.asarray(v, dtype=np.float32)
    alpha = np.float32(alpha)
    if not alpha > 0:
        raise ValueError("tensor scale must be positive")
    k = v.shape[-1]
    if k % 16:
        raise ValueError("last dimension must be a multiple of 16")
    blocks = v.reshape(v.shape[:-1] + (k // 16, 16))
    amax = np.max(np.abs(blocks), axis=-1)  # FP32, exact
    six_alpha = np.float32(np.float32(6.0) * alpha)  # fl32(6 * alpha)
    s = (amax / six_alpha).astype(np.float32)  # IEEE FP32 division
    scode = e4m3_encode(s)
    S = e4m3_decode(scode).astype(np.float32)  # exact
    d = (S * alpha).astype(np.float32)  # fl32(S * alpha)
    zero = scode == 0
    d_safe = np.where(zero, np.float32(1.0), d).astype(np.float32)
    q = (blocks / d_safe[..., None]).astype(np.float32)  # IEEE FP32 division
    codes = e2m1_encode(q)
    codes[zero] = 0
    codes = codes.reshape(v.shape)
    return pack_nibbles(codes), scode


def dequantize_nvfp4(packed, scodes, alpha) -> np.ndarray:
    """Exact FP64 value of NVFP4 data: e2m1(q) * e4m3(S) * alpha."""
    codes = unpack_nibbles(packed)
    vals = e2m1_decode(codes)
    k = vals.shape[-1]
    scale = e4m3_decode(scodes) * np.float64(np.float32(alpha))
    vals = vals.reshape(vals.shape[:-1] + (k // 16, 16)) * scale[..., None]
    return vals.reshape(codes.shape)
