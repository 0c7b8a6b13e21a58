"""MXFP8 quantiser of the oracle (test infrastructure only; see the package docstring).

The second precision variant of the routed experts: the pages list an FP8 checkpoint next
to the NVFP4 one ([P2] "Variants"; served with FP8 MoE kernels, [P2] "Launching the
server", "FP8 with TP8 on H200 or Blackwell").  They do not say how the FP8 values are
scaled.  Reading taken here: block-scaled W8A8 in the OCP Microscaling format MXFP8 --
E4M3 elements with one shared power-of-two scale per 32 consecutive values along the
contraction dimension, the scale stored as UE8M0 (an 8-bit biased exponent, bias 127, no
sign and no mantissa), for weights and activations alike, and no tensor scale.

Scale rule (reading; the MX format fixes the encoding, not how a scale is chosen): the
scale of a block is X = 2^e with e the smallest integer such that amax <= 448 * 2^e, so
that the block's largest magnitude maps inside E4M3's finite range and no value
saturates.  e is clamped to [-127, 127]; amax == 0 (and any amax below 448 * 2^-127)
gives e = -127, scale code 0.
Element rule: q_i = E4M3(v_i / X), round-to-nearest-even, sign kept (v_i / X is exact:
a division by a power of two).
Value: v ~= e4m3(q_i) * 2^(S - 127) for scale code S.

Steps are written from the format definitions; E4M3 rounding reuses this oracle's own
E4M3 encoder (non-negative magnitudes) with the sign bit added.
"""

from __future__ import annotations

import numpy as np

from .nvfp4 import E4M3_MAX, _E4M3_TABLE, e4m3_encode

MX_BLOCK = 32
UE8M0_BIAS = 127


def e4m3_encode_signed(v) -> np.ndarray:
    """FP32 -> signed E4M3 code (bit 7 = sign), round-to-nearest-even, saturating to 448.

    The sign bit copies the sign of the input: -0.0 and negatives that round to zero give
    code 0x80 (negative zero)."""
    v = np.asarray(v, dtype=np.float32)
    if np.any(~np.isfinite(v)):
        raise ValueError("e4m3_encode_signed expects finite input")
    mag = e4m3_encode(np.abs(v))
    return (mag | (np.signbit(v).astype(np.uint8) << 7)).astype(np.uint8)


def e4m3_decode_signed(codes) -> np.ndarray:
    """Signed E4M3 code -> exact value as float64 (codes 0x7F / 0xFF are NaN)."""
    c = np.asarray(codes, dtype=np.uint8)
    mag = _E4M3_TABLE[c & 0x7F]
    return np.where(c & 0x80, -mag, mag)


def scale_exponent(amax) -> np.ndarray:
    """e = smallest integer with amax <= 448 * 2^e, clamped to [-127, 127] (int64).

    amax: non-negative finite values.  From amax = f * 2^p with f in [0.5, 1):
    448 * 2^e = 0.875 * 2^(e + 9), so e = p - 9 when f <= 0.875, else p - 8."""
    a = np.asarray(amax, dtype=np.float64)
    if np.any(~np.isfinite(a)) or np.any(a < 0):
        raise ValueError("scale_exponent expects finite non-negative amax")
    f, p = np.frexp(a)
    e = np.where(f <= 0.875, p - 9, p - 8).astype(np.int64)
    e = np.where(a == 0, -UE8M0_BIAS, e)
    return np.clip(e, -UE8M0_BIAS, UE8M0_BIAS)


def ue8m0_decode(scodes) -> np.ndarray:
    """UE8M0 scale code -> 2^(code - 127) as float64 (code 255 is NaN)."""
    s = np.asarray(scodes, dtype=np.int64)
    out = np.ldexp(1.0, s - UE8M0_BIAS)
    return np.where(s == 255, np.nan, out)


def quantize_mxfp8(v):
    """MXFP8 of v along the last axis in blocks of 32.

    v: FP32 array [..., K], K a multiple of 32.
    Returns (codes uint8 [..., K] signed E4M3, scale codes uint8 [..., K/32] UE8M0)."""
    v = np.asarray(v, dtype=np.float32)
    k = v.shape[-1]
    if k % MX_BLOCK:
        raise ValueError("last dimension must be a multiple of 32")
    blocks = v.reshape(v.shape[:-1] + (k // MX_BLOCK, MX_BLOCK)).astype(np.float64)
    amax = np.max(np.abs(blocks), axis=-1)
    e = scale_exponent(amax)
    scaled = np.ldexp(blocks, -e[..., None])  # exact: multiplication by a power of two
    if np.any(np.abs(scaled) > E4M3_MAX):
        raise AssertionError("scale rule violated: a scaled value exceeds 448")
    # v / X is exactly representable in FP32 unless it falls below 2^-126, far under half
    # of E4M3's smallest step, where both it and its FP32 rounding encode to zero.
    codes = e4m3_encode_signed(scaled.astype(np.float32))
    return codes.reshape(v.shape), (e + UE8M0_BIAS).astype(np.uint8)


def dequantize_mxfp8(codes, scodes) -> np.ndarray:
    """Exact FP64 value of MXFP8 data: e4m3(q) * 2^(S - 127)."""
    vals = e4m3_decode_signed(codes)
    k = vals.shape[-1]
    scale = ue8m0_decode(scodes)
    vals = vals.reshape(vals.shape[:-1] + (k // MX_BLOCK, MX_BLOCK)) * scale[..., None]
    return vals.reshape(np.shape(codes))
