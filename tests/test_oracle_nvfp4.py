"""Pins of the oracle's NVFP4 quantiser against things other than itself.

* E4M3 decode/encode against torch's float8_e4m3fn conversion (a library routine that
  rounds to nearest even), exhaustively over every finite code, every midpoint between
  neighbouring codes and random values; saturation against the format's definition.
* E2M1 encode against ml_dtypes' float4_e2m1fn conversion (library routine), over the
  grid, the midpoints, their FP32 neighbours and random values.
* Q(v, alpha) against its defining properties: the scale is the nearest E4M3 of
  amax / (6 alpha), each code is the nearest E2M1 of v / d, inputs already on the grid
  round-trip exactly, and the zero / underflow / saturation special cases.
NVFP4 as used here: routed experts quantised to NVFP4, W4A4 on Blackwell (vLLM recipe
"reflection/Beam-1.0-501B-A23B", section "Variants").
"""

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import nvfp4 as q


def _torch_e4m3(vals):
    t = torch.from_numpy(np.asarray(vals, np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def test_e4m3_decode_table_matches_torch():
    codes = np.arange(0x7F, dtype=np.uint8)  # all non-negative finite codes
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(q.e4m3_decode(codes), ref)
    assert q.e4m3_decode(np.uint8(0x7E)) == 448.0
    assert q.e4m3_decode(np.uint8(0x01)) == 2.0 ** -9


def test_e4m3_encode_exhaustive_codes_and_midpoints():
    vals = q.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    np.testing.assert_array_equal(q.e4m3_encode(vals.astype(np.float32)), np.arange(0x7F, dtype=np.uint8))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)  # exact in FP32
    assert np.all(mids.astype(np.float64) == (vals[:-1] + vals[1:]) / 2)
    got = q.e4m3_encode(mids)
    np.testing.assert_array_equal(got, _torch_e4m3(mids))
    # ties go to the even code
    assert np.all(got % 2 == 0)
    below = np.nextafter(mids, np.float32(0))
    above = np.nextafter(mids, np.float32(1e9))
    np.testing.assert_array_equal(q.e4m3_encode(below), _torch_e4m3(below))
    np.testing.assert_array_equal(q.e4m3_encode(above), _torch_e4m3(above))


def test_e4m3_encode_random_and_saturation():
    rng = np.random.default_rng(7)
    v = np.concatenate([
        rng.uniform(0, 448, 200_000),
        np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448.0), 200_000)),
    ]).astype(np.float32)
    np.testing.assert_array_equal(q.e4m3_encode(v), _torch_e4m3(v))
    # satfinite: everything at or above 448 maps to the largest finite code, never NaN
    big = np.array([448.0, 450.0, 463.9, 464.0, 480.0, 1e6, 3e38], np.float32)
    assert np.all(q.e4m3_encode(big) == 0x7E)
    # underflow: below half the smallest subnormal rounds to zero; exactly half ties to 0
    assert q.e4m3_encode(np.float32(2.0 ** -10)) == 0
    assert q.e4m3_encode(np.float32(2.0 ** -10 * 1.0001)) == 1


def _ml_e2m1(vals):
    return np.asarray(vals, np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF


def test_e2m1_encode_against_ml_dtypes():
    grid = q.E2M1_VALUES.astype(np.float32)
    mids = ((q.E2M1_VALUES[:-1] + q.E2M1_VALUES[1:]) / 2).astype(np.float32)
    pts = np.concatenate([grid, mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(9)),
                          [6.5, 7.0, 7.5, 8.0, 100.0, 3e38]]).astype(np.float32)
    pts = np.concatenate([pts, -pts])
    rng = np.random.default_rng(3)
    pts = np.concatenate([pts, rng.uniform(-8, 8, 500_000).astype(np.float32)])
    np.testing.assert_array_equal(q.e2m1_encode(pts), _ml_e2m1(pts))
    # the tie list of the format: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    np.testing.assert_array_equal(q.e2m1_decode(q.e2m1_encode(ties)), [0, 1, 1, 2, 2, 4, 4])
    # sign kept, +-0 equal in value
    assert q.e2m1_encode(np.float32(-0.0)) == 8 and q.e2m1_decode(np.uint8(8)) == 0.0


def test_pack_nibbles_order():
    codes = np.array([[1, 2, 3, 4]], np.uint8)
    packed = q.pack_nibbles(codes)
    assert packed.tolist() == [[0x21, 0x43]]  # element 2i low nibble, 2i+1 high nibble
    np.testing.assert_array_equal(q.unpack_nibbles(packed), codes)


def test_quantize_nearest_properties():
    rng = np.random.default_rng(11)
    v = (rng.standard_normal((64, 256)) * rng.uniform(0.01, 10, (64, 1))).astype(np.float32)
    alpha = np.float32(0.05)
    packed, sf = q.quantize_nvfp4(v, alpha)
    codes = q.unpack_nibbles(packed).reshape(64, 16, 16)
    blocks = v.reshape(64, 16, 16)
    amax = np.abs(blocks).max(-1).astype(np.float64)
    s = np.float32(amax / np.float64(np.float32(6 * alpha)))
    table = q.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    # the scale is a nearest finite E4M3 value of s (s < 448 here)
    assert np.all(s < 448)
    dist = np.abs(table[None, None, :] - s.astype(np.float64)[..., None])
    chosen = q.e4m3_decode(sf)
    assert np.all(np.abs(chosen - s) <= dist.min(-1) + 0.0)
    # each code is a nearest E2M1 value of v / d (saturating at 6)
    d = (chosen.astype(np.float32) * alpha).astype(np.float32)
    r = (blocks / d[..., None]).astype(np.float64)
    val = q.e2m1_decode(codes)
    cand = np.concatenate([q.E2M1_VALUES, -q.E2M1_VALUES])
    best = np.abs(cand[None, None, None, :] - np.clip(r, -6, 6)[..., None]).min(-1)
    assert np.all(np.abs(val - np.clip(r, -6, 6)) <= best)


def test_quantize_grid_exact_roundtrip():
    rng = np.random.default_rng(5)
    alpha = np.float32(2.0 ** -7)
    # per block: a random scale code; values = e2m1 grid * S * alpha with one element at 6*S*alpha
    sc = rng.integers(8, 0x77, size=(32, 8)).astype(np.uint8)
    S = q.e4m3_decode(sc)
    codes = rng.integers(0, 16, size=(32, 8, 16)).astype(np.uint8)
    codes[..., 0] = 7  # +6 fixes amax = 6 * S * alpha, so s == S exactly
    v = (q.e2m1_decode(codes) * S[..., None] * float(alpha)).astype(np.float32).reshape(32, 128)
    packed, sf = q.quantize_nvfp4(v, alpha)
    np.testing.assert_array_equal(sf, sc)
    back = q.dequantize_nvfp4(packed, sf, alpha)
    np.testing.assert_array_equal(back, v.astype(np.float64))


def test_quantize_special_cases():
    z = np.zeros((2, 32), np.float32)
    packed, sf = q.quantize_nvfp4(z, np.float32(1.0))
    assert not packed.any() and not sf.any()
    # a block whose scale underflows to zero is all zero codes
    tiny = np.full((1, 16), 1e-6, np.float32)
    packed, sf = q.quantize_nvfp4(tiny, np.float32(1.0))  # s = 1.7e-7 -> E4M3 0
    assert sf[0, 0] == 0 and not packed.any()
    # a tensor scale that is too small saturates the block scale at 448, codes at +-6
    big = np.linspace(-10, 10, 16, dtype=np.float32)[None]
    packed, sf = q.quantize_nvfp4(big, np.float32(1e-4))
    assert sf[0, 0] == 0x7E
    codes = q.unpack_nibbles(packed)
    assert (codes[0, 0] == 0xF) and (codes[0, -1] == 0x7)
    # tensor scale of a weight: fl32(amax / 2688)
    w = np.array([[0.5, -2.0], [1.0, 0.25]], np.float32)
    assert q.tensor_scale(w) == np.float32(np.float32(2.0) / np.float32(2688.0))
