"""GPU NVFP4 quantiser (beam_moe_quantize_nvfp4) against the oracle quantiser, bit for bit.

NVFP4 routed experts, W4A4 on Blackwell (recipe "reflection/Beam-1.0-501B-A23B",
section "Variants").  Codes are compared with +0 and -0 identified (equal values)."""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

from oracle import nvfp4  # noqa: E402


@pytest.fixture(scope="module")
def bm():
    import sparse_moe_layer_fp32_b200 as m
    return m


def _gpu_q(bm, v, alpha=None):
    codes, sf, a = bm.beam_moe_quantize_nvfp4(torch.from_numpy(v).cuda(), alpha)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), sf.cpu().numpy(), a.cpu().numpy()[0]


def _norm(p):
    c = nvfp4.unpack_nibbles(p)
    c[c == 8] = 0
    return c


@pytest.mark.parametrize("rows,cols,scale", [(1, 16, 1.0), (7, 48, 0.02), (64, 5120, 0.02), (300, 1536, 3.0)])
def test_quantize_matches_oracle_given_alpha(bm, rows, cols, scale):
    rng = np.random.default_rng(rows * 7 + cols)
    v = (rng.standard_normal((rows, cols)) * scale).astype(np.float32)
    alpha = np.float32(np.abs(v).max() / 2688.0)
    codes, sf, a = _gpu_q(bm, v, float(alpha))
    rc, rs = nvfp4.quantize_nvfp4(v, alpha)
    assert a == alpha
    np.testing.assert_array_equal(sf, rs)
    np.testing.assert_array_equal(_norm(codes), _norm(rc))


def test_quantize_tensor_scale_on_device(bm):
    rng = np.random.default_rng(1)
    v = (rng.standard_normal((3072, 640)) * 0.02).astype(np.float32)
    codes, sf, a = _gpu_q(bm, v, None)
    assert a == nvfp4.tensor_scale(v)
    rc, rs = nvfp4.quantize_nvfp4(v, a)
    np.testing.assert_array_equal(sf, rs)
    np.testing.assert_array_equal(_norm(codes), _norm(rc))


def test_quantize_edge_blocks(bm):
    # zero block, underflowing block, saturating block, exact E2M1 midpoints, +-0, huge range
    blocks = [np.zeros(16), np.full(16, 1e-9), np.linspace(-1e4, 1e4, 16),
              np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 2) * np.repeat([1, -1], 8),
              np.array([-0.0] * 15 + [1.0]), np.array([6.0, 1e-30] + [3.0] * 14)]
    v = np.stack(blocks).astype(np.float32)
    for alpha in (1.0, 1.0 / 448, 1e-4, 3.7):
        codes, sf, _ = _gpu_q(bm, v, alpha)
        rc, rs = nvfp4.quantize_nvfp4(v, np.float32(alpha))
        np.testing.assert_array_equal(sf, rs)
        np.testing.assert_array_equal(_norm(codes), _norm(rc))


def test_quotients_near_every_e2m1_midpoint(bm):
    # v / d within a few ulp of each E2M1 rounding midpoint (and exactly on it where fl32
    # allows), for many block scales d: the quotients whose code depends on the last bit of
    # the IEEE quotient.
    rng = np.random.default_rng(77)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    rows = []
    for alpha in (np.float32(1.0), np.float32(0.37), np.float32(1e-3), np.float32(3.1e-5)):
        for sc in rng.choice(np.arange(8, 127), 12, replace=False):
            d = np.float32(nvfp4.e4m3_decode(np.uint8(sc)) * alpha)
            for m in mids:
                base = np.float32(m * d)
                cand = [base, np.nextafter(base, np.float32(0)), np.nextafter(base, np.float32(np.inf))]
                cand += [np.nextafter(cand[1], np.float32(0)), np.nextafter(cand[2], np.float32(np.inf))]
                row = np.zeros(16, np.float32)
                row[0] = np.float32(6.0 * d)  # amax: the block's scale code is sc again
                row[1:6] = cand
                row[6:11] = -np.array(cand, np.float32)
                row[11:] = rng.uniform(-6, 6, 5).astype(np.float32) * d
                rows.append((row, alpha))
    for alpha in sorted({a for _, a in rows}):
        v = np.stack([r for r, a in rows if a == alpha])
        codes, sf, _ = _gpu_q(bm, v, float(alpha))
        rc, rs = nvfp4.quantize_nvfp4(v, alpha)
        np.testing.assert_array_equal(sf, rs)
        np.testing.assert_array_equal(_norm(codes), _norm(rc))


def test_e2m1_e4m3_conversion_sweep(bm):
    # 7 x 2^24 (1.17e8) values spread over every block scale and every E2M1 interval: the
    # hardware conversions (cvt.rn.satfinite e2m1x2 / e4m3x2) and the quotient rounding
    # against the oracle rounding.
    rng = np.random.default_rng(2024)
    for _ in range(7):
        n = 1 << 24
        mag = np.exp(rng.uniform(np.log(1e-3), np.log(5e3), n // 16)).astype(np.float32)
        v = (rng.uniform(-1, 1, (n // 16, 16)) * mag[:, None]).astype(np.float32)
        alpha = np.float32(0.37)
        codes, sf, _ = _gpu_q(bm, v, float(alpha))
        rc, rs = nvfp4.quantize_nvfp4(v, alpha)
        np.testing.assert_array_equal(sf, rs)
        np.testing.assert_array_equal(_norm(codes), _norm(rc))


# ---------------------------------------------------------------- MXFP8 (beam_moe_quantize_mxfp8)
# The block-scaled FP8 variant of the experts (the recipe's FP8 checkpoint, read as MXFP8:
# E4M3 codes, one UE8M0 scale per 32 values).  Codes are compared bit for bit, the sign of
# zero included: both sides keep the input's sign.
def _gpu_mx(bm, v):
    codes, sf = bm.beam_moe_quantize_mxfp8(torch.from_numpy(v).cuda())
    torch.cuda.synchronize()
    return codes.cpu().numpy(), sf.cpu().numpy()


@pytest.mark.parametrize("rows,cols,scale", [(1, 32, 1.0), (7, 96, 0.02), (64, 5120, 0.02), (300, 1536, 3e5)])
def test_quantize_mxfp8_matches_oracle(bm, rows, cols, scale):
    from oracle import mxfp8
    rng = np.random.default_rng(rows * 11 + cols)
    v = (rng.standard_normal((rows, cols)) * scale).astype(np.float32)
    codes, sf = _gpu_mx(bm, v)
    rc, rs = mxfp8.quantize_mxfp8(v)
    np.testing.assert_array_equal(sf, rs)
    np.testing.assert_array_equal(codes, rc)


def test_quantize_mxfp8_edge_blocks(bm):
    from oracle import mxfp8
    e4 = mxfp8.e4m3_decode_signed(np.arange(0x7F, dtype=np.uint8))
    mids = (e4[:-1] + e4[1:]) / 2
    blocks = [np.zeros(32),                                   # amax 0 -> scale code 0
              np.full(32, 1e-42),                             # subnormal amax
              np.linspace(-3e38, 3e38, 32),                   # largest exponents
              np.array([448.0] + [-0.0] * 31) * 2.0 ** -20,   # exactly on a scale boundary, -0
              np.array([np.nextafter(np.float32(448.0), np.float32(1e9))] + [1.0] * 31),  # one ulp above
              np.concatenate([mids[-32:-1], [448.0]]),        # E4M3 midpoints with scale 2^0: ties to even
              np.concatenate([-mids[40:71], [-448.0]]) * 2.0 ** 7,
              np.array([1.0, -1e-30] * 16)]                   # negatives that round to zero
    v = np.stack(blocks).astype(np.float32)
    codes, sf = _gpu_mx(bm, v)
    rc, rs = mxfp8.quantize_mxfp8(v)
    np.testing.assert_array_equal(sf, rs)
    np.testing.assert_array_equal(codes, rc)
    assert sf[0, 0] == 0 and sf[3, 0] == 127 - 20 and sf[5, 0] == 127
    with pytest.raises(bm.BeamMoeError):
        bm.beam_moe_quantize_mxfp8(torch.zeros((2, 48), device="cuda"))


def test_hardware_conversions_swept_against_the_oracle_rounding(bm):
    # The quantisers expose the raw conversions when the block scale is one: an MXFP8 block
    # holding 448 (the E4M3 maximum) has scale 2^0, so its codes are E4M3(v); an NVFP4 block
    # with amax 6 and alpha 1 has d = E4M3(6 / 6) = 1, so its codes are E2M1(v).  Every code,
    # every midpoint between neighbours and the FP32 neighbours of each midpoint, both signs.
    from oracle import mxfp8
    e4 = mxfp8.e4m3_decode_signed(np.arange(0x7F, dtype=np.uint8))
    mids = ((e4[:-1] + e4[1:]) / 2).astype(np.float32)
    pos = np.concatenate([e4.astype(np.float32), mids, np.nextafter(mids, np.float32(0)),
                          np.nextafter(mids, np.float32(1e9))])
    vals = np.concatenate([pos, -pos]).astype(np.float32)
    n = (len(vals) + 30) // 31
    v = np.zeros((n, 32), np.float32)
    v[:, 0] = 448.0  # fixes the scale at 2^0
    v[:, 1:].reshape(-1)[: len(vals)] = vals
    codes, sf = _gpu_mx(bm, v)
    assert np.all(sf == 127)
    np.testing.assert_array_equal(codes, mxfp8.e4m3_encode_signed(v))
    # E2M1 through NVFP4 with d = 1
    e2 = nvfp4.E2M1_VALUES.astype(np.float32)
    m2 = ((e2[:-1] + e2[1:]) / 2).astype(np.float32)
    p2 = np.concatenate([e2, m2, np.nextafter(m2, np.float32(0)), np.nextafter(m2, np.float32(10))])
    vals2 = np.concatenate([p2, -p2]).astype(np.float32)
    n2 = (len(vals2) + 14) // 15
    w = np.zeros((n2, 16), np.float32)
    w[:, 0] = 6.0  # amax 6 with alpha 1: scale E4M3(1) = 1, d = 1
    w[:, 1:].reshape(-1)[: len(vals2)] = vals2
    c2, s2, a = _gpu_q(bm, w, 1.0)
    assert a == 1.0 and np.all(nvfp4.e4m3_decode(s2) == 1.0)
    np.testing.assert_array_equal(_norm(c2), _norm(nvfp4.quantize_nvfp4(w, np.float32(1.0))[0]))
    np.testing.assert_array_equal(_norm(c2).reshape(n2, 16), np.where(nvfp4.e2m1_encode(w) == 8, 0,
                                                                      nvfp4.e2m1_encode(w)))
