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


def test_e2m1_e4m3_conversion_sweep(bm):
    # 2^24 values per call spread over every block scale and every E2M1 interval: the
    # hardware conversions (cvt.rn.satfinite e2m1x2 / e4m3x2) against the oracle rounding.
    rng = np.random.default_rng(2024)
    for _ in range(2):
        n = 1 << 24
        mag = np.exp(rng.uniform(np.log(1e-3), np.log(5e3), n // 16)).astype(np.float32)
        v = (rng.uniform(-1, 1, (n // 16, 16)) * mag[:, None]).astype(np.float32)
        alpha = np.float32(0.37)
        codes, sf, _ = _gpu_q(bm, v, float(alpha))
        rc, rs = nvfp4.quantize_nvfp4(v, alpha)
        np.testing.assert_array_equal(sf, rs)
        np.testing.assert_array_equal(_norm(codes), _norm(rc))
