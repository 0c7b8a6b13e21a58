"""Pins of the oracle's MXFP8 quantiser and of the MXFP8 variant of the layer against things
other than themselves.

* Signed E4M3 encode/decode against torch's float8_e4m3fn conversion (a library routine
  that rounds to nearest even): every finite code of both signs, every midpoint between
  neighbours and its FP32 neighbours, random values, and the sign of zero.
* UE8M0 scale decode against ml_dtypes' float8_e8m0fnu (library routine), every code.
* The scale rule against a brute-force search over all exponents (the smallest e with
  amax <= 448 * 2^e), including amax exactly on and one ulp off every boundary.
* Quantisation: each code is the nearest E4M3 of v / 2^e (torch again), values already on
  the grid round-trip exactly, and the error stays within half an E4M3 step.
* The layer with MXFP8 experts: dense evaluation of every expert masked by the routing
  equals the sparse forward, grid-exact operands reduce the expert GEMMs to plain FP64
  matmuls, and a hand-worked two-expert example matches every intermediate written as a
  literal (scales, codes, SwiGLU values, A2 roundings, m, the RMS and the BF16 output).
The FP8 checkpoint is the second variant of the routed experts (vLLM recipe
"reflection/Beam-1.0-501B-A23B", section "Variants"); MXFP8 is the reading of its block
format (E4M3 values, one power-of-two scale per 32 values).
"""

import ml_dtypes
import numpy as np
import torch

import moe_inputs as mi
from oracle import moe, mxfp8 as mx


def _torch_e4m3(vals):
    t = torch.from_numpy(np.asarray(vals, np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def test_signed_e4m3_all_codes_midpoints_and_zero_sign():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    vals = mx.e4m3_decode_signed(codes)
    np.testing.assert_array_equal(vals, ref)
    np.testing.assert_array_equal(np.signbit(vals), np.signbit(ref))
    np.testing.assert_array_equal(mx.e4m3_encode_signed(vals.astype(np.float32)), codes)
    pos = mx.e4m3_decode_signed(np.arange(0x7F, dtype=np.uint8))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    for s in (1.0, -1.0):
        m = (s * mids).astype(np.float32)
        np.testing.assert_array_equal(mx.e4m3_encode_signed(m), _torch_e4m3(m))
        lo = np.nextafter(m, np.float32(0))
        hi = np.nextafter(m, np.float32(s * 1e9))
        np.testing.assert_array_equal(mx.e4m3_encode_signed(lo), _torch_e4m3(lo))
        np.testing.assert_array_equal(mx.e4m3_encode_signed(hi), _torch_e4m3(hi))
    # negative values that round to zero keep the sign bit, like the library conversion
    tiny = np.array([-0.0, -2.0 ** -11, -1e-30, 0.0, 2.0 ** -11], np.float32)
    np.testing.assert_array_equal(mx.e4m3_encode_signed(tiny), _torch_e4m3(tiny))
    assert list(mx.e4m3_encode_signed(tiny)) == [0x80, 0x80, 0x80, 0x00, 0x00]
    rng = np.random.default_rng(3)
    v = (rng.uniform(-448, 448, 100_000) * np.exp(rng.uniform(-12, 0, 100_000))).astype(np.float32)
    np.testing.assert_array_equal(mx.e4m3_encode_signed(v), _torch_e4m3(v))


def test_ue8m0_decode_matches_ml_dtypes():
    codes = np.arange(255, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    np.testing.assert_array_equal(mx.ue8m0_decode(codes), ref)
    assert np.isnan(mx.ue8m0_decode(np.uint8(255)))


def _brute_exponent(a: float) -> int:
    for e in range(-127, 128):
        if a <= 448.0 * 2.0 ** e:
            return e
    raise AssertionError("amax beyond 448 * 2^127")


def test_scale_exponent_brute_force():
    rng = np.random.default_rng(11)
    amax = [0.0, 1e-45, 2.0 ** -149, 2.0 ** -126, 448.0 * 2.0 ** -127, 3.4e38]
    amax += list(np.exp(rng.uniform(np.log(1e-38), np.log(1e38), 3000)).astype(np.float32))
    for e in range(-126, 120, 7):  # every boundary 448 * 2^e, exactly and one FP32 ulp either side
        b = np.float32(448.0 * 2.0 ** e)
        amax += [float(b), float(np.nextafter(b, np.float32(0))), float(np.nextafter(b, np.float32(np.inf)))]
    for m in (1.0, 1.5, 1.75, 1.875, 1.999):  # mantissas around 448's 1.75
        amax += [m * 2.0 ** p for p in range(-20, 20, 3)]
    amax = np.array(amax, np.float32).astype(np.float64)
    got = mx.scale_exponent(amax)
    ref = np.array([_brute_exponent(a) for a in amax])
    np.testing.assert_array_equal(got, ref)


def test_quantize_codes_are_nearest_e4m3_of_scaled_values():
    rng = np.random.default_rng(5)
    v = rng.normal(size=(64, 256)).astype(np.float32)
    v *= np.exp(rng.uniform(-30, 30, size=(64, 1))).astype(np.float32)  # very different row magnitudes
    v[3, 32:64] = 0.0                      # all-zero block
    v[4, 0:32] = 1e-42                     # subnormal block
    v[5, 64:96] = -448.0 * 2.0 ** -3       # exactly on a boundary
    codes, sc = mx.quantize_mxfp8(v)
    assert codes.shape == v.shape and sc.shape == (64, 8)
    e = sc.astype(np.int64) - 127
    blocks = v.reshape(64, 8, 32).astype(np.float64)
    scaled = (blocks / np.ldexp(1.0, e)[..., None]).astype(np.float32)  # exact division by 2^e
    np.testing.assert_array_equal(codes, _torch_e4m3(scaled).reshape(64, 256))
    # scale: amax within range, and the next smaller power of two would not hold it
    amax = np.abs(blocks).max(-1)
    assert np.all(amax <= 448.0 * np.ldexp(1.0, e))
    nz = amax > 448.0 * 2.0 ** -127
    assert np.all(amax[nz] > 448.0 * np.ldexp(1.0, e[nz] - 1))
    assert sc[3, 1] == 0 and np.all(codes[3, 32:64] == 0)
    assert sc[4, 0] == 0
    assert sc[5, 2] == 127 - 3 and np.all(codes[5, 64:96] == 0xFE)  # -448 = sign | 0x7E


def test_quantize_grid_roundtrip_and_error_bound():
    rng = np.random.default_rng(6)
    # on the grid: E4M3 values times 2^e, one element +-448 * 2^e per block -> exact
    codes = rng.integers(0, 256, size=(16, 128)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x10
    codes[:, ::32] = 0x7E
    e = rng.integers(-20, 20, size=(16, 4))
    vals = mx.e4m3_decode_signed(codes).reshape(16, 4, 32) * np.ldexp(1.0, e)[..., None]
    c2, s2 = mx.quantize_mxfp8(vals.reshape(16, 128).astype(np.float32))
    np.testing.assert_array_equal(c2, codes)
    np.testing.assert_array_equal(s2.astype(np.int64) - 127, e)
    np.testing.assert_array_equal(mx.dequantize_mxfp8(c2, s2), vals.reshape(16, 128))
    # error bound: half an E4M3 step at the scaled magnitude (2^-4 relative in the normal
    # range, 2^-10 absolute below 2^-6), times the block scale
    v = rng.normal(size=(32, 512)).astype(np.float32) * np.float32(0.02)
    c, s = mx.quantize_mxfp8(v)
    d = mx.dequantize_mxfp8(c, s)
    X = np.repeat(mx.ue8m0_decode(s), 32, axis=1)
    y = np.abs(v.astype(np.float64)) / X
    step_half = np.where(y >= 2.0 ** -6, np.ldexp(1.0, np.floor(np.log2(np.maximum(y, 2.0 ** -6))).astype(int) - 4),
                         2.0 ** -10)
    assert np.all(np.abs(d - v) <= step_half * X * (1 + 1e-12))


def _tiny_mx(seed=0):
    shape = mi.SHAPES["tiny"]
    xb, rb = mi.tokens(shape, seed)
    x = mi.bf16_bits_to_f32(xb).astype(np.float64)
    res = mi.bf16_bits_to_f32(rb).astype(np.float64)
    wr = mi.router_weight(shape, seed)
    g = mi.bf16_bits_to_f32(mi.gamma(shape, seed)).astype(np.float64)
    cache = moe.ExpertCache(lambda e: mi.expert_weights(shape, seed, e), fmt="mxfp8")
    return shape, x, res, wr, g, cache


def test_mxfp8_brute_force_dense_equals_sparse():
    shape, x, res, wr, g, cache = _tiny_mx()
    r = moe.moe_forward(x, res, wr, g, cache, shape.experts, shape.top_k, None, None)
    wfull = np.zeros((shape.tokens, shape.experts))
    for t in range(shape.tokens):
        for j in range(shape.top_k):
            wfull[t, r["ids"][t, j]] = r["w"][t, j]
    # A1 from the library E4M3 conversion of x / 2^e, e from the brute-force scale search
    xb = x.reshape(shape.tokens, -1, 32)
    e = np.array([[_brute_exponent(a) for a in row] for row in np.abs(xb).max(-1)])
    a1c = _torch_e4m3((xb / np.ldexp(1.0, e)[..., None]).astype(np.float32))
    a1 = (torch.from_numpy(a1c).view(torch.float8_e4m3fn).double().numpy() * np.ldexp(1.0, e)[..., None])
    a1 = a1.reshape(shape.tokens, shape.hidden)
    np.testing.assert_array_equal(r["a1_packed"], a1c.reshape(shape.tokens, shape.hidden))
    m = np.zeros((shape.tokens, shape.hidden))
    for ex in range(shape.experts):
        w_gu, w_d = cache.dequantized(ex)
        gg = a1 @ w_gu[: shape.inter].T
        uu = a1 @ w_gu[shape.inter:].T
        h = (gg * (1.0 / (1.0 + np.exp(-gg))) * uu).astype(np.float32)
        a2c, a2s = mx.quantize_mxfp8(h)
        m += wfull[:, ex:ex + 1] * (mx.dequantize_mxfp8(a2c, a2s) @ w_d.T)
    np.testing.assert_allclose(r["m"], m, rtol=0, atol=1e-12)
    # the routing is format-independent
    r4 = moe.moe_forward(x, res, wr, g, moe.ExpertCache(lambda e: mi.expert_weights(shape, 0, e)), shape.experts,
                         shape.top_k, np.float32(5.0 / 2688), np.float32(3.0 / 2688))
    np.testing.assert_array_equal(r["ids"], r4["ids"])


def test_mxfp8_grid_exact_expert_gemms_equal_fp64_matmul():
    rng = np.random.default_rng(10)
    rows, hidden, inter = 5, 64, 32

    def grid(shape):
        codes = rng.integers(0, 256, size=shape).astype(np.uint8)
        codes[(codes & 0x7F) == 0x7F] = 0x22
        codes[..., ::32] = 0x7E
        e = rng.integers(-12, -4, size=shape[:-1] + (shape[-1] // 32,))
        return (mx.e4m3_decode_signed(codes) * np.repeat(np.ldexp(1.0, e), 32, axis=-1)).astype(np.float32)

    x, w_gu, w_d = grid((rows, hidden)), grid((2 * inter, hidden)), grid((hidden, inter))
    q = moe.quantize_expert(w_gu, w_d, "mxfp8")
    deq = moe.dequantize_expert(q)
    np.testing.assert_array_equal(deq[0], w_gu)
    np.testing.assert_array_equal(deq[1], w_d)
    a1c, a1s = mx.quantize_mxfp8(x)
    r = moe.expert_forward(a1c, a1s, None, deq, None, "mxfp8")
    gg = x.astype(np.float64) @ w_gu[:inter].T.astype(np.float64)
    uu = x.astype(np.float64) @ w_gu[inter:].T.astype(np.float64)
    np.testing.assert_array_equal(r["h32"], (gg / (1 + np.exp(-gg)) * uu).astype(np.float32))
    a2 = mx.dequantize_mxfp8(r["a2_packed"], r["a2_sf"])
    np.testing.assert_allclose(r["y"], a2 @ w_d.T.astype(np.float64), rtol=1e-15, atol=0)


def test_hand_worked_two_expert_example_mxfp8():
    # T = 1, H = I = 32 (one MX block), E = 2, k = 2, residual 0, gamma 1.  x = 2 e0, router
    # rows +-0.5 e0 (logits +-1); expert 0: gate row 0 = up row 0 = e0, down[0, 0] = 1;
    # expert 1: gate row 0 = -e0, up row 0 = e0, down[1, 0] = 1.  Worked by hand:
    #   A1: amax 2 -> e = -7 (2 <= 448 * 2^-7 = 3.5, 2 > 448 * 2^-8), 2 / 2^-7 = 256 exact
    #   weights: amax 1 -> e = -8, 1 / 2^-8 = 256 exact: every operand is exact
    #   h0 = silu(2) * 2 = 4 sigmoid(2) = 3.52318831; e = -6; 3.5232 * 64 = 225.48 -> E4M3 224
    #        (step 16 in [128, 256)) -> 3.5
    #   h1 = silu(-2) * 2 = -4 sigmoid(-2) = -0.47681169; e = -9; * 512 = -244.13 -> -240 -> -0.46875
    #   m = (sigmoid(2) * 3.5, sigmoid(-2) * -0.46875) = (3.08278977, -0.05587637)
    #   rms = sqrt((m0^2 + m1^2) / 32 + 1e-6) = 0.54505582; out = (5.65591575, -0.10251495)
    #   BF16: 5.65625 (181 * 2^-5), -0.1025390625 (-210 * 2^-11)
    H = I = 32
    x = np.zeros((1, H)); x[0, 0] = 2.0
    wr = np.zeros((2, H), np.float32); wr[0, 0] = 0.5; wr[1, 0] = -0.5
    experts = {}
    for e, sign in ((0, 1.0), (1, -1.0)):
        w_gu = np.zeros((2 * I, H), np.float32)
        w_gu[0, 0] = sign
        w_gu[I, 0] = 1.0
        w_d = np.zeros((H, I), np.float32)
        w_d[e, 0] = 1.0
        experts[e] = (w_gu, w_d)
    cache = moe.ExpertCache(lambda e: experts[e], fmt="mxfp8")
    r = moe.moe_forward(x, np.zeros_like(x), wr, np.ones(H), cache, num_experts=2, top_k=2, alpha_a1=None,
                        alpha_a2=None)
    assert r["ids"].tolist() == [[0, 1]]
    np.testing.assert_allclose(r["w"][0], [0.8807970779778823, 0.11920292202211755], rtol=1e-15)
    assert r["a1_sf"][0, 0] == 127 - 7 and r["a1_packed"][0, 0] == 0x78  # 256 = 2^8: E4M3 (15 << 3) | 0
    assert not r["a1_packed"][0, 1:].any()
    q0 = cache.quantized(0)
    assert q0["w_gu_sf"][0, 0] == 127 - 8 and q0["w_gu"][0, 0] == 0x78 and q0["w_gu"][I, 0] == 0x78
    assert q0["w_gu"][0, 1:].sum() == 0 and q0["w_d_sf"][0, 0] == 127 - 8
    h0, h1 = r["h32"][0, 0, 0], r["h32"][0, 1, 0]
    assert abs(h0 - 3.52318831) < 1e-6 and abs(h1 - (-0.47681169)) < 1e-6
    y = r["y"][0]
    assert y[0, 0] == 3.5 and y[1, 1] == -0.46875 and not y[0, 1:].any() and y[1, 0] == 0
    m = r["m"][0]
    assert abs(m[0] - 3.08278977) < 1e-7 and abs(m[1] - (-0.05587637)) < 1e-7 and not m[2:].any()
    assert abs(r["out_pre"][0, 0] - 5.65591575) < 1e-7 and abs(r["out_pre"][0, 1] - (-0.10251495)) < 1e-7
    assert r["out"][0, 0] == 181 * 2.0 ** -5 and r["out"][0, 1] == -210 * 2.0 ** -11
