"""Pins of the C++ FP64 oracle (oracle/moe_oracle.cpp), the plain CPU statement of the layer,
against things other than itself, and its agreement with the numpy oracle (an independent
statement of the same steps: different rounding method, different loop structure).

* E4M3 and E2M1 encoders against the library conversions (torch float8_e4m3fn, ml_dtypes
  float4_e2m1fn): every code, every midpoint and its FP32 neighbours, random values;
  saturation and the sign of zero by definition.
* The hand-worked two-expert example (no page prints one): routing weights sigmoid(+-2),
  x quantised to 2.0625, m = (3.302989, -0.0558764), RMS 0.825866, out (4.0, -139 2^-11).
* BF16 rounding against torch.
* Routing invariants and special cases (zero router -> experts 0..k-1 at 1/k; k = E -> the
  full softmax), and the permutation's invariants.
* Quantisers, routing, permutation and the whole forward bit-exact / within 1e-12 of the
  numpy oracle on seeded tiny and mid-size layers, NVFP4 and MXFP8 experts.
Routing 8 of 256 experts and NVFP4 / FP8 experts: vLLM recipe "reflection/Beam-1.0-501B-A23B",
sections "Overview" and "Variants"; finalize and sandwich norm: vLLM PR "Day-0 support for
Reflection's Beam-1.0", section "Status".
"""

import dataclasses

import ml_dtypes
import numpy as np
import pytest
import torch

import moe_inputs as mi
from oracle import cpp, moe, mxfp8, nvfp4


@pytest.fixture(scope="module")
def L():
    return cpp.lib()


def _fp32_neighbours(v):
    v = np.asarray(v, np.float32)
    return np.concatenate([v, np.nextafter(v, np.float32(np.inf)), np.nextafter(v, np.float32(0))])


# ------------------------------------------------------------------ number formats
def test_e4m3_encoder_matches_torch(L):
    vals = np.array([L.orc_e4m3_decode(c) for c in range(127)])
    assert vals[0] == 0 and vals[1] == 2.0 ** -9 and vals[8] == 2.0 ** -6 and vals[126] == 448.0
    assert np.all(np.diff(vals) > 0)
    mids = (vals[:-1] + vals[1:]) / 2
    rng = np.random.default_rng(1)
    probe = np.concatenate([_fp32_neighbours(vals), _fp32_neighbours(mids),
                            rng.uniform(0, 448, 200_000).astype(np.float32),
                            np.exp2(rng.uniform(-12, 8.8, 200_000)).astype(np.float32)])
    probe = probe[(probe >= 0) & (probe <= 448)]
    ref = torch.from_numpy(probe).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([L.orc_e4m3_encode(float(p)) for p in probe], np.uint8)
    np.testing.assert_array_equal(got, ref)
    # saturating: anything past 448 is 448 (code 0x7E), never NaN
    for s in (448.0001, 464.0, 480.0, 1e6, 3.0e38):
        assert L.orc_e4m3_encode(s) == 0x7E


def test_e2m1_encoder_matches_ml_dtypes(L):
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    mids = (mags[:-1] + mags[1:]) / 2
    rng = np.random.default_rng(2)
    probe = np.concatenate([_fp32_neighbours(mags), _fp32_neighbours(mids), rng.uniform(-6, 6, 100_000)])
    probe = np.concatenate([probe, -probe]).astype(np.float32)
    ref = probe.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    got = np.array([L.orc_e2m1_encode(float(p)) for p in probe], np.uint8)
    np.testing.assert_array_equal(got & 7, ref & 7)  # magnitudes
    rounds_to_nonzero = (got & 7) != 0  # there the sign must agree too
    np.testing.assert_array_equal(got[rounds_to_nonzero], ref[rounds_to_nonzero])
    np.testing.assert_array_equal(got >> 3, np.signbit(probe).astype(np.uint8))  # sign of the input, zero too
    # saturating to 6, sign kept for values that round to zero
    assert L.orc_e2m1_encode(7.5) == 7 and L.orc_e2m1_encode(-100.0) == 15
    assert L.orc_e2m1_encode(-0.1) == 8 and L.orc_e2m1_encode(0.25) == 0 and L.orc_e2m1_encode(0.75) == 2


def test_bf16_rounding_matches_torch(L):
    rng = np.random.default_rng(3)
    z = np.concatenate([rng.standard_normal(20_000) * 10.0 ** rng.integers(-6, 6, 20_000),
                        np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8)])])
    got = np.array([L.orc_bf16_round(float(v)) for v in z])
    # torch rounds FP32 -> BF16; feed it values that are exact in FP32 so no double rounding
    z32 = z.astype(np.float32).astype(np.float64)
    got32 = np.array([L.orc_bf16_round(float(v)) for v in z32])
    ref = torch.from_numpy(z32.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(got32, ref)
    assert got[-3] == 1.0 and got[-2] == 1 + 2.0 ** -6 and got[-1] == -1.0  # ties to even


# ------------------------------------------------------------------ hand-worked example
def test_hand_worked_two_expert_example():
    H = I = 16
    x = np.zeros((1, H), np.float32)
    x[0, 0] = 2.0
    wr = np.zeros((2, H), np.float32)
    wr[0, 0], wr[1, 0] = 0.5, -0.5
    experts = {}
    for e, sign in ((0, 1.0), (1, -1.0)):
        w_gu = np.zeros((2 * I, H), np.float32)
        w_gu[0, 0], w_gu[I, 0] = sign, 1.0
        w_d = np.zeros((H, I), np.float32)
        w_d[e, 0] = 1.0
        experts[e] = (w_gu, w_d)
    bits = mi.f32_to_bf16_bits
    r = cpp.moe_forward(bits(x), bits(np.zeros_like(x)), wr, bits(np.ones(H, np.float32)), lambda e: experts[e],
                        top_k=2, inter=I, alpha_a1=1.0, alpha_a2=1.0)
    assert r["ids"].tolist() == [[0, 1]]
    np.testing.assert_allclose(r["w"][0], [0.8807970779778823, 0.11920292202211755], rtol=1e-15)
    m = r["m"][0]
    assert abs(m[0] - 3.302989) < 2e-6 and abs(m[1] - (-0.0558764)) < 2e-7 and not m[2:].any()
    assert abs(np.sqrt((m[0] ** 2 + m[1] ** 2) / 16 + 1e-6) - 0.825866) < 2e-6
    assert abs(r["out_pre"][0, 0] - 3.999425) < 3e-6 and abs(r["out_pre"][0, 1] - (-0.0676579)) < 3e-7
    out = mi.bf16_bits_to_f32(r["out_bf16"])[0]
    assert out[0] == 4.0 and out[1] == -139 * 2.0 ** -11 and not out[2:].any()
    # the quantised x of the example: scale 0.34375, x0 -> 6 * 0.34375 = 2.0625
    p, s = cpp.quantize_nvfp4(x, 1.0)
    assert nvfp4.e4m3_decode(s[0, 0]) == 0.34375 and (p[0, 0] & 15) == 7


# ------------------------------------------------------------------ routing
def test_routing_special_cases_and_invariants():
    rng = np.random.default_rng(4)
    x = mi.f32_to_bf16_bits(rng.standard_normal((5, 64)).astype(np.float32))
    _, ids, w, _ = cpp.route(x, np.zeros((16, 64), np.float32), 4)  # all logits equal
    assert (ids == np.arange(4)).all() and np.allclose(w, 0.25, rtol=0, atol=1e-15)
    wr = (rng.standard_normal((16, 64)) / 8).astype(np.float32)
    logits, ids, w, _ = cpp.route(x, wr, 16)  # k = E: the full softmax
    p = np.exp(logits - logits.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    np.testing.assert_allclose(np.take_along_axis(p, ids.astype(np.int64), 1), w, rtol=1e-14)
    assert np.all(np.diff(w, axis=1) <= 0)
    _, ids, w, _ = cpp.route(x, wr, 1)
    assert np.all(w == 1.0)
    for k in (2, 5):
        _, ids, w, _ = cpp.route(x, wr, k)
        np.testing.assert_allclose(w.sum(1), 1.0, rtol=1e-14)
        pm = cpp.permute(ids, 16)
        np.testing.assert_array_equal(pm["offsets"], np.concatenate([[0], np.cumsum(np.bincount(ids.ravel(),
                                                                                                   minlength=16))]))
        assert np.bincount(pm["perm_src"], minlength=5).tolist() == [k] * 5
        np.testing.assert_array_equal(pm["inv"][pm["perm_src"], pm["perm_slot"]], np.arange(5 * k))
        for e in range(16):
            seg = pm["perm_src"][pm["offsets"][e]:pm["offsets"][e + 1]]
            assert np.all(np.diff(seg) > 0)


# ------------------------------------------------------------------ agreement with the numpy oracle
def test_quantisers_bit_exact_against_numpy_oracle():
    rng = np.random.default_rng(5)
    v = (rng.standard_normal((64, 512)) * np.exp2(rng.integers(-20, 20, (64, 1)))).astype(np.float32)
    v[3, :16] = 0.0
    v[4, 16:32] = 1e-30
    v[5, 32:48] = -0.0
    a = np.float32(np.abs(v).max() / 2688)
    for alpha in (a, np.float32(1.0), np.float32(a * 1e-3)):
        p, s = cpp.quantize_nvfp4(v, alpha)
        rp, rs = nvfp4.quantize_nvfp4(v, alpha)
        np.testing.assert_array_equal(s, rs)
        np.testing.assert_array_equal(p, rp)
    c, s = cpp.quantize_mxfp8(v)
    rc, rs = mxfp8.quantize_mxfp8(v)
    np.testing.assert_array_equal(s, rs)
    np.testing.assert_array_equal(c, rc)


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp8"])
@pytest.mark.parametrize("name,tokens", [("tiny", 4), ("tiny", 37), ("mid", 9)])
def test_forward_agrees_with_numpy_oracle(fmt, name, tokens):
    shape = mi.SHAPES["tiny"] if name == "tiny" else mi.LayerShape("mid", 9, 512, 32, 4, 384)
    shape = dataclasses.replace(shape, tokens=tokens)
    seed = 7
    xb, rb = mi.tokens(shape, seed)
    wr = mi.router_weight(shape, seed)
    gb = mi.gamma(shape, seed)
    a1, a2 = (np.float32(4.0 / 2688), np.float32(2.0 / 2688)) if fmt == "nvfp4" else (None, None)
    get = lambda e: mi.expert_weights(shape, seed, e)  # noqa: E731
    r = cpp.moe_forward(xb, rb, wr, gb, get, shape.top_k, shape.inter, alpha_a1=a1 or 1.0, alpha_a2=a2 or 1.0,
                        eps=shape.rms_eps, fmt=fmt)
    ref = moe.moe_forward(mi.bf16_bits_to_f32(xb).astype(np.float64), mi.bf16_bits_to_f32(rb).astype(np.float64), wr,
                          mi.bf16_bits_to_f32(gb).astype(np.float64), moe.ExpertCache(get, fmt=fmt), shape.experts,
                          shape.top_k, a1, a2, shape.rms_eps)
    np.testing.assert_array_equal(r["ids"], ref["ids"])
    np.testing.assert_array_equal(r["near_tie"], ref["near_tie"])
    np.testing.assert_allclose(r["w"], ref["w"], rtol=1e-13)
    np.testing.assert_allclose(r["m"], ref["m"], rtol=0, atol=1e-12 * max(1.0, np.abs(ref["m"]).max()))
    np.testing.assert_allclose(r["out_pre"], ref["out_pre"], rtol=0, atol=1e-12)
    np.testing.assert_array_equal(mi.bf16_bits_to_f32(r["out_bf16"]).astype(np.float64), ref["out"])
    pm = cpp.permute(r["ids"], shape.experts)
    for key in ("offsets", "perm_src", "perm_slot", "inv"):
        np.testing.assert_array_equal(pm[key], ref[key])
