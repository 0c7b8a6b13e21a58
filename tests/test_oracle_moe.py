"""Pins of the oracle's MoE forward against things other than itself.

* A hand-worked 2-expert example (no page prints one), each intermediate derived by hand
  from the definitions and written here as a literal: the quantised x, the block scales,
  the SwiGLU values, the finalize sum, the RMS and the output.
* Brute force: every expert evaluated densely for every token, weighted by the routing
  (zero for unchosen experts), must equal the sparse grouped evaluation.
* Invariants of routing and permutation (weights sum to one, each token k times, offsets
  = exclusive scan of the histogram, inv o perm = identity, ascending tokens per expert).
* Special cases with textbook answers: zero router -> experts 0..k-1 with 1/k; k = E ->
  the full softmax; k = 1 -> weight 1; constant m -> RMSNorm closed form; grid-exact
  operands -> the expert GEMMs equal plain FP64 matmuls.
Routing: 8 of 256 experts (vLLM recipe "reflection/Beam-1.0-501B-A23B", "Overview");
finalize + sandwich norm (vLLM PR "Day-0 support for Reflection's Beam-1.0", "Status").
"""

import math

import numpy as np
import pytest
import torch

import moe_inputs as mi
from oracle import moe, nvfp4


# ------------------------------------------------------------------ hand-worked example
def _hand_example():
    """T=1, H=I=16, E=2, k=2, alpha_a1 = alpha_a2 = 1, residual 0, gamma 1.

    x = 2 e0; router rows +-0.5 e0 (logits +-1).  Expert 0: gate row 0 = e0, up row 0 = e0,
    down[h=0, i=0] = 1.  Expert 1: gate row 0 = -e0, up row 0 = e0, down[h=1, i=0] = 1.
    """
    H = I = 16
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
    cache = moe.ExpertCache(lambda e: experts[e])
    return x, wr, cache


def test_hand_worked_two_expert_example():
    x, wr, cache = _hand_example()
    r = moe.moe_forward(x, np.zeros_like(x), wr, np.ones(16), cache, num_experts=2, top_k=2,
                        alpha_a1=np.float32(1), alpha_a2=np.float32(1))
    # routing: logits +-1 -> w = (sigmoid(2), sigmoid(-2))
    assert r["ids"].tolist() == [[0, 1]]
    np.testing.assert_allclose(r["w"][0], [0.8807970779778823, 0.11920292202211755], rtol=1e-15)
    # x block: s = 2/6 -> E4M3 0.34375 (nearest of 0.3125 / 0.34375); 2/0.34375 = 5.8 -> 6
    assert nvfp4.e4m3_decode(r["a1_sf"][0, 0]) == 0.34375
    a1 = nvfp4.dequantize_nvfp4(r["a1_packed"], r["a1_sf"], 1.0)
    assert a1[0, 0] == 2.0625 and not a1[0, 1:].any()
    # weights: alpha_w = fl32(1/2688), block scale saturates to 448, code 6 -> 1.0000000186
    q0 = cache.quantized(0)
    assert q0["w_gu_alpha"] == np.float32(np.float32(1) / np.float32(2688))
    assert nvfp4.e4m3_decode(q0["w_gu_sf"][0, 0]) == 448.0
    one = 6 * 448 * float(np.float32(1) / np.float32(2688))
    assert abs(one - 1.0000000186) < 1e-10
    # SwiGLU values and their NVFP4 codes
    h0, h1 = r["h32"][0, 0, 0], r["h32"][0, 1, 0]
    assert abs(h0 - 3.774085) < 2e-6 and abs(h1 - (-0.479821)) < 2e-6
    # A2: 3.774/6 -> E4M3 0.625, 3.774/0.625 = 6.04 -> 6 -> 3.75; -0.4798/6 -> 0.078125 -> -0.46875
    y = r["y"][0]
    assert abs(y[0, 0] - 3.75 * one) < 1e-12 and abs(y[1, 1] - (-0.46875 * one)) < 1e-12
    m = r["m"][0]
    assert abs(m[0] - 3.302989) < 2e-6 and abs(m[1] - (-0.0558764)) < 2e-7 and not m[2:].any()
    rms = math.sqrt((m[0] ** 2 + m[1] ** 2) / 16 + 1e-6)
    assert abs(rms - 0.825866) < 2e-6
    assert abs(r["out_pre"][0, 0] - 3.999425) < 3e-6 and abs(r["out_pre"][0, 1] - (-0.0676579)) < 3e-7
    # BF16: 3.999425 -> 4.0 (step 2^-6); -0.0676579 -> -139 * 2^-11
    assert r["out"][0, 0] == 4.0 and r["out"][0, 1] == -139 * 2.0 ** -11


# ------------------------------------------------------------------ tiny-config helpers
def _tiny(seed=0, shape=None):
    shape = shape or mi.SHAPES["tiny"]
    xb, rb = mi.tokens(shape, seed)
    x = mi.bf16_bits_to_f32(xb).astype(np.float64)
    res = mi.bf16_bits_to_f32(rb).astype(np.float64)
    wr = mi.router_weight(shape, seed)
    g = mi.bf16_bits_to_f32(mi.gamma(shape, seed)).astype(np.float64)
    cache = moe.ExpertCache(lambda e: mi.expert_weights(shape, seed, e))
    return shape, x, res, wr, g, cache


def test_brute_force_dense_equals_sparse():
    shape, x, res, wr, g, cache = _tiny()
    a1s, a2s = np.float32(5.0 / 2688), np.float32(3.0 / 2688)
    r = moe.moe_forward(x, res, wr, g, cache, shape.experts, shape.top_k, a1s, a2s)
    # dense: every expert on every token, mixed by a [T, E] weight that is 0 off the top-k
    wfull = np.zeros((shape.tokens, shape.experts))
    for t in range(shape.tokens):
        for j in range(shape.top_k):
            wfull[t, r["ids"][t, j]] = r["w"][t, j]
    a1p, a1sf = nvfp4.quantize_nvfp4(x.astype(np.float32), a1s)
    a1 = nvfp4.dequantize_nvfp4(a1p, a1sf, a1s)
    m = np.zeros((shape.tokens, shape.hidden))
    for e in range(shape.experts):
        w_gu, w_d = cache.dequantized(e)
        gg = a1 @ w_gu[: shape.inter].T
        uu = a1 @ w_gu[shape.inter:].T
        h = (gg * (1.0 / (1.0 + np.exp(-gg))) * uu).astype(np.float32)
        a2p, a2sf = nvfp4.quantize_nvfp4(h, a2s)
        y = nvfp4.dequantize_nvfp4(a2p, a2sf, a2s) @ w_d.T
        m += wfull[:, e:e + 1] * y
    np.testing.assert_allclose(r["m"], m, rtol=0, atol=1e-12)


def test_routing_and_permutation_invariants():
    shape = mi.SHAPES["tiny"]
    rng = np.random.default_rng(0)
    for trial in range(20):
        t_count = int(rng.integers(1, 40))
        logits = rng.standard_normal((t_count, shape.experts))
        if trial % 3 == 0:
            logits = np.round(logits, 1)  # many exact ties
        ids, w, p = moe.route_topk(logits, shape.top_k)
        np.testing.assert_allclose(w.sum(1), 1.0, rtol=1e-14)
        assert np.all(np.diff(w, axis=1) <= 0)  # descending weight
        for t in range(t_count):
            assert len(set(ids[t].tolist())) == shape.top_k
            # brute force: no unchosen expert beats a chosen one; ties go to the lower index
            chosen = set(ids[t].tolist())
            for e in range(shape.experts):
                if e in chosen:
                    continue
                for c in chosen:
                    assert p[t, e] < p[t, c] or (p[t, e] == p[t, c] and c < e)
        # renormalised weights equal a softmax over the chosen logits
        sel = np.take_along_axis(logits, ids, 1)
        sm = np.exp(sel - sel.max(1, keepdims=True))
        np.testing.assert_allclose(w, sm / sm.sum(1, keepdims=True), rtol=1e-12)
        pm = moe.permute(ids, shape.experts)
        counts = np.array([(ids == e).sum() for e in range(shape.experts)])
        np.testing.assert_array_equal(pm["counts"], counts)
        offs = [0]
        for c in counts:
            offs.append(offs[-1] + c)
        np.testing.assert_array_equal(pm["offsets"], offs)
        # every token appears exactly k times; inv o perm = identity
        assert np.all(np.bincount(pm["perm_src"], minlength=t_count) == shape.top_k)
        r_idx = pm["inv"][pm["perm_src"], pm["perm_slot"]]
        np.testing.assert_array_equal(r_idx, np.arange(t_count * shape.top_k))
        for e in range(shape.experts):
            seg = pm["perm_src"][offs[e]:offs[e + 1]]
            assert np.all(np.diff(seg) > 0)  # ascending tokens within an expert
            assert np.all(ids[seg, pm["perm_slot"][offs[e]:offs[e + 1]]] == e)


def test_special_cases_routing():
    t_count, experts = 5, 16
    ids, w, _ = moe.route_topk(np.zeros((t_count, experts)), 4)
    assert ids.tolist() == [[0, 1, 2, 3]] * t_count and np.all(w == 0.25)
    logits = np.random.default_rng(1).standard_normal((t_count, experts))
    ids, w, p = moe.route_topk(logits, experts)  # k = E: the full softmax
    np.testing.assert_allclose(np.take_along_axis(p, ids, 1), w, rtol=1e-14)
    z = np.exp(logits - logits.max(1, keepdims=True))
    np.testing.assert_allclose(np.take_along_axis(z / z.sum(1, keepdims=True), ids, 1), w, rtol=1e-14)
    ids, w, _ = moe.route_topk(logits, 1)  # k = 1: the argmax with weight 1
    assert np.all(w == 1.0) and np.all(ids[:, 0] == logits.argmax(1))


def test_near_tie_mask():
    l = np.array([[3.0, 2.0, 1.0, 1.0 - 5e-6], [3.0, 2.0, 1.0, 0.5]])
    assert moe.near_tie_mask(l, 3).tolist() == [True, False]
    assert not moe.near_tie_mask(l, 4).any()


def test_rmsnorm_closed_form_and_bf16():
    t_count, k, hidden = 3, 2, 64
    c = np.array([0.5, -2.0, 1e-3])
    y = np.broadcast_to(c[:, None, None], (t_count, k, hidden)).copy()
    w = np.full((t_count, k), 0.5)
    gam = np.linspace(0.5, 1.5, hidden)
    pre, out, m = moe.finalize(y, w, np.zeros((t_count, hidden)), gam, 1e-6)
    expect = np.sign(c)[:, None] * gam[None, :] / np.sqrt(1 + 1e-6 / c[:, None] ** 2)
    np.testing.assert_allclose(pre, expect, rtol=1e-14)
    # BF16 rounding against torch's FP32 -> BF16 conversion (single rounding from FP32 values)
    v = np.random.default_rng(2).standard_normal(100_000).astype(np.float32) * 37
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(moe.bf16_round(v.astype(np.float64)), ref)


def test_next_prenorm_closed_form():
    # constant rows c -> gamma * sign(c) / sqrt(1 + eps / c^2); the output is rounded to BF16
    c = np.array([3.0, -0.25])
    out = np.broadcast_to(c[:, None], (2, 32)).copy()
    gam = np.linspace(0.5, 2.0, 32)
    pre, rounded = moe.next_prenorm(out, gam, 1e-6)
    expect = np.sign(c)[:, None] * gam[None, :] / np.sqrt(1 + 1e-6 / c[:, None] ** 2)
    np.testing.assert_allclose(pre, expect, rtol=1e-14)
    assert np.all(np.abs(rounded - pre) <= 2.0 ** -8 * np.abs(pre))  # half a BF16 ulp
    # scale invariance: RMSNorm(a x) = RMSNorm(x) for a > 0 (eps -> 0)
    x = np.random.default_rng(8).standard_normal((3, 64))
    np.testing.assert_allclose(moe.next_prenorm(4.0 * x, np.ones(64), 0.0)[0], moe.next_prenorm(x, np.ones(64), 0.0)[0],
                               rtol=1e-13)


def test_grid_exact_expert_gemms_equal_fp64_matmul():
    # Operands already on the E2M1 x E4M3 grid with power-of-two tensor scales quantise
    # losslessly, so steps 7 and 10 reduce to plain FP64 matmuls of the raw values.
    rng = np.random.default_rng(9)
    rows, hidden, inter = 6, 64, 32

    def grid(shape, alpha):
        sc = rng.integers(40, 60, size=shape[:-1] + (shape[-1] // 16,)).astype(np.uint8)
        codes = rng.integers(0, 16, size=shape).astype(np.uint8)
        codes[..., ::16] = 7
        S = np.repeat(nvfp4.e4m3_decode(sc), 16, axis=-1)
        return (nvfp4.e2m1_decode(codes) * S * float(alpha)).astype(np.float32)

    a1s = np.float32(2.0 ** -3)
    x = grid((rows, hidden), a1s)
    w_gu = grid((2 * inter, hidden), 2.0 ** -9)
    w_d = grid((hidden, inter), 2.0 ** -9)
    wa = np.float32(2.0 ** -9)
    gu_p, gu_s = nvfp4.quantize_nvfp4(w_gu, wa)
    d_p, d_s = nvfp4.quantize_nvfp4(w_d, wa)
    q = dict(w_gu=gu_p, w_gu_sf=gu_s, w_gu_alpha=wa, w_d=d_p, w_d_sf=d_s, w_d_alpha=wa)
    deq = moe.dequantize_expert(q)
    np.testing.assert_array_equal(deq[0], w_gu)
    np.testing.assert_array_equal(deq[1], w_d)
    a1p, a1sf = nvfp4.quantize_nvfp4(x, a1s)
    a2s = np.float32(0.01)
    r = moe.expert_forward(a1p, a1sf, a1s, deq, a2s)
    g = x.astype(np.float64) @ w_gu[:inter].T.astype(np.float64)
    u = x.astype(np.float64) @ w_gu[inter:].T.astype(np.float64)
    np.testing.assert_array_equal(r["h32"], (g / (1 + np.exp(-g)) * u).astype(np.float32))
    a2 = nvfp4.dequantize_nvfp4(r["a2_packed"], r["a2_sf"], a2s)
    np.testing.assert_allclose(r["y"], a2 @ w_d.T.astype(np.float64), rtol=1e-15, atol=0)


def test_subset_of_tokens_matches_batch():
    shape, x, res, wr, g, cache = _tiny(seed=3)
    a1s, a2s = np.float32(5.0 / 2688), np.float32(3.0 / 2688)
    full = moe.moe_forward(x, res, wr, g, cache, shape.experts, shape.top_k, a1s, a2s)
    sub = moe.moe_forward_tokens(x[[1, 3]], res[[1, 3]], wr, g, cache, shape.top_k, a1s, a2s)
    np.testing.assert_array_equal(sub["ids"], full["ids"][[1, 3]])
    np.testing.assert_array_equal(sub["out"], full["out"][[1, 3]])


def test_generator_bf16_matches_torch():
    v = np.random.default_rng(4).standard_normal(50_000).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(mi.f32_to_bf16_bits(v), ref)


def test_tensor_parallel_partials_sum_to_the_unsharded_layer():
    # Splitting every expert's intermediate features over W ranks partitions the sums of
    # the gate/up and down GEMMs; A2's quantisation blocks never straddle a shard.  So the
    # ranks' partial m add up to the unsharded m (FP64 rounding only), for both formats,
    # and W = 1 is the unsharded layer itself.
    shape, x, res, wr, g, cache = _tiny()
    a1s, a2s = np.float32(5.0 / 2688), np.float32(3.0 / 2688)
    full = moe.moe_forward(x, res, wr, g, cache, shape.experts, shape.top_k, a1s, a2s)
    for world in (1, 2, 4):
        tp = moe.moe_forward_tp(x, res, wr, g, cache, shape.top_k, a1s, a2s, world)
        np.testing.assert_array_equal(tp["ids"], full["ids"])
        np.testing.assert_allclose(tp["m"], full["m"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(tp["out_pre"], full["out_pre"], rtol=0, atol=1e-12)
        assert tp["m_parts"].shape == (world,) + full["m"].shape
        if world > 1:  # every rank contributes
            assert all(np.abs(tp["m_parts"][r]).max() > 0 for r in range(world))
    one = moe.moe_forward_tp(x, res, wr, g, cache, shape.top_k, a1s, a2s, 1)
    np.testing.assert_array_equal(one["m"], full["m"])
    cache8 = moe.ExpertCache(lambda e: mi.expert_weights(shape, 0, e), fmt="mxfp8")
    full8 = moe.moe_forward(x, res, wr, g, cache8, shape.experts, shape.top_k, None, None)
    tp8 = moe.moe_forward_tp(x, res, wr, g, cache8, shape.top_k, None, None, 4)
    np.testing.assert_allclose(tp8["m"], full8["m"], rtol=0, atol=1e-12)
    # the shard slices: gate rows, matching up rows, matching down columns
    w_gu, w_d = cache.dequantized(0)
    gu1, d1 = moe.shard_dequantized((w_gu, w_d), 1, 4)
    inter = w_gu.shape[0] // 2
    np.testing.assert_array_equal(gu1[: inter // 4], w_gu[inter // 4: inter // 2])
    np.testing.assert_array_equal(gu1[inter // 4:], w_gu[inter + inter // 4: inter + inter // 2])
    np.testing.assert_array_equal(d1, w_d[:, inter // 4: inter // 2])
    with pytest.raises(ValueError):
        moe.shard_dequantized((w_gu, w_d), 0, 3)


def test_expert_parallel_routed_rows_reproduce_the_unsharded_layer():
    # Experts split over W ranks, each rank with its own batch; only routed rows travel: each
    # rank routes and quantises its own tokens, sends each slot's row to the expert's owner
    # and finalizes its tokens from the rows that come back.  Every token's output is then
    # the unsharded layer's output for that token (W = 1 is the unsharded layer itself), the
    # rows each rank computes are its experts' share of all slots, and every rank sends
    # exactly its tokens' k slots.
    shape, x, res, wr, g, cache = _tiny()
    shape2, x2, res2, _, _, _ = _tiny(seed=5)
    a1s, a2s = np.float32(5.0 / 2688), np.float32(3.0 / 2688)
    xs, rs = [x, x2[:3]], [res, res2[:3]]
    full = moe.moe_forward(np.concatenate(xs), np.concatenate(rs), wr, g, cache, shape.experts, shape.top_k, a1s,
                           a2s)
    for world in (1, 2, 4):
        xw = xs if world == 2 else ([np.concatenate(xs)] if world == 1 else [x[:2], x[2:], x2[:1], x2[1:3]])
        rw = rs if world == 2 else ([np.concatenate(rs)] if world == 1 else [res[:2], res[2:], res2[:1], res2[1:3]])
        ep = moe.moe_forward_ep(xw, rw, wr, g, cache, shape.experts, shape.top_k, a1s, a2s, world)
        np.testing.assert_array_equal(np.concatenate([q["ids"] for q in ep["ranks"]]), full["ids"])
        np.testing.assert_allclose(np.concatenate([q["m"] for q in ep["ranks"]]), full["m"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(np.concatenate(ep["out_pre"]), full["out_pre"], rtol=0, atol=1e-12)
        np.testing.assert_array_equal(np.concatenate(ep["out"]), full["out"])
        e_loc = shape.experts // world
        hist = np.bincount(full["ids"].reshape(-1), minlength=shape.experts)
        np.testing.assert_array_equal(ep["received"], hist.reshape(world, e_loc).sum(1))
        np.testing.assert_array_equal(ep["counts"].sum(1), [len(v) * shape.top_k for v in xw])
        np.testing.assert_array_equal(ep["counts"].sum(0), hist)
    with pytest.raises(ValueError):
        moe.moe_forward_ep(xs, rs, wr, g, cache, shape.experts, shape.top_k, a1s, a2s, 3)
