"""GPU routing (beam_moe_route: FP32 router GEMM + softmax/top-k/renormalise) against the
oracle.  Router 5120 -> 256 (vLLM PR "Day-0 support for Reflection's Beam-1.0", section
"Status"); 8 of 256 experts (recipe "reflection/Beam-1.0-501B-A23B", section "Overview").
Expert ids must match exactly except at near-ties (8th/9th logit gap below 1e-5 relative),
which are counted."""

import dataclasses

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import moe_inputs as mi  # noqa: E402
from oracle import moe  # noqa: E402
from tests.gpu_util import bf16_to_f64, ids_match  # noqa: E402


@pytest.fixture(scope="module")
def bm():
    import sparse_moe_layer_fp32_b200 as m
    return m


CASES = [("tiny", 4), ("tiny", 1), ("tiny", 300), ("decode8", 8), ("decode8", 16), ("decode8", 17),
         ("decode8", 333), ("decode8", 1024), ("decode8", 4096)]


@pytest.mark.parametrize("name,tokens", CASES)
def test_route_matches_oracle(bm, name, tokens):
    shape = dataclasses.replace(mi.SHAPES[name], tokens=tokens)
    xb, _ = mi.tokens(shape, 5)
    wr = mi.router_weight(shape, 5)
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
    ids, w = bm.beam_moe_route(x, torch.from_numpy(wr).cuda(), shape.top_k)
    torch.cuda.synchronize()
    ids, w = ids.cpu().numpy(), w.cpu().numpy()
    logits = moe.router_logits(mi.bf16_bits_to_f32(xb).astype(np.float64), wr)
    rid, rw, _ = moe.route_topk(logits, shape.top_k)
    near = moe.near_tie_mask(logits, shape.top_k)
    bad = ids_match(ids, rid, logits, near)
    assert not bad, f"routing differs on tokens {bad[:10]}"
    ok = ~near
    same = np.all(ids == rid, axis=1) & ok
    np.testing.assert_allclose(w[same], rw[same], rtol=0, atol=2e-5)
    np.testing.assert_allclose(w.sum(1), 1.0, atol=1e-5)
    assert np.all((ids >= 0) & (ids < shape.experts))
    print(f"{name} T={tokens}: near-ties {int(near.sum())}")


def test_route_zero_router_ties(bm):
    # all logits equal: the lowest k expert indices, weight 1/k each
    shape = mi.SHAPES["decode8"]
    xb, _ = mi.tokens(shape, 1)
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
    ids, w = bm.beam_moe_route(x, torch.zeros((256, 5120), device="cuda"), 8)
    torch.cuda.synchronize()
    assert ids.cpu().numpy().tolist() == [list(range(8))] * 8
    np.testing.assert_allclose(w.cpu().numpy(), 1 / 8, rtol=1e-6)


@pytest.fixture(scope="module")
def router_layer(bm):
    # the full router shape (H 5120 -> 256, top-8) with small experts (I = 128): only the
    # routing buffers are read here
    from sparse_moe_layer_fp32_b200 import synthetic
    shape = dataclasses.replace(mi.SHAPES["decode8"], inter=128, tokens=5000)
    weights = synthetic.make_weights(shape, 5, threads=8)
    layer = bm.MoELayer(max_tokens=5000, hidden=shape.hidden, num_experts=shape.experts, top_k=shape.top_k,
                        inter=shape.inter, alpha_a1=0.002, alpha_a2=0.0002, **weights)
    yield shape, layer
    layer.close()


@pytest.mark.parametrize("tokens", [17, 32, 100, 640, 1024, 2500, 4095, 4096, 5000])
def test_router_modes_match_oracle(bm, router_layer, tokens):
    # SIMT FFMA over slices of H, and the tensor cores on the three-part BF16 split (below
    # 4096 tokens over token tiles x slices of H with partial logits; from 4096 one tile per
    # CTA with the top-k in the epilogue): both exact against the oracle except near-ties
    shape, layer = router_layer
    shape = dataclasses.replace(shape, tokens=tokens)
    xb, rb = mi.tokens(shape, 6)
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
    r = torch.from_numpy(rb.view(np.int16)).view(torch.bfloat16).cuda()
    logits = moe.router_logits(mi.bf16_bits_to_f32(xb).astype(np.float64), mi.router_weight(shape, 5))
    rid, rw, _ = moe.route_topk(logits, shape.top_k)
    near = moe.near_tie_mask(logits, shape.top_k)
    got = {}
    for mode in (bm.ROUTER_SIMT, bm.ROUTER_TENSOR, bm.ROUTER_AUTO):
        layer.set_router_mode(mode)
        layer.forward(x, r)
        layer.check()
        ids = layer.debug(bm.BUF_IDS).cpu().numpy().view(np.int32).reshape(tokens, shape.top_k)
        w = layer.debug(bm.BUF_WEIGHTS).cpu().numpy().view(np.float32).reshape(tokens, shape.top_k)
        assert not ids_match(ids, rid, logits, near), mode
        # neighbours with near-equal logits may swap slots: compare sorted weights.  The
        # logits are FP32-accurate (~1e-5 absolute at |l| ~ 3 after 5120 terms, the scale of
        # the near-tie margin), so the renormalised weights agree to ~1e-5
        keep = ~near
        np.testing.assert_allclose(np.sort(w[keep], 1), np.sort(rw[keep], 1), rtol=1e-4, atol=1e-5)
        got[mode] = ids
    layer.set_router_mode(bm.ROUTER_AUTO)
    with pytest.raises(bm.BeamMoeError):
        layer.set_router_mode(7)
