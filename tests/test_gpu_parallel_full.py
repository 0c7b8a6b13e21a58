"""Tensor- and expert-parallel layers at the full layer size (H 5120, 256 experts, top-8,
I 1536), with their ranks sharing one GPU, in the batch sizes bench.py times for them.

Expert parallelism (vLLM PR "Day-0 support for Reflection's Beam-1.0", section "Status":
attention data parallelism with MegaMoE): 4 ranks of 64 experts, each with its own batch
(8 tokens: the fused small-batch routing; 64 tokens: the sliced tensor-core router).  Every
rank's output is bit-identical to one handle holding all 256 experts run on that rank's
tokens: the routed rows travel and return exactly, and every row's arithmetic is the
single-GPU one.

Tensor parallelism (the same section: the TP all-reduce fused with the finalize; recipe
"reflection/Beam-1.0-501B-A23B": NVFP4 with TP4): 4 ranks of 384 intermediate features,
8 tokens (one-shot all-reduce) and 300 tokens (two-shot).  All ranks hold the same bits, the
two-shot and one-shot forms agree bit for bit on the same batch, and the output is close to
the single handle's (rel-L2 < 5e-3: each rank rounds its partial y to BF16).
"""

import dataclasses

import pytest
import torch

pytestmark = pytest.mark.gpu

import moe_inputs as mi  # noqa: E402
from tests.gpu_util import bf16_to_f64, compare_outputs  # noqa: E402

WORLD = 4


@pytest.fixture(scope="module")
def bm():
    import sparse_moe_layer_fp32_b200 as m
    return m


@pytest.fixture(scope="module")
def full():
    from sparse_moe_layer_fp32_b200 import synthetic
    return synthetic.make_weights(mi.SHAPES["decode8"], 0)


@pytest.fixture(scope="module")
def whole(bm, full):
    shape = mi.SHAPES["decode8"]
    a1, a2 = mi.activation_scales(shape)
    lay = bm.MoELayer(max_tokens=WORLD * 300, hidden=shape.hidden, num_experts=shape.experts, top_k=shape.top_k,
                      inter=shape.inter, alpha_a1=float(a1), alpha_a2=float(a2), **full)
    yield lay
    lay.close()


@pytest.mark.parametrize("tokens", [8, 64])
def test_ep_full_size_matches_single_gpu_bits(bm, full, whole, tokens):
    from sparse_moe_layer_fp32_b200 import synthetic, tp
    shape = dataclasses.replace(mi.SHAPES["decode8"], tokens=WORLD * tokens)
    a1, a2 = mi.activation_scales(mi.SHAPES["decode8"])
    e_loc = shape.experts // WORLD
    layers = []
    for r in range(WORLD):
        sh = tp.shard_experts(full, r, WORLD, shape.experts)
        layers.append(bm.MoELayer(max_tokens=WORLD * tokens, hidden=shape.hidden, num_experts=shape.experts,
                                  top_k=shape.top_k, inter=shape.inter, alpha_a1=float(a1), alpha_a2=float(a2),
                                  expert_begin=r * e_loc, expert_count=e_loc, **sh))
        del sh
    grp = tp.SharedGpuGroup(layers)
    xd, rd = synthetic.make_batch(shape, 11)
    xs = [xd[r * tokens:(r + 1) * tokens].contiguous() for r in range(WORLD)]
    rs = [rd[r * tokens:(r + 1) * tokens].contiguous() for r in range(WORLD)]
    for _ in range(2):  # the exchange regions are reused forward after forward
        outs = grp.forward(xs, rs)
        for lay in layers:
            lay.check()
        for r in range(WORLD):
            assert torch.equal(outs[r], whole.forward(xs[r], rs[r])), r
        whole.check()
    grp.close()


@pytest.mark.parametrize("tokens", [8, 300])
def test_tp_full_size_ranks_agree_and_match_single_gpu(bm, full, whole, tokens):
    from sparse_moe_layer_fp32_b200 import synthetic, tp
    shape = dataclasses.replace(mi.SHAPES["decode8"], tokens=tokens)
    a1, a2 = mi.activation_scales(mi.SHAPES["decode8"])
    layers = []
    for r in range(WORLD):
        sh = tp.shard_weights(full, r, WORLD, shape.inter)
        layers.append(bm.MoELayer(max_tokens=tokens, hidden=shape.hidden, num_experts=shape.experts,
                                  top_k=shape.top_k, inter=shape.inter // WORLD, alpha_a1=float(a1),
                                  alpha_a2=float(a2), **sh))
        del sh
    grp = tp.SharedGpuGroup(layers)
    xd, rd = synthetic.make_batch(shape, 12)
    outs = grp.forward(xd, rd)
    for lay in layers:
        lay.check()
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    if tokens >= bm.TP_TWO_SHOT_MIN_TOKENS:  # two-shot above; the one-shot form of the same batch
        for lay in layers:
            lay.set_tp_two_shot_tokens(2 ** 31 - 1)
        one = grp.forward(xd, rd)
        for lay in layers:
            lay.check()
        assert all(torch.equal(o, outs[0]) for o in one)
    rel, _ = compare_outputs(bf16_to_f64(outs[0]), bf16_to_f64(whole.forward(xd, rd)))
    whole.check()
    assert rel < 5e-3, rel
    grp.close()
