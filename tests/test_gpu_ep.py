"""Expert-parallel layer with attention data parallelism (beam_moe_create_ep*,
beam_moe_forward_ep through the C ABI) on one GPU.

The vLLM PR "Day-0 support for Reflection's Beam-1.0" (section "Status") pairs attention
data parallelism with the MegaMoE expert kernels; each rank owns E / W of the experts and
its own batch, and only routed rows travel: each rank routes and quantises its own tokens,
stores each slot's row into the activation tiles of its expert's rank, the rank computes the
rows it received and returns each output row to its source slot, and each rank finalizes
its own tokens.  One GPU holds every rank here (SharedGpuGroup): each of the four phases
runs for every rank before the next phase, so the exchange waits are satisfied when they
run.  Checks: each rank's output matches the oracle's expert-parallel layer at the layer's
tolerances and is bit-identical to a handle with all experts run on that rank's tokens;
repeated forwards repeat the bits; phases out of order, unequal expert ranges and the
single-GPU and tensor-parallel forwards are refused.
"""

import dataclasses

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import moe_inputs as mi  # noqa: E402
from oracle import moe  # noqa: E402
from tests.gpu_util import (ABS_MAX, REL_L2, a2_boundary_tokens, bf16_to_f64, compare_outputs,  # noqa: E402
                            oracle_layer_inputs)

SHAPES = {"tiny": mi.SHAPES["tiny"], "mid": mi.LayerShape("mid", 0, 512, 32, 4, 384)}


@pytest.fixture(scope="module")
def bm():
    import sparse_moe_layer_fp32_b200 as m
    return m


def _ep_layers(bm, shape, full, world, max_tokens, a1, a2, fmt):
    from sparse_moe_layer_fp32_b200 import tp
    E, e_loc = shape.experts, shape.experts // world
    layers = []
    for r in range(world):
        sh = tp.shard_experts(full, r, world, E)
        layers.append(bm.MoELayer(max_tokens=max_tokens, hidden=shape.hidden, num_experts=E, top_k=shape.top_k,
                                  inter=shape.inter, alpha_a1=float(a1), alpha_a2=float(a2), fmt=fmt,
                                  expert_begin=r * e_loc, expert_count=e_loc, **sh))
    return layers


@pytest.mark.parametrize("name,fmt,world,tokens,seed", [("tiny", "nvfp4", 2, 3, 40), ("mid", "nvfp4", 4, 2, 41),
                                                        ("mid", "nvfp4", 4, 80, 42), ("tiny", "mxfp8", 4, 70, 43),
                                                        ("mid", "mxfp8", 2, 300, 44), ("mid", "nvfp4", 2, 600, 45)])
def test_ep_matches_oracle_and_single_gpu_bits(bm, name, fmt, world, tokens, seed):
    from sparse_moe_layer_fp32_b200 import synthetic, tp
    shape = dataclasses.replace(SHAPES[name], tokens=world * tokens)  # every rank's batch together
    x, res, wr, g, cache = oracle_layer_inputs(shape, seed, fmt=fmt)
    if fmt == "nvfp4":
        a1 = np.float32(np.float32(np.abs(x).max()) / np.float32(2688))
        h = moe.moe_forward_tokens(x, res, wr, g, cache, shape.top_k, a1, np.float32(1.0))["h32"]
        a2 = np.float32(np.float32(np.abs(h).max()) / np.float32(2688))
    else:
        a1 = a2 = np.float32(1.0)
    full = synthetic.make_weights(shape, seed, threads=4, fmt=fmt)
    layers = _ep_layers(bm, shape, full, world, world * tokens, a1, a2, fmt)
    grp = tp.SharedGpuGroup(layers)
    xd, rd = synthetic.make_batch(shape, seed)
    xs = [xd[r * tokens:(r + 1) * tokens].contiguous() for r in range(world)]
    rs = [rd[r * tokens:(r + 1) * tokens].contiguous() for r in range(world)]
    outs = grp.forward(xs, rs)
    for lay in layers:
        lay.check()
    torch.cuda.synchronize()
    ref = moe.moe_forward_ep([x[r * tokens:(r + 1) * tokens] for r in range(world)],
                             [res[r * tokens:(r + 1) * tokens] for r in range(world)], wr, g, cache, shape.experts,
                             shape.top_k, a1 if fmt == "nvfp4" else None, a2 if fmt == "nvfp4" else None, world,
                             shape.rms_eps)
    # the same bits as one handle with every expert, run on each rank's own tokens; its A2
    # buffers show which tokens' A2 codes or scales sit on a rounding boundary, where the
    # GPU's FP32 h and the oracle's FP64 h may decide differently (both valid): like routing
    # near-ties, those tokens are counted and held to the relative-L2 bound only
    whole = bm.MoELayer(max_tokens=world * tokens, hidden=shape.hidden, num_experts=shape.experts, top_k=shape.top_k,
                        inter=shape.inter, alpha_a1=float(a1), alpha_a2=float(a2), fmt=fmt, **full)
    edge = np.zeros(world * tokens, bool)
    for r in range(world):
        assert torch.equal(outs[r], whole.forward(xs[r], rs[r])), r
        whole.check()
        sl = slice(r * tokens, (r + 1) * tokens)
        o = moe.moe_forward_tokens(x[sl], res[sl], wr, g, cache, shape.top_k, a1 if fmt == "nvfp4" else None,
                                   a2 if fmt == "nvfp4" else None, shape.rms_eps)
        edge[sl] = a2_boundary_tokens(whole, tokens, shape.top_k, shape.inter, o["h32"], a2, fmt, skip=o["near_tie"])
    whole.close()
    got = np.concatenate([bf16_to_f64(o) for o in outs])
    rel, _ = compare_outputs(got, np.concatenate(ref["out_pre"]), skip=ref["near_tie"])
    _, mx = compare_outputs(got, np.concatenate(ref["out_pre"]), skip=ref["near_tie"] | edge)
    assert rel <= REL_L2 and mx <= ABS_MAX, (rel, mx)
    assert edge.sum() <= max(2, 0.01 * world * tokens), int(edge.sum())
    for _ in range(2):  # the regions are reused forward after forward
        again = grp.forward(xs, rs)
        for o, a in zip(outs, again):
            assert torch.equal(o, a)
    for lay in layers:
        lay.check()
    # a handle that holds part of the experts runs only the expert-parallel forward, its
    # phases in order
    with pytest.raises(bm.BeamMoeError) as ei:
        layers[0].forward(xs[0], rs[0])
    assert ei.value.status == bm.ERR_INVALID_ARG
    with pytest.raises(bm.BeamMoeError):
        layers[0].forward_tp(xs[0], rs[0])
    with pytest.raises(bm.BeamMoeError):
        layers[0].forward_ep_phase(xs[0], rs[0], outs[0], 2)
    grp.close()


def test_ep_attach_refuses_unequal_expert_ranges(bm):
    from sparse_moe_layer_fp32_b200 import synthetic, tp
    shape = dataclasses.replace(SHAPES["tiny"], tokens=4)
    full = synthetic.make_weights(shape, 3, threads=2)
    # 16 experts over 2 ranks as 4 + 12: not the equal ranges the layout needs
    layers = []
    for begin, count in ((0, 4), (4, 12)):
        sh = dict(full)
        for key in ("w_gu", "w_gu_sf", "w_d", "w_d_sf", "w_gu_alpha", "w_d_alpha"):
            sh[key] = full[key][begin:begin + count].contiguous()
        layers.append(bm.MoELayer(max_tokens=8, hidden=shape.hidden, num_experts=shape.experts, top_k=shape.top_k,
                                  inter=shape.inter, alpha_a1=0.001, alpha_a2=0.0001, expert_begin=begin,
                                  expert_count=count, **sh))
    with pytest.raises(bm.BeamMoeError) as ei:
        tp.SharedGpuGroup(layers)
    assert ei.value.status == bm.ERR_INVALID_ARG
    for lay in layers:
        lay.close()


def test_ep_wait_gives_up_without_peer_and_group_recovers(bm):
    # Failure detection without a GPU fault: rank 1 never publishes its expert counts, so
    # rank 0's layout wait runs out (2 s): the error word says TIMEOUT, the layout leaves an
    # empty block list and the context stays usable; after a re-attach the group computes
    # the same bits as one handle with every expert.
    from sparse_moe_layer_fp32_b200 import synthetic, tp
    shape = dataclasses.replace(SHAPES["tiny"], tokens=2 * 4)
    full = synthetic.make_weights(shape, 5, threads=2)
    a1, a2 = 0.002, 0.0005
    layers = _ep_layers(bm, shape, full, 2, 8, a1, a2, "nvfp4")
    grp = tp.SharedGpuGroup(layers)
    xd, rd = synthetic.make_batch(shape, 5)
    xs = [xd[:4].contiguous(), xd[4:].contiguous()]
    rs = [rd[:4].contiguous(), rd[4:].contiguous()]
    out = torch.empty_like(rs[0])
    layers[0].forward_ep_phase(xs[0], rs[0], out, 0)
    layers[0].forward_ep_phase(xs[0], rs[0], out, 1)  # waits for rank 1's counts, which nothing sets
    with pytest.raises(bm.BeamMoeError) as ei:
        layers[0].check()
    assert ei.value.status == bm.ERR_TIMEOUT
    # phases run in order; rank 1 cannot start at phase 1
    with pytest.raises(bm.BeamMoeError) as ei:
        layers[1].forward_ep_phase(xs[1], rs[1], out, 1)
    assert ei.value.status == bm.ERR_INVALID_ARG
    regions = [lay.tp_region() for lay in layers]
    for r, lay in enumerate(layers):
        lay.tp_attach(r, 2, regions)
    outs = grp.forward(xs, rs)
    for lay in layers:
        lay.check()
    whole = bm.MoELayer(max_tokens=8, hidden=shape.hidden, num_experts=shape.experts, top_k=shape.top_k,
                        inter=shape.inter, alpha_a1=a1, alpha_a2=a2, **full)
    for r in range(2):
        assert torch.equal(outs[r], whole.forward(xs[r], rs[r])), r
    whole.close()
    grp.close()
