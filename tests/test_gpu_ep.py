"""Expert-parallel layer with attention data parallelism (beam_moe_create_ep*,
beam_moe_forward_ep through the C ABI) on one GPU.

The vLLM PR "Day-0 support for Reflection's Beam-1.0" (section "Status") pairs attention
data parallelism with the MegaMoE expert kernels; each rank owns E / W of the experts and
its own batch.  One GPU holds every rank here (SharedGpuGroup): each phase (dispatch;
routing of the gathered batch + the rank's experts + partial m; combine + finalize) runs
for every rank before the next phase, so the exchange waits are satisfied when they run.
Checks: each rank's output matches the oracle's expert-parallel layer (= the unsharded
layer on the concatenated batch) at the layer's tolerances and a single handle with all
experts closely; repeated forwards repeat the bits; handles holding part of the experts
refuse the single-GPU and tensor-parallel forwards.
"""

import dataclasses

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import moe_inputs as mi  # noqa: E402
from oracle import moe  # noqa: E402
from tests.gpu_util import ABS_MAX, REL_L2, bf16_to_f64, compare_outputs, oracle_layer_inputs  # noqa: E402

SHAPES = {"tiny": mi.SHAPES["tiny"], "mid": mi.LayerShape("mid", 0, 512, 32, 4, 384)}


@pytest.fixture(scope="module")
def bm():
    import sparse_moe_layer_fp32_b200 as m
    return m


@pytest.mark.parametrize("name,fmt,world,tokens,seed", [("tiny", "nvfp4", 2, 3, 40), ("mid", "nvfp4", 4, 2, 41),
                                                        ("mid", "nvfp4", 4, 80, 42), ("tiny", "mxfp8", 4, 70, 43),
                                                        ("mid", "mxfp8", 2, 300, 44)])
def test_ep_matches_oracle(bm, name, fmt, world, tokens, seed):
    from sparse_moe_layer_fp32_b200 import synthetic, tp
    shape = dataclasses.replace(SHAPES[name], tokens=world * tokens)  # the gathered batch
    x, res, wr, g, cache = oracle_layer_inputs(shape, seed, fmt=fmt)
    if fmt == "nvfp4":
        a1 = np.float32(np.float32(np.abs(x).max()) / np.float32(2688))
        h = moe.moe_forward_tokens(x, res, wr, g, cache, shape.top_k, a1, np.float32(1.0))["h32"]
        a2 = np.float32(np.float32(np.abs(h).max()) / np.float32(2688))
    else:
        a1 = a2 = np.float32(1.0)
    full = synthetic.make_weights(shape, seed, threads=4, fmt=fmt)
    E, e_loc = shape.experts, shape.experts // world
    layers = []
    for r in range(world):
        sh = tp.shard_experts(full, r, world, E)
        layers.append(bm.MoELayer(max_tokens=world * tokens, hidden=shape.hidden, num_experts=E,
                                  top_k=shape.top_k, inter=shape.inter, alpha_a1=float(a1), alpha_a2=float(a2),
                                  fmt=fmt, expert_begin=r * e_loc, expert_count=e_loc, **sh))
    grp = tp.SharedGpuGroup(layers)
    xd, rd = synthetic.make_batch(shape, seed)
    xs = [xd[r * tokens:(r + 1) * tokens].contiguous() for r in range(world)]
    rs = [rd[r * tokens:(r + 1) * tokens].contiguous() for r in range(world)]
    outs = grp.forward(xs, rs)
    for lay in layers:
        lay.check()
    torch.cuda.synchronize()
    ref = moe.moe_forward_ep([x[r * tokens:(r + 1) * tokens] for r in range(world)],
                             [res[r * tokens:(r + 1) * tokens] for r in range(world)], wr, g, cache, E, shape.top_k,
                             a1 if fmt == "nvfp4" else None, a2 if fmt == "nvfp4" else None, world, shape.rms_eps)
    got = np.concatenate([bf16_to_f64(o) for o in outs])
    rel, mx = compare_outputs(got, np.concatenate(ref["out_pre"]), skip=ref["near_tie"])
    assert rel <= REL_L2 and mx <= ABS_MAX, (rel, mx)
    whole = bm.MoELayer(max_tokens=world * tokens, hidden=shape.hidden, num_experts=E, top_k=shape.top_k,
                        inter=shape.inter, alpha_a1=float(a1), alpha_a2=float(a2), fmt=fmt, **full)
    rel1, _ = compare_outputs(got, bf16_to_f64(whole.forward(xd, rd)))
    assert rel1 < 5e-3, rel1
    whole.close()
    for _ in range(2):  # the gathered and partial buffers alternate by epoch
        again = grp.forward(xs, rs)
        for o, a in zip(outs, again):
            assert torch.equal(o, a)
    for lay in layers:
        lay.check()
    # a handle that holds part of the experts runs only the expert-parallel forward
    with pytest.raises(bm.BeamMoeError) as ei:
        layers[0].forward(xs[0], rs[0])
    assert ei.value.status == bm.ERR_INVALID_ARG
    with pytest.raises(bm.BeamMoeError):
        layers[0].forward_tp(xs[0], rs[0])
    grp.close()
