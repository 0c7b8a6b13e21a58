"""Tensor-parallel layer (experts split over ranks along the intermediate size, finalize fused
with its all-reduce: beam_moe_tp_* and beam_moe_forward_tp through the C ABI) on one GPU.

The vLLM PR "Day-0 support for Reflection's Beam-1.0" (section "Status") fuses Beam's TP
all-reduce with the sandwich norms and the MoE finalize; the recipe
"reflection/Beam-1.0-501B-A23B" runs NVFP4 with TP4 on Blackwell.  One GPU holds every rank
here (SharedGpuGroup): every rank's phase 0 runs before any rank's phase 1, so the exchange
waits are satisfied when they run.  Checks: all ranks produce identical bits; the output
matches the oracle's tensor-parallel layer (= the unsharded layer) at the layer's
tolerances and a single handle holding all experts closely; from 256 tokens on the
all-reduce is two-shot (each rank finishes its slice of the tokens, then gathers the
others'), and its bits equal the one-shot form's on the same batch; repeated forwards
(the exchange buffers alternate by epoch) repeat the bits; a peer that never publishes
makes the wait give up with a TIMEOUT status and the group recovers after a re-attach.
"""

import dataclasses

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import moe_inputs as mi  # noqa: E402
from oracle import moe  # noqa: E402
from tests.gpu_util import ABS_MAX, REL_L2, bf16_to_f64, compare_outputs, oracle_layer_inputs  # noqa: E402

# I = 512 splits into 2 or 4 slices of whole 128-feature gate/up tiles
SHAPE = mi.LayerShape("tp", 0, 512, 32, 4, 512)


@pytest.fixture(scope="module")
def bm():
    import sparse_moe_layer_fp32_b200 as m
    return m


def _scales(shape, x, res, wr, g, cache):
    a1 = np.float32(np.float32(np.abs(x).max()) / np.float32(2688))
    r = moe.moe_forward_tokens(x, res, wr, g, cache, shape.top_k, a1, np.float32(1.0))
    return a1, np.float32(np.float32(np.abs(r["h32"]).max()) / np.float32(2688))


def _group(bm, shape, full, world, tokens, fmt, a1, a2):
    from sparse_moe_layer_fp32_b200 import tp
    layers = []
    for r in range(world):
        sh = tp.shard_weights(full, r, world, shape.inter)
        layers.append(bm.MoELayer(max_tokens=tokens, hidden=shape.hidden, num_experts=shape.experts,
                                  top_k=shape.top_k, inter=shape.inter // world, alpha_a1=float(a1),
                                  alpha_a2=float(a2), fmt=fmt, **sh))
    return tp.SharedGpuGroup(layers)


@pytest.mark.parametrize("fmt,world,tokens,seed", [("nvfp4", 2, 5, 30), ("nvfp4", 4, 40, 31), ("nvfp4", 4, 300, 32),
                                                   ("mxfp8", 2, 7, 33), ("mxfp8", 4, 260, 34),
                                                   ("nvfp4", 2, 301, 35), ("nvfp4", 4, 257, 36)])
def test_tp_matches_oracle_and_ranks_agree(bm, fmt, world, tokens, seed):
    from sparse_moe_layer_fp32_b200 import synthetic
    shape = dataclasses.replace(SHAPE, tokens=tokens)
    x, res, wr, g, cache = oracle_layer_inputs(shape, seed, fmt=fmt)
    a1, a2 = _scales(shape, x, res, wr, g, cache) if fmt == "nvfp4" else (1.0, 1.0)
    full = synthetic.make_weights(shape, seed, threads=4, fmt=fmt)
    grp = _group(bm, shape, full, world, tokens, fmt, a1, a2)
    xd, rd = synthetic.make_batch(shape, seed)
    outs = grp.forward(xd, rd)
    for lay in grp.layers:
        lay.check()
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o, outs[0])  # every rank holds the same output
    if tokens >= bm.TP_TWO_SHOT_MIN_TOKENS:  # two-shot; the one-shot form of the same batch: the same bits
        for lay in grp.layers:
            lay.set_tp_two_shot_tokens(2 ** 31 - 1)
        one = grp.forward(xd, rd)
        for lay in grp.layers:
            lay.check()
            lay.set_tp_two_shot_tokens(bm.TP_TWO_SHOT_MIN_TOKENS)
        for o in one:
            assert torch.equal(o, outs[0])
    ref = moe.moe_forward_tp(x, res, wr, g, cache, shape.top_k, a1 if fmt == "nvfp4" else None,
                             a2 if fmt == "nvfp4" else None, world, shape.rms_eps)
    got = bf16_to_f64(outs[0])
    rel, mx = compare_outputs(got, ref["out_pre"], skip=ref["near_tie"])
    assert rel <= REL_L2 and mx <= ABS_MAX, (rel, mx)
    # one handle with all the experts computes the same layer (the partial sums of y are
    # rounded to BF16 per rank instead of once)
    whole = bm.MoELayer(max_tokens=tokens, hidden=shape.hidden, num_experts=shape.experts, top_k=shape.top_k,
                        inter=shape.inter, alpha_a1=float(a1), alpha_a2=float(a2), fmt=fmt, **full)
    o1 = bf16_to_f64(whole.forward(xd, rd))
    whole.check()
    rel1, _ = compare_outputs(got, o1)
    assert rel1 < 5e-3, rel1
    whole.close()
    # epochs alternate the exchange buffers: repeated forwards repeat the bits
    for _ in range(3):
        again = grp.forward(xd, rd)
        for o in again:
            assert torch.equal(o, outs[0])
    for lay in grp.layers:
        lay.check()
    grp.close()


def test_tp_wait_gives_up_without_peer_and_group_recovers(bm):
    # Failure detection without a GPU fault: rank 1 never publishes its partial sums, so
    # rank 0's exchange wait runs out (2 s), the error word says TIMEOUT and the context
    # stays usable; after a re-attach the group computes again.
    from sparse_moe_layer_fp32_b200 import synthetic
    shape = dataclasses.replace(SHAPE, tokens=4)
    full = synthetic.make_weights(shape, 0, threads=2, fmt="mxfp8")
    grp = _group(bm, shape, full, 2, 4, "mxfp8", 1.0, 1.0)
    xd, rd = synthetic.make_batch(shape, 0)
    l0, l1 = grp.layers
    out = torch.empty_like(rd)
    l0.forward_tp_phase(xd, rd, out, 0)
    l0.forward_tp_phase(xd, rd, out, 1)  # waits for rank 1's flag, which nothing sets
    with pytest.raises(bm.BeamMoeError) as ei:
        l0.check()
    assert ei.value.status == bm.ERR_TIMEOUT
    # phases must alternate; a phase 1 without its phase 0 is refused on the host
    with pytest.raises(bm.BeamMoeError) as ei:
        l1.forward_tp_phase(xd, rd, out, 1)
    assert ei.value.status == bm.ERR_INVALID_ARG
    regions = [lay.tp_region() for lay in grp.layers]
    for r, lay in enumerate(grp.layers):
        lay.tp_attach(r, 2, regions)
    outs = grp.forward(xd, rd)
    for lay in grp.layers:
        lay.check()
    assert torch.equal(outs[0], outs[1])
    whole = bm.MoELayer(max_tokens=4, hidden=shape.hidden, num_experts=shape.experts, top_k=shape.top_k,
                        inter=shape.inter, fmt="mxfp8", **full)
    rel, _ = compare_outputs(bf16_to_f64(outs[0]), bf16_to_f64(whole.forward(xd, rd)))
    assert rel < 5e-3
    whole.close()
    # a region list that does not hold the handle's own region at its rank is refused
    with pytest.raises(bm.BeamMoeError):
        l0.tp_attach(1, 2, regions)
    grp.close()
