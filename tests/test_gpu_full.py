"""Full-size workloads (H 5120, 256 experts, top-8) through beam_moe_forward, in the launch
configuration bench.py times.

* Sampled tokens against oracle outputs stored by tests/golden/make_full_size_golden.py
  (each token's output depends only on that token, so a sample of the batch is exact):
  routing ids exact except near-ties, outputs within relative L2 1e-2 and absolute 5e-2.
* Whole-batch properties that hold at any size: ids distinct and in range, weights sum to
  one, offsets = histogram prefix sum, the permutation bit-exact against the oracle's
  permutation of the GPU ids (every token exactly k times, ascending tokens per expert),
  finite outputs.
Workloads: decode verify (7 draft + 1, recipe "reflection/Beam-1.0-501B-A23B", section
"DFlash2 speculative decoding"), 128 x 8 batched verify and the 8 x 2K / 32K prefills
(vLLM PR "Day-0 support for Reflection's Beam-1.0", section "Validation").
"""

import os

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import moe_inputs as mi  # noqa: E402
from oracle import moe  # noqa: E402
from tests.gpu_util import ABS_MAX, REL_L2, bf16_to_f64, buf, compare_outputs, ids_match  # noqa: E402

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.fixture(scope="module")
def bm():
    import sparse_moe_layer_fp32_b200 as m
    return m


@pytest.fixture(scope="module")
def weights_i1536():
    from sparse_moe_layer_fp32_b200 import synthetic
    return synthetic.make_weights(mi.SHAPES["decode8"], 0)


def _check_workload(bm, shape, weights, fmt="nvfp4"):
    from sparse_moe_layer_fp32_b200 import synthetic
    suffix = "" if fmt == "nvfp4" else f"_{fmt}"
    gold = np.load(os.path.join(GOLDEN, f"full_{shape.name}{suffix}.npz"))
    assert str(gold["experts_format"]) == fmt if "experts_format" in gold else fmt == "nvfp4"
    layer = synthetic.make_layer(shape, weights, fmt=fmt)
    x, res = synthetic.make_batch(shape, 0)
    out = layer.forward(x, res)
    layer.check()
    T, k, E = shape.tokens, shape.top_k, shape.experts
    ids = buf(layer, bm.BUF_IDS, np.int32).reshape(T, k)
    w = buf(layer, bm.BUF_WEIGHTS, np.float32).reshape(T, k)
    offsets = buf(layer, bm.BUF_OFFSETS, np.int32)
    perm = buf(layer, bm.BUF_PERM, np.int32)
    inv = buf(layer, bm.BUF_INV, np.int32).reshape(T, k)
    out_np = bf16_to_f64(out)
    # ---- sampled tokens against the stored oracle outputs
    toks = gold["tokens"]
    near = gold["near_tie"]
    bad = ids_match(ids[toks], gold["ids"].astype(np.int64), gold["logits"].astype(np.float64), near)
    assert not bad, f"routing differs at sampled tokens {toks[bad]}"
    rel, mx = compare_outputs(out_np[toks], gold["out_pre"].astype(np.float64), skip=near)
    assert rel <= REL_L2 and mx <= ABS_MAX, (rel, mx)
    # ---- whole-batch properties
    assert np.all((ids >= 0) & (ids < E))
    assert np.all(np.sort(ids, 1)[:, 1:] != np.sort(ids, 1)[:, :-1])
    np.testing.assert_allclose(w.sum(1), 1.0, atol=1e-5)
    assert np.all(np.diff(w, axis=1) <= 1e-7)
    pm = moe.permute(ids.astype(np.int64), E)
    np.testing.assert_array_equal(offsets, pm["offsets"])
    np.testing.assert_array_equal(perm, pm["perm_src"])
    np.testing.assert_array_equal(inv, pm["inv"])
    assert np.isfinite(out_np).all()
    layer.close()
    return int(near.sum()), rel, mx, int((np.diff(offsets) > 0).sum())


@pytest.mark.parametrize("name", ["decode8", "spec1024", "prefill16k", "prefill32k_skew"])
def test_full_size_workload(bm, weights_i1536, name):
    shape = mi.SHAPES[name]
    weights = dict(weights_i1536)
    if shape.skew:
        weights["router_w"] = torch.from_numpy(mi.router_weight(shape, 0)).cuda()
    near, rel, mx, used = _check_workload(bm, shape, weights)
    print(f"{name}: sampled near-ties {near}, rel-L2 {rel:.2e}, max abs {mx:.2e}, experts used {used}")


def test_full_size_page_implied_intermediate(bm):
    from sparse_moe_layer_fp32_b200 import synthetic
    shape = mi.SHAPES["decode8_i2560"]
    weights = synthetic.make_weights(shape, 0)
    near, rel, mx, used = _check_workload(bm, shape, weights)
    print(f"decode8_i2560: rel-L2 {rel:.2e}, max abs {mx:.2e}, experts used {used}")


@pytest.mark.parametrize("name", ["decode8", "prefill16k"])
def test_full_size_workload_mxfp8_experts(bm, name):
    # the block-scaled FP8 variant of the experts (MXFP8), same routing and finalize
    from sparse_moe_layer_fp32_b200 import synthetic
    shape = mi.SHAPES[name]
    weights = synthetic.make_weights(shape, 0, fmt="mxfp8")
    near, rel, mx, used = _check_workload(bm, shape, weights, fmt="mxfp8")
    del weights
    torch.cuda.empty_cache()
    print(f"{name} mxfp8: sampled near-ties {near}, rel-L2 {rel:.2e}, max abs {mx:.2e}, experts used {used}")
