"""Full-size workloads (H 5120, 256 experts, top-8) through beam_moe_forward, in the launch
configuration bench.py times.

* Routing of the WHOLE batch against the oracle's (FP64 logits of every token, computed
  here in chunks): ids exact except near-ties (8th/9th logit gap below 1e-5 relative; their
  count is printed), weights per (token, expert) within 1e-5.
* Sampled tokens against oracle outputs stored by tests/golden/make_full_size_golden.py
  (each token's output depends only on that token, so a sample of the batch is exact):
  whole rows of 8 tokens, and 320 columns (every 256-column output tile) of at least 256
  tokens that include the first and last row of every used expert's last, ragged 128-row
  block; outputs within relative L2 1e-2 and absolute 5e-2.
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
from tests.gpu_util import (ABS_MAX, REL_L2, bf16_to_f64, buf, compare_outputs, ids_match_sel,  # noqa: E402
                            oracle_batch_routing, weights_by_expert)

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
    assert str(gold["experts_format"]) == fmt
    layer = synthetic.make_layer(shape, weights, fmt=fmt)
    xb, rb = mi.tokens(shape, 0)
    x, res = synthetic.bf16_tensor(xb), synthetic.bf16_tensor(rb)
    out = layer.forward(x, res)
    layer.check()
    T, k, E = shape.tokens, shape.top_k, shape.experts
    ids = buf(layer, bm.BUF_IDS, np.int32).reshape(T, k)
    w = buf(layer, bm.BUF_WEIGHTS, np.float32).reshape(T, k)
    offsets = buf(layer, bm.BUF_OFFSETS, np.int32)
    perm = buf(layer, bm.BUF_PERM, np.int32)
    inv = buf(layer, bm.BUF_INV, np.int32).reshape(T, k)
    out_np = bf16_to_f64(out)
    # ---- routing of every token against the oracle's
    r_ids, r_w, r_lsel, near_all = oracle_batch_routing(xb, mi.router_weight(shape, 0), k)
    bad = ids_match_sel(ids, r_ids, r_lsel, near_all)
    assert not bad, f"routing differs from the oracle at {len(bad)} tokens, e.g. {bad[:8]}"
    keep = np.nonzero(~near_all)[0]
    g_ids, g_w = weights_by_expert(ids.astype(np.int64), w.astype(np.float64), keep)
    o_ids, o_w = weights_by_expert(r_ids, r_w, keep)
    np.testing.assert_array_equal(g_ids, o_ids)
    np.testing.assert_allclose(g_w, o_w, rtol=0, atol=1e-5)
    # ---- sampled tokens against the stored oracle outputs: whole rows ...
    tf = gold["tokens_full"]
    near_f = gold["near_tie_full"]
    np.testing.assert_array_equal(gold["ids_full"].astype(np.int64)[~near_f], r_ids[tf][~near_f])
    rel_f, mx_f = compare_outputs(out_np[tf], gold["out_pre_full"].astype(np.float64), skip=near_f)
    assert rel_f <= REL_L2 and mx_f <= ABS_MAX, (rel_f, mx_f)
    # ... and 320 columns of >= 256 tokens
    toks, cols = gold["tokens"], gold["cols"]
    near = gold["near_tie"]
    np.testing.assert_array_equal(gold["ids"].astype(np.int64)[~near], r_ids[toks][~near])
    assert not ids_match_sel(ids[toks], gold["ids"].astype(np.int64), gold["logits_sel"], near)
    rel, mx = compare_outputs(out_np[toks][:, cols], gold["out_cols"].astype(np.float64), skip=near)
    assert rel <= REL_L2 and mx <= ABS_MAX, (rel, mx)
    # every used expert's last 128-row block has sampled rows
    pm = moe.permute(ids.astype(np.int64), E)
    sampled = np.zeros(T, bool)
    sampled[toks] = True
    for e in np.nonzero(pm["counts"])[0]:
        lo = int(pm["offsets"][e]) + (int(pm["counts"][e]) - 1) // 128 * 128
        assert sampled[pm["perm_src"][lo:int(pm["offsets"][e + 1])]].any(), e
    # ---- whole-batch properties
    assert np.all((ids >= 0) & (ids < E))
    assert np.all(np.sort(ids, 1)[:, 1:] != np.sort(ids, 1)[:, :-1])
    np.testing.assert_allclose(w.sum(1), 1.0, atol=1e-5)
    assert np.all(np.diff(w, axis=1) <= 1e-7)
    np.testing.assert_array_equal(offsets, pm["offsets"])
    np.testing.assert_array_equal(perm, pm["perm_src"])
    np.testing.assert_array_equal(inv, pm["inv"])
    assert np.isfinite(out_np).all()
    layer.close()
    return dict(near_ties=int(near_all.sum()), sampled=len(toks), rel=max(rel, rel_f), max_abs=max(mx, mx_f),
                used=int((np.diff(offsets) > 0).sum()))


@pytest.mark.parametrize("name", ["decode8", "spec1024", "prefill16k", "prefill32k_skew"])
def test_full_size_workload(bm, weights_i1536, name):
    shape = mi.SHAPES[name]
    weights = dict(weights_i1536)
    if shape.skew:
        weights["router_w"] = torch.from_numpy(mi.router_weight(shape, 0)).cuda()
    r = _check_workload(bm, shape, weights)
    print(f"{name}: {r}")


def test_full_size_page_implied_intermediate(bm):
    from sparse_moe_layer_fp32_b200 import synthetic
    shape = mi.SHAPES["decode8_i2560"]
    weights = synthetic.make_weights(shape, 0)
    r = _check_workload(bm, shape, weights)
    print(f"decode8_i2560: {r}")


@pytest.mark.parametrize("name", ["decode8", "prefill16k"])
def test_full_size_workload_mxfp8_experts(bm, name):
    # the block-scaled FP8 variant of the experts (MXFP8), same routing and finalize
    from sparse_moe_layer_fp32_b200 import synthetic
    shape = mi.SHAPES[name]
    weights = synthetic.make_weights(shape, 0, fmt="mxfp8")
    r = _check_workload(bm, shape, weights, fmt="mxfp8")
    del weights
    torch.cuda.empty_cache()
    print(f"{name} mxfp8: {r}")
