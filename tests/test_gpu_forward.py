"""Whole-layer GPU forward (beam_moe_forward through the C ABI) against the oracle, stage by
stage and end to end, on small shapes that still span several tiles and ragged tails.

Each stage is checked on the GPU's own previous-stage output, so one stage's rounding does
not cascade into the next check:
  routing ids/w      exact except near-ties
  offsets/perm/inv   bit-exact vs the oracle permutation of the GPU ids
  A1 codes/scales    bit-exact vs the oracle quantiser on the permuted x rows
  A2 (SwiGLU NVFP4)  code mismatch rate (GPU FP32 h vs oracle FP64 h may straddle a
                     rounding boundary) and dequantised relative L2
  y                  relative L2 vs the oracle down GEMM of the GPU's A2
  out                vs the oracle finalize of the GPU's y, and end to end vs the oracle
Sources: router 5120 -> 256 and the fused finalize/sandwich norm (vLLM PR "Day-0 support
for Reflection's Beam-1.0", section "Status"); 8 of 256 experts and NVFP4 W4A4 experts
(recipe "reflection/Beam-1.0-501B-A23B", sections "Overview" and "Variants")."""

import dataclasses

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import moe_inputs as mi  # noqa: E402
from oracle import moe, nvfp4  # noqa: E402
from tests.gpu_util import (ABS_MAX, REL_L2, bf16_to_f64, buf, compare_outputs, ids_match, norm_zero,  # noqa: E402
                            oracle_layer_inputs, sf_rows, tile_rows, to_np)


@pytest.fixture(scope="module")
def bm():
    import sparse_moe_layer_fp32_b200 as m
    return m


# (name, shape) — tiny is the workload of the same name; "mid" spans 2-3 output tiles and
# 2 K tiles per GEMM with an intermediate size that needs K padding (384 -> 512).
SHAPES = {
    "tiny": mi.SHAPES["tiny"],
    "mid": mi.LayerShape("mid", 0, 512, 32, 4, 384),
}


def _scales(shape, x, res, wr, g, cache):
    a1 = np.float32(np.float32(np.abs(x).max()) / np.float32(2688))
    r = moe.moe_forward_tokens(x, res, wr, g, cache, shape.top_k, a1, np.float32(1.0))
    return a1, np.float32(np.float32(np.abs(r["h32"]).max()) / np.float32(2688))


def _run(bm, shape, tokens, seed, max_tokens=None):
    from sparse_moe_layer_fp32_b200 import synthetic
    shape = dataclasses.replace(shape, tokens=tokens)
    x, res, wr, g, cache = oracle_layer_inputs(shape, seed)
    a1, a2 = _scales(shape, x, res, wr, g, cache)
    weights = synthetic.make_weights(shape, seed, threads=4)
    layer = bm.MoELayer(max_tokens=max_tokens or max(tokens, 1), hidden=shape.hidden, num_experts=shape.experts,
                        top_k=shape.top_k, inter=shape.inter, alpha_a1=float(a1), alpha_a2=float(a2), **weights)
    xd, rd = synthetic.make_batch(shape, seed)
    out = layer.forward(xd, rd)
    layer.check()
    ref = moe.moe_forward(x, res, wr, g, cache, shape.experts, shape.top_k, a1, a2, shape.rms_eps)
    return shape, layer, weights, out, ref, (x, res, wr, g, cache, a1, a2)


@pytest.mark.parametrize("name,tokens,seed", [("tiny", 4, 0), ("tiny", 1, 1), ("tiny", 37, 2), ("tiny", 1500, 3),
                                              ("mid", 200, 4), ("mid", 7, 5), ("mid", 4500, 13),
                                              ("tiny", 19500, 14)])
def test_forward_stages_and_end_to_end(bm, name, tokens, seed):
    shape, layer, weights, out, ref, (x, res, wr, g, cache, a1, a2) = _run(bm, SHAPES[name], tokens, seed)
    T, E, k, H, I = tokens, shape.experts, shape.top_k, shape.hidden, shape.inter
    Ip = (I + 255) // 256 * 256
    # ---- routing
    ids = buf(layer, bm.BUF_IDS, np.int32).reshape(T, k)
    w = buf(layer, bm.BUF_WEIGHTS, np.float32).reshape(T, k)
    near = ref["near_tie"]
    assert not ids_match(ids, ref["ids"], ref["logits"], near)
    np.testing.assert_allclose(w.sum(1), 1.0, atol=1e-5)
    # ---- permutation of the GPU ids: bit-exact
    pm = moe.permute(ids.astype(np.int64), E)
    offsets = buf(layer, bm.BUF_OFFSETS, np.int32)
    perm = buf(layer, bm.BUF_PERM, np.int32)
    inv = buf(layer, bm.BUF_INV, np.int32).reshape(T, k)
    sfb = buf(layer, bm.BUF_SFBLOCK, np.int32)
    np.testing.assert_array_equal(offsets, pm["offsets"])
    np.testing.assert_array_equal(perm, pm["perm_src"])
    np.testing.assert_array_equal(inv, pm["inv"])
    nblk = np.array([(c + 127) // 128 for c in pm["counts"]])
    np.testing.assert_array_equal(sfb, np.concatenate([[0], np.cumsum(nblk)]))
    # ---- A1: bit-exact
    a1p = tile_rows(buf(layer, bm.BUF_A1, np.uint8), sfb, offsets, H)
    a1s = sf_rows(buf(layer, bm.BUF_A1, np.uint8), sfb, offsets, H)
    rp, rs = nvfp4.quantize_nvfp4(x[perm].astype(np.float32), a1)
    np.testing.assert_array_equal(a1s, rs)
    np.testing.assert_array_equal(norm_zero(a1p), norm_zero(rp))
    # ---- A2 and y from the GPU's own inputs
    a2p = tile_rows(buf(layer, bm.BUF_A2, np.uint8), sfb, offsets, Ip)[:, : I // 2]
    a2s = sf_rows(buf(layer, bm.BUF_A2, np.uint8), sfb, offsets, Ip)[:, : I // 16]
    y = to_np(layer.debug(bm.BUF_Y).view(torch.bfloat16).float()).reshape(T * k, H).astype(np.float64)
    mism, n_codes = 0, 0
    y_ref = np.zeros_like(y)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if lo == hi:
            continue
        deq = cache.dequantized(e)
        r = moe.expert_forward(a1p[lo:hi], a1s[lo:hi], a1, deq, a2)
        c_gpu = nvfp4.unpack_nibbles(norm_zero(a2p[lo:hi]))
        c_ref = nvfp4.unpack_nibbles(norm_zero(r["a2_packed"]))
        mism += int((c_gpu != c_ref).sum()) + int((a2s[lo:hi] != r["a2_sf"]).sum())
        n_codes += c_gpu.size
        y_ref[lo:hi] = nvfp4.dequantize_nvfp4(a2p[lo:hi], a2s[lo:hi], a2) @ deq[1].T
        d_gpu = nvfp4.dequantize_nvfp4(a2p[lo:hi], a2s[lo:hi], a2)
        d_ref = nvfp4.dequantize_nvfp4(r["a2_packed"], r["a2_sf"], a2)
        assert np.linalg.norm(d_gpu - d_ref) <= 1e-2 * max(np.linalg.norm(d_ref), 1e-30)
    assert mism <= max(2, 1e-3 * n_codes), f"A2 mismatches {mism} of {n_codes}"
    rel_y = np.linalg.norm(y - y_ref) / max(np.linalg.norm(y_ref), 1e-30)
    assert rel_y < 5e-3, rel_y
    # ---- finalize of the GPU's own y, w, inv
    out_np = bf16_to_f64(out)
    pre, _, _ = moe.finalize(y[inv], w.astype(np.float64), res, g, shape.rms_eps)
    assert np.all(np.abs(out_np - pre) <= 2.0 ** -8 * np.maximum(np.abs(pre), 1.0))
    # ---- end to end
    rel, mx = compare_outputs(out_np, ref["out_pre"], skip=near)
    assert rel <= REL_L2 and mx <= ABS_MAX, (rel, mx)
    assert layer.launches() > 0
    layer.close()


def test_forward_edge_cases(bm):
    from sparse_moe_layer_fp32_b200 import synthetic
    shape = dataclasses.replace(SHAPES["tiny"], tokens=6)
    weights = synthetic.make_weights(shape, 0, threads=2)
    layer = bm.MoELayer(max_tokens=6, hidden=shape.hidden, num_experts=shape.experts, top_k=shape.top_k,
                        inter=shape.inter, alpha_a1=0.0012, alpha_a2=0.00012, **weights)
    x, r = synthetic.make_batch(shape, 0)
    out = layer.forward(x, r)
    # in place: out == residual
    r2 = r.clone()
    layer.forward(x, r2, out=r2)
    torch.cuda.synchronize()
    assert torch.equal(out, r2)
    # zero tokens is a no-op; more than max_tokens is rejected before launching
    layer.forward(x[:0], r[:0])
    with pytest.raises(bm.BeamMoeError) as ei:
        bm.beam_moe_forward(layer.handle, torch.cat([x, x[:1]]), torch.cat([r, r[:1]]), torch.empty_like(
            torch.cat([r, r[:1]])), 7)
    assert ei.value.status == bm.ERR_INVALID_ARG
    # repeated calls are deterministic
    o1 = layer.forward(x, r)
    o2 = layer.forward(x, r)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    layer.check()
    layer.close()


def test_bounded_wait_reports_timeout_and_context_survives(bm):
    # Failure detection without a GPU fault: a wait that nothing completes gives up after
    # 50 ms, the error word says TIMEOUT, and the next forward still runs correctly.
    from sparse_moe_layer_fp32_b200 import synthetic
    shape = dataclasses.replace(SHAPES["tiny"], tokens=4)
    weights = synthetic.make_weights(shape, 0, threads=2)
    layer = bm.MoELayer(max_tokens=4, hidden=shape.hidden, num_experts=shape.experts, top_k=shape.top_k,
                        inter=shape.inter, alpha_a1=0.0012, alpha_a2=0.00012, **weights)
    x, r = synthetic.make_batch(shape, 0)
    before = layer.forward(x, r)
    layer.check()
    bm.beam_moe_debug_wait_timeout(layer.handle, 50_000_000)
    with pytest.raises(bm.BeamMoeError) as ei:
        layer.check()
    assert ei.value.status == bm.ERR_TIMEOUT
    layer.check()  # the error word was cleared by the check that reported it
    after = layer.forward(x, r)
    layer.check()
    assert torch.equal(before, after)
    with pytest.raises(bm.BeamMoeError):
        bm.beam_moe_debug_wait_timeout(layer.handle, 0)
    layer.close()


@pytest.mark.parametrize("name,tokens,seed", [("tiny", 5, 7), ("tiny", 300, 8), ("mid", 9, 9)])
def test_forward_with_fused_next_prenorm(bm, name, tokens, seed):
    # The next sublayer's sandwich pre-norm fused into the finalize: out is unchanged and
    # next_x = bf16(RMSNorm(out) * gamma_next), checked on the GPU's own out (one BF16
    # rounding apart) and end to end against the oracle.
    shape, layer, weights, out_plain, ref, (x, res, wr, g, cache, a1, a2) = _run(bm, SHAPES[name], tokens, seed)
    from sparse_moe_layer_fp32_b200 import synthetic
    xd, rd = synthetic.make_batch(shape, seed)
    g_next_bits = mi.gamma(dataclasses.replace(shape, name="next"), seed + 100)
    g_next = synthetic.bf16_tensor(g_next_bits)
    out, next_x = layer.forward_prenorm(xd, rd, g_next, 1e-6)
    layer.check()
    torch.cuda.synchronize()
    assert torch.equal(out, out_plain)
    gn = mi.bf16_bits_to_f32(g_next_bits).astype(np.float64)
    pre, _ = moe.next_prenorm(bf16_to_f64(out), gn, 1e-6)
    nx = bf16_to_f64(next_x)
    assert np.all(np.abs(nx - pre) <= 2.0 ** -7 * np.maximum(np.abs(pre), 2.0 ** -6))
    pre_ref, _ = moe.next_prenorm(ref["out"], gn, 1e-6)
    rel, mx = compare_outputs(nx, pre_ref, skip=ref["near_tie"])
    assert rel <= REL_L2 and mx <= ABS_MAX, (rel, mx)
    with pytest.raises(bm.BeamMoeError):
        layer.forward_prenorm(xd, rd, g_next, 1e-6, next_x=rd)  # next_x may not alias residual
    layer.close()


# ---------------------------------------------------------------- MXFP8 experts
# The block-scaled FP8 variant (the recipe's FP8 checkpoint, section "Variants", read as
# MXFP8: E4M3 values and one power-of-two scale per 32 values for weights, A1 and A2),
# created with beam_moe_create_mxfp8.  Stages as above: routing and permutation are the
# format-independent kernels; A1 is bit-exact (codes and scales, sign of zero included);
# A2 codes may differ where the GPU's FP32 SwiGLU and the oracle's FP64 one straddle a
# rounding boundary; y, finalize and the end-to-end output at the layer's tolerances.
@pytest.mark.parametrize("name,tokens,seed", [("tiny", 4, 20), ("tiny", 37, 21), ("tiny", 1500, 22), ("mid", 7, 23),
                                              ("mid", 200, 24), ("mid", 4500, 25)])
def test_forward_mxfp8_stages_and_end_to_end(bm, name, tokens, seed):
    from oracle import mxfp8
    from sparse_moe_layer_fp32_b200 import synthetic
    shape = dataclasses.replace(SHAPES[name], tokens=tokens)
    x, res, wr, g, cache = oracle_layer_inputs(shape, seed, fmt="mxfp8")
    weights = synthetic.make_weights(shape, seed, threads=4, fmt="mxfp8")
    layer = bm.MoELayer(max_tokens=tokens, hidden=shape.hidden, num_experts=shape.experts, top_k=shape.top_k,
                        inter=shape.inter, fmt="mxfp8", **weights)
    assert bm.beam_moe_expert_format(layer.handle) == bm.FMT_MXFP8
    xd, rd = synthetic.make_batch(shape, seed)
    out = layer.forward(xd, rd)
    layer.check()
    ref = moe.moe_forward(x, res, wr, g, cache, shape.experts, shape.top_k, None, None, shape.rms_eps)
    T, E, k, H, I = tokens, shape.experts, shape.top_k, shape.hidden, shape.inter
    ids = buf(layer, bm.BUF_IDS, np.int32).reshape(T, k)
    w = buf(layer, bm.BUF_WEIGHTS, np.float32).reshape(T, k)
    near = ref["near_tie"]
    assert not ids_match(ids, ref["ids"], ref["logits"], near)
    pm = moe.permute(ids.astype(np.int64), E)
    offsets = buf(layer, bm.BUF_OFFSETS, np.int32)
    perm = buf(layer, bm.BUF_PERM, np.int32)
    inv = buf(layer, bm.BUF_INV, np.int32).reshape(T, k)
    sfb = buf(layer, bm.BUF_SFBLOCK, np.int32)
    np.testing.assert_array_equal(offsets, pm["offsets"])
    np.testing.assert_array_equal(perm, pm["perm_src"])
    np.testing.assert_array_equal(inv, pm["inv"])
    # ---- A1 = MX(x rows): bit-exact
    a1c = tile_rows(buf(layer, bm.BUF_A1, np.uint8), sfb, offsets, H, values_per_byte=1)
    a1s = sf_rows(buf(layer, bm.BUF_A1, np.uint8), sfb, offsets, H, block=32)
    rc, rs = mxfp8.quantize_mxfp8(x[perm].astype(np.float32))
    np.testing.assert_array_equal(a1s, rs)
    np.testing.assert_array_equal(a1c, rc)
    # ---- A2 and y from the GPU's own A1
    a2c = tile_rows(buf(layer, bm.BUF_A2, np.uint8), sfb, offsets, I, values_per_byte=1)
    a2s = sf_rows(buf(layer, bm.BUF_A2, np.uint8), sfb, offsets, I, block=32)
    y = to_np(layer.debug(bm.BUF_Y).view(torch.bfloat16).float()).reshape(T * k, H).astype(np.float64)
    mism, n_codes = 0, 0
    y_ref = np.zeros_like(y)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if lo == hi:
            continue
        deq = cache.dequantized(e)
        r = moe.expert_forward(a1c[lo:hi], a1s[lo:hi], None, deq, None, "mxfp8")
        mism += int((a2c[lo:hi] != r["a2_packed"]).sum()) + int((a2s[lo:hi] != r["a2_sf"]).sum())
        n_codes += a2c[lo:hi].size
        d_gpu = mxfp8.dequantize_mxfp8(a2c[lo:hi], a2s[lo:hi])
        d_ref = mxfp8.dequantize_mxfp8(r["a2_packed"], r["a2_sf"])
        assert np.linalg.norm(d_gpu - d_ref) <= 1e-2 * max(np.linalg.norm(d_ref), 1e-30)
        y_ref[lo:hi] = d_gpu @ deq[1].T
    assert mism <= max(2, 5e-3 * n_codes), f"A2 mismatches {mism} of {n_codes}"
    rel_y = np.linalg.norm(y - y_ref) / max(np.linalg.norm(y_ref), 1e-30)
    assert rel_y < 5e-3, rel_y
    out_np = bf16_to_f64(out)
    pre, _, _ = moe.finalize(y[inv], w.astype(np.float64), res, g, shape.rms_eps)
    assert np.all(np.abs(out_np - pre) <= 2.0 ** -8 * np.maximum(np.abs(pre), 1.0))
    rel, mx = compare_outputs(out_np, ref["out_pre"], skip=near)
    assert rel <= REL_L2 and mx <= ABS_MAX, (rel, mx)
    layer.close()


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp8"])
def test_forward_host_buffers_match_device_path(bm, fmt):
    # beam_moe_forward_host: x uploads on the caller's stream, the residual on the handle's
    # copy stream (overlapping routing and GEMMs, the finalize waits for it), out comes back
    # on the caller's stream.  Same bits as the device-buffer forward, call after call with
    # changing batch sizes (the staging buffers are reused), pinned or pageable host memory.
    from sparse_moe_layer_fp32_b200 import synthetic
    shape = dataclasses.replace(SHAPES["mid"], tokens=300)
    weights = synthetic.make_weights(shape, 3, threads=4, fmt=fmt)
    if fmt == "nvfp4":
        layer = bm.MoELayer(max_tokens=300, hidden=shape.hidden, num_experts=shape.experts, top_k=shape.top_k,
                            inter=shape.inter, alpha_a1=0.002, alpha_a2=0.0002, **weights)
    else:
        layer = bm.MoELayer(max_tokens=300, hidden=shape.hidden, num_experts=shape.experts, top_k=shape.top_k,
                            inter=shape.inter, fmt="mxfp8", **weights)
    xd, rd = synthetic.make_batch(shape, 3)
    for T, pinned in [(300, True), (7, True), (300, False), (64, True), (1, False)]:
        xh, rh = xd[:T].cpu(), rd[:T].cpu()
        oh = torch.empty_like(rh)
        if pinned:
            xh, rh, oh = xh.pin_memory(), rh.pin_memory(), oh.pin_memory()
        layer.forward_host(xh, rh, oh)
        torch.cuda.synchronize()
        ref = layer.forward(xd[:T], rd[:T])
        torch.cuda.synchronize()
        assert torch.equal(oh, ref.cpu()), (T, pinned)
    layer.check()
    layer.close()


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp8"])
def test_forward_host_in_parts_matches_device_path(bm, fmt):
    # beam_moe_forward_host of a batch of 2 parts or more: each part uploads, computes and
    # copies back on its own schedule, with the whole batch's router (forms, slices and the
    # K order of each token tile), finalize and GEMM forms.  Same bits as the device-buffer
    # forward of the whole batch, for parts of 256 and 512 tokens, ragged last parts (one of
    # 188 tokens: the small-batch A1 writer inside it), call after call.
    from sparse_moe_layer_fp32_b200 import synthetic
    shape = dataclasses.replace(SHAPES["mid"], tokens=700)
    weights = synthetic.make_weights(shape, 5, threads=4, fmt=fmt)
    kw = dict(alpha_a1=0.002, alpha_a2=0.0002) if fmt == "nvfp4" else dict(fmt="mxfp8")
    layer = bm.MoELayer(max_tokens=700, hidden=shape.hidden, num_experts=shape.experts, top_k=shape.top_k,
                        inter=shape.inter, **kw, **weights)
    xd, rd = synthetic.make_batch(shape, 5)
    with pytest.raises(bm.BeamMoeError):
        layer.set_host_chunk_tokens(100)  # parts align with the router's token tiles
    for chunk, T in [(256, 700), (512, 700), (256, 512), (256, 511), (0, 700), (256, 700)]:
        layer.set_host_chunk_tokens(chunk)
        xh, rh = xd[:T].cpu().pin_memory(), rd[:T].cpu().pin_memory()
        oh = torch.empty_like(rh).pin_memory()
        layer.forward_host(xh, rh, oh)
        torch.cuda.synchronize()
        layer.check()
        ref = layer.forward(xd[:T], rd[:T])
        torch.cuda.synchronize()
        assert torch.equal(oh, ref.cpu()), (chunk, T)
    layer.check()
    layer.close()


def test_profiled_sections_and_launch_counts(bm):
    """Per-kernel timing of a forward (beam_moe_profile_enable / _read): one named section per
    kernel launched, in launch order, ending with the finalize; the output is the same bits
    with timing on."""
    from sparse_moe_layer_fp32_b200 import synthetic
    shape = dataclasses.replace(SHAPES["mid"], tokens=300)
    weights = synthetic.make_weights(shape, 31, threads=4)
    layer = bm.MoELayer(max_tokens=300, hidden=shape.hidden, num_experts=shape.experts, top_k=shape.top_k,
                        inter=shape.inter, alpha_a1=0.01, alpha_a2=0.01, **weights)
    for T in (8, 40, 255, 256, 300):
        x, r = synthetic.make_batch(dataclasses.replace(shape, tokens=T), T)
        x, r = x.cuda(), r.cuda()
        plain = layer.forward(x, r)
        layer.check()
        layer.profile(True)
        timed = layer.forward(x, r)
        sections = layer.kernel_times()
        layer.profile(False)
        layer.check()
        assert torch.equal(plain, timed), T
        names = [n for n, _ in sections]
        assert names[-1] == "finalize" and names.count("quant_a1") == 1 and "gemm_experts" in names, names
        assert all(ms >= 0 for _, ms in sections)
        assert layer.launches() == len(names), (T, names)
    layer.close()


@pytest.mark.parametrize("tokens", [8, 300])
def test_forward_replays_from_a_cuda_graph(bm, tokens):
    # The forward enqueues only kernels on the caller's stream (no allocation, no host sync),
    # so it can be captured in a CUDA graph once and replayed; each replay gives the eager
    # forward's bits, and replays of new inputs copied into the captured buffers follow them.
    from sparse_moe_layer_fp32_b200 import synthetic
    shape = dataclasses.replace(SHAPES["mid"], tokens=tokens)
    weights = synthetic.make_weights(shape, 9, threads=4)
    layer = bm.MoELayer(max_tokens=tokens, hidden=shape.hidden, num_experts=shape.experts, top_k=shape.top_k,
                        inter=shape.inter, alpha_a1=0.002, alpha_a2=0.0002, **weights)
    x0, r0 = synthetic.make_batch(shape, 9)
    x1, r1 = synthetic.make_batch(shape, 10)
    x, r = x0.cuda().clone(), r0.cuda().clone()
    out = torch.empty_like(r)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        layer.forward(x, r, out)
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer.forward(x, r, out)
    for xs, rs in [(x0, r0), (x1, r1), (x0, r0)]:
        x.copy_(xs.cuda())
        r.copy_(rs.cuda())
        g.replay()
        torch.cuda.synchronize()
        layer.check()
        assert torch.equal(out, layer.forward(xs.cuda(), rs.cuda()))
    del g
    layer.close()
