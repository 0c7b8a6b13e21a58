"""Stage-by-stage parity on EVERY row at the layer's real contraction sizes: H = 5120 and
I = 1536, so the gate/up GEMM runs its full 20 K steps of 256 values (40 of 128 for MXFP8)
and the down GEMM 6 (12), through the shared-memory ring several times per tile, with
about 512 rows per expert (four 128-row blocks, the last one ragged).  32 experts instead
of 256 keep the oracle's FP64 GEMMs to seconds; the kernels and their tiling are those of
the full layer.

Each stage is checked on the GPU's own previous-stage output:
  routing ids/w      exact except near-ties (whole batch against the oracle's FP64 routing)
  offsets/perm/inv   bit-exact vs the oracle permutation of the GPU ids
  A1 codes/scales    bit-exact vs the oracle quantiser on the permuted x rows
  A2 (SwiGLU)        code mismatch rate and dequantised relative L2 per expert
  y                  relative L2 vs the oracle down GEMM of the GPU's A2
  out                vs the oracle finalize of the GPU's y, and end to end vs the oracle
                     (its own A2 and routing weights) on every token that is not a near-tie
Sources: router 5120 -> 256 and the fused finalize / sandwich norm (vLLM PR "Day-0
support for Reflection's Beam-1.0", section "Status"); NVFP4 W4A4 experts and the FP8
checkpoint (recipe "reflection/Beam-1.0-501B-A23B", section "Variants")."""

import dataclasses

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import moe_inputs as mi  # noqa: E402
from oracle import moe, mxfp8, nvfp4  # noqa: E402
from tests.gpu_util import (ABS_MAX, REL_L2, bf16_to_f64, buf, compare_outputs, ids_match_sel,  # noqa: E402
                            norm_zero, oracle_batch_routing, sf_rows, tile_rows, to_np)


@pytest.fixture(scope="module")
def bm():
    import sparse_moe_layer_fp32_b200 as m
    return m


def _deq_act(codes, sf, alpha, fmt):
    if fmt == "mxfp8":
        return mxfp8.dequantize_mxfp8(codes, sf)
    return nvfp4.dequantize_nvfp4(codes, sf, alpha)


@pytest.mark.parametrize("fmt,tokens,seed", [("nvfp4", 2048, 0), ("mxfp8", 1500, 0)])
def test_full_k_stages_on_every_row(bm, fmt, tokens, seed):
    from sparse_moe_layer_fp32_b200 import synthetic
    shape = dataclasses.replace(mi.SHAPES["prefill2k_e32"], tokens=tokens)
    T, E, k, H, I = shape.tokens, shape.experts, shape.top_k, shape.hidden, shape.inter
    mx = fmt == "mxfp8"
    kv = 128 if mx else 256
    Ip = (I + kv - 1) // kv * kv
    xb, rb = mi.tokens(shape, seed)
    res = mi.bf16_bits_to_f32(rb).astype(np.float64)
    x32 = mi.bf16_bits_to_f32(xb)
    wr = mi.router_weight(shape, seed)
    g = mi.bf16_bits_to_f32(mi.gamma(shape, seed)).astype(np.float64)
    a1, a2 = (None, None) if mx else mi.activation_scales(shape)
    weights = synthetic.make_weights(shape, seed, threads=8, fmt=fmt)
    layer = synthetic.make_layer(shape, weights, fmt=fmt)
    del weights
    out = layer.forward(synthetic.bf16_tensor(xb), synthetic.bf16_tensor(rb))
    layer.check()
    # ---- routing of every token
    ids = buf(layer, bm.BUF_IDS, np.int32).reshape(T, k).astype(np.int64)
    w = buf(layer, bm.BUF_WEIGHTS, np.float32).reshape(T, k).astype(np.float64)
    r_ids, r_w, r_lsel, near = oracle_batch_routing(xb, wr, k)
    assert not ids_match_sel(ids, r_ids, r_lsel, near)
    # ---- permutation of the GPU ids: bit-exact
    pm = moe.permute(ids, E)
    offsets = buf(layer, bm.BUF_OFFSETS, np.int32)
    perm = buf(layer, bm.BUF_PERM, np.int32)
    inv = buf(layer, bm.BUF_INV, np.int32).reshape(T, k)
    sfb = buf(layer, bm.BUF_SFBLOCK, np.int32)
    np.testing.assert_array_equal(offsets, pm["offsets"])
    np.testing.assert_array_equal(perm, pm["perm_src"])
    np.testing.assert_array_equal(inv, pm["inv"])
    assert any(c % 128 for c in pm["counts"] if c), "no ragged last block"
    # ---- A1: bit-exact on every row
    vpb, blk = (1, 32) if mx else (2, 16)
    a1c = tile_rows(buf(layer, bm.BUF_A1, np.uint8), sfb, offsets, H, values_per_byte=vpb)
    a1s = sf_rows(buf(layer, bm.BUF_A1, np.uint8), sfb, offsets, H, block=blk)
    if mx:
        rc, rs = mxfp8.quantize_mxfp8(x32[perm])
        np.testing.assert_array_equal(a1c, rc)
    else:
        rc, rs = nvfp4.quantize_nvfp4(x32[perm], a1)
        np.testing.assert_array_equal(norm_zero(a1c), norm_zero(rc))
    np.testing.assert_array_equal(a1s, rs)
    del rc, rs
    # ---- A2, y (from the GPU's own A1 / A2) and the oracle's own m, expert by expert
    a2c = tile_rows(buf(layer, bm.BUF_A2, np.uint8), sfb, offsets, Ip, values_per_byte=vpb)[:, : I // vpb]
    a2s = sf_rows(buf(layer, bm.BUF_A2, np.uint8), sfb, offsets, Ip, block=blk)[:, : I // blk]
    y = to_np(layer.debug(bm.BUF_Y).view(torch.bfloat16).float()).reshape(T * k, H)
    w_ref = np.zeros((T, E))
    np.put_along_axis(w_ref, r_ids, r_w, axis=1)
    m_ref = np.zeros((T, H))
    cache = moe.ExpertCache(lambda e: mi.expert_weights(shape, seed, e), keep=1, fmt=fmt)
    mism = n_codes = 0
    y_err2 = y_ref2 = 0.0
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if lo == hi:
            continue
        deq = cache.dequantized(e)
        r = moe.expert_forward(a1c[lo:hi], a1s[lo:hi], a1, deq, a2, fmt)
        if mx:
            mism += int((a2c[lo:hi] != r["a2_packed"]).sum())
            n_codes += a2c[lo:hi].size
        else:
            c_gpu = nvfp4.unpack_nibbles(norm_zero(a2c[lo:hi]))
            mism += int((c_gpu != nvfp4.unpack_nibbles(norm_zero(r["a2_packed"]))).sum())
            n_codes += c_gpu.size
        mism += int((a2s[lo:hi] != r["a2_sf"]).sum())
        d_gpu = _deq_act(a2c[lo:hi], a2s[lo:hi], a2, fmt)
        d_ref = _deq_act(r["a2_packed"], r["a2_sf"], a2, fmt)
        assert np.linalg.norm(d_gpu - d_ref) <= 1e-2 * max(np.linalg.norm(d_ref), 1e-30), e
        y_ref = d_gpu @ deq[1].T
        y_err2 += float(np.sum((y[lo:hi] - y_ref) ** 2))
        y_ref2 += float(np.sum(y_ref ** 2))
        tok = perm[lo:hi]  # each token at most once per expert
        m_ref[tok] += w_ref[tok, e][:, None] * r["y"]
    assert mism <= max(2, (5e-3 if mx else 1e-3) * n_codes), f"A2 mismatches {mism} of {n_codes}"
    rel_y = np.sqrt(y_err2 / max(y_ref2, 1e-30))
    assert rel_y < 5e-3, rel_y
    # ---- finalize of the GPU's own y, w, inv (in chunks of tokens)
    out_np = bf16_to_f64(out)
    for t0 in range(0, T, 256):
        t1 = min(T, t0 + 256)
        pre, _, _ = moe.finalize(y[inv[t0:t1]].astype(np.float64), w[t0:t1], res[t0:t1], g, shape.rms_eps)
        assert np.all(np.abs(out_np[t0:t1] - pre) <= 2.0 ** -8 * np.maximum(np.abs(pre), 1.0)), t0
    # ---- end to end against the oracle on every token that is not a near-tie
    pre_ref, _, _ = moe.finalize(m_ref[:, None, :], np.ones((T, 1)), res, g, shape.rms_eps)
    rel, mx_abs = compare_outputs(out_np, pre_ref, skip=near)
    assert rel <= REL_L2 and mx_abs <= ABS_MAX, (rel, mx_abs)
    print(f"{fmt} T={T}: near-ties {int(near.sum())}, A2 mismatches {mism}/{n_codes}, y rel-L2 {rel_y:.2e}, "
          f"out rel-L2 {rel:.2e} max abs {mx_abs:.2e}")
    layer.close()
