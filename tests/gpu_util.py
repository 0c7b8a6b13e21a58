"""Helpers of the GPU parity tests: reading the library's internal buffers back into the
oracle's layouts, and the output comparison at the layer's tolerances."""

import numpy as np
import torch

import moe_inputs as mi
import sparse_moe_layer_fp32_b200 as bm
from oracle import moe, mxfp8, nvfp4

# Output tolerance of the layer against the oracle: relative L2 1e-2 and per-element
# absolute 5e-2 (tokens whose 8th/9th logit gap is a near-tie are excluded and counted).
REL_L2 = 1e-2
ABS_MAX = 5e-2


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def buf(layer, which, dtype):
    return to_np(layer.debug(which)).view(dtype)


ACT_CODE_BYTES = 16384  # codes of one activation unit (128 rows x 128 bytes)


def act_unit_bytes(block: int) -> int:
    """Bytes of one activation unit (one 128-row block, one K step): the codes, then the
    scales (NVFP4, block 16: 128 rows x 16; MXFP8, block 32: one 512-byte atom)."""
    return ACT_CODE_BYTES + (128 * 16 if block == 16 else 512)


def sf_rows(units: np.ndarray, sf_block: np.ndarray, offsets: np.ndarray, kcols: int, block: int = 16) -> np.ndarray:
    """Activation units (beam_moe.h layouts) -> row-major scales [rows, kcols/block] in
    permuted row order: block = 16 (NVFP4, each K step's 128 rows x 16 scales after its
    codes) or 32 (MXFP8, a 512-byte atom of 4 scales per row after each K step's codes)."""
    experts = len(offsets) - 1
    rows = int(offsets[-1])
    n_sc = kcols // block
    kgroups = n_sc // 4
    out = np.zeros((rows, n_sc), np.uint8)
    s = np.arange(n_sc)
    unit = act_unit_bytes(block)
    for e in range(experts):
        n = int(offsets[e + 1] - offsets[e])
        if n == 0:
            continue
        i = np.arange(n)
        blk = sf_block[e] + i // 128
        m = i % 128
        if block == 16:
            off = ((blk[:, None] * (n_sc // 16) + s[None, :] // 16) * unit + ACT_CODE_BYTES + m[:, None] * 16
                   + s[None, :] % 16)
        else:
            off = ((blk[:, None] * kgroups + s[None, :] // 4) * unit + ACT_CODE_BYTES + (m[:, None] % 32) * 16
                   + (m[:, None] // 32) * 4 + s[None, :] % 4)
        out[offsets[e]:offsets[e + 1]] = units[off]
    return out


def tile_rows(units: np.ndarray, sf_block: np.ndarray, offsets: np.ndarray, kcols: int,
              values_per_byte: int = 2) -> np.ndarray:
    """Activation units (beam_moe.h layout) -> codes [rows, kcols / values_per_byte] in
    permuted row order (2: packed NVFP4; 1: MXFP8).  A unit holds 128 code bytes of each row."""
    experts = len(offsets) - 1
    rows = int(offsets[-1])
    row_bytes = kcols // values_per_byte
    k_tiles = row_bytes // 128
    out = np.zeros((rows, row_bytes), np.uint8)
    j = np.arange(row_bytes)
    unit = act_unit_bytes(16 if values_per_byte == 2 else 32)
    for e in range(experts):
        n = int(offsets[e + 1] - offsets[e])
        if n == 0:
            continue
        i = np.arange(n)
        blk = (sf_block[e] + i // 128)[:, None]
        m = (i % 128)[:, None]
        off = ((blk * k_tiles + j[None, :] // 128) * unit + m * 128 + ((((j[None, :] % 128) // 16) ^ (m % 8)) * 16)
               + j[None, :] % 16)
        out[offsets[e]:offsets[e + 1]] = units[off]
    return out


def norm_zero(packed: np.ndarray) -> np.ndarray:
    """Map the E2M1 negative zero (code 8) to +0 in packed bytes (+-0 are equal values)."""
    c = nvfp4.unpack_nibbles(packed)
    c[c == 8] = 0
    return nvfp4.pack_nibbles(c)


def compare_outputs(gpu_out: np.ndarray, ref_pre: np.ndarray, skip=None):
    """Returns (rel_l2, max_abs) of the GPU output against the oracle's, rows in skip excluded."""
    keep = np.ones(gpu_out.shape[0], bool) if skip is None else ~np.asarray(skip, bool)
    g, r = gpu_out[keep], ref_pre[keep]
    if g.size == 0:
        return 0.0, 0.0
    rel = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30))
    return rel, float(np.max(np.abs(g - r)))


def ids_match(gpu_ids: np.ndarray, ref_ids: np.ndarray, logits: np.ndarray, near: np.ndarray, rel=1e-5):
    """Routing equality except at near-ties.  Slots whose logits are within the near-tie
    gap of a neighbour may swap order; everything else must match exactly."""
    bad = []
    for t in range(ref_ids.shape[0]):
        if near[t]:
            continue
        if set(gpu_ids[t].tolist()) != set(ref_ids[t].tolist()):
            bad.append(t)
            continue
        if not np.array_equal(gpu_ids[t], ref_ids[t]):
            lv = logits[t, ref_ids[t]]
            gap = np.abs(np.diff(lv))
            tol = rel * np.maximum(np.maximum(np.abs(lv[:-1]), np.abs(lv[1:])), 1.0)
            # every position that differs must sit next to a near-equal neighbour
            diff = np.nonzero(gpu_ids[t] != ref_ids[t])[0]
            if not all((j > 0 and gap[j - 1] < tol[j - 1]) or (j < len(gap) and gap[j] < tol[j]) for j in diff):
                bad.append(t)
    return bad


def ids_match_sel(gpu_ids: np.ndarray, ref_ids: np.ndarray, logits_sel: np.ndarray, near: np.ndarray, rel=1e-5):
    """ids_match with the oracle's logits of its chosen experts only (logits_sel[t, j] is the
    logit of ref_ids[t, j]), which is all the order check needs."""
    t_count, k = ref_ids.shape
    dense = np.zeros((t_count, int(max(ref_ids.max(), gpu_ids.max())) + 1), np.float64)
    np.put_along_axis(dense, ref_ids.astype(np.int64), logits_sel, axis=1)
    return ids_match(gpu_ids, ref_ids, dense, near, rel)


def oracle_batch_routing(x_bits: np.ndarray, router_w: np.ndarray, k: int, chunk: int = 4096):
    """The oracle's routing of a whole batch (FP64 logits, computed in chunks of tokens):
    ids [T, k], w [T, k], the chosen logits [T, k] and the near-tie mask [T]."""
    t_count = x_bits.shape[0]
    ids = np.empty((t_count, k), np.int64)
    w = np.empty((t_count, k), np.float64)
    lsel = np.empty((t_count, k), np.float64)
    near = np.empty(t_count, bool)
    for t0 in range(0, t_count, chunk):
        t1 = min(t_count, t0 + chunk)
        logits = moe.router_logits(mi.bf16_bits_to_f32(x_bits[t0:t1]), router_w)
        i, ww, _ = moe.route_topk(logits, k)
        ids[t0:t1], w[t0:t1] = i, ww
        lsel[t0:t1] = np.take_along_axis(logits, i, axis=1)
        near[t0:t1] = moe.near_tie_mask(logits, k)
    return ids, w, lsel, near


def weights_by_expert(ids: np.ndarray, w: np.ndarray, rows) -> tuple:
    """(ids, w) of the given rows with each row's slots sorted by expert id, so routing
    weights compare per (token, expert) whatever the slot order."""
    o = np.argsort(ids[rows], axis=1, kind="stable")
    return np.take_along_axis(ids[rows], o, 1), np.take_along_axis(w[rows], o, 1)


def oracle_layer_inputs(shape: mi.LayerShape, seed: int, weights_fp32=None, tokens=None, fmt: str = "nvfp4"):
    """Oracle-side inputs of a workload: x, residual (FP64 of BF16), W_r, gamma, expert cache."""
    xb, rb = mi.tokens(shape, seed) if tokens is None else tokens
    x = mi.bf16_bits_to_f32(xb).astype(np.float64)
    res = mi.bf16_bits_to_f32(rb).astype(np.float64)
    wr = mi.router_weight(shape, seed)
    g = mi.bf16_bits_to_f32(mi.gamma(shape, seed)).astype(np.float64)
    getter = weights_fp32 or (lambda e: mi.expert_weights(shape, seed, e))
    return x, res, wr, g, moe.ExpertCache(getter, keep=16, fmt=fmt)


# Relative width of the band around a rounding boundary inside which the GPU and the oracle
# may decide an A2 code or scale differently: the GPU's h comes from FP32 tensor-core sums of
# up to H exact products and an FP32 SiLU, the oracle's from FP64 (typically ~1e-6 apart).
A2_BOUNDARY_DELTA = 1e-4


def _boundary(encode, v, delta=A2_BOUNDARY_DELTA):
    """True where v scaled by (1 - delta) and by (1 + delta) encode differently."""
    v = np.asarray(v, np.float64)
    return encode((v * (1 - delta)).astype(np.float32)) != encode((v * (1 + delta)).astype(np.float32))


def a2_boundary_rows(gpu_codes, gpu_sf, h32, alpha2, fmt, delta=A2_BOUNDARY_DELTA):
    """Rows whose GPU A2 differs from the oracle's quantisation of the oracle's own h.

    gpu_codes / gpu_sf: the GPU's A2 of those rows (packed NVFP4 nibbles or E4M3 bytes, and
    scale codes); h32: the oracle's FP32 h [R, I].  Every difference must be a decision at a
    rounding boundary: a differing scale where the block's scale input moved by +-delta
    (relative) encodes to two codes, a differing code (in a block whose scales agree) where
    its quotient moved by +-delta does; both decisions are then valid at FP32 precision.
    Any other difference fails.  Returns a bool mask [R] of the rows that differ."""
    h = np.asarray(h32, np.float32)
    R, I = h.shape
    if fmt == "mxfp8":
        oc, osf = mxfp8.quantize_mxfp8(h)
        blocks = h.reshape(R, I // 32, 32).astype(np.float64)
        amax = np.abs(blocks).max(axis=-1)
        sb = (mxfp8.scale_exponent(amax * (1 - delta)) != mxfp8.scale_exponent(amax * (1 + delta)))
        q = np.ldexp(blocks, -mxfp8.scale_exponent(amax)[..., None]).reshape(R, I)
        cb = _boundary(mxfp8.e4m3_encode_signed, q, delta)
        gc, oc2, blk = np.asarray(gpu_codes), oc, 32
    else:
        pc, osf = nvfp4.quantize_nvfp4(h, alpha2)
        blocks = h.reshape(R, I // 16, 16)
        six_alpha = np.float32(np.float32(6.0) * np.float32(alpha2))
        s_in = (np.abs(blocks).max(axis=-1) / six_alpha).astype(np.float32)
        sb = _boundary(nvfp4.e4m3_encode, s_in, delta)
        d = (nvfp4.e4m3_decode(osf).astype(np.float32) * np.float32(alpha2)).astype(np.float32)
        q = (blocks / np.where(d == 0, np.float32(1), d)[..., None]).astype(np.float32).reshape(R, I)
        cb = _boundary(lambda v: nvfp4.e2m1_encode(np.abs(v)), q, delta)
        # +-0 compare equal; a nonzero code's sign is the value's sign on both sides
        gc, oc2, blk = nvfp4.unpack_nibbles(norm_zero(gpu_codes)), nvfp4.unpack_nibbles(norm_zero(pc)), 16
    s_diff = np.asarray(gpu_sf) != osf
    assert np.all(sb[s_diff]), "an A2 scale differs away from a rounding boundary"
    c_diff = (gc != oc2) & ~np.repeat(s_diff, blk, axis=1)
    assert np.all(cb[c_diff]), "an A2 code differs away from a rounding boundary"
    return s_diff.any(axis=1) | c_diff.any(axis=1)


def a2_boundary_tokens(layer, T, k, I, h32_tok, alpha2, fmt, skip=None):
    """Tokens of the layer's last forward (T tokens) whose A2 rows differ from the oracle's at
    rounding boundaries only (a2_boundary_rows; other differences fail).  h32_tok: the
    oracle's h [T, k, I] in slot order; tokens in skip (routing near-ties) are not compared."""
    mx = fmt == "mxfp8"
    kv, vpb, blk = (128, 1, 32) if mx else (256, 2, 16)
    Ip = (I + kv - 1) // kv * kv
    offsets = buf(layer, bm.BUF_OFFSETS, np.int32)
    sfb = buf(layer, bm.BUF_SFBLOCK, np.int32)
    inv = buf(layer, bm.BUF_INV, np.int32).reshape(-1, k)[:T]
    codes = tile_rows(buf(layer, bm.BUF_A2, np.uint8), sfb, offsets, Ip, values_per_byte=vpb)[:, : I // vpb]
    sf = sf_rows(buf(layer, bm.BUF_A2, np.uint8), sfb, offsets, Ip, block=blk)[:, : I // blk]
    keep = np.ones(T, bool) if skip is None else ~np.asarray(skip, bool)
    tok = np.nonzero(keep)[0]
    rows = inv[tok].reshape(-1)
    diff = a2_boundary_rows(codes[rows], sf[rows], np.asarray(h32_tok)[tok].reshape(-1, I), alpha2, fmt)
    out = np.zeros(T, bool)
    out[tok] = diff.reshape(-1, k).any(axis=1)
    return out
