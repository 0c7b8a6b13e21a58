"""Writes tests/golden/full_<workload>.npz: oracle outputs on sampled tokens of each
full-size workload, for the GPU parity tests (the oracle needs seconds per expert at
H = 5120, so it runs here once instead of on every GPU test run).

Each token's output depends only on that token (routing and experts are per token), so a
sample of rows of the whole batch is checked exactly.  Two samples per workload:

* tokens_full: up to 8 tokens with their whole output rows (out_pre [n, H]);
* tokens: at least 256 tokens (every token of smaller batches) with the output at 320
  columns (cols: 16 per 256-column output tile of the down GEMM, at both ends of each
  32-column half of every 64-column epilogue group).  The tokens are chosen from the
  oracle's routing of the whole batch so that every expert that receives rows has the
  first and the last row of its last 128-row block (the ragged one) in the sample; the
  rest are seeded random tokens.

A name ending in "_mxfp8" is the same workload with the MXFP8 variant of the experts.
Calls only the oracle and the seeded generator.
Run: python tests/golden/make_full_size_golden.py [name ...]
"""

import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402
from oracle import moe  # noqa: E402

SEED = 0
FULL_ROWS = {
    "decode8": list(range(8)),
    "spec1024": [0, 1, 137, 511, 512, 777, 1022, 1023],
    "prefill16k": [0, 1, 4095, 8191, 8192, 12000, 16382, 16383],
    "prefill32k_skew": [0, 1, 9999, 16383, 16384, 25000, 32766, 32767],
    "decode8_i2560": list(range(8)),
    "decode8_mxfp8": list(range(8)),
    "prefill16k_mxfp8": [0, 1, 4095, 8191, 8192, 12000, 16382, 16383],
}
MIN_SAMPLE = 256
CHUNK = 4096


def sample_columns(hidden: int) -> np.ndarray:
    within = np.array([0, 31, 32, 63, 64, 95, 96, 127, 128, 159, 160, 191, 192, 223, 224, 255])
    return (np.arange(hidden // 256)[:, None] * 256 + within[None, :]).reshape(-1)


def batch_routing(shape, seed):
    """The oracle's routing of the whole batch (FP64 logits in chunks of tokens)."""
    wr = mi.router_weight(shape, seed)
    ids = np.empty((shape.tokens, shape.top_k), np.int64)
    for t0 in range(0, shape.tokens, CHUNK):
        t1 = min(shape.tokens, t0 + CHUNK)
        xb, _ = mi.tokens(shape, seed, t0, t1)
        logits = moe.router_logits(mi.bf16_bits_to_f32(xb), wr)
        ids[t0:t1] = moe.route_topk(logits, shape.top_k)[0]
    return ids


def choose_tokens(shape, seed, ids):
    if shape.tokens <= MIN_SAMPLE:
        return np.arange(shape.tokens)
    pm = moe.permute(ids, shape.experts)
    off, src = pm["offsets"], pm["perm_src"]
    chosen = set()
    for e in range(shape.experts):
        c = int(off[e + 1] - off[e])
        if c == 0:
            continue
        last_block_first = int(off[e]) + (c - 1) // 128 * 128
        chosen.add(int(src[last_block_first]))
        chosen.add(int(src[int(off[e + 1]) - 1]))
    rng = np.random.default_rng(np.random.SeedSequence([seed, 991, shape.tokens]))
    while len(chosen) < MIN_SAMPLE:
        chosen.add(int(rng.integers(shape.tokens)))
    return np.array(sorted(chosen), np.int64)


def oracle_rows(shape, fmt, toks, cache):
    xs, rs = [], []
    for t in toks:
        xb, rb = mi.tokens(shape, SEED, int(t), int(t) + 1)
        xs.append(xb[0])
        rs.append(rb[0])
    x = mi.bf16_bits_to_f32(np.stack(xs)).astype(np.float64)
    res = mi.bf16_bits_to_f32(np.stack(rs)).astype(np.float64)
    wr = mi.router_weight(shape, SEED)
    g = mi.bf16_bits_to_f32(mi.gamma(shape, SEED)).astype(np.float64)
    a1, a2 = mi.activation_scales(shape) if fmt == "nvfp4" else (np.float32(1.0), np.float32(1.0))
    return moe.moe_forward_tokens(x, res, wr, g, cache, shape.top_k, a1, a2, shape.rms_eps), a1, a2


def make(name):
    fmt = "mxfp8" if name.endswith("_mxfp8") else "nvfp4"
    shape = mi.SHAPES[name[: -len("_mxfp8")] if fmt == "mxfp8" else name]
    t0 = time.time()
    toks = choose_tokens(shape, SEED, batch_routing(shape, SEED))
    full = np.array(FULL_ROWS[name], np.int64)
    cache = moe.ExpertCache(lambda e: mi.expert_weights(shape, SEED, e), keep=4, fmt=fmt)
    # experts in ascending order, each quantised once: moe_forward_tokens visits np.unique(ids)
    r, a1, a2 = oracle_rows(shape, fmt, toks, cache)
    rf, _, _ = oracle_rows(shape, fmt, full, cache)
    cols = sample_columns(shape.hidden)
    k = shape.top_k
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), f"full_{name}.npz")
    np.savez_compressed(
        path, tokens=toks, ids=r["ids"].astype(np.int16), w=r["w"],
        logits_sel=np.take_along_axis(r["logits"], r["ids"], axis=1), near_tie=r["near_tie"],
        cols=cols.astype(np.int32), out_cols=r["out_pre"][:, cols].astype(np.float32),
        tokens_full=full, ids_full=rf["ids"].astype(np.int16),
        logits_sel_full=np.take_along_axis(rf["logits"], rf["ids"], axis=1), near_tie_full=rf["near_tie"],
        out_pre_full=rf["out_pre"].astype(np.float32),
        seed=SEED, alpha_a1=a1, alpha_a2=a2, experts_format=fmt, top_k=k)
    print(f"{name}: {len(toks)} sampled tokens, {len(np.unique(r['ids']))} experts, "
          f"{int(r['near_tie'].sum())} near-ties, {time.time() - t0:.0f}s -> {path}", flush=True)


if __name__ == "__main__":
    for n in (sys.argv[1:] or list(FULL_ROWS)):
        make(n)
