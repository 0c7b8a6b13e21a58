"""Writes tests/golden/full_<workload>.npz: oracle outputs on sampled tokens of each
full-size workload, for the GPU parity tests (the oracle needs seconds per expert at
H = 5120, so it runs here once instead of on every GPU test run).

Each token's output depends only on that token (routing and experts are per token), so a
sample of rows of the whole batch is checked exactly.  A name ending in "_mxfp8" is the
same workload with the MXFP8 variant of the experts.  Calls only the oracle and the
seeded generator.  Run: python tests/golden/make_full_size_golden.py [name ...]
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
SAMPLES = {
    "decode8": list(range(8)),
    "spec1024": [0, 1, 137, 511, 512, 777, 1022, 1023],
    "prefill16k": [0, 1, 4095, 8191, 8192, 12000, 16382, 16383],
    "prefill32k_skew": [0, 1, 9999, 16383, 16384, 25000, 32766, 32767],
    "decode8_i2560": list(range(8)),
    "decode8_mxfp8": list(range(8)),
    "prefill16k_mxfp8": [0, 1, 4095, 8191, 8192, 12000, 16382, 16383],
}


def make(name):
    fmt = "mxfp8" if name.endswith("_mxfp8") else "nvfp4"
    shape = mi.SHAPES[name[: -len("_mxfp8")] if fmt == "mxfp8" else name]
    toks = SAMPLES[name]
    xs, rs = [], []
    for t in toks:
        xb, rb = mi.tokens(shape, SEED, t, t + 1)
        xs.append(xb[0])
        rs.append(rb[0])
    xb, rb = np.stack(xs), np.stack(rs)
    x = mi.bf16_bits_to_f32(xb).astype(np.float64)
    res = mi.bf16_bits_to_f32(rb).astype(np.float64)
    wr = mi.router_weight(shape, SEED)
    g = mi.bf16_bits_to_f32(mi.gamma(shape, SEED)).astype(np.float64)
    a1, a2 = mi.activation_scales(shape) if fmt == "nvfp4" else (np.float32(1.0), np.float32(1.0))
    cache = moe.ExpertCache(lambda e: mi.expert_weights(shape, SEED, e), keep=4, fmt=fmt)
    t0 = time.time()
    r = moe.moe_forward_tokens(x, res, wr, g, cache, shape.top_k, a1, a2, shape.rms_eps)
    out_bits = (np.asarray(r["out"], np.float32).view(np.uint32) >> 16).astype(np.uint16)
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), f"full_{name}.npz")
    np.savez_compressed(
        path, tokens=np.array(toks, np.int64), ids=r["ids"].astype(np.int16), w=r["w"],
        logits=r["logits"].astype(np.float32), near_tie=r["near_tie"], out_pre=r["out_pre"].astype(np.float32),
        out_bf16=out_bits, seed=SEED, alpha_a1=a1, alpha_a2=a2, experts_format=fmt)
    print(f"{name}: {len(np.unique(r['ids']))} experts, {time.time() - t0:.0f}s -> {path}", flush=True)


if __name__ == "__main__":
    for n in (sys.argv[1:] or list(SAMPLES)):
        make(n)
