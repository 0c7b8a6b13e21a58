"""Writes tests/golden/act_scales.json: the static FP32 activation tensor scales.

The layer quantises its activations with static tensor scales (alpha_a1 for the expert
inputs, alpha_a2 for the SwiGLU outputs), as NVFP4 W4A4 serving does with calibrated
scales (vLLM recipe "reflection/Beam-1.0-501B-A23B", section "Variants": NVFP4 routed
experts run W4A4 on Blackwell).  Calibration: amax over a seed-1 batch of the workload's
distribution, divided by 2688 (= 6 * 448, the largest NVFP4 magnitude at unit scale).
alpha_a1 comes from the generated x; alpha_a2 from the oracle's FP32 SwiGLU outputs h.

Calls only the oracle and the seeded generator.  Run: python tests/golden/calibrate_act_scales.py
"""

import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402
from oracle import moe  # noqa: E402

CAL_SEED = 1
CAL_TOKENS = {"tiny": 4, "decode8": 16, "decode8_i2560": 8}


def calibrate(shape, n_tokens):
    import dataclasses
    shp = dataclasses.replace(shape, tokens=max(n_tokens, shape.tokens if shape.tokens < 64 else n_tokens))
    xb, rb = mi.tokens(shp, CAL_SEED, 0, n_tokens)
    x = mi.bf16_bits_to_f32(xb)
    a1 = np.float32(np.float32(np.abs(x).max()) / np.float32(2688.0))
    res = mi.bf16_bits_to_f32(rb).astype(np.float64)
    wr = mi.router_weight(shp, CAL_SEED)
    g = mi.bf16_bits_to_f32(mi.gamma(shp, CAL_SEED)).astype(np.float64)
    cache = moe.ExpertCache(lambda e: mi.expert_weights(shp, CAL_SEED, e), keep=8)
    # alpha_a2 does not affect h (h is formed before A2 is quantised); pass a placeholder
    r = moe.moe_forward_tokens(x.astype(np.float64), res, wr, g, cache, shp.top_k, a1, np.float32(1.0))
    a2 = np.float32(np.float32(np.abs(r["h32"]).max()) / np.float32(2688.0))
    return float(a1), float(a2)


def main():
    table = {}
    for name, n in CAL_TOKENS.items():
        s = mi.SHAPES[name]
        key = f"h{s.hidden}_e{s.experts}_k{s.top_k}_i{s.inter}"
        a1, a2 = calibrate(s, n)
        table[key] = {"alpha_a1": a1, "alpha_a2": a2, "calibration": f"seed {CAL_SEED}, {n} tokens"}
        print(key, table[key], flush=True)
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "act_scales.json")
    with open(out, "w") as f:
        json.dump(table, f, indent=1, sort_keys=True)
        f.write("\n")


if __name__ == "__main__":
    main()
