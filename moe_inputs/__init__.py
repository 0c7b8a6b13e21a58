"""Seeded synthetic inputs of the sparse MoE layer, shared by the oracle side and the CUDA side.

This module only draws random numbers and casts dtypes; it holds none of the layer's
arithmetic (no routing, no quantisation, no GEMM, no normalisation).  Every tensor has its
own seeded stream: numpy's PCG64 seeded by SeedSequence([seed, tensor_id, index]), so any
expert's weights can be regenerated alone, bit for bit, on any machine with the same numpy.

Workloads (shapes from the pages: hidden 5120 and 256 experts in the router shape of the
vLLM PR "Day-0 support for Reflection's Beam-1.0", section "Status"; 8 of 256 experts in
the vLLM recipe "reflection/Beam-1.0-501B-A23B", section "Overview"; token counts follow
its workloads: 7 draft + 1 verify token in "DFlash2 speculative decoding", 128 sequences
at concurrency 128 and the 8 x 2K / 32K prefills in the PR's "Validation" section):

  x, residual ~ N(0, 1) rounded to BF16 (round-to-nearest-even)
  router W_r  ~ N(0, 1/H) FP32 (std 1/sqrt(H), so logits are ~N(0, 1))
  expert W    ~ N(0, 0.02^2) FP32, then quantised to NVFP4 by each side's own quantiser
  gamma       = 1 + 0.1 N(0, 1), rounded to BF16
  skewed routing (32K prefill): x[:, 0] = 1 and W_r[e, 0] = 2 log p(rank_e) with
  p(r) proportional to r^-1.1 over ranks 1..E, ranks a seeded permutation of the experts.
"""

from __future__ import annotations

import dataclasses
import json
import os

import numpy as np

TID_X, TID_RESIDUAL, TID_ROUTER, TID_GAMMA, TID_W_GU, TID_W_D, TID_SKEW = 1, 2, 3, 4, 5, 6, 7


@dataclasses.dataclass(frozen=True)
class LayerShape:
    name: str
    tokens: int
    hidden: int
    experts: int
    top_k: int
    inter: int
    skew: bool = False
    rms_eps: float = 1e-6

    @property
    def rows(self) -> int:
        return self.tokens * self.top_k


SHAPES = {
    s.name: s
    for s in [
        LayerShape("tiny", 4, 256, 16, 2, 128),
        LayerShape("decode8", 8, 5120, 256, 8, 1536),
        LayerShape("spec1024", 1024, 5120, 256, 8, 1536),
        LayerShape("prefill16k", 16384, 5120, 256, 8, 1536),
        LayerShape("prefill32k_skew", 32768, 5120, 256, 8, 1536, skew=True),
        # intermediate size implied by the pages' checkpoint sizes (a labelled extra)
        LayerShape("decode8_i2560", 8, 5120, 256, 8, 2560),
        # profiling case: the decode step's per-expert shapes with 32 experts, so that a
        # multi-pass profiler capture holds a few GB (weights still far larger than L2)
        LayerShape("decode8_e32", 8, 5120, 32, 8, 1536),
        # profiling case: the 8 x 2K prefill's rows per expert (512) with 32 experts
        LayerShape("prefill2k_e32", 2048, 5120, 32, 8, 1536),
        # profiling case: the 8 x 2K prefill's token count (per-token kernels see the full
        # batch: x 168 MB, A1 377 MB, y 1.34 GB, all larger than L2) with 32 experts' weights
        LayerShape("prefill16k_e32", 16384, 5120, 32, 8, 1536),
    ]
}


def _rng(seed: int, tid: int, idx: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed), int(tid), int(idx)]))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """FP32 -> BF16 bit patterns (uint16), round-to-nearest-even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """BF16 bit patterns -> exact FP32 values."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def skew_bias(shape: LayerShape, seed: int) -> np.ndarray:
    """Per-expert logit bias of the skewed workload, FP32 [E]."""
    ranks = _rng(seed, TID_SKEW).permutation(shape.experts) + 1
    p = ranks.astype(np.float64) ** -1.1
    p /= p.sum()
    return (2.0 * np.log(p)).astype(np.float32)


def tokens(shape: LayerShape, seed: int, t_begin: int = 0, t_end: int | None = None):
    """x and residual as BF16 bit patterns [T, H] (rows t_begin..t_end of the batch)."""
    t_end = shape.tokens if t_end is None else t_end
    out = []
    for tid in (TID_X, TID_RESIDUAL):
        # one stream per row, so any row range is reproducible on its own
        rows = np.empty((t_end - t_begin, shape.hidden), np.float32)
        for i, t in enumerate(range(t_begin, t_end)):
            rows[i] = _rng(seed, tid, t).standard_normal(shape.hidden, dtype=np.float32)
        if tid == TID_X and shape.skew:
            rows[:, 0] = 1.0
        out.append(f32_to_bf16_bits(rows))
    return out[0], out[1]


def router_weight(shape: LayerShape, seed: int) -> np.ndarray:
    w = _rng(seed, TID_ROUTER).standard_normal((shape.experts, shape.hidden), dtype=np.float32)
    w *= np.float32(1.0 / np.sqrt(shape.hidden))
    if shape.skew:
        w[:, 0] = skew_bias(shape, seed)
    return w


def gamma(shape: LayerShape, seed: int) -> np.ndarray:
    g = np.float32(1.0) + np.float32(0.1) * _rng(seed, TID_GAMMA).standard_normal(shape.hidden, dtype=np.float32)
    return f32_to_bf16_bits(g)


def expert_weights(shape: LayerShape, seed: int, e: int):
    """FP32 weights of expert e: w_gu [2I, H] (rows 0..I-1 gate, I..2I-1 up), w_d [H, I]."""
    w_gu = _rng(seed, TID_W_GU, e).standard_normal((2 * shape.inter, shape.hidden), dtype=np.float32)
    w_gu *= np.float32(0.02)
    w_d = _rng(seed, TID_W_D, e).standard_normal((shape.hidden, shape.inter), dtype=np.float32)
    w_d *= np.float32(0.02)
    return w_gu, w_d


_SCALES_FILE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "tests", "golden", "act_scales.json")


def activation_scales(shape: LayerShape):
    """Static FP32 activation tensor scales (alpha_a1, alpha_a2) of a workload.

    They were calibrated once on a seed-1 batch (amax / 2688) by the committed script
    tests/golden/calibrate_act_scales.py and are read here as stored data.
    """
    with open(_SCALES_FILE) as f:
        table = json.load(f)
    key = f"h{shape.hidden}_e{shape.experts}_k{shape.top_k}_i{shape.inter}"
    if key not in table:
        # the scales depend on the x and weight distributions, not on the expert count
        key = next(k for k in table if k.startswith(f"h{shape.hidden}_") and k.endswith(f"_k{shape.top_k}_i{shape.inter}"))
    a1, a2 = table[key]["alpha_a1"], table[key]["alpha_a2"]
    return np.float32(a1), np.float32(a2)
