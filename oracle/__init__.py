"""CPU oracle for the Beam-style sparse MoE layer forward — TEST INFRASTRUCTURE ONLY.

This package is the plain, slow, obviously-correct definition that the CUDA path is
checked against.  Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline``
/ ``--impl reference`` legs of ``bench.py`` may import it.  The product library never
imports, links or executes anything in here, and this package imports nothing from the
product package: the two share no code.  The only module both sides use is the seeded
input generator ``moe_inputs``, which holds none of the layer's arithmetic.

Sources (web pages, cited by title and section):
  [P1] vLLM PR #61978 "Day-0 support for Reflection's Beam-1.0", sections "Status"
       (router GEMM kernels for (5120, 256); fused sandwich norms and MoE finalize) and
       "Remaining work" (moe_finalize.cu).
  [P2] vLLM recipe "reflection/Beam-1.0-501B-A23B", sections "Overview" (8 of 256
       routed experts) and "Variants" (NVFP4 routed experts, W4A4 on Blackwell; the
       router stays un-quantised).
  [P3] "vLLM adds day-zero Reflection Beam serving ...", section "Agents worked on the
       serving path" (specialised FP32 router kernel; fused normalisation/residual).
The pages fix the shapes and the precisions above; the rest (softmax over all experts,
renormalisation over the chosen k, SwiGLU, NVFP4 = E2M1 + one E4M3 scale per 16 values +
an FP32 tensor scale, post-RMSNorm with eps 1e-6) is the stated convention of the layer
this repository implements.

Precision: every floating-point step is FP64 except the NVFP4 quantiser, whose steps are
IEEE FP32 operations by definition (so codes are reproducible bit for bit).  The MXFP8
variant of the experts (``mxfp8.py``: E4M3 values, one power-of-two scale per 32 values)
needs no FP32 step: its scaling is exact.

Parity status: every function here is pinned by ``tests/test_oracle_*.py`` (library
routines for the rounding, closed forms, brute force and invariants).  No function is
"parity unpinned".
"""

from .nvfp4 import (  # noqa: F401
    E2M1_VALUES,
    e2m1_encode,
    e2m1_decode,
    e4m3_encode,
    e4m3_decode,
    tensor_scale,
    quantize_nvfp4,
    dequantize_nvfp4,
    pack_nibbles,
    unpack_nibbles,
)
from .mxfp8 import (  # noqa: F401
    e4m3_encode_signed,
    e4m3_decode_signed,
    scale_exponent,
    ue8m0_decode,
    quantize_mxfp8,
    dequantize_mxfp8,
)
from .moe import (  # noqa: F401
    router_logits,
    route_topk,
    near_tie_mask,
    permute,
    expert_forward,
    finalize,
    next_prenorm,
    moe_forward,
    moe_forward_tokens,
    shard_dequantized,
    moe_forward_tp,
    moe_forward_ep,
)
