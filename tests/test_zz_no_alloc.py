"""beam_moe_route_static: routing for callers that cannot allocate device memory.

Some callers of this library cannot call cudaMalloc, for example a plugin inside a host
engine that owns all device memory and only hands the plugin its inputs and outputs, or a
latency-critical loop that must not allocate (nor risk the device synchronisation an
allocation can bring) once it is running.  beam_moe_route_static serves them: its logits
scratch is a fixed array compiled into the library, so the caller passes only x, the
router weights and the outputs.  The pages have no counterpart of this entry point.

The test calls it through the C ABI several times in a row, on different shapes (among
them the two that fill the array exactly with 2 and 1 slices of H), and checks each result
against the allocating entry point beam_moe_route at the routing tolerance of the other GPU
tests (ids equal, weights within 2e-5).  Shapes whose logits do not fit the array, including
those between the accepted token ranges, must be rejected.  This file is collected last.
"""

import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import moe_inputs as mi  # noqa: E402


def _inputs(name, tokens, seed):
    shape = mi.SHAPES[name]
    xb, _ = mi.tokens(shape, seed, 0, tokens)
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
    wr = torch.from_numpy(mi.router_weight(shape, seed)).cuda()
    return shape, x, wr


def _route_static(bm, x, wr, top_k):
    t_count, hidden = x.shape
    ids = torch.full((t_count, top_k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((t_count, top_k), -1.0, dtype=torch.float32, device="cuda")
    st = bm.lib().beam_moe_route_static(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(wr.data_ptr()), t_count,
                                        hidden, wr.shape[0], top_k, ctypes.c_void_p(ids.data_ptr()),
                                        ctypes.c_void_p(w.data_ptr()),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, ids, w


def test_route_static_matches_route_on_consecutive_calls():
    import sparse_moe_layer_fp32_b200 as bm

    results = []
    for name, tokens, seed in (("decode8", 8, 11), ("spec1024", 1024, 12), ("prefill16k", 4096, 14),
                               ("prefill16k", 8192, 15)):
        shape, x, wr = _inputs(name, tokens, seed)
        st, ids, w = _route_static(bm, x, wr, shape.top_k)
        assert st == bm.OK, bm.status_string(st)
        results.append((shape, x, wr, ids.clone(), w.clone()))
    torch.cuda.synchronize()
    for shape, x, wr, ids, w in results:
        ref_ids, ref_w = bm.beam_moe_route(x, wr, shape.top_k)
        torch.cuda.synchronize()
        assert torch.equal(ids, ref_ids)
        np.testing.assert_allclose(w.cpu().numpy(), ref_w.cpu().numpy(), rtol=0, atol=2e-5)


def test_route_static_rejects_shapes_beyond_its_array():
    import sparse_moe_layer_fp32_b200 as bm

    shape, x, wr = _inputs("decode8", 8, 13)
    # 16384 tokens x 256 experts of logits need 16 MiB, twice the fixed array: rejected
    # before anything is enqueued, so the (too short) pointers are never read
    st = bm.lib().beam_moe_route_static(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(wr.data_ptr()), 16384,
                                        5120, 256, 8, ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(x.data_ptr()),
                                        None)
    assert st == bm.ERR_UNSUPPORTED
    assert bm.beam_moe_route_workspace_bytes(16384, 5120, 256) > 8 << 20
    # between the accepted ranges: 1025..1152 tokens are summed over 8 slices of H, 4097..4672
    # over 2, so their logits need more than the array holds although 4096 and 8192 fit
    for tokens in (1025, 1100, 1152, 2049, 2304, 4097, 4672, 8193):
        st = bm.lib().beam_moe_route_static(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(wr.data_ptr()), tokens,
                                            5120, 256, 8, ctypes.c_void_p(x.data_ptr()),
                                            ctypes.c_void_p(x.data_ptr()), None)
        assert st == bm.ERR_UNSUPPORTED, tokens
        assert bm.beam_moe_route_workspace_bytes(tokens, 5120, 256) > 8 << 20, tokens
    for tokens in (1024, 1153, 2048, 2305, 4096, 4673, 8192):
        assert bm.beam_moe_route_workspace_bytes(tokens, 5120, 256) <= 8 << 20, tokens
