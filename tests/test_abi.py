"""The C-ABI library loads and exports every symbol that include/beam_moe.h declares;
host-side argument checks answer without touching a GPU."""

import ctypes
import os
import re

import pytest


def _declared(repo_root):
    text = open(os.path.join(repo_root, "include", "beam_moe.h")).read()
    return sorted(set(re.findall(r"BEAM_MOE_API\s+[\w\s\*]+?\b(beam_moe_\w+)\s*\(", text)))


def test_header_declares_the_binding_names(repo_root):
    import sparse_moe_layer_fp32_b200 as pkg
    assert _declared(repo_root) == sorted(pkg.EXPORTED)


def test_header_constants_match_the_binding(repo_root):
    import sparse_moe_layer_fp32_b200 as pkg
    text = open(os.path.join(repo_root, "include", "beam_moe.h")).read()
    m = re.search(r"#define BEAM_MOE_TP_TWO_SHOT_MIN_TOKENS (\d+)", text)
    assert m and int(m.group(1)) == pkg.TP_TWO_SHOT_MIN_TOKENS
    m = re.search(r"#define BEAM_MOE_HOST_CHUNK_TOKENS (\d+)", text)
    assert m and int(m.group(1)) == pkg.HOST_CHUNK_TOKENS


def test_library_exports_every_declared_symbol(repo_root):
    import sparse_moe_layer_fp32_b200 as pkg
    lib = ctypes.CDLL(pkg.LIB_PATH)
    for name in _declared(repo_root):
        assert hasattr(lib, name), name


def test_host_side_validation_without_gpu():
    import sparse_moe_layer_fp32_b200 as pkg
    lib = pkg.lib()
    assert pkg.status_string(pkg.OK) == "ok"
    assert "unsupported" in pkg.status_string(pkg.ERR_UNSUPPORTED)
    # null handle / arguments are rejected before any CUDA call
    assert lib.beam_moe_forward(None, None, None, None, 1, None) == pkg.ERR_INVALID_ARG
    assert lib.beam_moe_check(None, None) == pkg.ERR_INVALID_ARG
    assert lib.beam_moe_last_launch_count(None) == 0
    lib.beam_moe_destroy(None)
    h = ctypes.c_void_p()
    assert lib.beam_moe_create(None, None, None, ctypes.byref(h)) == pkg.ERR_INVALID_ARG
    # unsupported shapes are reported as such
    assert lib.beam_moe_route(None, None, 4, 100, 256, 8, None, None, None, None) == pkg.ERR_UNSUPPORTED
    assert lib.beam_moe_route(None, None, 4, 5120, 256, 17, None, None, None, None) == pkg.ERR_UNSUPPORTED
    assert lib.beam_moe_route(None, None, -1, 5120, 256, 8, None, None, None, None) == pkg.ERR_INVALID_ARG
    assert lib.beam_moe_route(None, None, 0, 5120, 256, 8, None, None, None, None) == pkg.OK
    assert lib.beam_moe_quantize_nvfp4(None, 4, 24, ctypes.c_float(1.0), None, None, None, None) == pkg.ERR_INVALID_ARG
    assert lib.beam_moe_quantize_nvfp4(None, 4, 32, ctypes.c_float(-1.0), None, None, None, None) == pkg.ERR_INVALID_ARG
    # workspace size of the routing entry point (host arithmetic only)
    assert lib.beam_moe_route_workspace_bytes(8, 5120, 256) == 8 * 256 * 4
    assert lib.beam_moe_route_workspace_bytes(0, 5120, 256) == 0
    assert lib.beam_moe_route_workspace_bytes(1024, 5120, 256) % (1024 * 256 * 4) == 0


def test_host_side_validation_of_the_variant_and_parallel_entry_points():
    # MXFP8 experts, tensor and expert parallelism, router mode: argument errors are answered
    # on the host, before any CUDA call
    import sparse_moe_layer_fp32_b200 as pkg
    lib = pkg.lib()
    h = ctypes.c_void_p()
    bad = pkg.ERR_INVALID_ARG
    assert lib.beam_moe_create_mxfp8(None, None, None, ctypes.byref(h)) == bad
    assert lib.beam_moe_create_ep(None, None, 0, 8, None, ctypes.byref(h)) == bad
    assert lib.beam_moe_create_ep_mxfp8(None, None, 0, 8, None, ctypes.byref(h)) == bad
    cfg = pkg.BeamMoeConfig(8, 5120, 256, 8, 1536, 1e-6, 1.0, 1.0)
    w = pkg.BeamMoeWeights()  # all null
    assert lib.beam_moe_create_ep(ctypes.byref(cfg), ctypes.byref(w), 0, 0, None, ctypes.byref(h)) == bad
    assert lib.beam_moe_create_mxfp8(ctypes.byref(cfg), ctypes.byref(pkg.BeamMoeWeightsMxfp8()), None,
                                     ctypes.byref(h)) == bad
    assert lib.beam_moe_quantize_mxfp8(None, 4, 48, None, None, None) == bad      # cols % 32
    assert lib.beam_moe_quantize_mxfp8(None, -1, 64, None, None, None) == bad
    assert lib.beam_moe_quantize_mxfp8(None, 0, 64, None, None, None) == pkg.OK  # empty: nothing to do
    assert lib.beam_moe_quantize_mxfp8(None, 4, 64, None, None, None) == bad      # null buffers
    assert lib.beam_moe_expert_format(None) == -1
    assert lib.beam_moe_set_router_mode(None, pkg.ROUTER_AUTO) == bad
    assert lib.beam_moe_set_tp_two_shot_tokens(None, 256) == bad
    assert lib.beam_moe_set_host_chunk_tokens(None, 4096) == bad
    assert lib.beam_moe_tp_region_bytes(None) == 0
    p = ctypes.c_void_p()
    assert lib.beam_moe_tp_region(None, ctypes.byref(p)) == bad
    assert lib.beam_moe_tp_attach(None, 0, 2, None, None) == bad
    assert lib.beam_moe_forward_tp(None, None, None, None, 4, None) == bad
    assert lib.beam_moe_forward_tp_phase(None, None, None, None, 4, 3, None) == bad  # phase 0, 1 or 2
    assert lib.beam_moe_forward_ep(None, None, None, None, 4, None) == bad
    assert lib.beam_moe_forward_ep_phase(None, None, None, None, 4, 4, None) == bad  # phase 0 .. 3
    assert lib.beam_moe_ipc_export(None, None) == bad
    assert lib.beam_moe_ipc_import(None, ctypes.byref(p)) == bad
    assert lib.beam_moe_ipc_close(None) == bad
