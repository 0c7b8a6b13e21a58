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
