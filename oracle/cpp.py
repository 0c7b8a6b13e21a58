"""ctypes binding of the C++ oracle (oracle/moe_oracle.cpp) -- test infrastructure only.

The C++ oracle is the plain FP64 CPU statement of the layer; the numpy modules of this
package are a second, independent statement of the same steps, and the tests check the two
against each other and against the same pins.  build() compiles it with g++ and OpenMP into
oracle/libmoe_oracle.so (no CUDA involved)."""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_DIR = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_DIR, "moe_oracle.cpp")
LIB = os.path.join(_DIR, "libmoe_oracle.so")
EXPERT_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p)
_lib = None


def build(verbose: bool = False) -> str:
    """Compiles the oracle if the library is missing or older than its source."""
    if os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", SRC, "-o", LIB]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    return LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB)
        vp, i32, i64, f32, f64, u8 = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                                      ctypes.c_double, ctypes.c_uint8)
        L.orc_e4m3_encode.restype, L.orc_e4m3_encode.argtypes = u8, [f32]
        L.orc_e4m3_encode_signed.restype, L.orc_e4m3_encode_signed.argtypes = u8, [f32]
        L.orc_e4m3_decode.restype, L.orc_e4m3_decode.argtypes = f64, [u8]
        L.orc_e2m1_encode.restype, L.orc_e2m1_encode.argtypes = u8, [f32]
        L.orc_e2m1_decode.restype, L.orc_e2m1_decode.argtypes = f64, [u8]
        L.orc_bf16_round.restype, L.orc_bf16_round.argtypes = f64, [f64]
        L.orc_tensor_scale.restype, L.orc_tensor_scale.argtypes = f32, [vp, i64]
        L.orc_quantize_nvfp4.restype, L.orc_quantize_nvfp4.argtypes = None, [vp, i64, i64, f32, vp, vp]
        L.orc_quantize_mxfp8.restype, L.orc_quantize_mxfp8.argtypes = None, [vp, i64, i64, vp, vp]
        L.orc_route.restype, L.orc_route.argtypes = None, [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp]
        L.orc_permute.restype, L.orc_permute.argtypes = None, [vp, i32, i32, i32, vp, vp, vp, vp, vp]
        L.orc_moe_forward.restype = ctypes.c_int
        L.orc_moe_forward.argtypes = [i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, f32, f32, f64, EXPERT_FN, vp,
                                      vp, vp, vp, vp, vp, vp]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def quantize_nvfp4(v, alpha):
    v = np.ascontiguousarray(v, np.float32)
    rows, cols = v.reshape(-1, v.shape[-1]).shape
    packed = np.empty(v.shape[:-1] + (cols // 2,), np.uint8)
    sf = np.empty(v.shape[:-1] + (cols // 16,), np.uint8)
    lib().orc_quantize_nvfp4(_p(v), rows, cols, float(np.float32(alpha)), _p(packed), _p(sf))
    return packed, sf


def quantize_mxfp8(v):
    v = np.ascontiguousarray(v, np.float32)
    rows, cols = v.reshape(-1, v.shape[-1]).shape
    codes = np.empty(v.shape, np.uint8)
    sf = np.empty(v.shape[:-1] + (cols // 32,), np.uint8)
    lib().orc_quantize_mxfp8(_p(v), rows, cols, _p(codes), _p(sf))
    return codes, sf


def route(x_bits, router_w, k):
    """Steps 1-4: (logits [T, E], ids [T, k], w [T, k], near_tie [T])."""
    x = np.ascontiguousarray(x_bits, np.uint16)
    wr = np.ascontiguousarray(router_w, np.float32)
    T, H = x.shape
    E = wr.shape[0]
    logits = np.empty((T, E), np.float64)
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    near = np.empty(T, np.uint8)
    lib().orc_route(_p(x), _p(wr), T, H, E, k, _p(logits), _p(ids), _p(w), _p(near))
    return logits, ids, w, near.astype(bool)


def permute(ids, num_experts):
    ids = np.ascontiguousarray(ids, np.int32)
    T, k = ids.shape
    counts = np.empty(num_experts, np.int64)
    offsets = np.empty(num_experts + 1, np.int64)
    src = np.empty(T * k, np.int32)
    slot = np.empty(T * k, np.int32)
    inv = np.empty((T, k), np.int32)
    lib().orc_permute(_p(ids), T, k, num_experts, _p(counts), _p(offsets), _p(src), _p(slot), _p(inv))
    return dict(counts=counts, offsets=offsets, perm_src=src, perm_slot=slot, inv=inv)


def moe_forward(x_bits, residual_bits, router_w, gamma_bits, expert_fp32, top_k, inter, alpha_a1=1.0, alpha_a2=1.0,
                eps=1e-6, fmt="nvfp4"):
    """The layer forward of T tokens (steps 1-4, 6-13).  expert_fp32(e) -> (w_gu [2I, H],
    w_d [H, I]) FP32.  Returns dict(ids, w, near_tie, m, out_pre, out_bf16 bits)."""
    x = np.ascontiguousarray(x_bits, np.uint16)
    res = np.ascontiguousarray(residual_bits, np.uint16)
    wr = np.ascontiguousarray(router_w, np.float32)
    g = np.ascontiguousarray(gamma_bits, np.uint16)
    T, H = x.shape
    E = wr.shape[0]
    err = []

    def cb(_ctx, e, p_gu, p_d):
        try:
            w_gu, w_d = expert_fp32(int(e))
            ctypes.memmove(p_gu, np.ascontiguousarray(w_gu, np.float32).ctypes.data, 2 * inter * H * 4)
            ctypes.memmove(p_d, np.ascontiguousarray(w_d, np.float32).ctypes.data, H * inter * 4)
            return 0
        except Exception as ex:  # reported after the call
            err.append(ex)
            return 1

    fn = EXPERT_FN(cb)
    ids = np.empty((T, top_k), np.int32)
    w = np.empty((T, top_k), np.float64)
    near = np.empty(T, np.uint8)
    m = np.empty((T, H), np.float64)
    pre = np.empty((T, H), np.float64)
    out = np.empty((T, H), np.uint16)
    rc = lib().orc_moe_forward(T, H, E, top_k, inter, 1 if fmt == "mxfp8" else 0, _p(x), _p(res), _p(wr), _p(g),
                               float(np.float32(alpha_a1)), float(np.float32(alpha_a2)), float(eps), fn, None,
                               _p(ids), _p(w), _p(near), _p(m), _p(pre), _p(out))
    if rc != 0:
        raise RuntimeError(f"expert weights callback failed: {err[0] if err else rc}")
    return dict(ids=ids, w=w, near_tie=near.astype(bool), m=m, out_pre=pre, out_bf16=out)
