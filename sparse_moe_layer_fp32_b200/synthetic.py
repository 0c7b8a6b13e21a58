"""Synthetic layers and batches on the GPU: seeded FP32 weights from ``moe_inputs``,
quantised by this library's own quantisers (beam_moe_quantize_nvfp4, or
beam_moe_quantize_mxfp8 for the MXFP8 variant of the experts)."""

from __future__ import annotations

import ctypes
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import moe_inputs as mi

from . import MoELayer, _check, _ptr, _stream, lib


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def make_weights(shape: mi.LayerShape, seed: int = 0, device="cuda", threads: int = 16, stream=None,
                 fmt: str = "nvfp4"):
    """All layer weights as CUDA tensors in the C-ABI layout (NVFP4 or MXFP8 experts)."""
    E, H, I = shape.experts, shape.hidden, shape.inter
    if fmt == "mxfp8":
        return _make_weights_mx(shape, seed, device, threads, stream)
    out = dict(
        router_w=torch.from_numpy(mi.router_weight(shape, seed)).to(device),
        gamma=bf16_tensor(mi.gamma(shape, seed), device),
        w_gu=torch.empty((E, 2 * I, H // 2), dtype=torch.uint8, device=device),
        w_gu_sf=torch.empty((E, 2 * I, H // 16), dtype=torch.uint8, device=device),
        w_gu_alpha=torch.empty(E, dtype=torch.float32, device=device),
        w_d=torch.empty((E, H, I // 2), dtype=torch.uint8, device=device),
        w_d_sf=torch.empty((E, H, I // 16), dtype=torch.uint8, device=device),
        w_d_alpha=torch.empty(E, dtype=torch.float32, device=device),
    )
    fn = lib().beam_moe_quantize_nvfp4
    st = _stream(stream)

    def quant(src, codes, sf, alpha):
        _check(fn(_ptr(src), src.shape[0], src.shape[1], ctypes.c_float(-1.0), _ptr(codes), _ptr(sf), _ptr(alpha),
                  st), "beam_moe_quantize_nvfp4")

    window = max(2 * threads, 4)
    with ThreadPoolExecutor(threads) as ex:
        for e0 in range(0, E, window):
            futs = [ex.submit(mi.expert_weights, shape, seed, e) for e in range(e0, min(E, e0 + window))]
            for i, f in enumerate(futs):
                e = e0 + i
                w_gu, w_d = f.result()
                g = torch.from_numpy(w_gu).to(device)
                d = torch.from_numpy(w_d).to(device)
                quant(g, out["w_gu"][e], out["w_gu_sf"][e], out["w_gu_alpha"][e:e + 1])
                quant(d, out["w_d"][e], out["w_d_sf"][e], out["w_d_alpha"][e:e + 1])
    torch.cuda.synchronize()
    return out


def _make_weights_mx(shape: mi.LayerShape, seed: int, device, threads: int, stream):
    E, H, I = shape.experts, shape.hidden, shape.inter
    out = dict(
        router_w=torch.from_numpy(mi.router_weight(shape, seed)).to(device),
        gamma=bf16_tensor(mi.gamma(shape, seed), device),
        w_gu=torch.empty((E, 2 * I, H), dtype=torch.uint8, device=device),
        w_gu_sf=torch.empty((E, 2 * I, H // 32), dtype=torch.uint8, device=device),
        w_d=torch.empty((E, H, I), dtype=torch.uint8, device=device),
        w_d_sf=torch.empty((E, H, I // 32), dtype=torch.uint8, device=device),
    )
    fn = lib().beam_moe_quantize_mxfp8
    st = _stream(stream)

    def quant(src, codes, sf):
        _check(fn(_ptr(src), src.shape[0], src.shape[1], _ptr(codes), _ptr(sf), st), "beam_moe_quantize_mxfp8")

    window = max(2 * threads, 4)
    with ThreadPoolExecutor(threads) as ex:
        for e0 in range(0, E, window):
            futs = [ex.submit(mi.expert_weights, shape, seed, e) for e in range(e0, min(E, e0 + window))]
            for i, f in enumerate(futs):
                e = e0 + i
                w_gu, w_d = f.result()
                quant(torch.from_numpy(w_gu).to(device), out["w_gu"][e], out["w_gu_sf"][e])
                quant(torch.from_numpy(w_d).to(device), out["w_d"][e], out["w_d_sf"][e])
    torch.cuda.synchronize()
    return out


def make_layer(shape: mi.LayerShape, weights: dict, max_tokens: int | None = None, stream=None,
               fmt: str = "nvfp4") -> MoELayer:
    if fmt == "mxfp8":
        return MoELayer(max_tokens=max_tokens or shape.tokens, hidden=shape.hidden, num_experts=shape.experts,
                        top_k=shape.top_k, inter=shape.inter, rms_eps=shape.rms_eps, stream=stream, fmt="mxfp8",
                        **weights)
    a1, a2 = mi.activation_scales(shape)
    return MoELayer(max_tokens=max_tokens or shape.tokens, hidden=shape.hidden, num_experts=shape.experts,
                    top_k=shape.top_k, inter=shape.inter, alpha_a1=float(a1), alpha_a2=float(a2),
                    rms_eps=shape.rms_eps, stream=stream, **weights)


def make_batch(shape: mi.LayerShape, seed: int = 0, device="cuda"):
    """x, residual [T, H] bf16 CUDA tensors."""
    xb, rb = mi.tokens(shape, seed)
    return bf16_tensor(xb, device), bf16_tensor(rb, device)
