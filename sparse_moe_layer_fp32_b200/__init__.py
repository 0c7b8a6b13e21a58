"""Python binding of libbeam_moe.so: the Beam-style sparse MoE layer forward on a B200.

Argument marshalling only: every step of the layer runs in the library's CUDA kernels.
PyTorch provides device memory and streams.  The functions keep the C names
(beam_moe_create, beam_moe_forward, ...); ``MoELayer`` wraps a handle.  Importing this
package never falls back to anything: if the library is missing it raises.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbeam_moe.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_OOM, ERR_TIMEOUT, ERR_DEVICE = range(7)
(BUF_LOGITS, BUF_IDS, BUF_WEIGHTS, BUF_OFFSETS, BUF_PERM, BUF_INV, BUF_SFBLOCK, BUF_A1, BUF_A2,
 BUF_Y) = range(10)

EXPORTED = [
    "beam_moe_create", "beam_moe_forward", "beam_moe_forward_host", "beam_moe_route",
    "beam_moe_route_workspace_bytes", "beam_moe_quantize_nvfp4", "beam_moe_debug_copy", "beam_moe_check",
    "beam_moe_last_launch_count", "beam_moe_status_string", "beam_moe_destroy", "beam_moe_profile_enable",
    "beam_moe_profile_read", "beam_moe_kernel_name", "beam_moe_route_static", "beam_moe_debug_wait_timeout",
    "beam_moe_forward_prenorm", "beam_moe_create_mxfp8", "beam_moe_quantize_mxfp8",
    "beam_moe_expert_format", "beam_moe_tp_region_bytes", "beam_moe_tp_region", "beam_moe_tp_attach",
    "beam_moe_forward_tp", "beam_moe_forward_tp_phase", "beam_moe_ipc_export", "beam_moe_ipc_import",
    "beam_moe_ipc_close", "beam_moe_create_ep", "beam_moe_create_ep_mxfp8", "beam_moe_forward_ep",
    "beam_moe_forward_ep_phase", "beam_moe_set_router_mode", "beam_moe_set_tp_two_shot_tokens",
    "beam_moe_set_host_chunk_tokens",
]
IPC_HANDLE_BYTES = 64
FMT_NVFP4, FMT_MXFP8 = 0, 1
FORMATS = {"nvfp4": FMT_NVFP4, "mxfp8": FMT_MXFP8}


class BeamMoeConfig(ctypes.Structure):
    _fields_ = [("max_tokens", ctypes.c_int32), ("hidden", ctypes.c_int32), ("num_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("inter", ctypes.c_int32), ("rms_eps", ctypes.c_float),
                ("alpha_a1", ctypes.c_float), ("alpha_a2", ctypes.c_float)]


class BeamMoeWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("router_w", "w_gu", "w_gu_sf", "w_gu_alpha", "w_d", "w_d_sf", "w_d_alpha", "gamma")]


class BeamMoeWeightsMxfp8(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("router_w", "w_gu", "w_gu_sf", "w_d", "w_d_sf", "gamma")]


class BeamMoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run sparse_moe_layer_fp32_b200.build.build() "
                          "(needs nvcc with sm_100a support)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    sig = {
        "beam_moe_create": (i32, [ctypes.POINTER(BeamMoeConfig), ctypes.POINTER(BeamMoeWeights), vp,
                                  ctypes.POINTER(vp)]),
        "beam_moe_forward": (i32, [vp, vp, vp, vp, i32, vp]),
        "beam_moe_forward_host": (i32, [vp, vp, vp, vp, i32, vp]),
        "beam_moe_route": (i32, [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp]),
        "beam_moe_route_workspace_bytes": (i64, [i32, i32, i32]),
        "beam_moe_quantize_nvfp4": (i32, [vp, i64, i64, f32, vp, vp, vp, vp]),
        "beam_moe_debug_copy": (i32, [vp, i32, vp, sz, ctypes.POINTER(sz), vp]),
        "beam_moe_check": (i32, [vp, vp]),
        "beam_moe_last_launch_count": (i32, [vp]),
        "beam_moe_status_string": (ctypes.c_char_p, [i32]),
        "beam_moe_destroy": (None, [vp]),
        "beam_moe_profile_enable": (i32, [vp, i32]),
        "beam_moe_set_router_mode": (i32, [vp, i32]),
        "beam_moe_set_tp_two_shot_tokens": (i32, [vp, i32]),
        "beam_moe_set_host_chunk_tokens": (i32, [vp, i32]),
        "beam_moe_profile_read": (i32, [vp, ctypes.POINTER(f32), i32, ctypes.POINTER(i32)]),
        "beam_moe_kernel_name": (ctypes.c_char_p, [vp, i32]),
        "beam_moe_route_static": (i32, [vp, vp, i32, i32, i32, i32, vp, vp, vp]),
        "beam_moe_debug_wait_timeout": (i32, [vp, i64, vp]),
        "beam_moe_forward_prenorm": (i32, [vp, vp, vp, vp, vp, vp, f32, i32, vp]),
        "beam_moe_create_mxfp8": (i32, [ctypes.POINTER(BeamMoeConfig), ctypes.POINTER(BeamMoeWeightsMxfp8), vp,
                                        ctypes.POINTER(vp)]),
        "beam_moe_quantize_mxfp8": (i32, [vp, i64, i64, vp, vp, vp]),
        "beam_moe_expert_format": (i32, [vp]),
        "beam_moe_tp_region_bytes": (i64, [vp]),
        "beam_moe_tp_region": (i32, [vp, ctypes.POINTER(vp)]),
        "beam_moe_tp_attach": (i32, [vp, i32, i32, ctypes.POINTER(vp), vp]),
        "beam_moe_forward_tp": (i32, [vp, vp, vp, vp, i32, vp]),
        "beam_moe_forward_tp_phase": (i32, [vp, vp, vp, vp, i32, i32, vp]),
        "beam_moe_ipc_export": (i32, [vp, vp]),
        "beam_moe_ipc_import": (i32, [vp, ctypes.POINTER(vp)]),
        "beam_moe_ipc_close": (i32, [vp]),
        "beam_moe_create_ep": (i32, [ctypes.POINTER(BeamMoeConfig), ctypes.POINTER(BeamMoeWeights), i32, i32, vp,
                                     ctypes.POINTER(vp)]),
        "beam_moe_create_ep_mxfp8": (i32, [ctypes.POINTER(BeamMoeConfig), ctypes.POINTER(BeamMoeWeightsMxfp8), i32,
                                           i32, vp, ctypes.POINTER(vp)]),
        "beam_moe_forward_ep": (i32, [vp, vp, vp, vp, i32, vp]),
        "beam_moe_forward_ep_phase": (i32, [vp, vp, vp, vp, i32, i32, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def lib():
    return _lib


def status_string(status: int) -> str:
    return _lib.beam_moe_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != OK:
        raise BeamMoeError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


# ------------------------------------------------------------------ C names
def beam_moe_create(cfg: BeamMoeConfig, weights: BeamMoeWeights, stream=None) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(_lib.beam_moe_create(ctypes.byref(cfg), ctypes.byref(weights), _stream(stream), ctypes.byref(h)),
           "beam_moe_create")
    return h


def beam_moe_create_mxfp8(cfg: BeamMoeConfig, weights: BeamMoeWeightsMxfp8, stream=None) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(_lib.beam_moe_create_mxfp8(ctypes.byref(cfg), ctypes.byref(weights), _stream(stream), ctypes.byref(h)),
           "beam_moe_create_mxfp8")
    return h


def beam_moe_create_ep(cfg: BeamMoeConfig, weights, expert_begin: int, expert_count: int, stream=None):
    """Expert-parallel handle: weights (BeamMoeWeights or BeamMoeWeightsMxfp8) of experts
    [expert_begin, expert_begin + expert_count) of cfg.num_experts."""
    h = ctypes.c_void_p()
    fn = _lib.beam_moe_create_ep_mxfp8 if isinstance(weights, BeamMoeWeightsMxfp8) else _lib.beam_moe_create_ep
    _check(fn(ctypes.byref(cfg), ctypes.byref(weights), int(expert_begin), int(expert_count), _stream(stream),
              ctypes.byref(h)), "beam_moe_create_ep")
    return h


def beam_moe_forward_ep(h, x, residual, out, num_tokens: int, stream=None):
    _check(_lib.beam_moe_forward_ep(h, _ptr(x), _ptr(residual), _ptr(out), int(num_tokens), _stream(stream)),
           "beam_moe_forward_ep")


def beam_moe_forward_ep_phase(h, x, residual, out, num_tokens: int, phase: int, stream=None):
    _check(_lib.beam_moe_forward_ep_phase(h, _ptr(x), _ptr(residual), _ptr(out), int(num_tokens), int(phase),
                                          _stream(stream)), "beam_moe_forward_ep_phase")


def beam_moe_expert_format(h) -> int:
    return int(_lib.beam_moe_expert_format(h))


def beam_moe_tp_region_bytes(h) -> int:
    return int(_lib.beam_moe_tp_region_bytes(h))


def beam_moe_tp_region(h) -> int:
    """Device address of the handle's tensor-parallel exchange region (allocated on first use)."""
    p = ctypes.c_void_p()
    _check(_lib.beam_moe_tp_region(h, ctypes.byref(p)), "beam_moe_tp_region")
    return int(p.value)


def beam_moe_tp_attach(h, rank: int, world: int, regions, stream=None):
    arr = (ctypes.c_void_p * world)(*[int(r) for r in regions])
    _check(_lib.beam_moe_tp_attach(h, int(rank), int(world), arr, _stream(stream)), "beam_moe_tp_attach")


def beam_moe_forward_tp(h, x, residual, out, num_tokens: int, stream=None):
    _check(_lib.beam_moe_forward_tp(h, _ptr(x), _ptr(residual), _ptr(out), int(num_tokens), _stream(stream)),
           "beam_moe_forward_tp")


def beam_moe_forward_tp_phase(h, x, residual, out, num_tokens: int, phase: int, stream=None):
    _check(_lib.beam_moe_forward_tp_phase(h, _ptr(x), _ptr(residual), _ptr(out), int(num_tokens), int(phase),
                                          _stream(stream)), "beam_moe_forward_tp_phase")


def beam_moe_ipc_export(dev_ptr: int) -> bytes:
    buf = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    _check(_lib.beam_moe_ipc_export(ctypes.c_void_p(int(dev_ptr)), buf), "beam_moe_ipc_export")
    return buf.raw


def beam_moe_ipc_import(handle: bytes) -> int:
    p = ctypes.c_void_p()
    _check(_lib.beam_moe_ipc_import(ctypes.create_string_buffer(bytes(handle), IPC_HANDLE_BYTES), ctypes.byref(p)),
           "beam_moe_ipc_import")
    return int(p.value)


def beam_moe_ipc_close(dev_ptr: int):
    _check(_lib.beam_moe_ipc_close(ctypes.c_void_p(int(dev_ptr))), "beam_moe_ipc_close")


def beam_moe_forward(h, x, residual, out, num_tokens: int, stream=None):
    _check(_lib.beam_moe_forward(h, _ptr(x), _ptr(residual), _ptr(out), int(num_tokens), _stream(stream)),
           "beam_moe_forward")


def beam_moe_forward_prenorm(h, x, residual, out, next_x, next_gamma, next_eps: float, num_tokens: int, stream=None):
    _check(_lib.beam_moe_forward_prenorm(h, _ptr(x), _ptr(residual), _ptr(out), _ptr(next_x), _ptr(next_gamma),
                                         ctypes.c_float(next_eps), int(num_tokens), _stream(stream)),
           "beam_moe_forward_prenorm")


def beam_moe_forward_host(h, x_host, residual_host, out_host, num_tokens: int, stream=None):
    _check(_lib.beam_moe_forward_host(h, _ptr(x_host), _ptr(residual_host), _ptr(out_host), int(num_tokens),
                                      _stream(stream)), "beam_moe_forward_host")


def beam_moe_route_workspace_bytes(num_tokens: int, hidden: int, num_experts: int) -> int:
    return int(_lib.beam_moe_route_workspace_bytes(num_tokens, hidden, num_experts))


def beam_moe_route(x, router_w, top_k: int, stream=None):
    """Returns (ids [T, k] int32, w [T, k] float32) for x [T, H] bf16, router_w [E, H] fp32."""
    t_count, hidden = x.shape
    experts = router_w.shape[0]
    ws = torch.empty(max(beam_moe_route_workspace_bytes(t_count, hidden, experts) // 4, 1), dtype=torch.float32,
                     device=x.device)
    ids = torch.empty((t_count, top_k), dtype=torch.int32, device=x.device)
    w = torch.empty((t_count, top_k), dtype=torch.float32, device=x.device)
    _check(_lib.beam_moe_route(_ptr(x), _ptr(router_w), t_count, hidden, experts, top_k, _ptr(ws), _ptr(ids),
                               _ptr(w), _stream(stream)), "beam_moe_route")
    return ids, w


def beam_moe_quantize_nvfp4(src, alpha: float | None = None, stream=None):
    """NVFP4 of a 2-D FP32 CUDA tensor: (codes uint8 [r, c/2], scales uint8 [r, c/16], alpha fp32 [1])."""
    rows, cols = src.shape
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=src.device)
    sf = torch.empty((rows, cols // 16), dtype=torch.uint8, device=src.device)
    alpha_out = torch.empty(1, dtype=torch.float32, device=src.device)
    a = -1.0 if alpha is None else float(alpha)
    _check(_lib.beam_moe_quantize_nvfp4(_ptr(src.contiguous()), rows, cols, ctypes.c_float(a), _ptr(codes),
                                        _ptr(sf), _ptr(alpha_out), _stream(stream)), "beam_moe_quantize_nvfp4")
    return codes, sf, alpha_out


def beam_moe_quantize_mxfp8(src, stream=None):
    """MXFP8 of a 2-D FP32 CUDA tensor: (codes uint8 [r, c] E4M3, scales uint8 [r, c/32] UE8M0)."""
    rows, cols = src.shape
    codes = torch.empty((rows, cols), dtype=torch.uint8, device=src.device)
    sf = torch.empty((rows, cols // 32), dtype=torch.uint8, device=src.device)
    _check(_lib.beam_moe_quantize_mxfp8(_ptr(src.contiguous()), rows, cols, _ptr(codes), _ptr(sf), _stream(stream)),
           "beam_moe_quantize_mxfp8")
    return codes, sf


def beam_moe_debug_copy(h, which: int, stream=None) -> torch.Tensor:
    size = ctypes.c_size_t(0)
    _check(_lib.beam_moe_debug_copy(h, which, None, 0, ctypes.byref(size), _stream(stream)), "beam_moe_debug_copy")
    out = torch.empty(max(size.value, 1), dtype=torch.uint8, device="cuda")
    _check(_lib.beam_moe_debug_copy(h, which, _ptr(out), size.value, None, _stream(stream)), "beam_moe_debug_copy")
    return out[: size.value]


def beam_moe_check(h, stream=None):
    _check(_lib.beam_moe_check(h, _stream(stream)), "beam_moe_check")


def beam_moe_last_launch_count(h) -> int:
    return int(_lib.beam_moe_last_launch_count(h))


def beam_moe_destroy(h):
    _lib.beam_moe_destroy(h)


def beam_moe_debug_wait_timeout(h, limit_ns: int, stream=None):
    _check(_lib.beam_moe_debug_wait_timeout(h, int(limit_ns), _stream(stream)), "beam_moe_debug_wait_timeout")


ROUTER_AUTO, ROUTER_SIMT, ROUTER_TENSOR = 0, 1, 2


def beam_moe_set_router_mode(h, mode: int):
    _check(_lib.beam_moe_set_router_mode(h, int(mode)), "beam_moe_set_router_mode")


TP_TWO_SHOT_MIN_TOKENS = 256  # BEAM_MOE_TP_TWO_SHOT_MIN_TOKENS
HOST_CHUNK_TOKENS = 4096  # BEAM_MOE_HOST_CHUNK_TOKENS


def beam_moe_set_tp_two_shot_tokens(h, min_tokens: int):
    _check(_lib.beam_moe_set_tp_two_shot_tokens(h, int(min_tokens)), "beam_moe_set_tp_two_shot_tokens")


def beam_moe_set_host_chunk_tokens(h, tokens: int):
    _check(_lib.beam_moe_set_host_chunk_tokens(h, int(tokens)), "beam_moe_set_host_chunk_tokens")


def beam_moe_profile_enable(h, enable: bool = True):
    _check(_lib.beam_moe_profile_enable(h, 1 if enable else 0), "beam_moe_profile_enable")


def beam_moe_profile_read(h):
    """[(kernel name, ms)] of the last profiled forward, in launch order."""
    buf = (ctypes.c_float * 32)()
    n = ctypes.c_int32(0)
    _check(_lib.beam_moe_profile_read(h, buf, 32, ctypes.byref(n)), "beam_moe_profile_read")
    return [(_lib.beam_moe_kernel_name(h, i).decode(), float(buf[i])) for i in range(n.value)]


# ------------------------------------------------------------------ handle wrapper
class MoELayer:
    """Owns a beam_moe handle.  Weight tensors are CUDA tensors in the C-ABI layout.

    fmt="nvfp4" (beam_moe_create): NVFP4 experts with tensor scales w_gu_alpha / w_d_alpha
    and the activation scales alpha_a1 / alpha_a2.  fmt="mxfp8" (beam_moe_create_mxfp8):
    MXFP8 experts; the alphas are not used."""

    def __init__(self, *, max_tokens, hidden, num_experts, top_k, inter, router_w, w_gu, w_gu_sf, w_d, w_d_sf,
                 gamma, alpha_a1=1.0, alpha_a2=1.0, w_gu_alpha=None, w_d_alpha=None, rms_eps=1e-6, fmt="nvfp4",
                 expert_begin=None, expert_count=None, stream=None):
        if fmt not in FORMATS:
            raise ValueError(f"unknown expert format {fmt!r}")
        self.fmt = fmt
        self.cfg = BeamMoeConfig(max_tokens, hidden, num_experts, top_k, inter, rms_eps, float(alpha_a1),
                                 float(alpha_a2))
        self.hidden, self.top_k = hidden, top_k
        if fmt == "mxfp8":
            ws = [router_w, w_gu, w_gu_sf, w_d, w_d_sf, gamma]
            wts = BeamMoeWeightsMxfp8(*[t.data_ptr() for t in ws])
        else:
            if w_gu_alpha is None or w_d_alpha is None:
                raise ValueError("NVFP4 experts need w_gu_alpha and w_d_alpha")
            ws = [router_w, w_gu, w_gu_sf, w_gu_alpha, w_d, w_d_sf, w_d_alpha, gamma]
            wts = BeamMoeWeights(*[t.data_ptr() for t in ws])
        self.expert_parallel = expert_count is not None
        if self.expert_parallel:  # this layer holds experts [expert_begin, expert_begin + expert_count)
            self.handle = beam_moe_create_ep(self.cfg, wts, expert_begin or 0, expert_count, stream)
        elif fmt == "mxfp8":
            self.handle = beam_moe_create_mxfp8(self.cfg, wts, stream)
        else:
            self.handle = beam_moe_create(self.cfg, wts, stream)

    def forward(self, x, residual, out=None, stream=None):
        out = torch.empty_like(residual) if out is None else out
        beam_moe_forward(self.handle, x, residual, out, x.shape[0], stream)
        return out

    def forward_prenorm(self, x, residual, next_gamma, next_eps=1e-6, out=None, next_x=None, stream=None):
        """(out, next_x): the layer output and the next sublayer's pre-normed input."""
        out = torch.empty_like(residual) if out is None else out
        next_x = torch.empty_like(residual) if next_x is None else next_x
        beam_moe_forward_prenorm(self.handle, x, residual, out, next_x, next_gamma, next_eps, x.shape[0], stream)
        return out, next_x

    def forward_host(self, x_host, residual_host, out_host, stream=None):
        beam_moe_forward_host(self.handle, x_host, residual_host, out_host, x_host.shape[0], stream)
        return out_host

    def debug(self, which: int, stream=None) -> torch.Tensor:
        return beam_moe_debug_copy(self.handle, which, stream)

    def check(self, stream=None):
        beam_moe_check(self.handle, stream)

    def launches(self) -> int:
        return beam_moe_last_launch_count(self.handle)

    def profile(self, enable: bool = True):
        beam_moe_profile_enable(self.handle, enable)

    # ---- tensor parallelism (this layer holds one rank's slice of the experts; see tp.py)
    def tp_region(self) -> int:
        return beam_moe_tp_region(self.handle)

    def tp_attach(self, rank: int, world: int, regions, stream=None):
        beam_moe_tp_attach(self.handle, rank, world, regions, stream)

    def forward_tp(self, x, residual, out=None, stream=None):
        out = torch.empty_like(residual) if out is None else out
        beam_moe_forward_tp(self.handle, x, residual, out, x.shape[0], stream)
        return out

    def forward_tp_phase(self, x, residual, out, phase: int, stream=None):
        beam_moe_forward_tp_phase(self.handle, x, residual, out, x.shape[0], phase, stream)
        return out

    def forward_ep(self, x, residual, out=None, stream=None):
        out = torch.empty_like(residual) if out is None else out
        beam_moe_forward_ep(self.handle, x, residual, out, x.shape[0], stream)
        return out

    def forward_ep_phase(self, x, residual, out, phase: int, stream=None):
        beam_moe_forward_ep_phase(self.handle, x, residual, out, x.shape[0], phase, stream)
        return out

    def set_router_mode(self, mode: int):
        beam_moe_set_router_mode(self.handle, mode)

    def set_tp_two_shot_tokens(self, min_tokens: int):
        beam_moe_set_tp_two_shot_tokens(self.handle, min_tokens)

    def set_host_chunk_tokens(self, tokens: int):
        """Part size of forward_host (0: never split a batch)."""
        beam_moe_set_host_chunk_tokens(self.handle, tokens)

    def kernel_times(self):
        return beam_moe_profile_read(self.handle)

    def close(self):
        if self.handle:
            beam_moe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
