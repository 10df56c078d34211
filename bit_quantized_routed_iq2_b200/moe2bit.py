"""ctypes binding of libmoe2bit.so (the C ABI in include/moe2bit.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. Device buffers are torch tensors (torch provides device memory and
streams); they are passed to the library as raw pointers. If the shared library
is missing the import of a call raises; there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
SO_PATH = os.path.join(_HERE, "libmoe2bit.so")

MOE_F32, MOE_BF16 = 0, 1
STATUS = {
    0: "MOE_OK",
    1: "MOE_ERR_INVALID_ARG",
    2: "MOE_ERR_UNSUPPORTED_SHAPE",
    3: "MOE_ERR_WORKSPACE_TOO_SMALL",
    4: "MOE_ERR_CUDA",
    5: "MOE_ERR_TIMEOUT",
}

# Every symbol include/moe2bit.h declares.
EXPORTS = (
    "moe_workspace_size", "moe_route", "moe_expert_ffn", "moe_layer_forward", "moe_status_string",
    "moe_debug_dequant_iq2", "moe_debug_dequant_q2k", "moe_debug_grid", "moe_profile_enable", "moe_profile_read",
    "moe_layer_forward_noalloc",
)
NOALLOC_SCRATCH_BYTES = 32 << 20
KERNEL_NAMES = ("router_logits", "topk", "permute", "active", "gateup", "down", "shared_gateup", "shared_down",
                "combine", "prep", "prefill_gateup", "prefill_down", "hquant")
K_COUNT = 16


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}")
        self.status = status


class Desc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("hidden", "inter", "n_experts", "top_k", "shared_inter")]


class Weights(ctypes.Structure):
    _fields_ = [
        (n, ctypes.c_void_p)
        for n in ("router_w", "router_bias", "gate_codes", "gate_d", "up_codes", "up_d",
                  "down_codes", "down_dd", "sh_gate", "sh_up", "sh_down")
    ]


_lib = None


def load() -> ctypes.CDLL:
    """Load the in-tree library. Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(SO_PATH):
        raise ImportError(
            f"{SO_PATH} is missing: build it with `python -m bit_quantized_routed_iq2_b200.build` "
            "(there is no CPU fallback)"
        )
    L = ctypes.CDLL(SO_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    pd, pw = ctypes.POINTER(Desc), ctypes.POINTER(Weights)
    L.moe_workspace_size.argtypes = [pd, i32, ctypes.POINTER(sz)]
    L.moe_route.argtypes = [pd, vp, vp, vp, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_expert_ffn.argtypes = [pd, pw, vp, i32, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_layer_forward.argtypes = [pd, pw, vp, i32, i32, vp, vp, vp, sz, vp]
    L.moe_status_string.argtypes = [i32]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_debug_dequant_iq2.argtypes = [vp, vp, i64, vp, vp]
    L.moe_debug_dequant_q2k.argtypes = [vp, vp, i64, vp, vp]
    L.moe_debug_grid.argtypes = [vp]
    L.moe_debug_grid.restype = None
    L.moe_layer_forward_noalloc.argtypes = [pd, pw, vp, i32, i32, vp, vp, vp]
    L.moe_profile_enable.argtypes = [i32]
    L.moe_profile_read.argtypes = [vp, vp]
    for name in EXPORTS:
        if name not in ("moe_debug_grid",):
            getattr(L, name).restype = ctypes.c_int32 if name != "moe_status_string" else ctypes.c_char_p
    _lib = L
    return L


def _ptr(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _check(rc: int, where: str):
    if rc != 0:
        raise MoeError(rc, where)


def _dtype_of(x) -> int:
    import torch

    if x.dtype == torch.float32:
        return MOE_F32
    if x.dtype in (torch.bfloat16, torch.int16, torch.uint16):
        return MOE_BF16
    raise TypeError("activations must be float32 or bfloat16")


def status_string(code: int) -> str:
    return load().moe_status_string(code).decode()


def desc_of(H: int, I: int, E: int, k: int, Is: int) -> Desc:
    return Desc(H, I, E, k, Is)


def workspace_size(desc: Desc, max_tokens: int) -> int:
    n = ctypes.c_size_t(0)
    _check(load().moe_workspace_size(ctypes.byref(desc), max_tokens, ctypes.byref(n)), "moe_workspace_size")
    return int(n.value)


def profile_enable(on: bool):
    _check(load().moe_profile_enable(1 if on else 0), "moe_profile_enable")


def profile_read() -> dict:
    """{kernel name: (total ms, launches)} since the last read; waits for the events."""
    ms = (ctypes.c_float * K_COUNT)()
    n = (ctypes.c_int32 * K_COUNT)()
    _check(load().moe_profile_read(ms, n), "moe_profile_read")
    return {KERNEL_NAMES[i]: (float(ms[i]), int(n[i])) for i in range(len(KERNEL_NAMES)) if n[i]}


def debug_grid() -> bytes:
    buf = (ctypes.c_uint8 * 2048)()
    load().moe_debug_grid(buf)
    return bytes(buf)


def debug_dequant_iq2(codes, d, out, stream=None):
    nb = codes.numel() // 64
    _check(load().moe_debug_dequant_iq2(_ptr(codes), _ptr(d), nb, _ptr(out), _stream(stream)), "moe_debug_dequant_iq2")


def debug_dequant_q2k(codes, dd, out, stream=None):
    nb = codes.numel() // 80
    _check(load().moe_debug_dequant_q2k(_ptr(codes), _ptr(dd), nb, _ptr(out), _stream(stream)), "moe_debug_dequant_q2k")


@dataclass
class DeviceLayer:
    """Device-resident planes of one layer (torch tensors) plus the ABI structs."""

    desc: Desc
    tensors: dict

    @property
    def weights(self) -> Weights:
        t = self.tensors
        return Weights(*[_ptr(t.get(n)) for n in (
            "router_w", "router_bias", "gate_codes", "gate_d", "up_codes", "up_d",
            "down_codes", "down_dd", "sh_gate", "sh_up", "sh_down")])


def to_device(lw, device="cuda") -> DeviceLayer:
    """Upload host planes (numpy, the layout documented in include/moe2bit.h)."""
    import numpy as np
    import torch

    def up(a, dt):
        if a is None:
            return None
        return torch.from_numpy(np.ascontiguousarray(a).view(dt)).to(device)

    t = {
        "router_w": up(lw.router_w, np.int16),
        "router_bias": None if lw.router_bias is None else up(lw.router_bias, np.float32),
        "gate_codes": up(lw.gate_codes, np.uint8),
        "gate_d": up(lw.gate_d, np.int16),
        "up_codes": up(lw.up_codes, np.uint8),
        "up_d": up(lw.up_d, np.int16),
        "down_codes": up(lw.down_codes, np.uint8),
        "down_dd": up(lw.down_dd, np.int32),
        "sh_gate": up(lw.sh_gate, np.int16) if lw.Is else None,
        "sh_up": up(lw.sh_up, np.int16) if lw.Is else None,
        "sh_down": up(lw.sh_down, np.int16) if lw.Is else None,
    }
    return DeviceLayer(desc_of(lw.H, lw.I, lw.E, lw.k, lw.Is), t)


def route(desc: Desc, router_w, router_bias, x, topk_idx, topk_w, offsets, perm, inv, ws, stream=None):
    T = x.shape[0]
    _check(load().moe_route(ctypes.byref(desc), _ptr(router_w), _ptr(router_bias), _ptr(x), _dtype_of(x), T,
                            _ptr(topk_idx), _ptr(topk_w), _ptr(offsets), _ptr(perm), _ptr(inv),
                            _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "moe_route")


def expert_ffn(layer: DeviceLayer, x, topk_w, offsets, perm, inv, residual, y, ws, stream=None):
    T = x.shape[0]
    w = layer.weights
    _check(load().moe_expert_ffn(ctypes.byref(layer.desc), ctypes.byref(w), _ptr(x), _dtype_of(x), T,
                                 _ptr(topk_w), _ptr(offsets), _ptr(perm), _ptr(inv), _ptr(residual), _ptr(y),
                                 _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "moe_expert_ffn")


def layer_forward(layer: DeviceLayer, x, residual, y, ws, stream=None):
    T = x.shape[0]
    w = layer.weights
    _check(load().moe_layer_forward(ctypes.byref(layer.desc), ctypes.byref(w), _ptr(x), _dtype_of(x), T,
                                    _ptr(residual), _ptr(y), _ptr(ws), ws.numel() * ws.element_size(),
                                    _stream(stream)), "moe_layer_forward")


def layer_forward_noalloc(layer: DeviceLayer, x, residual, y, stream=None):
    """The whole layer with the library's own fixed scratch array (no workspace
    argument); see moe_layer_forward_noalloc in include/moe2bit.h."""
    T = x.shape[0]
    w = layer.weights
    _check(load().moe_layer_forward_noalloc(ctypes.byref(layer.desc), ctypes.byref(w), _ptr(x), _dtype_of(x), T,
                                            _ptr(residual), _ptr(y), _stream(stream)), "moe_layer_forward_noalloc")


def alloc_workspace(desc: Desc, max_tokens: int, device="cuda"):
    import torch

    n = workspace_size(desc, max_tokens)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)
