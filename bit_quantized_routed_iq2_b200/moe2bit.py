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
# MOE2BIT_SO may name another build of the same library (the bounds-checked libmoe2bit_bc.so in its tests)
SO_PATH = os.environ.get("MOE2BIT_SO") or os.path.join(_HERE, "libmoe2bit.so")

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
    "moe_layer_forward_noalloc", "moe_read_status", "moe_read_status_noalloc", "moe_debug_inject",
    "moe_debug_gemv_operands_iq2", "moe_debug_gemv_operands_q2k", "moe_debug_tc_operands_iq2",
    "moe_debug_tc_operands_q2k", "moe_quantize_q2k", "moe_quantize_iq2",
    "moe_prefetch_layer", "moe_debug_bounds_check_build", "moe_debug_bounds_violations",
    "moe_cache_bytes", "moe_cache_create", "moe_cache_destroy", "moe_cache_read_stats", "moe_layer_forward_cached",
    "moe_workspace_size_mxfp4", "moe_layer_forward_mxfp4", "moe_debug_dequant_mxfp4",
    "moe_workspace_size_q4", "moe_layer_forward_q4", "moe_debug_dequant_q4", "moe_layer_forward_next",
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


class CacheStats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("calls", "hits", "misses", "bytes_copied")]


class Weights(ctypes.Structure):
    _fields_ = [
        (n, ctypes.c_void_p)
        for n in ("router_w", "router_bias", "gate_codes", "gate_d", "up_codes", "up_d",
                  "down_codes", "down_dd", "sh_gate", "sh_up", "sh_down")
    ]


class MxWeights(ctypes.Structure):
    """moe_mxfp4_weights (router, MXFP4 code and E8M0 scale planes, shared expert); the same
    pointer layout serves moe_q4_weights (code planes and fp16 d planes)."""

    _fields_ = [(n, ctypes.c_void_p) for n in (
        "router_w", "router_bias", "gate_codes", "gate_scales", "up_codes", "up_scales",
        "down_codes", "down_scales", "sh_gate", "sh_up", "sh_down")]


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
    L.moe_layer_forward_next.argtypes = [pd, pw, vp, i32, i32, vp, vp, vp, vp, sz, vp]
    L.moe_status_string.argtypes = [i32]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_debug_dequant_iq2.argtypes = [vp, vp, i64, vp, vp]
    L.moe_debug_dequant_q2k.argtypes = [vp, vp, i64, vp, vp]
    L.moe_workspace_size_mxfp4.argtypes = [pd, i32, ctypes.POINTER(sz)]
    L.moe_layer_forward_mxfp4.argtypes = [pd, ctypes.POINTER(MxWeights), vp, i32, i32, vp, vp, vp, sz, vp]
    L.moe_debug_dequant_mxfp4.argtypes = [vp, vp, i64, vp, vp]
    L.moe_workspace_size_q4.argtypes = [pd, i32, ctypes.POINTER(sz)]
    L.moe_layer_forward_q4.argtypes = [pd, ctypes.POINTER(MxWeights), vp, i32, i32, vp, vp, vp, sz, vp]
    L.moe_debug_dequant_q4.argtypes = [vp, vp, i64, vp, vp]
    L.moe_debug_gemv_operands_iq2.argtypes = [vp, i64, vp, vp, vp]
    L.moe_debug_gemv_operands_q2k.argtypes = [vp, i64, vp, vp, vp]
    L.moe_debug_tc_operands_iq2.argtypes = [vp, vp, i64, vp, vp]
    L.moe_debug_tc_operands_q2k.argtypes = [vp, vp, i64, vp, vp]
    L.moe_prefetch_layer.argtypes = [pd, pw, vp]
    L.moe_debug_bounds_check_build.argtypes = []
    L.moe_debug_bounds_violations.argtypes = [ctypes.POINTER(ctypes.c_uint64)]
    L.moe_cache_bytes.argtypes = [pd, i32, ctypes.POINTER(sz)]
    L.moe_cache_create.argtypes = [pd, pw, i32, vp, sz, ctypes.POINTER(vp)]
    L.moe_cache_destroy.argtypes = [vp]
    L.moe_cache_read_stats.argtypes = [vp, ctypes.POINTER(CacheStats)]
    L.moe_layer_forward_cached.argtypes = [vp, pw, vp, i32, i32, vp, vp, vp, sz, vp]
    L.moe_quantize_q2k.argtypes = [vp, i64, vp, vp, vp]
    L.moe_quantize_iq2.argtypes = [vp, i64, vp, vp, vp]
    L.moe_debug_grid.argtypes = [vp]
    L.moe_debug_grid.restype = None
    L.moe_layer_forward_noalloc.argtypes = [pd, pw, vp, i32, i32, vp, vp, vp]
    L.moe_read_status.argtypes = [vp, ctypes.POINTER(i32), vp]
    L.moe_read_status_noalloc.argtypes = [ctypes.POINTER(i32), vp]
    L.moe_debug_inject.argtypes = [i32, i64]
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


def quantize_q2k(w, codes, dd, stream=None):
    """fp32 device weights (numel % 256 == 0) -> Q2K codes [nb][80] u8 and dd [nb] (int32 view)."""
    nb = w.numel() // 256
    _check(load().moe_quantize_q2k(_ptr(w), nb, _ptr(codes), _ptr(dd), _stream(stream)), "moe_quantize_q2k")


def quantize_iq2(w, codes, d, stream=None):
    """fp32 device weights -> IQ2 codes [nb][64] u8 and d [nb] (int16 view of fp16 bits)."""
    nb = w.numel() // 256
    _check(load().moe_quantize_iq2(_ptr(w), nb, _ptr(codes), _ptr(d), _stream(stream)), "moe_quantize_iq2")


def bounds_violations() -> int:
    """Violations counted by the bounds-checked build since the last read (-1 from a normal build)."""
    L = load()
    if not L.moe_debug_bounds_check_build():
        return -1
    v = ctypes.c_uint64(0)
    _check(L.moe_debug_bounds_violations(ctypes.byref(v)), "moe_debug_bounds_violations")
    return int(v.value)


def debug_gemv_operands_iq2(codes, w, odd, stream=None):
    nb = codes.numel() // 64
    _check(load().moe_debug_gemv_operands_iq2(_ptr(codes), nb, _ptr(w), _ptr(odd), _stream(stream)),
           "moe_debug_gemv_operands_iq2")


def debug_gemv_operands_q2k(codes, scq, m, stream=None):
    nb = codes.numel() // 80
    _check(load().moe_debug_gemv_operands_q2k(_ptr(codes), nb, _ptr(scq), _ptr(m), _stream(stream)),
           "moe_debug_gemv_operands_q2k")


def debug_tc_operands_iq2(codes, d, out, stream=None):
    nb = codes.numel() // 64
    _check(load().moe_debug_tc_operands_iq2(_ptr(codes), _ptr(d), nb, _ptr(out), _stream(stream)),
           "moe_debug_tc_operands_iq2")


def debug_tc_operands_q2k(codes, dd, out, stream=None):
    nb = codes.numel() // 80
    _check(load().moe_debug_tc_operands_q2k(_ptr(codes), _ptr(dd), nb, _ptr(out), _stream(stream)),
           "moe_debug_tc_operands_q2k")


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


def layer_forward(layer: DeviceLayer, x, residual, y, ws, stream=None, y_next=None):
    """moe_layer_forward; with y_next (bf16 [T][H]) moe_layer_forward_next, which also writes bf16(y) there."""
    T = x.shape[0]
    w = layer.weights
    if y_next is None:
        _check(load().moe_layer_forward(ctypes.byref(layer.desc), ctypes.byref(w), _ptr(x), _dtype_of(x), T,
                                        _ptr(residual), _ptr(y), _ptr(ws), ws.numel() * ws.element_size(),
                                        _stream(stream)), "moe_layer_forward")
    else:
        _check(load().moe_layer_forward_next(ctypes.byref(layer.desc), ctypes.byref(w), _ptr(x), _dtype_of(x), T,
                                             _ptr(residual), _ptr(y), _ptr(y_next), _ptr(ws),
                                             ws.numel() * ws.element_size(), _stream(stream)),
               "moe_layer_forward_next")


def prefetch_layer(layer: DeviceLayer, stream=None):
    """L2 prefetch of the layer's router and shared expert (moe_prefetch_layer)."""
    w = layer.weights
    _check(load().moe_prefetch_layer(ctypes.byref(layer.desc), ctypes.byref(w), _stream(stream)), "moe_prefetch_layer")


def layer_forward_noalloc(layer: DeviceLayer, x, residual, y, stream=None):
    """The whole layer with the library's own fixed scratch array (no workspace
    argument); see moe_layer_forward_noalloc in include/moe2bit.h."""
    T = x.shape[0]
    w = layer.weights
    _check(load().moe_layer_forward_noalloc(ctypes.byref(layer.desc), ctypes.byref(w), _ptr(x), _dtype_of(x), T,
                                            _ptr(residual), _ptr(y), _stream(stream)), "moe_layer_forward_noalloc")


@dataclass
class MxDeviceLayer:
    """Device planes of a layer with MXFP4 routed experts."""

    desc: Desc
    tensors: dict

    @property
    def weights(self) -> "MxWeights":
        t = self.tensors
        return MxWeights(*[_ptr(t.get(n)) for n in (
            "router_w", "router_bias", "gate_codes", "gate_scales", "up_codes", "up_scales",
            "down_codes", "down_scales", "sh_gate", "sh_up", "sh_down")])


def to_device_mxfp4(lw, device="cuda") -> MxDeviceLayer:
    """Upload the host planes of an MXFP4 layer (synth.MxLayerWeights layout)."""
    import numpy as np
    import torch

    def up(a, dt):
        if a is None:
            return None
        return torch.from_numpy(np.ascontiguousarray(a).view(dt)).to(device)

    t = {
        "router_w": up(lw.router_w, np.int16),
        "router_bias": None if lw.router_bias is None else up(lw.router_bias, np.float32),
        "gate_codes": up(lw.gate_codes, np.uint8), "gate_scales": up(lw.gate_scales, np.uint8),
        "up_codes": up(lw.up_codes, np.uint8), "up_scales": up(lw.up_scales, np.uint8),
        "down_codes": up(lw.down_codes, np.uint8), "down_scales": up(lw.down_scales, np.uint8),
        "sh_gate": up(lw.sh_gate, np.int16) if lw.Is else None,
        "sh_up": up(lw.sh_up, np.int16) if lw.Is else None,
        "sh_down": up(lw.sh_down, np.int16) if lw.Is else None,
    }
    return MxDeviceLayer(desc_of(lw.H, lw.I, lw.E, lw.k, lw.Is), t)


def to_device_q4(lw, device="cuda") -> MxDeviceLayer:
    """Upload the host planes of a Q4-style layer (synth.Q4LayerWeights layout). The fp16 d planes
    travel as their bytes (the upload of to_device_mxfp4 views every scale plane as bytes)."""
    return to_device_mxfp4(lw, device)


def layer_forward_q4(layer: MxDeviceLayer, x, residual, y, ws, stream=None):
    T = x.shape[0]
    w = layer.weights
    _check(load().moe_layer_forward_q4(ctypes.byref(layer.desc), ctypes.byref(w), _ptr(x), _dtype_of(x), T,
                                       _ptr(residual), _ptr(y), _ptr(ws), ws.numel() * ws.element_size(),
                                       _stream(stream)), "moe_layer_forward_q4")


def debug_dequant_q4(codes, d, out, stream=None):
    nb = codes.numel() // 16
    _check(load().moe_debug_dequant_q4(_ptr(codes), _ptr(d), nb, _ptr(out), _stream(stream)), "moe_debug_dequant_q4")


def workspace_size_mxfp4(desc: Desc, max_tokens: int) -> int:
    n = ctypes.c_size_t(0)
    _check(load().moe_workspace_size_mxfp4(ctypes.byref(desc), max_tokens, ctypes.byref(n)), "moe_workspace_size_mxfp4")
    return int(n.value)


def alloc_workspace_mxfp4(desc: Desc, max_tokens: int, device="cuda"):
    import torch

    return torch.empty(max(workspace_size_mxfp4(desc, max_tokens), 16), dtype=torch.uint8, device=device)


def layer_forward_mxfp4(layer: MxDeviceLayer, x, residual, y, ws, stream=None):
    T = x.shape[0]
    w = layer.weights
    _check(load().moe_layer_forward_mxfp4(ctypes.byref(layer.desc), ctypes.byref(w), _ptr(x), _dtype_of(x), T,
                                          _ptr(residual), _ptr(y), _ptr(ws), ws.numel() * ws.element_size(),
                                          _stream(stream)), "moe_layer_forward_mxfp4")


def debug_dequant_mxfp4(codes, scales, out, stream=None):
    nb = codes.numel() // 16
    _check(load().moe_debug_dequant_mxfp4(_ptr(codes), _ptr(scales), nb, _ptr(out), _stream(stream)),
           "moe_debug_dequant_mxfp4")


def read_status(ws, stream=None) -> int:
    """Device status word of the last call that used workspace `ws` (0 = MOE_OK);
    synchronises `stream`."""
    v = ctypes.c_int32(-1)
    _check(load().moe_read_status(_ptr(ws), ctypes.byref(v), _stream(stream)), "moe_read_status")
    return int(v.value)


def read_status_noalloc(stream=None) -> int:
    """Device status word of the last moe_layer_forward_noalloc on this device."""
    v = ctypes.c_int32(-1)
    _check(load().moe_read_status_noalloc(ctypes.byref(v), _stream(stream)), "moe_read_status_noalloc")
    return int(v.value)


def debug_inject(mode: int, wait_limit_cycles: int = 0):
    """Fault injection for tests (see moe_debug_inject in include/moe2bit.h)."""
    _check(load().moe_debug_inject(mode, wait_limit_cycles), "moe_debug_inject")


class ExpertCache:
    """Host-resident routed experts with `n_slots` of them cached on the GPU
    (moe_cache_create in include/moe2bit.h). The host planes are copied once
    into page-locked memory owned by this object; the slot memory is a device
    tensor owned by this object."""

    ROUTED = ("gate_codes", "gate_d", "up_codes", "up_d", "down_codes", "down_dd")

    def __init__(self, lw, n_slots: int, device="cuda"):
        import numpy as np
        import torch

        self.desc = desc_of(lw.H, lw.I, lw.E, lw.k, lw.Is)
        self.host = {}
        for name in self.ROUTED:
            a = np.ascontiguousarray(getattr(lw, name))
            self.host[name] = torch.from_numpy(a.view(np.uint8).reshape(-1)).pin_memory()
        n = ctypes.c_size_t(0)
        _check(load().moe_cache_bytes(ctypes.byref(self.desc), n_slots, ctypes.byref(n)), "moe_cache_bytes")
        self.slot_mem = torch.empty(int(n.value), dtype=torch.uint8, device=device)
        pool = Weights()
        for name in self.ROUTED:
            setattr(pool, name, self.host[name].data_ptr())
        h = ctypes.c_void_p()
        _check(load().moe_cache_create(ctypes.byref(self.desc), ctypes.byref(pool), n_slots, _ptr(self.slot_mem),
                                       int(n.value), ctypes.byref(h)), "moe_cache_create")
        self.handle = h
        self.n_slots = n_slots

    def forward(self, layer: "DeviceLayer", x, residual, y, ws, stream=None):
        """The layer with the routed planes from the cache; `layer` supplies the
        device router and shared expert."""
        T = x.shape[0]
        w = layer.weights
        _check(load().moe_layer_forward_cached(self.handle, ctypes.byref(w), _ptr(x), _dtype_of(x), T, _ptr(residual),
                                               _ptr(y), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
               "moe_layer_forward_cached")

    def stats(self) -> dict:
        st = CacheStats()
        _check(load().moe_cache_read_stats(self.handle, ctypes.byref(st)), "moe_cache_read_stats")
        return {n: int(getattr(st, n)) for n, _ in CacheStats._fields_}

    def close(self):
        if getattr(self, "handle", None):
            load().moe_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def to_device_shared_only(lw, device="cuda") -> "DeviceLayer":
    """Device copies of the router and shared expert only (the routed planes
    stay on the host, for ExpertCache)."""
    import numpy as np
    import torch

    def up(a, dt):
        return None if a is None else torch.from_numpy(np.ascontiguousarray(a).view(dt)).to(device)

    t = {"router_w": up(lw.router_w, np.int16),
         "router_bias": None if lw.router_bias is None else up(lw.router_bias, np.float32),
         "sh_gate": up(lw.sh_gate, np.int16) if lw.Is else None,
         "sh_up": up(lw.sh_up, np.int16) if lw.Is else None,
         "sh_down": up(lw.sh_down, np.int16) if lw.Is else None}
    return DeviceLayer(desc_of(lw.H, lw.I, lw.E, lw.k, lw.Is), t)


def alloc_workspace(desc: Desc, max_tokens: int, device="cuda"):
    import torch

    n = workspace_size(desc, max_tokens)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)
