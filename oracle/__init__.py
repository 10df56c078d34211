"""CPU oracle for the routed 2-bit MoE FFN layer (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library and
its binding) never touches it. The arithmetic lives in ``moeref.c``; this file
only marshals numpy arrays into it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")          # single-threaded build
_SO_OMP = os.path.join(_HERE, "liboracle_omp.so")  # the same source with OpenMP on
_lib = None
_openmp = os.environ.get("MOEREF_OPENMP", "1") != "0"

F32, BF16 = 0, 1


class Desc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("hidden", "inter", "n_experts", "top_k", "shared_inter")]


class Weights(ctypes.Structure):
    _fields_ = [
        (n, ctypes.c_void_p)
        for n in (
            "router_w", "router_bias", "gate_codes", "gate_d", "up_codes", "up_d",
            "down_codes", "down_dd", "sh_gate", "sh_up", "sh_down",
        )
    ] + [("expert_format", ctypes.c_int32)] + [
        (n, ctypes.c_void_p) for n in ("gate_scales", "up_scales", "down_scales")
    ]


FMT_IQ2_Q2K, FMT_MXFP4, FMT_Q4, FMT_MXFP4_A8 = 0, 1, 2, 3


def build(force: bool = False, openmp: bool | None = None) -> str:
    """Compile the oracle: plain C99, -O2, no fast-math, no FMA contraction.

    Two builds of the one source: ``liboracle.so`` (single thread) and
    ``liboracle_omp.so`` (-fopenmp: independent tokens, assignments, rows and
    blocks spread over threads; every output is still computed by one thread
    with the same sequential loop, so both builds return identical bits).
    ``openmp=None`` builds both and returns the path of the one in use."""
    src = os.path.join(_HERE, "moeref.c")
    base = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c99", "-fPIC", "-shared"]
    for so, extra in ((_SO, ["-Wno-unknown-pragmas"]), (_SO_OMP, ["-fopenmp"])):
        if openmp is not None and (so == _SO_OMP) != openmp:
            continue
        if force or not os.path.exists(so) or os.path.getmtime(so) < os.path.getmtime(src):
            subprocess.check_call([*base, *extra, "-o", so, src, "-lm"])
    if openmp is None:
        return _SO_OMP if _openmp else _SO
    return _SO_OMP if openmp else _SO


def use_openmp(on: bool) -> None:
    """Select the build that lib() loads (before its first call)."""
    global _openmp
    if _lib is not None and on != _openmp:
        raise RuntimeError("the oracle library is already loaded")
    _openmp = on


def threads() -> int:
    """Threads the loaded build may use (1 for the single-threaded build)."""
    if not _openmp:
        return 1
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n and n.isdigit() else (os.cpu_count() or 1)


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build(openmp=_openmp))
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        L.moeref_f16_to_f64.restype = ctypes.c_double
        L.moeref_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.moeref_bf16_to_f64.restype = ctypes.c_double
        L.moeref_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.moeref_splitmix64_next.restype = ctypes.c_uint64
        L.moeref_splitmix64_next.argtypes = [ctypes.POINTER(ctypes.c_uint64)]
        L.moeref_grid.argtypes = [vp]
        L.moeref_dequant_iq2.argtypes = [vp, vp, i64, vp]
        L.moeref_dequant_q2k.argtypes = [vp, vp, i64, vp]
        L.moeref_e2m1.restype = ctypes.c_double
        L.moeref_e2m1.argtypes = [ctypes.c_uint]
        L.moeref_dequant_mxfp4.argtypes = [vp, vp, i64, vp]
        L.moeref_dequant_q4.argtypes = [vp, vp, i64, vp]
        L.moeref_e4m3_decode.restype = ctypes.c_double
        L.moeref_e4m3_decode.argtypes = [ctypes.c_uint]
        L.moeref_e4m3_encode.restype = ctypes.c_uint
        L.moeref_e4m3_encode.argtypes = [ctypes.c_double]
        L.moeref_quant_mxfp8.argtypes = [vp, i64, vp, vp]
        L.moeref_route.argtypes = [i32, i32, i32, vp, vp, vp, i32, i32, vp, vp, vp]
        L.moeref_permute.argtypes = [i32, i32, i32, vp, vp, vp, vp]
        L.moeref_f32_to_f16.restype = ctypes.c_uint16
        L.moeref_f32_to_f16.argtypes = [ctypes.c_float]
        L.moeref_quantize_q2k.argtypes = [vp, i64, vp, vp]
        L.moeref_quantize_iq2.argtypes = [vp, i64, vp, vp]
        L.moeref_expert_ffn.argtypes = [ctypes.POINTER(Desc), ctypes.POINTER(Weights), vp, i32, i32, vp, vp, vp, vp]
        L.moeref_layer_forward.argtypes = [ctypes.POINTER(Desc), ctypes.POINTER(Weights), vp, i32, i32, vp, vp, vp, vp]
        _lib = L
    return _lib


def _p(a):
    if a is None:
        return None
    assert isinstance(a, np.ndarray) and a.flags["C_CONTIGUOUS"], "arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(x: np.ndarray) -> int:
    if x.dtype == np.float32:
        return F32
    if x.dtype == np.uint16:
        return BF16
    raise TypeError("activations are fp32 or bf16 bit patterns (uint16)")


def _check(rc: int):
    if rc != 0:
        raise RuntimeError(f"oracle returned status {rc}")


def splitmix64(state: int, n: int) -> list[int]:
    s = ctypes.c_uint64(state)
    return [int(lib().moeref_splitmix64_next(ctypes.byref(s))) for _ in range(n)]


def grid() -> np.ndarray:
    out = np.zeros((256, 8), np.uint8)
    lib().moeref_grid(_p(out))
    return out


def f16_to_f64(h: int) -> float:
    return float(lib().moeref_f16_to_f64(h))


def dequant_iq2(codes: np.ndarray, d: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8).reshape(-1, 64)
    d = np.ascontiguousarray(d, np.uint16).reshape(-1)
    assert codes.shape[0] == d.shape[0]
    out = np.zeros(codes.shape[0] * 256, np.float32)
    lib().moeref_dequant_iq2(_p(codes), _p(d), codes.shape[0], _p(out))
    return out


def dequant_q2k(codes: np.ndarray, dd: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8).reshape(-1, 80)
    dd = np.ascontiguousarray(dd, np.uint32).reshape(-1)
    assert codes.shape[0] == dd.shape[0]
    out = np.zeros(codes.shape[0] * 256, np.float32)
    lib().moeref_dequant_q2k(_p(codes), _p(dd), codes.shape[0], _p(out))
    return out


def e2m1(c: int) -> float:
    """The value of one FP4 E2M1 element code (OCP MX v1.0)."""
    return float(lib().moeref_e2m1(int(c)))


def dequant_mxfp4(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """MXFP4 blocks (codes [nb][16] u8, E8M0 scales [nb] u8) -> fp32 [nb * 32]."""
    codes = np.ascontiguousarray(codes, np.uint8).reshape(-1, 16)
    scales = np.ascontiguousarray(scales, np.uint8).reshape(-1)
    assert codes.shape[0] == scales.shape[0]
    out = np.zeros(codes.shape[0] * 32, np.float32)
    lib().moeref_dequant_mxfp4(_p(codes), _p(scales), codes.shape[0], _p(out))
    return out


def e4m3_decode(c: int) -> float:
    """The value of one FP8 E4M3 code (OCP MX v1.0 element type; NaN for S.1111.111)."""
    return float(lib().moeref_e4m3_decode(int(c)))


def e4m3_encode(v: float) -> int:
    """Nearest finite E4M3 code to ``v`` (ties to the even code, saturating at 448)."""
    return int(lib().moeref_e4m3_encode(float(v)))


def quant_mxfp8(v: np.ndarray):
    """Values (a multiple of 32, blocks along the flattened array, float64) ->
    (E4M3 codes [nb][32] u8, E8M0 scale bytes [nb] u8) by the MX block rule."""
    v = np.ascontiguousarray(v, np.float64).reshape(-1)
    assert v.size % 32 == 0
    nb = v.size // 32
    el = np.zeros((nb, 32), np.uint8)
    sc = np.zeros(nb, np.uint8)
    lib().moeref_quant_mxfp8(_p(v), nb, _p(el), _p(sc))
    return el, sc


def dequant_q4(codes: np.ndarray, d: np.ndarray) -> np.ndarray:
    """Q4-style blocks (codes [nb][16] u8, fp16 d [nb]) -> fp32 [nb * 32]."""
    codes = np.ascontiguousarray(codes, np.uint8).reshape(-1, 16)
    d = np.ascontiguousarray(d, np.uint16).reshape(-1)
    assert codes.shape[0] == d.shape[0]
    out = np.zeros(codes.shape[0] * 32, np.float32)
    lib().moeref_dequant_q4(_p(codes), _p(d), codes.shape[0], _p(out))
    return out


def f32_to_f16(v: float) -> int:
    return int(lib().moeref_f32_to_f16(float(v)))


def quantize_q2k(w: np.ndarray):
    """Float weights (a multiple of 256, blocks along the flattened array) ->
    (codes [nb][80] u8, dd [nb] u32)."""
    w = np.ascontiguousarray(w, np.float32).reshape(-1)
    assert w.size % 256 == 0
    nb = w.size // 256
    codes = np.zeros((nb, 80), np.uint8)
    dd = np.zeros(nb, np.uint32)
    lib().moeref_quantize_q2k(_p(w), nb, _p(codes), _p(dd))
    return codes, dd


def quantize_iq2(w: np.ndarray):
    """Float weights -> (codes [nb][64] u8, d [nb] fp16 bits)."""
    w = np.ascontiguousarray(w, np.float32).reshape(-1)
    assert w.size % 256 == 0
    nb = w.size // 256
    codes = np.zeros((nb, 64), np.uint8)
    d = np.zeros(nb, np.uint16)
    lib().moeref_quantize_iq2(_p(w), nb, _p(codes), _p(d))
    return codes, d


def route(router_w, router_bias, x, k: int, want_logits: bool = False):
    x = np.ascontiguousarray(x)
    T, H = x.shape
    E = router_w.shape[0]
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    logits = np.zeros((T, E), np.float64) if want_logits else None
    rb = None if router_bias is None else np.ascontiguousarray(router_bias, np.float32)
    _check(lib().moeref_route(H, E, k, _p(np.ascontiguousarray(router_w)), _p(rb), _p(x), _dtype_code(x), T,
                              _p(idx), _p(w), _p(logits)))
    return (idx, w, logits) if want_logits else (idx, w)


def permute(idx: np.ndarray, E: int):
    idx = np.ascontiguousarray(idx, np.int32)
    T, k = idx.shape
    offsets = np.zeros(E + 1, np.int32)
    perm = np.zeros(T * k, np.int32)
    inv = np.zeros(T * k, np.int32)
    _check(lib().moeref_permute(T, k, E, _p(idx), _p(offsets), _p(perm), _p(inv)))
    return offsets, perm, inv


def _structs(lw, act_mxfp8: bool = False):
    """Oracle structs of a layer; a layer with ``fmt == "mxfp4"`` carries MXFP4
    code planes and E8M0 scale planes instead of the IQ2 / Q2K planes.
    ``act_mxfp8`` (MXFP4 layers only) quantises the routed experts' activations
    to MXFP8 before each contraction (the block-scaled FP4 x FP8 reading)."""
    desc = Desc(lw.H, lw.I, lw.E, lw.k, lw.Is)
    fmt = getattr(lw, "fmt", "iq2")
    assert not act_mxfp8 or fmt == "mxfp4", "MXFP8 activations go with MXFP4 weights"
    mx = fmt in ("mxfp4", "q4")
    arrs = (lw.router_w, lw.router_bias, lw.gate_codes, None if mx else lw.gate_d, lw.up_codes,
            None if mx else lw.up_d, lw.down_codes, None if mx else lw.down_dd, lw.sh_gate, lw.sh_up, lw.sh_down)
    keep = [np.ascontiguousarray(a) if a is not None else None for a in arrs]
    sc = [np.ascontiguousarray(getattr(lw, n)) for n in ("gate_scales", "up_scales", "down_scales")] if mx else []
    keep += sc
    code = FMT_MXFP4_A8 if act_mxfp8 else {"mxfp4": FMT_MXFP4, "q4": FMT_Q4}.get(fmt, FMT_IQ2_Q2K)
    W = Weights(*[_p(a) for a in keep[:11]], code,
                *([_p(a) for a in sc] if mx else [None, None, None]))
    return desc, W, keep


def expert_ffn(lw, x, idx, w, residual=None, act_mxfp8: bool = False) -> np.ndarray:
    x = np.ascontiguousarray(x)
    T = x.shape[0]
    desc, W, keep = _structs(lw, act_mxfp8)
    y = np.zeros((T, lw.H), np.float32)
    res = None if residual is None else np.ascontiguousarray(residual, np.float32)
    _check(lib().moeref_expert_ffn(ctypes.byref(desc), ctypes.byref(W), _p(x), _dtype_code(x), T,
                                   _p(np.ascontiguousarray(idx, np.int32)),
                                   _p(np.ascontiguousarray(w, np.float32)), _p(res), _p(y)))
    return y


def layer_forward(lw, x, residual=None, act_mxfp8: bool = False):
    x = np.ascontiguousarray(x)
    T = x.shape[0]
    desc, W, keep = _structs(lw, act_mxfp8)
    y = np.zeros((T, lw.H), np.float32)
    idx = np.zeros((T, lw.k), np.int32)
    w = np.zeros((T, lw.k), np.float32)
    res = None if residual is None else np.ascontiguousarray(residual, np.float32)
    _check(lib().moeref_layer_forward(ctypes.byref(desc), ctypes.byref(W), _p(x), _dtype_code(x), T,
                                      _p(res), _p(y), _p(idx), _p(w)))
    return y, idx, w
