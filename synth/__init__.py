"""Seeded synthetic inputs for the routed 2-bit MoE FFN layer.

This module only draws random numbers and arranges them in the input planes
(see ``moegen.c`` for the generator and the recipes). It contains none of the
layer's arithmetic, so the CPU oracle and the CUDA library can both be fed from
it without sharing any computation.

Shapes and value recipes follow the five synthetic workloads of the routed
MoE layer of the ds4 engine ("ds4 : analyse pratique pour un usage documenté",
section « Support de modèles et choix de quantification »: routed experts in
2-bit, gate/up IQ2_XXS-style, down Q2_K-style, router and shared expert
unquantized).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libmoegen.so")
_lib = None

# tensor ids of the per-tensor streams
T_ROUTER_W, T_ROUTER_B, T_GATE_CODES, T_GATE_D, T_UP_CODES, T_UP_D = 0, 1, 2, 3, 4, 5
T_DOWN_CODES, T_DOWN_DD, T_SH_GATE, T_SH_UP, T_SH_DOWN, T_X, T_RESID = 6, 7, 8, 9, 10, 11, 12

T_MX_GATE_CODES, T_MX_GATE_E, T_MX_UP_CODES, T_MX_UP_E, T_MX_DOWN_CODES, T_MX_DOWN_E = 13, 14, 15, 16, 17, 18

IQ2_BLOCK_BYTES = 64  # code bytes per 256-weight block (plus one fp16 d)
Q2K_BLOCK_BYTES = 80  # code bytes per 256-weight block (plus one u32 d|dmin)
QK = 256


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "moegen.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", _SO, src, "-lm"]
        )
    return _SO


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        u64, i64, i32, vp, dbl = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_double
        L.moegen_seed.restype = u64
        L.moegen_seed.argtypes = [u64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32]
        L.moegen_splitmix64_at.restype = u64
        L.moegen_splitmix64_at.argtypes = [u64, u64]
        for name in ("moegen_bytes",):
            getattr(L, name).argtypes = [u64, vp, i64]
        for name in ("moegen_normal_f32", "moegen_normal_bf16", "moegen_f16_scale", "moegen_q2k_dd"):
            getattr(L, name).argtypes = [u64, vp, i64, dbl]
        L.moegen_permutation.argtypes = [u64, vp, i32]
        L.moegen_zipf_bias.argtypes = [u64, vp, i32, dbl]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def seed(cfg_seed: int, layer: int, tensor: int, expert: int = 0) -> int:
    return int(lib().moegen_seed(cfg_seed, layer, tensor, expert))


def rand_bytes(s: int, shape) -> np.ndarray:
    out = np.empty(shape, dtype=np.uint8)
    lib().moegen_bytes(s, _p(out), out.size)
    return out


def normal_f32(s: int, shape, std: float) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    lib().moegen_normal_f32(s, _p(out), out.size, std)
    return out


def normal_bf16(s: int, shape, std: float) -> np.ndarray:
    out = np.empty(shape, dtype=np.uint16)
    lib().moegen_normal_bf16(s, _p(out), out.size, std)
    return out


def f16_scale(s: int, shape, base: float) -> np.ndarray:
    out = np.empty(shape, dtype=np.uint16)
    lib().moegen_f16_scale(s, _p(out), out.size, base)
    return out


def q2k_dd(s: int, shape, base: float) -> np.ndarray:
    out = np.empty(shape, dtype=np.uint32)
    lib().moegen_q2k_dd(s, _p(out), out.size, base)
    return out


def permutation(s: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    lib().moegen_permutation(s, _p(out), n)
    return out


def zipf_bias(s: int, n: int, exponent: float) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    lib().moegen_zipf_bias(s, _p(out), n, exponent)
    return out


@dataclass(frozen=True)
class Config:
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    Is: int
    x_dtype: str  # "f32" or "bf16"
    x_std: float
    zipf: bool
    layers: int = 1
    seed: int = 0


# The five synthetic workloads. "N(0,0.5)" of the prefill case is read as
# variance 0.5 (std sqrt(0.5)); the tiny case's shared-expert width equals I.
CONFIGS = {
    "tiny": Config("tiny", 4, 256, 128, 8, 2, 128, "f32", 1.0, False, 1, 0xD5400001),
    "decode1": Config("decode1", 1, 7168, 2048, 256, 8, 2048, "bf16", 1.0, False, 1, 0xD5400002),
    "decode32": Config("decode32", 32, 7168, 2048, 256, 8, 2048, "bf16", 1.0, True, 1, 0xD5400003),
    "prefill": Config("prefill", 2048, 7168, 2048, 256, 8, 2048, "bf16", math.sqrt(0.5), False, 1, 0xD5400004),
    "stack": Config("stack", 16, 7168, 2048, 256, 8, 2048, "bf16", 1.0, True, 8, 0xD5400005),
}

IQ2_D_BASE_NUM = 1.0 / 67.1  # weight rms ~ 1/sqrt(K) for the IQ2-style planes
Q2K_D_BASE_NUM = 1.0 / 13.9  # weight rms ~ 1/sqrt(K) for the Q2K-style planes


@dataclass
class LayerWeights:
    """Host planes of one layer, in the library's layout (structure of arrays).

    gate/up: codes [E][I*H/256][64] u8, d [E][I*H/256] fp16 bits
    down:    codes [E][H*I/256][80] u8, dd [E][H*I/256] u32 (fp16 d | fp16 dmin << 16)
    router:  w [E][H] bf16 bits, bias [E] f32 or None
    shared:  gate/up [Is][H] bf16 bits, down [H][Is] bf16 bits
    """

    H: int
    I: int
    E: int
    k: int
    Is: int
    router_w: np.ndarray
    router_bias: np.ndarray | None
    gate_codes: np.ndarray
    gate_d: np.ndarray
    up_codes: np.ndarray
    up_d: np.ndarray
    down_codes: np.ndarray
    down_dd: np.ndarray
    sh_gate: np.ndarray
    sh_up: np.ndarray
    sh_down: np.ndarray
    extra: dict = field(default_factory=dict)


def make_layer(cfg: Config | dict, layer: int = 0, cfg_seed: int | None = None, experts=None) -> LayerWeights:
    """Generate one layer. ``experts`` (optional iterable) limits generation of the
    routed planes to those experts; the others stay zero (used to keep host memory
    small when only a few experts are read)."""
    if isinstance(cfg, dict):
        cfg = Config(**cfg)
    cs = cfg.seed if cfg_seed is None else cfg_seed
    H, I, E, Is = cfg.H, cfg.I, cfg.E, cfg.Is
    assert (I * H) % QK == 0
    nb = I * H // QK
    rw = normal_bf16(seed(cs, layer, T_ROUTER_W), (E, H), 1.28 / math.sqrt(H))
    rb = zipf_bias(seed(cs, layer, T_ROUTER_B), E, 1.1) if cfg.zipf else None
    gate_codes = np.zeros((E, nb, IQ2_BLOCK_BYTES), np.uint8)
    up_codes = np.zeros((E, nb, IQ2_BLOCK_BYTES), np.uint8)
    gate_d = np.zeros((E, nb), np.uint16)
    up_d = np.zeros((E, nb), np.uint16)
    down_codes = np.zeros((E, nb, Q2K_BLOCK_BYTES), np.uint8)
    down_dd = np.zeros((E, nb), np.uint32)
    iq2_base = IQ2_D_BASE_NUM / math.sqrt(H)
    q2k_base = Q2K_D_BASE_NUM / math.sqrt(I)
    for e in range(E) if experts is None else sorted(set(int(v) for v in experts)):
        lib().moegen_bytes(seed(cs, layer, T_GATE_CODES, e), _p(gate_codes[e]), gate_codes[e].size)
        lib().moegen_bytes(seed(cs, layer, T_UP_CODES, e), _p(up_codes[e]), up_codes[e].size)
        lib().moegen_bytes(seed(cs, layer, T_DOWN_CODES, e), _p(down_codes[e]), down_codes[e].size)
        lib().moegen_f16_scale(seed(cs, layer, T_GATE_D, e), _p(gate_d[e]), nb, iq2_base)
        lib().moegen_f16_scale(seed(cs, layer, T_UP_D, e), _p(up_d[e]), nb, iq2_base)
        lib().moegen_q2k_dd(seed(cs, layer, T_DOWN_DD, e), _p(down_dd[e]), nb, q2k_base)
    sg = normal_bf16(seed(cs, layer, T_SH_GATE), (Is, H), 1.0 / math.sqrt(H))
    su = normal_bf16(seed(cs, layer, T_SH_UP), (Is, H), 1.0 / math.sqrt(H))
    sd = normal_bf16(seed(cs, layer, T_SH_DOWN), (H, Is), 1.0 / math.sqrt(max(Is, 1)))
    return LayerWeights(H, I, E, cfg.k, Is, rw, rb, gate_codes, gate_d, up_codes, up_d, down_codes, down_dd, sg, su, sd)


@dataclass
class MxLayerWeights:
    """Host planes of one layer with MXFP4 routed experts (library layout).

    gate/up: codes [E][I][H/2] u8 (two E2M1 elements per byte, low nibble first),
             scales [E][I][H/32] u8 (E8M0)
    down:    codes [E][H][I/2] u8, scales [E][H][I/32] u8
    router and shared expert: as LayerWeights (the same streams as make_layer)
    """

    H: int
    I: int
    E: int
    k: int
    Is: int
    router_w: np.ndarray
    router_bias: np.ndarray | None
    gate_codes: np.ndarray
    gate_scales: np.ndarray
    up_codes: np.ndarray
    up_scales: np.ndarray
    down_codes: np.ndarray
    down_scales: np.ndarray
    sh_gate: np.ndarray
    sh_up: np.ndarray
    sh_down: np.ndarray
    fmt: str = "mxfp4"


# mean square of the 16 E2M1 values (uniform codes): (0 + .25 + 1 + 2.25 + 4 + 9 + 16 + 36) / 8
MX_ELEM_MS = 8.5625


def mx_scale_exponent(K: int) -> int:
    """E8M0 exponent that puts the weight RMS near 1/sqrt(K) for uniform codes."""
    return 127 + int(round(math.log2(1.0 / (math.sqrt(MX_ELEM_MS) * math.sqrt(K)))))


def mx_scales(s: int, shape, K: int) -> np.ndarray:
    """E8M0 scale bytes: the exponent of mx_scale_exponent(K) plus a uniform jitter of -1, 0 or +1."""
    return (mx_scale_exponent(K) - 1 + rand_bytes(s, shape) % 3).astype(np.uint8)


def make_layer_mxfp4(cfg: Config | dict, layer: int = 0, cfg_seed: int | None = None, experts=None) -> MxLayerWeights:
    """One layer with MXFP4 routed experts: uniform random code bytes, scales from
    mx_scales; router and shared expert from the streams of make_layer."""
    if isinstance(cfg, dict):
        cfg = Config(**cfg)
    cs = cfg.seed if cfg_seed is None else cfg_seed
    H, I, E, Is = cfg.H, cfg.I, cfg.E, cfg.Is
    assert H % 32 == 0 and I % 32 == 0
    rw = normal_bf16(seed(cs, layer, T_ROUTER_W), (E, H), 1.28 / math.sqrt(H))
    rb = zipf_bias(seed(cs, layer, T_ROUTER_B), E, 1.1) if cfg.zipf else None
    gc = np.zeros((E, I, H // 2), np.uint8)
    uc = np.zeros((E, I, H // 2), np.uint8)
    dc = np.zeros((E, H, I // 2), np.uint8)
    gs = np.zeros((E, I, H // 32), np.uint8)
    us = np.zeros((E, I, H // 32), np.uint8)
    ds = np.zeros((E, H, I // 32), np.uint8)
    for e in range(E) if experts is None else sorted(set(int(v) for v in experts)):
        lib().moegen_bytes(seed(cs, layer, T_MX_GATE_CODES, e), _p(gc[e]), gc[e].size)
        lib().moegen_bytes(seed(cs, layer, T_MX_UP_CODES, e), _p(uc[e]), uc[e].size)
        lib().moegen_bytes(seed(cs, layer, T_MX_DOWN_CODES, e), _p(dc[e]), dc[e].size)
        gs[e] = mx_scales(seed(cs, layer, T_MX_GATE_E, e), gs[e].shape, H)
        us[e] = mx_scales(seed(cs, layer, T_MX_UP_E, e), us[e].shape, H)
        ds[e] = mx_scales(seed(cs, layer, T_MX_DOWN_E, e), ds[e].shape, I)
    sg = normal_bf16(seed(cs, layer, T_SH_GATE), (Is, H), 1.0 / math.sqrt(H))
    su = normal_bf16(seed(cs, layer, T_SH_UP), (Is, H), 1.0 / math.sqrt(H))
    sd = normal_bf16(seed(cs, layer, T_SH_DOWN), (H, Is), 1.0 / math.sqrt(max(Is, 1)))
    return MxLayerWeights(H, I, E, cfg.k, Is, rw, rb, gc, gs, uc, us, dc, ds, sg, su, sd)


T_Q4_GATE_CODES, T_Q4_GATE_D, T_Q4_UP_CODES, T_Q4_UP_D, T_Q4_DOWN_CODES, T_Q4_DOWN_D = 19, 20, 21, 22, 23, 24
# mean square of q - 8 for uniform 4-bit codes: (sum of (q-8)^2, q = 0..15) / 16
Q4_ELEM_MS = 21.5


@dataclass
class Q4LayerWeights:
    """Host planes of one layer with Q4-style routed experts (library layout).

    gate/up: codes [E][I][H/2] u8 (two 4-bit codes per byte, low nibble first), d [E][I][H/32] fp16 bits
    down:    codes [E][H][I/2] u8, d [E][H][I/32] fp16 bits
    router and shared expert: as LayerWeights (the same streams as make_layer)
    """

    H: int
    I: int
    E: int
    k: int
    Is: int
    router_w: np.ndarray
    router_bias: np.ndarray | None
    gate_codes: np.ndarray
    gate_scales: np.ndarray
    up_codes: np.ndarray
    up_scales: np.ndarray
    down_codes: np.ndarray
    down_scales: np.ndarray
    sh_gate: np.ndarray
    sh_up: np.ndarray
    sh_down: np.ndarray
    fmt: str = "q4"


def make_layer_q4(cfg: Config | dict, layer: int = 0, cfg_seed: int | None = None, experts=None) -> Q4LayerWeights:
    """One layer with Q4-style routed experts: uniform random code bytes, fp16 scales from the
    f16_scale recipe with base 1 / (sqrt(Q4_ELEM_MS) sqrt(K)); router and shared expert from the
    streams of make_layer."""
    if isinstance(cfg, dict):
        cfg = Config(**cfg)
    cs = cfg.seed if cfg_seed is None else cfg_seed
    H, I, E, Is = cfg.H, cfg.I, cfg.E, cfg.Is
    assert H % 32 == 0 and I % 32 == 0
    rw = normal_bf16(seed(cs, layer, T_ROUTER_W), (E, H), 1.28 / math.sqrt(H))
    rb = zipf_bias(seed(cs, layer, T_ROUTER_B), E, 1.1) if cfg.zipf else None
    gc = np.zeros((E, I, H // 2), np.uint8)
    uc = np.zeros((E, I, H // 2), np.uint8)
    dc = np.zeros((E, H, I // 2), np.uint8)
    gd = np.zeros((E, I, H // 32), np.uint16)
    ud = np.zeros((E, I, H // 32), np.uint16)
    dd = np.zeros((E, H, I // 32), np.uint16)
    bh, bi = 1.0 / math.sqrt(Q4_ELEM_MS * H), 1.0 / math.sqrt(Q4_ELEM_MS * I)
    for e in range(E) if experts is None else sorted(set(int(v) for v in experts)):
        lib().moegen_bytes(seed(cs, layer, T_Q4_GATE_CODES, e), _p(gc[e]), gc[e].size)
        lib().moegen_bytes(seed(cs, layer, T_Q4_UP_CODES, e), _p(uc[e]), uc[e].size)
        lib().moegen_bytes(seed(cs, layer, T_Q4_DOWN_CODES, e), _p(dc[e]), dc[e].size)
        lib().moegen_f16_scale(seed(cs, layer, T_Q4_GATE_D, e), _p(gd[e]), gd[e].size, bh)
        lib().moegen_f16_scale(seed(cs, layer, T_Q4_UP_D, e), _p(ud[e]), ud[e].size, bh)
        lib().moegen_f16_scale(seed(cs, layer, T_Q4_DOWN_D, e), _p(dd[e]), dd[e].size, bi)
    sg = normal_bf16(seed(cs, layer, T_SH_GATE), (Is, H), 1.0 / math.sqrt(H))
    su = normal_bf16(seed(cs, layer, T_SH_UP), (Is, H), 1.0 / math.sqrt(H))
    sd = normal_bf16(seed(cs, layer, T_SH_DOWN), (H, Is), 1.0 / math.sqrt(max(Is, 1)))
    return Q4LayerWeights(H, I, E, cfg.k, Is, rw, rb, gc, gd, uc, ud, dc, dd, sg, su, sd)


def make_token(cfg: Config, t: int, attempt: int = 0, layer: int = 0, cfg_seed: int | None = None) -> np.ndarray:
    """One token's activations (H,), fp32 or bf16 bits; ``attempt`` selects the
    redraw stream used when a token is rejected for a near-tie in the router."""
    cs = cfg.seed if cfg_seed is None else cfg_seed
    s = seed(cs, layer, T_X, t + (attempt << 24))
    if cfg.x_dtype == "f32":
        return normal_f32(s, (cfg.H,), cfg.x_std)
    return normal_bf16(s, (cfg.H,), cfg.x_std)


def make_x(cfg: Config, T: int | None = None, layer: int = 0, cfg_seed: int | None = None) -> np.ndarray:
    T = cfg.T if T is None else T
    return np.stack([make_token(cfg, t, 0, layer, cfg_seed) for t in range(T)]) if T else np.zeros(
        (0, cfg.H), np.float32 if cfg.x_dtype == "f32" else np.uint16
    )


def make_x_fast(cfg: Config, T: int, layer: int = 0, cfg_seed: int | None = None) -> np.ndarray:
    """All tokens from one stream (bench inputs, no near-tie screening)."""
    cs = cfg.seed if cfg_seed is None else cfg_seed
    s = seed(cs, layer, T_X, 0xFFFFFF)
    if cfg.x_dtype == "f32":
        return normal_f32(s, (T, cfg.H), cfg.x_std)
    return normal_bf16(s, (T, cfg.H), cfg.x_std)


def make_residual(cfg: Config, T: int, cfg_seed: int | None = None) -> np.ndarray:
    cs = cfg.seed if cfg_seed is None else cfg_seed
    return normal_f32(seed(cs, 0, T_RESID), (T, cfg.H), 1.0)


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (a layout change, not arithmetic)."""
    return (a.astype(np.uint32) << 16).view(np.float32)
