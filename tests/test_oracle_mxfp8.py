"""Pins of the oracle's MXFP8 activation quantiser and of the MXFP4 x MXFP8
layer (no GPU needed).

What they rest on: the OCP MX v1.0 E4M3 encoding and block rule (values and
hand-encoded blocks in tests/golden/mxfp8_worked.txt), a library conversion to
float8_e4m3fn for the element rounding, and a dense float64 MoE whose
activation quantiser is written independently (numpy exponents, the library's
float8 rounding).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mxfp8_worked.txt")


def _golden():
    table, blocks, cur = {}, {}, None
    for line in open(GOLDEN):
        f = line.split()
        if not f or f[0].startswith("#"):
            continue
        if f[0] == "e4m3":
            table[int(f[1], 16)] = float(f[2])
        elif f[0] == "block":
            cur = {"v": np.zeros(32), "scale": None, "el": {}}
            blocks[f[1]] = cur
        elif f[0] == "v":
            cur["v"][int(f[1])] = float(f[2])
        elif f[0] == "scale":
            cur["scale"] = int(f[1], 16)
        elif f[0] == "el":
            cur["el"][int(f[1])] = int(f[2], 16)
    return table, blocks


def _same(a, b):
    if math.isnan(b):
        return math.isnan(a)
    return a == b and math.copysign(1.0, a) == math.copysign(1.0, b)


def test_e4m3_values_are_the_specification_encoding():
    table, _ = _golden()
    for c, v in table.items():
        assert _same(oracle.e4m3_decode(c), v), (hex(c), oracle.e4m3_decode(c), v)


def test_e4m3_decoder_matches_library_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        assert _same(oracle.e4m3_decode(c), float(lib[c])), hex(c)


def test_e4m3_encoder_matches_library_rounding_in_range():
    # the library rounds to nearest even; in range (|v| below the 464 midpoint) no saturation is involved
    rng = np.random.default_rng(11)
    v = np.concatenate([rng.standard_normal(4000) * 60.0, rng.standard_normal(4000) * 3e-3,
                        rng.uniform(-463.0, 463.0, 4000), [0.0, -0.0, 2.0 ** -10, 3 * 2.0 ** -10, -2.0 ** -9]])
    lib = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(x) for x in v], np.uint8)
    assert np.array_equal(got, lib)


def test_e4m3_encoder_ties_and_saturation():
    assert oracle.e4m3_encode(1 + 2.0 ** -4) == 0x38      # halfway 1 .. 1.125: even code (1)
    assert oracle.e4m3_encode(1 + 3 * 2.0 ** -4) == 0x3A  # halfway 1.125 .. 1.25: even code (1.25)
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00          # halfway 0 .. 2^-9: even code (0)
    assert oracle.e4m3_encode(3 * 2.0 ** -10) == 0x02      # halfway 2^-9 .. 2^-8: even code
    assert oracle.e4m3_encode(500.0) == 0x7E and oracle.e4m3_encode(-1e30) == 0xFE
    assert oracle.e4m3_encode(-0.0) == 0x80 and oracle.e4m3_encode(-1e-30) == 0x80
    for c in list(range(0x7F)) + list(range(0x80, 0xFF)):  # every finite code round-trips
        assert oracle.e4m3_encode(oracle.e4m3_decode(c)) == c, hex(c)


def test_hand_encoded_blocks():
    _, blocks = _golden()
    for name, b in blocks.items():
        el, sc = oracle.quant_mxfp8(b["v"])
        assert sc[0] == b["scale"], (name, sc[0], b["scale"])
        for i in range(32):
            assert el[0, i] == b["el"].get(i, 0), (name, i, hex(el[0, i]))


def test_block_rule_bounds_and_independence():
    rng = np.random.default_rng(5)
    v = rng.standard_normal(32 * 64) * np.repeat(2.0 ** rng.integers(-20, 20, 64), 32)
    el, sc = oracle.quant_mxfp8(v)
    dec = np.array([oracle.e4m3_decode(c) for c in el.reshape(-1)]).reshape(-1, 32)
    X = sc.astype(np.int64) - 127
    q = dec * np.exp2(X)[:, None]
    b = v.reshape(-1, 32)
    amax = np.abs(b).max(1)
    # the block maximum lands in [256, 512) before rounding, so no element needs a larger exponent
    assert np.all((amax / np.exp2(X) >= 256) & (amax / np.exp2(X) < 512))
    # half an E4M3 step: 2^-4 relative in the normal range, 2^-10 * 2^X among the subnormals;
    # a block maximum above 448 saturates (at most 512 - 448 before scaling)
    tol = np.maximum(np.abs(b) * 2.0 ** -4, np.exp2(X - 10)[:, None])
    sat = np.abs(b) / np.exp2(X)[:, None] > 448
    assert np.all((np.abs(q - b) <= tol) | sat)
    # blocks do not interact
    el1, sc1 = oracle.quant_mxfp8(v[32 * 7:32 * 8])
    assert np.array_equal(el1[0], el[7]) and sc1[0] == sc[7]


def _mx8_independent(v):
    """MX block rule written apart from the oracle: numpy exponents, the library's float8 rounding."""
    b = np.asarray(v, np.float64).reshape(-1, 32)
    amax = np.abs(b).max(1)
    _, e2 = np.frexp(amax)
    X = np.where(amax > 0, e2 - 1 - 8, -127).clip(-127, 127).astype(np.float64)
    s = np.clip(b / np.exp2(X)[:, None], -448.0, 448.0)
    q = torch.from_numpy(s).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    return (q * np.exp2(X)[:, None]).reshape(np.shape(v))


def _silu(z):
    return z / (1.0 + np.exp(-z))


@pytest.mark.parametrize("Is", [0, 64])
def test_mxfp4_a8_layer_matches_dense_library_moe(Is):
    cfg = synth.Config("mx8_tiny", 5, 256, 64, 8, 2, Is, "bf16", 1.0, False, 1, 0x4D38)
    lw = synth.make_layer_mxfp4(cfg)
    x = synth.make_x(cfg)
    res = synth.make_residual(cfg, cfg.T)
    y, idx, w = oracle.layer_forward(lw, x, res, act_mxfp8=True)
    E, I, H = lw.E, lw.I, lw.H
    Wg = oracle.dequant_mxfp4(lw.gate_codes.reshape(-1, 16), lw.gate_scales.reshape(-1)).reshape(E, I, H)
    Wu = oracle.dequant_mxfp4(lw.up_codes.reshape(-1, 16), lw.up_scales.reshape(-1)).reshape(E, I, H)
    Wd = oracle.dequant_mxfp4(lw.down_codes.reshape(-1, 16), lw.down_scales.reshape(-1)).reshape(E, H, I)
    Wg, Wu, Wd = (a.astype(np.float64) for a in (Wg, Wu, Wd))
    x64 = synth.bf16_bits_to_f32(x).astype(np.float64)
    xq = _mx8_independent(x64)
    ref = np.zeros((cfg.T, H))
    for t in range(cfg.T):
        for j in range(cfg.k):
            e = idx[t, j]
            h = _silu(Wg[e] @ xq[t]) * (Wu[e] @ xq[t])
            ref[t] += float(w[t, j]) * (Wd[e] @ _mx8_independent(h))
    if Is:  # the shared expert takes the exact activations
        sg = synth.bf16_bits_to_f32(lw.sh_gate).astype(np.float64)
        su = synth.bf16_bits_to_f32(lw.sh_up).astype(np.float64)
        sd = synth.bf16_bits_to_f32(lw.sh_down).astype(np.float64)
        ref += (_silu(x64 @ sg.T) * (x64 @ su.T)) @ sd.T
    ref += res.astype(np.float64)
    assert float(np.max(np.abs(y - ref)) / np.max(np.abs(ref))) < 1e-6
    # the quantised activations change the result: the pin distinguishes the two formats
    y_exact, _, _ = oracle.layer_forward(lw, x, res)
    assert float(np.max(np.abs(y - y_exact)) / np.max(np.abs(y_exact))) > 1e-4
