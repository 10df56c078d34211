"""Pins of the oracle's MXFP4 expert format (no GPU needed).

What they rest on: the OCP MX v1.0 table of FP4 E2M1 values and the E8M0
scale definition (tests/golden/mxfp4_worked.txt, with a block decoded by hand),
and a dense float64 MoE over library matmuls for the layer built on the
(pinned) decoder.
"""
import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mxfp4_worked.txt")


def _golden():
    table, block, expect = {}, None, {}
    for line in open(GOLDEN):
        f = line.split()
        if not f or f[0].startswith("#"):
            continue
        if f[0] == "e2m1":
            table[int(f[1])] = float(f[2])
        elif f[0] == "block":
            block = [int(v, 16) for v in f[1:]]
        elif f[0] == "expect":
            expect[int(f[1])] = float(f[2])
    return table, block, expect


def test_e2m1_values_are_the_specification_table():
    table, _, _ = _golden()
    assert sorted(table) == list(range(16))
    for c, v in table.items():
        got = oracle.e2m1(c)
        assert got == v and math.copysign(1.0, got) == math.copysign(1.0, v), (c, got, v)


def test_e8m0_scales_are_exact_powers_of_two():
    # every element code 2 (value 1): the block decodes to 2^(E - 127) exactly
    for E in (1, 100, 119, 127, 128, 200, 254):
        codes = np.full((1, 16), 0x22, np.uint8)
        out = oracle.dequant_mxfp4(codes, np.array([E], np.uint8))
        assert np.all(out == np.float32(2.0 ** (E - 127))), E


def test_hand_decoded_block():
    _, block, expect = _golden()
    out = oracle.dequant_mxfp4(np.array([block[1:]], np.uint8), np.array([block[0]], np.uint8))
    for i, v in expect.items():
        assert out[i] == np.float32(v) and math.copysign(1.0, out[i]) == math.copysign(1.0, v), (i, out[i], v)


def test_nibble_order_and_block_independence():
    # two blocks: swapping the two nibbles of a byte swaps the two elements; blocks do not mix
    rng = np.random.default_rng(7)
    codes = rng.integers(0, 256, (2, 16), dtype=np.uint8)
    scales = np.array([120, 130], np.uint8)
    a = oracle.dequant_mxfp4(codes, scales).reshape(2, 32)
    sw = ((codes >> 4) | (codes << 4)).astype(np.uint8)
    b = oracle.dequant_mxfp4(sw, scales).reshape(2, 32)
    assert np.array_equal(a[:, 0::2], b[:, 1::2]) and np.array_equal(a[:, 1::2], b[:, 0::2])
    one = oracle.dequant_mxfp4(codes[1:], scales[1:])
    assert np.array_equal(one, a[1])


def _dense_mx(lw):
    E, I, H = lw.E, lw.I, lw.H
    Wg = oracle.dequant_mxfp4(lw.gate_codes.reshape(-1, 16), lw.gate_scales.reshape(-1)).reshape(E, I, H)
    Wu = oracle.dequant_mxfp4(lw.up_codes.reshape(-1, 16), lw.up_scales.reshape(-1)).reshape(E, I, H)
    Wd = oracle.dequant_mxfp4(lw.down_codes.reshape(-1, 16), lw.down_scales.reshape(-1)).reshape(E, H, I)
    return Wg.astype(np.float64), Wu.astype(np.float64), Wd.astype(np.float64)


def _silu(z):
    return z / (1.0 + np.exp(-z))


@pytest.mark.parametrize("Is", [0, 64])
def test_mxfp4_layer_matches_dense_library_moe(Is):
    cfg = synth.Config("mx_tiny", 3, 256, 64, 8, 2, Is, "f32", 1.0, False, 1, 0x4D58)
    lw = synth.make_layer_mxfp4(cfg)
    x = synth.make_x(cfg)
    res = synth.make_residual(cfg, cfg.T)
    y, idx, w = oracle.layer_forward(lw, x, res)
    Wg, Wu, Wd = _dense_mx(lw)
    x64 = x.astype(np.float64)
    ref = np.zeros((cfg.T, cfg.H))
    for t in range(cfg.T):
        for j in range(cfg.k):
            e = idx[t, j]
            ref[t] += float(w[t, j]) * (Wd[e] @ (_silu(Wg[e] @ x64[t]) * (Wu[e] @ x64[t])))
    if Is:
        sg = synth.bf16_bits_to_f32(lw.sh_gate).astype(np.float64)
        su = synth.bf16_bits_to_f32(lw.sh_up).astype(np.float64)
        sd = synth.bf16_bits_to_f32(lw.sh_down).astype(np.float64)
        ref += (_silu(x64 @ sg.T) * (x64 @ su.T)) @ sd.T
    ref += res.astype(np.float64)
    assert float(np.max(np.abs(y - ref)) / np.max(np.abs(ref))) < 1e-6
    # routing does not depend on the expert format: the IQ2 layer of the same config routes alike
    _, idx2, w2 = oracle.layer_forward(synth.make_layer(cfg), x, res)
    assert np.array_equal(idx, idx2) and np.array_equal(w, w2)
