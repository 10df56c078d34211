"""Pins of the oracle's Q4-style expert format (no GPU needed): a block
decoded by hand (tests/golden/q4_worked.txt), the affine law in the code and
the scaling law in d, and a dense float64 MoE over the decoded weights."""
import os

import numpy as np

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "q4_worked.txt")


def test_hand_decoded_block():
    block, expect = None, {}
    for line in open(GOLDEN):
        f = line.split()
        if not f or f[0].startswith("#"):
            continue
        if f[0] == "block":
            block = [int(v, 16) for v in f[1:]]
        elif f[0] == "expect":
            expect[int(f[1])] = float(f[2])
    out = oracle.dequant_q4(np.array([block[1:]], np.uint8), np.array([block[0]], np.uint16))
    for i, v in expect.items():
        assert out[i] == np.float32(v), (i, out[i], v)


def test_affine_in_code_and_linear_in_scale():
    # every code q at every position: w = d (q - 8) with d = 0.75 (fp16 0x3A00), and doubling d doubles w
    codes = np.zeros((16, 16), np.uint8)
    for q in range(16):
        codes[q] = q | (q << 4)
    w1 = oracle.dequant_q4(codes, np.full(16, 0x3A00, np.uint16)).reshape(16, 32)
    w2 = oracle.dequant_q4(codes, np.full(16, 0x3E00, np.uint16)).reshape(16, 32)  # 1.5
    for q in range(16):
        assert np.all(w1[q] == np.float32(0.75 * (q - 8)))
    assert np.array_equal(w2, 2 * w1)


def test_q4_layer_matches_dense_library_moe():
    cfg = synth.Config("q4_tiny", 3, 256, 64, 8, 2, 64, "f32", 1.0, False, 1, 0x5134)
    lw = synth.make_layer_q4(cfg)
    x = synth.make_x(cfg)
    res = synth.make_residual(cfg, cfg.T)
    y, idx, w = oracle.layer_forward(lw, x, res)
    E, I, H = cfg.E, cfg.I, cfg.H
    Wg = oracle.dequant_q4(lw.gate_codes.reshape(-1, 16), lw.gate_scales.reshape(-1)).reshape(E, I, H).astype(np.float64)
    Wu = oracle.dequant_q4(lw.up_codes.reshape(-1, 16), lw.up_scales.reshape(-1)).reshape(E, I, H).astype(np.float64)
    Wd = oracle.dequant_q4(lw.down_codes.reshape(-1, 16), lw.down_scales.reshape(-1)).reshape(E, H, I).astype(np.float64)
    silu = lambda z: z / (1.0 + np.exp(-z))
    x64 = x.astype(np.float64)
    ref = np.zeros((cfg.T, H))
    for t in range(cfg.T):
        for j in range(cfg.k):
            e = idx[t, j]
            ref[t] += float(w[t, j]) * (Wd[e] @ (silu(Wg[e] @ x64[t]) * (Wu[e] @ x64[t])))
    sg = synth.bf16_bits_to_f32(lw.sh_gate).astype(np.float64)
    su = synth.bf16_bits_to_f32(lw.sh_up).astype(np.float64)
    sd = synth.bf16_bits_to_f32(lw.sh_down).astype(np.float64)
    ref += (silu(x64 @ sg.T) * (x64 @ su.T)) @ sd.T + res.astype(np.float64)
    assert float(np.max(np.abs(y - ref)) / np.max(np.abs(ref))) < 1e-6
