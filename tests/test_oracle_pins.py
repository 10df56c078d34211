"""Pins of the CPU oracle to facts outside itself (no GPU needed).

Each pin names what it rests on: a published value, a hand-worked example
(tests/golden/), an invariant that the format or the mathematics fixes, or a
reduction to a library routine (numpy / scipy float64).
"""
import hashlib
import math
import os
from fractions import Fraction

import numpy as np
import pytest
from scipy.special import softmax

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- splitmix64
def test_splitmix64_published_first_outputs():
    # splitmix64 (Steele, Lea, Flood, OOPSLA 2014) from state 0: the widely
    # published first three outputs of the reference generator.
    assert oracle.splitmix64(0, 3) == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


# ----------------------------------------------------------------------- grid
def test_grid_invariants():
    g = oracle.grid()
    assert g.shape == (256, 8)
    assert set(np.unique(g).tolist()) <= {8, 25, 43}
    assert len({bytes(r) for r in g}) == 256, "rows must be distinct"
    # every row is a base-3 word over {8,25,43}: the three levels all occur
    assert set(np.unique(g).tolist()) == {8, 25, 43}


def test_grid_first_row_from_generator():
    # Row 0 is the first accepted draw: c = (next() >> 32) mod 6561 of the
    # generator seeded with 0x4951325F47524944, digits least significant first.
    c = (oracle.splitmix64(0x4951325F47524944, 1)[0] >> 32) % 6561
    digits = [(c // 3**e) % 3 for e in range(8)]
    assert oracle.grid()[0].tolist() == [(8, 25, 43)[v] for v in digits]


def test_grid_regression_hash():
    # Regression pin (not a parity pin): recorded at first generation.
    h = hashlib.sha256(oracle.grid().tobytes()).hexdigest()
    assert h == "f7984473e4e3901291569559d48feccd32473efa5803db64bfffed66f3d8fdda"


# ---------------------------------------------------------- golden dequant
def _load_golden():
    cases = []
    cur = None
    for line in open(os.path.join(GOLDEN, "dequant_worked.txt")):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        tok = line.split()
        if tok[0] == "case":
            cur = {"name": tok[1], "fmt": tok[2], "d": int(tok[3].split("=")[1], 16), "set": [], "expect": []}
            cases.append(cur)
        elif tok[0] == "set":
            cur["set"].append((int(tok[1]), [int(b, 16) for b in tok[2:]]))
        elif tok[0] == "expect":
            cur["expect"].append((int(tok[1]), float(tok[2]), int(tok[3], 16) if len(tok) > 3 else None))
    return cases


@pytest.mark.parametrize("case", _load_golden(), ids=lambda c: c["name"])
def test_dequant_worked_examples(case):
    nbytes = 64 if case["fmt"] == "iq2" else 80
    codes = np.zeros(nbytes, np.uint8)
    for off, bs in case["set"]:
        codes[off:off + len(bs)] = bs
    if case["fmt"] == "iq2":
        out = oracle.dequant_iq2(codes, np.array([case["d"]], np.uint16))
    else:
        out = oracle.dequant_q2k(codes, np.array([case["d"]], np.uint32))
    for i, val, bits in case["expect"]:
        assert out[i] == np.float32(val), (case["name"], i, out[i], val)
        if bits is not None:
            assert int(out[i:i + 1].view(np.uint32)[0]) == bits


# --------------------------------------------------------- format invariants
def _pack_iq2(idx, sigma, ls):
    """Pack fields [8 sub-blocks][4 groups] into the 64 code bytes."""
    b = np.zeros(64, np.uint8)
    for s in range(8):
        b[8 * s:8 * s + 4] = idx[s]
        v = int(ls[s]) << 28
        for j in range(4):
            v |= int(sigma[s][j]) << (7 * j)
        b[8 * s + 4:8 * s + 8] = np.frombuffer(np.uint32(v).tobytes(), np.uint8)
    return b


def _f16(bits):
    return oracle.f16_to_f64(int(bits))


def test_iq2_fields_recovered_from_values():
    """Random fields -> bytes -> oracle values -> fields: the magnitude pattern
    is the chosen grid row times d(2ls+1)/8, the signs of elements 0..6 are the
    sigma bits, and element 7 makes the count of negatives even."""
    rng = np.random.default_rng(1)
    g = oracle.grid()
    for _ in range(300):
        idx = rng.integers(0, 256, (8, 4))
        sigma = rng.integers(0, 128, (8, 4))
        ls = rng.integers(0, 16, 8)
        d = int(rng.integers(0x0400, 0x7800))  # normal fp16, positive
        w = oracle.dequant_iq2(_pack_iq2(idx, sigma, ls), np.array([d], np.uint16)).astype(np.float64)
        dv = _f16(d)
        for s in range(8):
            for j in range(4):
                vals = w[32 * s + 8 * j:32 * s + 8 * j + 8]
                mag = np.abs(vals) * 8.0 / (dv * (2 * ls[s] + 1))
                assert np.array_equal(mag, g[idx[s, j]].astype(np.float64))
                neg = vals < 0
                assert neg.sum() % 2 == 0
                assert [bool((sigma[s, j] >> e) & 1) for e in range(7)] == neg[:7].tolist()


def test_iq2_scaling_laws():
    """Doubling d doubles every value exactly; ls enters as the odd factor 2ls+1."""
    rng = np.random.default_rng(2)
    codes = rng.integers(0, 256, 64).astype(np.uint8)
    codes[4::8] = codes[4::8]  # keep
    for s in range(8):
        codes[8 * s + 7] &= 0x0F  # ls = 0 everywhere
    w1 = oracle.dequant_iq2(codes, np.array([0x3C00], np.uint16))
    w2 = oracle.dequant_iq2(codes, np.array([0x4000], np.uint16))
    assert np.array_equal(w2, 2 * w1)
    for ls in range(16):
        c2 = codes.copy()
        for s in range(8):
            c2[8 * s + 7] |= ls << 4
        w = oracle.dequant_iq2(c2, np.array([0x3C00], np.uint16))
        assert np.array_equal(w.astype(np.float64), (2 * ls + 1) * w1.astype(np.float64))


def test_q2k_exhaustive_exact_rounding():
    """All (sc, m, q) for several (d, dmin), against exact rational arithmetic
    rounded once to fp32: the value is the correctly rounded d*sc*q - dmin*m."""
    pairs = [(0x3C00, 0x3800), (0x3555, 0x0001), (0x1234, 0x2F00), (0x0001, 0x7BFF), (0x03FF, 0x03FF)]
    for d, dm in pairs:
        for sc in range(16):
            for m in range(16):
                codes = np.zeros(80, np.uint8)
                codes[0] = sc | (m << 4)
                codes[16] = 0b11100100  # q = 0,1,2,3 for weights 0..3
                out = oracle.dequant_q2k(codes, np.array([d | (dm << 16)], np.uint32))
                for q in range(4):
                    exact = Fraction(_f16(d)) * sc * q - Fraction(_f16(dm)) * m
                    assert out[q] == np.float32(float(exact)), (d, dm, sc, m, q)


def test_q2k_affine_in_q():
    rng = np.random.default_rng(3)
    for _ in range(50):
        codes = rng.integers(0, 256, 80).astype(np.uint8)
        dd = np.array([int(rng.integers(0x0400, 0x5000)) | int(rng.integers(0x0400, 0x5000)) << 16], np.uint32)
        w = oracle.dequant_q2k(codes, dd).astype(np.float64)
        d, dm = _f16(int(dd[0]) & 0xFFFF), _f16(int(dd[0]) >> 16)
        for s in range(16):
            sc, m = codes[s] & 15, codes[s] >> 4
            qs = [(codes[16 + i // 4] >> (2 * (i % 4))) & 3 for i in range(16 * s, 16 * s + 16)]
            for i, q in zip(range(16 * s, 16 * s + 16), qs):
                # exact in fp32 whenever the two terms share a binade range; compare in double
                assert abs(w[i] - (d * sc * q - dm * m)) <= 2.0 ** -20 * max(1.0, abs(w[i]))


# ---------------------------------------------------------------- routing
def _router_case(T=16, H=64, E=12, k=3, seed=7, bias=False):
    rng = np.random.default_rng(seed)
    w = synth.normal_bf16(seed * 101 + 1, (E, H), 1.0 / math.sqrt(H))
    x = rng.standard_normal((T, H)).astype(np.float32)
    b = rng.standard_normal(E).astype(np.float32) if bias else None
    return w, b, x


@pytest.mark.parametrize("bias", [False, True])
def test_route_matches_library_sort_and_softmax(bias):
    w, b, x = _router_case(bias=bias)
    k = 3
    idx, tw, logits = oracle.route(w, b, x, k, want_logits=True)
    L = x.astype(np.float64) @ synth.bf16_bits_to_f32(w).astype(np.float64).T
    if b is not None:
        L = L + b.astype(np.float64)
    assert np.allclose(logits, L, rtol=1e-13, atol=1e-13)
    order = np.argsort(-L, axis=1, kind="stable")[:, :k]
    assert np.array_equal(idx, order)
    full = softmax(L, axis=1)
    sel = np.take_along_axis(full, order, axis=1)
    ref = sel / sel.sum(axis=1, keepdims=True)
    assert np.allclose(tw, ref, rtol=0, atol=2e-7)
    assert np.allclose(tw.astype(np.float64).sum(axis=1), 1.0, atol=1e-6)


def test_route_k_equals_E_is_plain_softmax():
    w, b, x = _router_case(E=6, k=6)
    idx, tw, logits = oracle.route(w, None, x, 6, want_logits=True)
    full = softmax(logits, axis=1)
    assert np.allclose(tw, np.take_along_axis(full, idx, axis=1), atol=2e-7)


def test_route_ties_break_to_lower_index():
    H, E = 8, 5
    w = np.zeros((E, H), np.uint16)  # all logits 0 -> full tie
    x = np.ones((2, H), np.float32)
    idx, tw = oracle.route(w, None, x, 3)
    assert idx.tolist() == [[0, 1, 2], [0, 1, 2]]
    assert np.allclose(tw, 1.0 / 3.0)


# ------------------------------------------------------------ permutation
def test_permute_matches_stable_argsort():
    rng = np.random.default_rng(5)
    T, k, E = 37, 4, 9
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    offsets, perm, inv = oracle.permute(idx, E)
    flat = idx.ravel()
    assert np.array_equal(perm, np.argsort(flat, kind="stable"))
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
    assert np.array_equal(inv[perm], np.arange(T * k))
    assert offsets[-1] == T * k


def test_permute_empty():
    offsets, perm, inv = oracle.permute(np.zeros((0, 2), np.int32), 4)
    assert offsets.tolist() == [0, 0, 0, 0, 0]


# ------------------------------------------------------------------- FFN
def _dense(lw):
    """Dequantise every matrix of a layer to float64 dense arrays via the
    (separately pinned) oracle dequantisers."""
    E, I, H = lw.E, lw.I, lw.H
    Wg = oracle.dequant_iq2(lw.gate_codes, lw.gate_d).reshape(E, I, H).astype(np.float64)
    Wu = oracle.dequant_iq2(lw.up_codes, lw.up_d).reshape(E, I, H).astype(np.float64)
    Wd = oracle.dequant_q2k(lw.down_codes, lw.down_dd).reshape(E, H, I).astype(np.float64)
    return Wg, Wu, Wd


def _silu(z):
    return z / (1.0 + np.exp(-z))


def _dense_moe(lw, x64, idx, w, residual=None):
    """Textbook dense MoE over library float64 matmuls."""
    Wg, Wu, Wd = _dense(lw)
    y = np.zeros((x64.shape[0], lw.H))
    for t in range(x64.shape[0]):
        for j in range(idx.shape[1]):
            e = idx[t, j]
            h = _silu(Wg[e] @ x64[t]) * (Wu[e] @ x64[t])
            y[t] += float(w[t, j]) * (Wd[e] @ h)
    if lw.Is:
        sg = synth.bf16_bits_to_f32(lw.sh_gate).astype(np.float64)
        su = synth.bf16_bits_to_f32(lw.sh_up).astype(np.float64)
        sd = synth.bf16_bits_to_f32(lw.sh_down).astype(np.float64)
        y += (_silu(x64 @ sg.T) * (x64 @ su.T)) @ sd.T
    if residual is not None:
        y += residual.astype(np.float64)
    return y


def _tiny(**over):
    cfg = synth.CONFIGS["tiny"]
    if over:
        cfg = synth.Config(**{**cfg.__dict__, **over})
    return cfg, synth.make_layer(cfg), synth.make_x(cfg)


def _normwise(a, ref):
    return float(np.max(np.abs(a - ref)) / max(np.max(np.abs(ref)), 1e-30))


def test_layer_forward_matches_dense_library_moe():
    cfg, lw, x = _tiny()
    res = synth.make_residual(cfg, cfg.T)
    y, idx, w = oracle.layer_forward(lw, x, res)
    ref = _dense_moe(lw, x.astype(np.float64), idx, w, res)
    assert _normwise(y.astype(np.float64), ref) < 1e-6  # fp32 output rounding only


def test_expert_ffn_bf16_inputs_and_flattened_blocks():
    # H=256, I=128: the down matrix has K=128 < 256 so its blocks span two rows.
    cfg, lw, _ = _tiny(x_dtype="bf16")
    x = synth.make_x(cfg)
    assert x.dtype == np.uint16
    idx, w = oracle.route(lw.router_w, lw.router_bias, x, cfg.k)
    y = oracle.expert_ffn(lw, x, idx, w)
    ref = _dense_moe(lw, synth.bf16_bits_to_f32(x).astype(np.float64), idx, w)
    assert _normwise(y.astype(np.float64), ref) < 1e-6


def test_single_expert_is_dense_swiglu_ffn():
    cfg, lw, x = _tiny(E=1, k=1, Is=0)
    y, idx, w = oracle.layer_forward(lw, x)
    assert np.all(idx == 0) and np.all(w == 1.0)
    Wg, Wu, Wd = _dense(lw)
    x64 = x.astype(np.float64)
    ref = (_silu(x64 @ Wg[0].T) * (x64 @ Wu[0].T)) @ Wd[0].T
    assert _normwise(y.astype(np.float64), ref) < 1e-6


def test_zero_scales_leave_only_shared_expert():
    cfg, lw, x = _tiny()
    lw.gate_d[:] = 0
    lw.up_d[:] = 0
    lw.down_dd[:] = 0
    y, idx, w = oracle.layer_forward(lw, x)
    x64 = x.astype(np.float64)
    sg = synth.bf16_bits_to_f32(lw.sh_gate).astype(np.float64)
    su = synth.bf16_bits_to_f32(lw.sh_up).astype(np.float64)
    sd = synth.bf16_bits_to_f32(lw.sh_down).astype(np.float64)
    ref = (_silu(x64 @ sg.T) * (x64 @ su.T)) @ sd.T
    assert _normwise(y.astype(np.float64), ref) < 1e-6


def test_zero_input_gives_residual():
    cfg, lw, x = _tiny()
    res = synth.make_residual(cfg, cfg.T)
    y, _, _ = oracle.layer_forward(lw, np.zeros_like(x), res)
    assert np.array_equal(y, res)


def test_expert_relabelling_invariance():
    cfg, lw, x = _tiny()
    y0, idx0, w0 = oracle.layer_forward(lw, x)
    p = np.random.default_rng(9).permutation(cfg.E)  # new expert p[e] <- old e
    lw2 = synth.make_layer(cfg)
    for name in ("gate_codes", "gate_d", "up_codes", "up_d", "down_codes", "down_dd", "router_w"):
        src = getattr(lw, name)
        dst = getattr(lw2, name)
        dst[p] = src
    y1, idx1, w1 = oracle.layer_forward(lw2, x)
    assert np.array_equal(idx1, p[idx0])
    assert np.array_equal(y1, y0)


def test_token_permutation_equivariance():
    cfg, lw, x = _tiny()
    y0, _, _ = oracle.layer_forward(lw, x)
    p = np.array([2, 0, 3, 1])
    y1, _, _ = oracle.layer_forward(lw, np.ascontiguousarray(x[p]))
    assert np.array_equal(y1, y0[p])


# ------------------------------------------------------- OpenMP build identity
def test_openmp_build_returns_identical_bits(tmp_path):
    """The OpenMP build spreads independent outputs over threads; each output is
    still one sequential loop, so its bits equal the single-threaded build's."""
    import subprocess
    import sys

    code = r'''
import os, sys, numpy as np
sys.path.insert(0, sys.argv[1])
import oracle, synth
sys.path.insert(0, os.path.join(sys.argv[1], "tests"))
cfg = synth.Config("omp_pin", 9, 512, 256, 8, 3, 64, "bf16", 1.0, True, 1, 0x0B5E)
lw = synth.make_layer(cfg)
x = synth.make_x(cfg)
y, idx, w = oracle.layer_forward(lw, x, synth.make_residual(cfg, cfg.T))
np.savez(sys.argv[2], y=y, idx=idx, w=w)
'''
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    outs = {}
    for flag in ("0", "1"):
        out = str(tmp_path / f"o{flag}.npz")
        env = dict(os.environ, MOEREF_OPENMP=flag, OMP_NUM_THREADS="4")
        subprocess.check_call([sys.executable, "-c", code, root, out], env=env)
        outs[flag] = np.load(out)
    for key in ("y", "idx", "w"):
        assert np.array_equal(outs["0"][key], outs["1"][key]), key
