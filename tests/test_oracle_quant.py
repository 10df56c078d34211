"""Pins of the oracle's quantisers (float weights -> the two block formats).

The quantisers are this project's plain rules (round-to-nearest for Q2K, an
exhaustive codebook search for IQ2, no importance matrix); these checks tie
them to facts outside themselves: a hand-worked block, an exact
encode -> decode -> encode round trip through the separately pinned decoder,
a float64 brute-force search, and numpy's fp16 rounding.
"""
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_f32_to_f16_matches_numpy():
    rng = np.random.default_rng(0)
    vals = np.concatenate([rng.standard_normal(4000).astype(np.float32) * s
                           for s in (1e-8, 1e-6, 1e-4, 1e-2, 1, 100, 1e4)])
    edges = np.float32([0, -0.0, 2**-24, 2**-25, 2**-25 * 1.0000001, 65504, 65519.99, 6.1e-5, 3 * 2**-26,
                        -65504, 1 - 2**-12, 1 + 2**-11, 1 + 3 * 2**-11])
    for v in np.concatenate([vals, edges]):
        if abs(float(v)) < 65520:
            assert oracle.f32_to_f16(v) == int(np.float16(v).view(np.uint16)), v


def _golden_q2k():
    for line in open(os.path.join(GOLDEN, "quantize_worked.txt")):
        line = line.split("#", 1)[0].strip()
        if line.startswith("q2k_pattern"):
            kv = dict(t.split("=") for t in line.split()[1:])
            return int(kv["scale_byte"], 16), int(kv["q_byte"], 16), int(kv["dd"], 16)
    raise AssertionError("fixture missing")


def test_q2k_worked_block():
    sc_byte, q_byte, dd_ref = _golden_q2k()
    w = (0.5 * (np.arange(256) % 4)).astype(np.float32)
    codes, dd = oracle.quantize_q2k(w)
    assert int(dd[0]) == dd_ref
    assert (codes[0, :16] == sc_byte).all()
    assert (codes[0, 16:] == q_byte).all()
    # and the decoder gives the weights back to within one fp16 rounding of d
    rec = oracle.dequant_q2k(codes, dd)
    assert np.max(np.abs(rec - w)) <= 1.5 * 2**-11 * 1.5


def _iq2_representable_codes(seed, nb):
    """Random IQ2 blocks whose decoded weights the quantiser must encode back
    exactly: every sub-block has a group on a codebook row that contains 43
    (so its largest magnitude is 43 * (2ls+1) * d / 8) and sub-block 0 has
    ls = 15 (so the block maximum fixes d)."""
    grid = oracle.grid()
    rows43 = np.nonzero((grid == 43).any(axis=1))[0]
    codes = synth.rand_bytes(seed, (nb, 64)).copy()
    pick = synth.rand_bytes(seed + 1, (nb, 8))
    for b in range(nb):
        for s in range(8):
            codes[b, 8 * s] = rows43[pick[b, s] % len(rows43)]
        codes[b, 7] |= 0xF0  # ls = 15 in sub-block 0 (bits 28..31 of its word)
    d = np.full(nb, 0x2A00, np.uint16)  # 0.046875: every product below stays exact in fp32
    return codes, d


def test_iq2_encode_decode_encode_round_trip():
    codes, d = _iq2_representable_codes(31, 300)
    w = oracle.dequant_iq2(codes, d)
    c2, d2 = oracle.quantize_iq2(w)
    assert np.array_equal(d2, d)
    assert np.array_equal(c2, codes)


def test_iq2_search_picks_the_least_error_row():
    """The chosen row minimises the group error, recomputed here in float64
    over all 256 rows with the format's sign rule (fp32 near-ties allowed)."""
    rng = np.random.default_rng(5)
    w = (rng.standard_normal(256 * 40) * 0.03).astype(np.float32)
    codes, d = oracle.quantize_iq2(w)
    grid = oracle.grid().astype(np.float64)
    W = w.reshape(-1, 8, 4, 8).astype(np.float64)  # [block][sub][group][elem]
    for b in range(codes.shape[0]):
        df = float(np.float16(d[b].view(np.float16)))
        for s in range(8):
            v = int.from_bytes(codes[b, 8 * s + 4:8 * s + 8].tobytes(), "little")
            c = df * (2 * (v >> 28) + 1) / 8
            for j in range(4):
                g = W[b, s, j]
                a = np.abs(g)
                neg = g < 0
                flip = -1
                if neg.sum() % 2:
                    flip = int(np.argmin(a))
                sgn = np.where(np.arange(8) == flip, -1.0, 1.0)
                errs = ((a[None, :] - sgn[None, :] * c * grid) ** 2).sum(axis=1)
                chosen = errs[codes[b, 8 * s + j]]
                assert chosen <= errs.min() * (1 + 1e-5) + 1e-12, (b, s, j)
                # and the stored signs are w's, with the flipped element reversed
                sig = (v >> (7 * j)) & 127
                want = [int(neg[e]) ^ int(e == flip) for e in range(7)]
                assert [(sig >> e) & 1 for e in range(7)] == want


@pytest.mark.parametrize("fmt", ["q2k", "iq2"])
def test_quantise_then_decode_error_is_bounded(fmt):
    """Statistical sanity of the plain rules on Gaussian weights: the relative
    RMS reconstruction error of 2-bit codes lies in a plausible band."""
    rng = np.random.default_rng(9)
    w = (rng.standard_normal(256 * 256) * 0.02).astype(np.float32)
    if fmt == "q2k":
        rec = oracle.dequant_q2k(*oracle.quantize_q2k(w))
    else:
        rec = oracle.dequant_iq2(*oracle.quantize_iq2(w))
    rel = np.sqrt(np.mean((rec - w) ** 2)) / np.sqrt(np.mean(w ** 2))
    assert 0.1 < rel < 0.6, rel
