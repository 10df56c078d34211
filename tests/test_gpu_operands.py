"""The hot paths' own operand builders against the oracle, element by element.

The decode GEMVs turn codes into int8 MMA operands (IQ2: level * sign and the
sub-block's 2ls+1; Q2K: sc * q and m) and the grouped GEMM turns them into fp16
tiles in tensor memory. Each builder runs here through its debug entry point
(the same device functions and tables as the kernels) on random blocks and on
every IQ2 (grid row, sign field, scale) group, and must agree exactly:
  - int8 path: w * odd == 8 * oracle(d = 1) as integers; sc * q == oracle(d = 1,
    dmin = 0) and -m == oracle(d = 0, dmin = 1);
  - fp16 path: IQ2 = sign * fp16(fp16(d * odd * 2^10 / 8) * level), Q2K =
    fp16(the oracle's fp32 weight), both rounding to nearest even.
"""
import numpy as np
import pytest

import oracle
import synth
from bit_quantized_routed_iq2_b200 import build as moebuild
from bit_quantized_routed_iq2_b200 import moe2bit

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    moebuild.build()
    moe2bit.load()
    return torch


def _t(torch, a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    elif a.dtype == np.uint32:
        a = a.view(np.int32)
    return torch.from_numpy(a).cuda()


def exhaustive_iq2_codes():
    """Every (grid row, sign field) pair under every scale ls, one group each."""
    pairs = np.array([(r, s) for r in range(256) for s in range(128)])
    ngroups = len(pairs) * 16
    nb = ngroups // 32
    codes = np.zeros((nb, 64), np.uint8)
    g = 0
    for ls in range(16):
        for r, s in pairs:
            b, within = divmod(g, 32)
            sb, j = divmod(within, 4)
            codes[b, 8 * sb + j] = r
            v = int.from_bytes(codes[b, 8 * sb + 4:8 * sb + 8].tobytes(), "little")
            v |= (int(s) << (7 * j)) | (ls << 28)
            codes[b, 8 * sb + 4:8 * sb + 8] = np.frombuffer(np.uint32(v & 0xFFFFFFFF).tobytes(), np.uint8)
            g += 1
    return codes


@pytest.fixture(scope="module")
def iq2_codes():
    rnd = synth.rand_bytes(21, (50_001, 64))
    return np.concatenate([rnd, exhaustive_iq2_codes()])


def _iq2_factors(codes):
    """(level * sign, 2ls + 1) of every weight, factored from the oracle's d = 1 values
    (8 w = odd * level * sign, and the factorisation over odd <= 31, level in {8, 25, 43} is unique)."""
    nb = codes.shape[0]
    w8 = (oracle.dequant_iq2(codes, np.full(nb, 0x3C00, np.uint16)).astype(np.float64) * 8).round().astype(np.int64)
    levels = np.array([8, 25, 43])
    lv = np.zeros_like(w8)
    odd = np.zeros_like(w8)
    for L in levels:
        q, r = np.divmod(np.abs(w8), L)
        ok = (r == 0) & (q % 2 == 1) & (q <= 31)
        lv[ok] = L
        odd[ok] = q[ok]
    assert (lv > 0).all()
    return lv * np.sign(w8), odd


def test_gemv_operands_iq2_exact(torch_cuda, iq2_codes):
    torch = torch_cuda
    codes = iq2_codes
    nb = codes.shape[0]
    w = torch.zeros(nb * 256, dtype=torch.int8, device="cuda")
    odd = torch.zeros(nb * 8, dtype=torch.uint8, device="cuda")
    moe2bit.debug_gemv_operands_iq2(_t(torch, codes), w, odd)
    torch.cuda.synchronize()
    gw = w.cpu().numpy().astype(np.int64)
    godd = odd.cpu().numpy().astype(np.int64)
    ref_w, ref_odd = _iq2_factors(codes)
    assert np.array_equal(gw, ref_w)
    assert np.array_equal(np.repeat(godd, 32), ref_odd)


def test_gemv_operands_q2k_exact(torch_cuda):
    torch = torch_cuda
    nb = 100_003
    codes = synth.rand_bytes(22, (nb, 80))
    scq = torch.zeros(nb * 256, dtype=torch.int16, device="cuda")
    m = torch.zeros(nb * 16, dtype=torch.uint8, device="cuda")
    moe2bit.debug_gemv_operands_q2k(_t(torch, codes), scq, m)
    torch.cuda.synchronize()
    one = np.uint32(0x3C00)
    ref_scq = oracle.dequant_q2k(codes, np.full(nb, one, np.uint32))            # d = 1, dmin = 0
    ref_m = -oracle.dequant_q2k(codes, np.full(nb, one << np.uint32(16), np.uint32))  # d = 0, dmin = 1
    assert np.array_equal(scq.cpu().numpy().astype(np.float32), ref_scq)
    assert np.array_equal(np.repeat(m.cpu().numpy().astype(np.float32), 16), ref_m)


def _f16_bits(a):
    return np.asarray(a, np.float16).view(np.uint16)


def test_tc_operands_iq2_rounding_rule(torch_cuda, iq2_codes):
    torch = torch_cuda
    codes = iq2_codes
    nb = codes.shape[0]
    # |d| from 2^-10 to 2^7, both signs; the largest scales overflow to inf, as in the kernel
    b = synth.rand_bytes(23, (nb, 2)).view(np.uint16).reshape(-1)
    e = 5 + (b >> 10) % 17  # biased exponent 5..21
    d = ((b & 0x83FF) | (e << 10)).astype(np.uint16)
    out = torch.zeros(nb * 256, dtype=torch.int16, device="cuda")
    moe2bit.debug_tc_operands_iq2(_t(torch, codes), _t(torch, d), out)
    torch.cuda.synchronize()
    got = out.cpu().numpy().view(np.uint16)
    lvs, odd = _iq2_factors(codes)
    dv = np.repeat(d.view(np.float16).astype(np.float32), 256)
    s16 = (dv * np.float32(128.0) * odd.astype(np.float32)).astype(np.float16)  # fp32 product is exact
    mag = (s16.astype(np.float32) * np.abs(lvs).astype(np.float32)).astype(np.float16)
    ref = np.where(lvs < 0, -mag, mag)
    assert np.array_equal(got, _f16_bits(ref))
    # and the value is the oracle's weight times 2^10 up to those two roundings
    w = oracle.dequant_iq2(codes, d).astype(np.float64) * 1024
    fin = np.isfinite(ref.astype(np.float64)) & (np.abs(w) > 2.0**-10)
    rel = np.abs(ref.astype(np.float64)[fin] - w[fin]) / np.abs(w[fin])
    assert rel.max() <= 2 * 2.0**-11 + 2.0**-22


def test_tc_operands_q2k_rounding_rule(torch_cuda):
    torch = torch_cuda
    nb = 100_003
    codes = synth.rand_bytes(24, (nb, 80))
    raw = synth.rand_bytes(25, (nb, 4)).view(np.uint16).reshape(nb, 2)
    raw[(raw & 0x7C00) == 0x7C00] &= 0xBFFF  # finite scales only
    dd = (raw[:, 0].astype(np.uint32) | (raw[:, 1].astype(np.uint32) << 16))
    out = torch.zeros(nb * 256, dtype=torch.int16, device="cuda")
    moe2bit.debug_tc_operands_q2k(_t(torch, codes), _t(torch, dd), out)
    torch.cuda.synchronize()
    ref = oracle.dequant_q2k(codes, dd).astype(np.float16)  # fp32 weight rounded to nearest even
    assert np.array_equal(out.cpu().numpy().view(np.uint16), _f16_bits(ref))
