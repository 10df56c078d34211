"""The GPU quantisers against the oracle's, byte for byte.

Both implement the same plain rules (include/moe2bit.h, moe_quantize_*) with
every decision in unfused fp32 round-to-nearest arithmetic, so the codes and
scales must be identical: on Gaussian weights of several scales (a ragged
number of blocks), on weights with exact zeros and repeated values, on a whole
expert matrix, and on decoded codes, which the IQ2 rule maps back to the same
codes.
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


def _weights(seed, nb, std):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal(nb * 256) * std).astype(np.float32)
    w[::97] = 0.0          # exact zeros
    w[5::131] = -0.0
    w[7:7 + 40] = w[6]      # a run of equal values (ties in the searches)
    return w


def _gpu_q2k(torch, w):
    nb = w.size // 256
    codes = torch.zeros((nb, 80), dtype=torch.uint8, device="cuda")
    dd = torch.zeros(nb, dtype=torch.int32, device="cuda")
    moe2bit.quantize_q2k(torch.from_numpy(w).cuda(), codes, dd)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), dd.cpu().numpy().view(np.uint32)


def _gpu_iq2(torch, w):
    nb = w.size // 256
    codes = torch.zeros((nb, 64), dtype=torch.uint8, device="cuda")
    d = torch.zeros(nb, dtype=torch.int16, device="cuda")
    moe2bit.quantize_iq2(torch.from_numpy(w).cuda(), codes, d)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), d.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("std", [1e-4, 0.02, 3.0])
def test_quantize_q2k_matches_oracle(torch_cuda, std):
    w = _weights(1, 3001, std)
    gc, gd = _gpu_q2k(torch_cuda, w)
    rc, rd = oracle.quantize_q2k(w)
    assert np.array_equal(gd, rd)
    assert np.array_equal(gc, rc)


@pytest.mark.parametrize("std", [1e-4, 0.02, 3.0])
def test_quantize_iq2_matches_oracle(torch_cuda, std):
    w = _weights(2, 1501, std)
    gc, gd = _gpu_iq2(torch_cuda, w)
    rc, rd = oracle.quantize_iq2(w)
    assert np.array_equal(gd, rd)
    assert np.array_equal(gc, rc)


def test_quantize_whole_expert_matrix(torch_cuda):
    """One expert's gate matrix and down matrix at the decode shapes (2048 x 7168
    and 7168 x 2048 weights), blocks along rows."""
    rng = np.random.default_rng(3)
    w = (rng.standard_normal(2048 * 7168) / np.sqrt(7168)).astype(np.float32)
    gc, gd = _gpu_iq2(torch_cuda, w)
    rc, rd = oracle.quantize_iq2(w)
    assert np.array_equal(gd, rd) and np.array_equal(gc, rc)
    gc, gd = _gpu_q2k(torch_cuda, w)
    rc, rd = oracle.quantize_q2k(w)
    assert np.array_equal(gd, rd) and np.array_equal(gc, rc)


def test_quantize_iq2_inverts_the_decoder(torch_cuda):
    """Decoded IQ2 blocks whose scales the rule recovers exactly (every
    sub-block holds a 43 level, sub-block 0 has ls = 15) quantise back to the
    same codes on the GPU."""
    grid = oracle.grid()
    rows43 = np.nonzero((grid == 43).any(axis=1))[0]
    nb = 700
    codes = synth.rand_bytes(41, (nb, 64)).copy()
    pick = synth.rand_bytes(42, (nb, 8))
    for b in range(nb):
        for s in range(8):
            codes[b, 8 * s] = rows43[pick[b, s] % len(rows43)]
        codes[b, 7] |= 0xF0
    d = np.full(nb, 0x2A00, np.uint16)
    w = oracle.dequant_iq2(codes, d)
    gc, gd = _gpu_iq2(torch_cuda, w)
    assert np.array_equal(gd, d)
    assert np.array_equal(gc, codes)
