"""Pins of the fp32 -> bf16 round-to-nearest-even rule that the next-layer
input is checked against (no GPU needed): hand-worked values around ties, the
sign and zero cases, and the library conversion of the same values."""
import numpy as np
import torch

from helpers import bf16_rne_bits


def test_hand_values():
    v = np.array([
        1.0,
        1 + 2.0 ** -8,                 # halfway between 1 and 1 + 2^-7: ties to the even code, 1
        1 + 3 * 2.0 ** -8,             # halfway between 1 + 2^-7 and 1 + 2^-6: ties to the even code
        1 + 2.0 ** -8 + 2.0 ** -20,    # just above a tie: rounds up
        1 + 2.0 ** -8 - 2.0 ** -20,    # just below a tie: rounds down
        2 - 2.0 ** -9,                 # halfway to 2 from the largest code below it: carries into the exponent
        -2.5,
        0.0,
        -0.0,
    ], np.float32)
    want = np.array([0x3F80, 0x3F80, 0x3F82, 0x3F81, 0x3F80, 0x4000, 0xC020, 0x0000, 0x8000], np.uint16)
    assert np.array_equal(bf16_rne_bits(v), want)


def test_agrees_with_library_conversion():
    rng = np.random.default_rng(7)
    v = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 100,
                        rng.standard_normal(20000).astype(np.float32) * 1e-30,
                        # exact ties: bf16 values plus half their spacing
                        ((rng.integers(0x0080, 0x7F00, 4000).astype(np.uint32) << 16) | 0x8000).view(np.float32)])
    lib = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bf16_rne_bits(v), lib)
