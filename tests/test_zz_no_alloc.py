"""moe_layer_forward_noalloc: the layer for callers that cannot allocate.

Some callers of this library cannot hand it a workspace: a plugin whose host
engine gives out no device memory, or a serving loop that must not allocate
after start-up. For them the library keeps its own fixed scratch array and
offers one extra entry point. These checks run it through the C ABI against the
regular entry point (same tolerance as the other layer tests), twice in a row
because calls share the array and must not depend on what the previous call
left in it. This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

import synth
from bit_quantized_routed_iq2_b200 import build as moebuild
from bit_quantized_routed_iq2_b200 import moe2bit
from helpers import FFN_TOL, normwise, screened_x

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    moebuild.build()
    moe2bit.load()
    return torch


def _x_dev(torch, x):
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


CASES = {
    "tiny": synth.CONFIGS["tiny"],
    "small": synth.Config("small", 37, 512, 256, 16, 4, 64, "bf16", 1.0, False, 1, 0x5A11),
    "decode32": synth.CONFIGS["decode32"],
    # the decode path (bf16, T <= 16): TMA-fed GEMVs and the shared expert on the side stream, which
    # writes its part of the scratch while routing runs on the caller's stream
    "decode_t1": synth.Config("decode_t1", 1, 7168, 2048, 16, 8, 2048, "bf16", 1.0, False, 1, 0x5A31),
    "decode_t8": synth.Config("decode_t8", 8, 7168, 2048, 16, 8, 2048, "bf16", 1.0, True, 1, 0x5A32),
}


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_workspace_entry_point(torch_cuda, name):
    torch = torch_cuda
    cfg = CASES[name]
    lw = synth.make_layer(cfg)
    x = screened_x(cfg, lw)
    dl = moe2bit.to_device(lw)
    xd = _x_dev(torch, x)
    res = torch.from_numpy(synth.make_residual(cfg, cfg.T)).cuda()
    y_ref = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device="cuda")
    ws = moe2bit.alloc_workspace(dl.desc, cfg.T)
    moe2bit.layer_forward(dl, xd, res, y_ref, ws)
    outs = []
    for _ in range(2):  # two calls in a row share the scratch array
        y = torch.full((cfg.T, cfg.H), float("nan"), dtype=torch.float32, device="cuda")
        moe2bit.layer_forward_noalloc(dl, xd, res, y)
        torch.cuda.synchronize()
        assert moe2bit.read_status_noalloc() == 0
        outs.append(y.cpu().numpy())
    ref = y_ref.cpu().numpy()
    for got in outs:
        assert np.all(np.isfinite(got))
        assert normwise(got, ref) <= FFN_TOL


def test_noalloc_rejects_oversize_before_launch(torch_cuda):
    lib = moe2bit.load()
    d = moe2bit.desc_of(7168, 2048, 256, 8, 2048)
    need = moe2bit.workspace_size(d, 2048)
    assert need > moe2bit.NOALLOC_SCRATCH_BYTES
    fake = 1 << 40  # never dereferenced: the size check comes first
    w = moe2bit.Weights(*([fake] * 11))
    rc = lib.moe_layer_forward_noalloc(ctypes.byref(d), ctypes.byref(w), fake, 1, 2048, None, fake, None)
    assert rc == 3  # MOE_ERR_WORKSPACE_TOO_SMALL
    # the documented capacity: a 32-token decode batch at these shapes fits
    assert moe2bit.workspace_size(d, 32) <= moe2bit.NOALLOC_SCRATCH_BYTES
