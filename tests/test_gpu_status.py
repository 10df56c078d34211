"""Device-side failures reach the caller as a status (no fault, trap or hang).

A bounded wait is made to run out on purpose: the decode gate/up GEMV's
producer is told to issue no loads (moe_debug_inject), so its consumers' waits
on shared-memory barriers never complete and give up after a short limit. The
call then reports MOE_ERR_TIMEOUT through moe_read_status, and the next call,
with injection off, clears the word and computes normally again.
"""
import numpy as np
import pytest

import oracle
import synth
from bit_quantized_routed_iq2_b200 import build as moebuild
from bit_quantized_routed_iq2_b200 import moe2bit
from helpers import FFN_TOL, normwise, screened_x

pytestmark = pytest.mark.gpu

MOE_ERR_TIMEOUT = 5


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    moebuild.build()
    moe2bit.load()
    return torch


def _x_dev(torch, x):
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("T", [1, 3])
def test_bounded_wait_timeout_reaches_the_caller(torch_cuda, T):
    torch = torch_cuda
    cfg = synth.Config("status", T, 1024, 512, 16, 4, 64, "bf16", 1.0, False, 1, 0x57A7 + T)
    lw = synth.make_layer(cfg)
    x = screened_x(cfg, lw)
    dl = moe2bit.to_device(lw)
    xd = _x_dev(torch, x)
    y = torch.zeros((T, cfg.H), dtype=torch.float32, device="cuda")
    ws = moe2bit.alloc_workspace(dl.desc, T)
    moe2bit.debug_inject(1, 100_000)  # ~50 us at B200 clocks
    try:
        moe2bit.layer_forward(dl, xd, None, y, ws)
        status = moe2bit.read_status(ws)
    finally:
        moe2bit.debug_inject(0)
    assert status == MOE_ERR_TIMEOUT
    # the context is still usable: the next call clears the word and is correct
    moe2bit.layer_forward(dl, xd, None, y, ws)
    assert moe2bit.read_status(ws) == 0
    ref, _, _ = oracle.layer_forward(lw, x)
    assert normwise(y.cpu().numpy(), ref) <= FFN_TOL


def test_status_is_clear_after_normal_calls(torch_cuda):
    torch = torch_cuda
    for T in (1, 40):
        cfg = synth.Config("status_ok", T, 1024, 512, 8, 2, 128, "bf16", 1.0, False, 1, 0x57B0 + T)
        lw = synth.make_layer(cfg)
        x = screened_x(cfg, lw)
        dl = moe2bit.to_device(lw)
        y = torch.empty((T, cfg.H), dtype=torch.float32, device="cuda")
        ws = moe2bit.alloc_workspace(dl.desc, T)
        ws.fill_(0xA5)  # a stale word from an earlier user of the memory must not survive the call
        moe2bit.layer_forward(dl, _x_dev(torch, x), None, y, ws)
        assert moe2bit.read_status(ws) == 0, T


def test_status_is_clear_after_the_plain_path(torch_cuda):
    # shapes with I below 256 (the tiny configuration, fp32 x) run the plain kernels, which have no bounded
    # waits; the call must still clear a stale status word, through both layer entry points
    torch = torch_cuda
    cfg = synth.CONFIGS["tiny"]
    lw = synth.make_layer(cfg)
    x = screened_x(cfg, lw)
    dl = moe2bit.to_device(lw)
    xd = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    y = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device="cuda")
    ws = moe2bit.alloc_workspace(dl.desc, cfg.T)
    ws.fill_(0xA5)
    moe2bit.layer_forward(dl, xd, None, y, ws)
    assert moe2bit.read_status(ws) == 0
    ws.fill_(0xA5)
    yb = torch.empty((cfg.T, cfg.H), dtype=torch.int16, device="cuda")
    moe2bit.layer_forward(dl, xd, None, y, ws, y_next=yb)
    assert moe2bit.read_status(ws) == 0
    ref, _, _ = oracle.layer_forward(lw, x)
    assert normwise(y.cpu().numpy(), ref) <= FFN_TOL
