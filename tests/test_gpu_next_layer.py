"""moe_layer_forward_next: the layer that also writes the next layer's bf16 input.

Chained layers keep the residual stream y in fp32 and take its bf16 rounding
(nearest, ties to even) as the next input. The entry point writes that rounding
itself: fused into the combine kernel on the decode path with bf16 inputs, by a
cast kernel after the combine elsewhere. The checks: y is bit-identical to
moe_layer_forward's, and y_next is bit-identical to the round-to-nearest-even
of y, computed from y's bits by the rule written out in numpy (tests/helpers.py,
pinned on hand values in test_bf16_rule.py), on every path that ends a layer.
"""
import dataclasses

import numpy as np
import pytest

import synth
from bit_quantized_routed_iq2_b200 import build as moebuild
from bit_quantized_routed_iq2_b200 import moe2bit
from helpers import bf16_rne_bits, screened_x

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
    # decode, bf16, shared expert on the side stream: the routed combine stores both outputs
    "decode_t1": synth.Config("decode_t1", 1, 7168, 2048, 16, 8, 2048, "bf16", 1.0, False, 1, 0x4E01),
    "decode_t16_zipf": synth.Config("decode_t16_zipf", 16, 7168, 2048, 32, 8, 2048, "bf16", 1.0, True, 1, 0x4E02),
    # decode without the side stream: fp32 activations, or no shared expert (cast kernel after the combine)
    "decode_f32_t4": synth.Config("decode_f32_t4", 4, 7168, 2048, 16, 8, 2048, "f32", 1.0, False, 1, 0x4E03),
    "decode_noshared_t2": synth.Config("decode_noshared_t2", 2, 7168, 2048, 16, 8, 0, "bf16", 1.0, False, 1,
                                       0x4E04),
    # the grouped GEMM (more than 16 tokens) and the plain path of the tiny shape
    "prefill_t37": synth.Config("prefill_t37", 37, 512, 256, 16, 4, 64, "bf16", 1.0, False, 1, 0x4E05),
    "tiny": synth.CONFIGS["tiny"],
}


@pytest.mark.parametrize("name", list(CASES))
def test_next_layer_input_is_bf16_of_y(torch_cuda, name):
    torch = torch_cuda
    cfg = CASES[name]
    lw = synth.make_layer(cfg)
    x = screened_x(cfg, lw)
    dl = moe2bit.to_device(lw)
    xd = _x_dev(torch, x)
    res = torch.from_numpy(synth.make_residual(cfg, cfg.T)).cuda()
    ws = moe2bit.alloc_workspace(dl.desc, cfg.T)
    y_ref = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device="cuda")
    moe2bit.layer_forward(dl, xd, res, y_ref, ws)
    y = torch.full((cfg.T, cfg.H), float("nan"), dtype=torch.float32, device="cuda")
    yb = torch.full((cfg.T, cfg.H), -1, dtype=torch.int16, device="cuda")
    moe2bit.layer_forward(dl, xd, res, y, ws, y_next=yb)
    torch.cuda.synchronize()
    assert moe2bit.read_status(ws) == 0
    got_y = y.cpu().numpy()
    assert np.array_equal(got_y.view(np.uint32), y_ref.cpu().numpy().view(np.uint32))
    assert np.array_equal(yb.cpu().numpy().view(np.uint16), bf16_rne_bits(got_y))


def test_chained_layers_alternate_input_buffers(torch_cuda):
    # three layers: each takes the previous one's y_next, with the residual stream y carried in place; the
    # same chain with the bf16 rounding done on the host from y gives the same bits
    torch = torch_cuda
    cfg = CASES["decode_t16_zipf"]
    layers = [moe2bit.to_device(synth.make_layer(dataclasses.replace(cfg, seed=cfg.seed + l))) for l in range(3)]
    x0 = _x_dev(torch, screened_x(cfg, synth.make_layer(cfg)))
    res = torch.from_numpy(synth.make_residual(cfg, cfg.T)).cuda()
    ws = moe2bit.alloc_workspace(layers[0].desc, cfg.T)
    bufs = [torch.empty((cfg.T, cfg.H), dtype=torch.int16, device="cuda") for _ in range(2)]
    y = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device="cuda")
    cur = x0
    for l, dl in enumerate(layers):
        nxt = bufs[l % 2]
        moe2bit.layer_forward(dl, cur, res if l == 0 else y, y, ws, y_next=nxt)
        cur = nxt.view(torch.bfloat16)
    torch.cuda.synchronize()
    assert moe2bit.read_status(ws) == 0
    y2 = torch.empty_like(y)
    cur = x0
    for l, dl in enumerate(layers):
        moe2bit.layer_forward(dl, cur, res if l == 0 else y2, y2, ws)
        torch.cuda.synchronize()
        host = bf16_rne_bits(y2.cpu().numpy())
        cur = torch.from_numpy(host.view(np.int16)).cuda().view(torch.bfloat16)
    torch.cuda.synchronize()
    assert np.array_equal(y.cpu().numpy().view(np.uint32), y2.cpu().numpy().view(np.uint32))
