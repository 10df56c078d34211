"""Block-32 routed experts on the GPU against the oracle: MXFP4
(moe_layer_forward_mxfp4) and the Q4-style format (moe_layer_forward_q4).

Element decoding bit-for-bit (as values) through moe_debug_dequant_mxfp4; the
layer within the normwise bound of the 2-bit path (FFN_TOL) at small shapes
(one and several tokens, fp32 and bf16 activations, with and without a shared
expert, uneven routing) and at the one-token decode shape (H=7168, I=2048,
E=256, k=8, I_s=2048). Above 16 tokens (the block-scaled grouped GEMM) against
the oracle with MXFP8 activations, at small shapes with ragged and multi-tile
experts and on sampled tokens of the 2048-token prefill shape; the Q4-style
format above 16 tokens (the dequantising grouped GEMM) against the exact oracle.
"""
import numpy as np
import pytest

import oracle
import synth
from bit_quantized_routed_iq2_b200 import moe2bit
from helpers import FFN_TOL, near_tie_tokens, normwise, screened_x

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    moe2bit.load()
    return torch


def _x_dev(torch, x):
    t = torch.from_numpy(np.ascontiguousarray(x).view(np.int16) if x.dtype == np.uint16 else x).cuda()
    return t.view(torch.bfloat16) if x.dtype == np.uint16 else t


def test_dequant_matches_oracle(torch_cuda):
    torch = torch_cuda
    nb = 4096
    codes = synth.rand_bytes(0x4D5801, (nb, 16))
    scales = (1 + synth.rand_bytes(0x4D5802, (nb,)) % 254).astype(np.uint8)  # every E in [1, 254]
    # every element code at least once per byte position
    codes[:256] = np.arange(256, dtype=np.uint8)[:, None]
    out = torch.empty(nb * 32, dtype=torch.float32, device="cuda")
    moe2bit.debug_dequant_mxfp4(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(), out)
    torch.cuda.synchronize()
    ref = oracle.dequant_mxfp4(codes, scales)
    # equal as values (the GPU's integer operands give +0 where the format's code 8 means -0)
    assert np.array_equal(out.cpu().numpy(), ref)


def _mx_forward(torch, dl, x, residual=None):
    T = x.shape[0]
    y = torch.full((T, dl.desc.hidden), float("nan"), dtype=torch.float32, device="cuda")
    res = None if residual is None else torch.from_numpy(np.ascontiguousarray(residual)).cuda()
    ws = moe2bit.alloc_workspace_mxfp4(dl.desc, T)
    moe2bit.layer_forward_mxfp4(dl, _x_dev(torch, x), res, y, ws)
    torch.cuda.synchronize()
    assert moe2bit.read_status(ws) == 0
    return y.cpu().numpy()


CASES = {
    "t1_bf16": dict(T=1, x_dtype="bf16", Is=128, zipf=False),
    "t2_f32_noshared": dict(T=2, x_dtype="f32", Is=0, zipf=False),
    "t5_bf16_zipf": dict(T=5, x_dtype="bf16", Is=128, zipf=True),
    "t16_bf16_zipf": dict(T=16, x_dtype="bf16", Is=128, zipf=True),
    "t16_f32": dict(T=16, x_dtype="f32", Is=64, zipf=False),
}


@pytest.mark.parametrize("name", list(CASES))
def test_mxfp4_layer_small(torch_cuda, name):
    c = CASES[name]
    cfg = synth.Config("mx_" + name, c["T"], 1024, 512, 16, 4, c["Is"], c["x_dtype"], 1.0, c["zipf"], 1,
                       0x4D58A0 + len(name))
    lw = synth.make_layer_mxfp4(cfg)
    x = screened_x(cfg, lw)
    res = synth.make_residual(cfg, cfg.T)
    y = _mx_forward(torch_cuda, moe2bit.to_device_mxfp4(lw), x, res)
    ref, _, _ = oracle.layer_forward(lw, x, res)
    assert normwise(y, ref) <= FFN_TOL, (name, normwise(y, ref))


def test_mxfp4_rejects_unsupported_shapes(torch_cuda):
    import ctypes

    desc = moe2bit.desc_of(1280, 512, 16, 4, 0)  # hidden not a multiple of 512
    with pytest.raises(RuntimeError):
        moe2bit.workspace_size_mxfp4(desc, 1)
    desc = moe2bit.desc_of(1024, 512, 16, 4, 0)
    assert moe2bit.workspace_size_mxfp4(desc, 16) > 0
    # above 16 tokens MXFP4 takes the block-scaled grouped GEMM; its workspace covers the GEMV step too
    assert moe2bit.workspace_size_mxfp4(desc, 300) >= moe2bit.workspace_size_mxfp4(desc, 16)
    # the Q4-style format takes the dequantising grouped GEMM above 16 tokens; its shared-expert GEMMs need
    # I_s % 128 == 0 there
    n = ctypes.c_size_t(0)
    assert moe2bit.load().moe_workspace_size_q4(ctypes.byref(desc), 16, ctypes.byref(n)) == 0
    assert moe2bit.load().moe_workspace_size_q4(ctypes.byref(desc), 300, ctypes.byref(n)) == 0
    odd = moe2bit.desc_of(1024, 512, 16, 4, 64)
    assert moe2bit.load().moe_workspace_size_q4(ctypes.byref(odd), 16, ctypes.byref(n)) == 0
    assert moe2bit.load().moe_workspace_size_q4(ctypes.byref(odd), 17, ctypes.byref(n)) != 0
    with pytest.raises(RuntimeError):
        moe2bit.workspace_size_mxfp4(odd, 17)


# More than 16 tokens: FP4 weights x MXFP8 activations on the block-scaled tensor cores; the oracle takes
# the same activation quantisation (act_mxfp8). Tiles hold up to 112 tokens of one expert.
MANY = {
    "t17_bf16": dict(T=17, x_dtype="bf16", Is=128, zipf=False, E=16, k=4),
    "t40_bf16_zipf": dict(T=40, x_dtype="bf16", Is=128, zipf=True, E=16, k=4),
    "t200_f32_zipf_noshared": dict(T=200, x_dtype="f32", Is=0, zipf=True, E=8, k=2),
    "t300_bf16": dict(T=300, x_dtype="bf16", Is=256, zipf=False, E=4, k=2),
}


@pytest.mark.parametrize("name", list(MANY))
def test_mxfp4_layer_many_tokens(torch_cuda, name):
    c = MANY[name]
    cfg = synth.Config("mxg_" + name, c["T"], 1024, 512, c["E"], c["k"], c["Is"], c["x_dtype"], 1.0, c["zipf"], 1,
                       0x4D47A0 + len(name))
    lw = synth.make_layer_mxfp4(cfg)
    x = screened_x(cfg, lw)
    res = synth.make_residual(cfg, cfg.T)
    y = _mx_forward(torch_cuda, moe2bit.to_device_mxfp4(lw), x, res)
    ref, idx, _ = oracle.layer_forward(lw, x, res, act_mxfp8=True)
    if name.startswith("t300") or name.startswith("t200"):  # an expert spans several tiles (ragged last one)
        assert np.bincount(idx.reshape(-1), minlength=cfg.E).max() > 112
    assert normwise(y, ref) <= FFN_TOL, (name, normwise(y, ref))
    # against the exact-activation oracle the FP8 rounding of x and h shows (a few 1e-2 normwise at most)
    exact, _, _ = oracle.layer_forward(lw, x, res)
    assert normwise(y, exact) < 0.1


@pytest.mark.slow
def test_mxfp4_prefill_shape_sampled(torch_cuda):
    """H=7168, I=2048, E=256, k=8, I_s=2048, 2048 bf16 tokens (every expert active): the GPU runs the whole
    batch in the launch configuration the benchmark times; the oracle checks a sample of tokens (a token's
    output depends on that token alone)."""
    cfg = synth.CONFIGS["prefill"]
    lw = synth.make_layer_mxfp4(cfg)
    x = synth.make_x_fast(cfg, cfg.T)
    y = _mx_forward(torch_cuda, moe2bit.to_device_mxfp4(lw), x)
    cand = np.array([0, 1, 2, 3, 777, 778, 1500, 1501, cfg.T - 2, cfg.T - 1])
    _, _, logits = oracle.route(lw.router_w, lw.router_bias, x[cand], cfg.k, want_logits=True)
    rows = np.setdiff1d(cand, cand[near_tie_tokens(logits, cfg.k)])[:5]  # routing decided in any precision
    assert rows.size == 5
    ref, _, _ = oracle.layer_forward(lw, x[rows], act_mxfp8=True)
    assert normwise(y[rows], ref) <= FFN_TOL, normwise(y[rows], ref)


@pytest.mark.slow
def test_mxfp4_decode1_shape(torch_cuda):
    """H=7168, I=2048, E=256, k=8, I_s=2048, one bf16 token: the routed experts'
    planes are generated (the others stay zero and are never read)."""
    cfg = synth.CONFIGS["decode1"]
    base = synth.make_layer(cfg, experts=[])
    x = screened_x(cfg, base)
    idx, _ = oracle.route(base.router_w, base.router_bias, x, cfg.k)
    lw = synth.make_layer_mxfp4(cfg, experts=np.unique(idx))
    y = _mx_forward(torch_cuda, moe2bit.to_device_mxfp4(lw), x)
    ref, ridx, _ = oracle.layer_forward(lw, x)
    assert np.array_equal(np.sort(ridx, axis=1), np.sort(idx, axis=1))
    assert normwise(y, ref) <= FFN_TOL, normwise(y, ref)


# ------------------------------------------------------------------ Q4-style
def test_q4_dequant_matches_oracle(torch_cuda):
    torch = torch_cuda
    nb = 4096
    codes = synth.rand_bytes(0x513401, (nb, 16))
    codes[:256] = np.arange(256, dtype=np.uint8)[:, None]
    d = synth.f16_scale(0x513402, (nb,), 0.01)
    d[:4] = [0x3C00, 0xBC00, 0x0001, 0x7BFF]  # 1, -1, the smallest subnormal, the largest finite
    out = torch.empty(nb * 32, dtype=torch.float32, device="cuda")
    moe2bit.debug_dequant_q4(torch.from_numpy(codes).cuda(), torch.from_numpy(d.view(np.int16)).cuda(), out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), oracle.dequant_q4(codes, d))


def _q4_forward(torch, dl, x, residual=None):
    T = x.shape[0]
    y = torch.full((T, dl.desc.hidden), float("nan"), dtype=torch.float32, device="cuda")
    res = None if residual is None else torch.from_numpy(np.ascontiguousarray(residual)).cuda()
    n = ctypes_size_q4(dl.desc, T)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    moe2bit.layer_forward_q4(dl, _x_dev(torch, x), res, y, ws)
    torch.cuda.synchronize()
    assert moe2bit.read_status(ws) == 0
    return y.cpu().numpy()


def ctypes_size_q4(desc, T):
    import ctypes

    n = ctypes.c_size_t(0)
    assert moe2bit.load().moe_workspace_size_q4(ctypes.byref(desc), T, ctypes.byref(n)) == 0
    return max(int(n.value), 16)


@pytest.mark.parametrize("name", ["t1_bf16", "t5_bf16_zipf", "t16_f32"])
def test_q4_layer_small(torch_cuda, name):
    c = CASES[name]
    cfg = synth.Config("q4_" + name, c["T"], 1024, 512, 16, 4, c["Is"], c["x_dtype"], 1.0, c["zipf"], 1,
                       0x5134A0 + len(name))
    lw = synth.make_layer_q4(cfg)
    x = screened_x(cfg, lw)
    res = synth.make_residual(cfg, cfg.T)
    y = _q4_forward(torch_cuda, moe2bit.to_device_q4(lw), x, res)
    ref, _, _ = oracle.layer_forward(lw, x, res)
    assert normwise(y, ref) <= FFN_TOL, (name, normwise(y, ref))


@pytest.mark.slow
def test_q4_decode1_shape(torch_cuda):
    cfg = synth.CONFIGS["decode1"]
    base = synth.make_layer(cfg, experts=[])
    x = screened_x(cfg, base)
    idx, _ = oracle.route(base.router_w, base.router_bias, x, cfg.k)
    lw = synth.make_layer_q4(cfg, experts=np.unique(idx))
    y = _q4_forward(torch_cuda, moe2bit.to_device_q4(lw), x)
    ref, _, _ = oracle.layer_forward(lw, x)
    assert normwise(y, ref) <= FFN_TOL, normwise(y, ref)


# More than 16 tokens with Q4-style experts: the dequantising grouped GEMM (fp16 weight tiles in TMEM,
# tcgen05.mma kind::f16) against the exact oracle.
@pytest.mark.parametrize("name", ["t17_bf16", "t40_bf16_zipf", "t200_f32_zipf_noshared", "t300_bf16"])
def test_q4_layer_many_tokens(torch_cuda, name):
    c = MANY[name]
    cfg = synth.Config("q4g_" + name, c["T"], 1024, 512, c["E"], c["k"], c["Is"], c["x_dtype"], 1.0, c["zipf"], 1,
                       0x5147A0 + len(name))
    lw = synth.make_layer_q4(cfg)
    x = screened_x(cfg, lw)
    res = synth.make_residual(cfg, cfg.T)
    y = _q4_forward(torch_cuda, moe2bit.to_device_q4(lw), x, res)
    ref, _, _ = oracle.layer_forward(lw, x, res)
    assert normwise(y, ref) <= FFN_TOL, (name, normwise(y, ref))


@pytest.mark.slow
def test_q4_prefill_shape_sampled(torch_cuda):
    """The 2048-token prefill shape with Q4-style experts (every expert active); sampled tokens against the
    oracle as in test_mxfp4_prefill_shape_sampled."""
    cfg = synth.CONFIGS["prefill"]
    lw = synth.make_layer_q4(cfg)
    x = synth.make_x_fast(cfg, cfg.T)
    y = _q4_forward(torch_cuda, moe2bit.to_device_q4(lw), x)
    cand = np.array([0, 1, 2, 3, 777, 778, 1500, 1501, cfg.T - 2, cfg.T - 1])
    _, _, logits = oracle.route(lw.router_w, lw.router_bias, x[cand], cfg.k, want_logits=True)
    rows = np.setdiff1d(cand, cand[near_tie_tokens(logits, cfg.k)])[:5]
    assert rows.size == 5
    ref, _, _ = oracle.layer_forward(lw, x[rows])
    assert normwise(y[rows], ref) <= FFN_TOL, normwise(y[rows], ref)


def test_mxfp4_many_tokens_need_32_byte_code_planes(torch_cuda):
    """Above 16 tokens the unpacking copy of the FP4 codes needs 32-byte plane bases: a plane that is 16-byte
    but not 32-byte aligned is rejected on the host (MOE_ERR_INVALID_ARG) before anything is enqueued, while
    the one-token GEMVs accept it and give the same result as the aligned plane."""
    torch = torch_cuda
    import ctypes

    cfg = synth.Config("mx_align", 40, 1024, 512, 8, 2, 0, "bf16", 1.0, False, 1, 0x4D4131)
    lw = synth.make_layer_mxfp4(cfg)
    dl = moe2bit.to_device_mxfp4(lw)
    g = dl.tensors["gate_codes"]
    buf = torch.empty(g.numel() + 64, dtype=torch.uint8, device="cuda")
    off = (32 - buf.data_ptr() % 32) % 32 + 16  # 16 (mod 32)
    shifted = buf[off:off + g.numel()]
    shifted.copy_(g.reshape(-1))
    assert shifted.data_ptr() % 32 == 16
    x = screened_x(cfg, lw)
    xd = _x_dev(torch, x)
    y = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device="cuda")
    ws = moe2bit.alloc_workspace_mxfp4(dl.desc, cfg.T)
    w = dl.weights
    w.gate_codes = shifted.data_ptr()
    L = moe2bit.load()
    rc = L.moe_layer_forward_mxfp4(ctypes.byref(dl.desc), ctypes.byref(w), xd.data_ptr(), 1, cfg.T, None,
                                   y.data_ptr(), ws.data_ptr(), ws.numel(), None)
    assert rc == 1  # MOE_ERR_INVALID_ARG
    # one token: the GEMVs take the 16-byte aligned plane
    y1 = torch.empty((1, cfg.H), dtype=torch.float32, device="cuda")
    y2 = torch.empty((1, cfg.H), dtype=torch.float32, device="cuda")
    assert L.moe_layer_forward_mxfp4(ctypes.byref(dl.desc), ctypes.byref(w), xd.data_ptr(), 1, 1, None,
                                     y1.data_ptr(), ws.data_ptr(), ws.numel(), None) == 0
    moe2bit.layer_forward_mxfp4(dl, xd[:1], None, y2, ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
