"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Dequantisation, router indices and the permutation must be bit-exact; router
weights within TOPK_W_TOL; layer outputs within FFN_TOL normwise.
"""
import numpy as np
import pytest

import oracle
import synth
from bit_quantized_routed_iq2_b200 import build as moebuild
from bit_quantized_routed_iq2_b200 import moe2bit
from helpers import FFN_TOL, TOPK_W_TOL, elementwise, normwise, screened_x

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    moebuild.build()
    moe2bit.load()
    return torch


def _t(torch, a, dtype=None):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    elif a.dtype == np.uint32:
        a = a.view(np.int32)
    return torch.from_numpy(a).cuda()


def _x_dev(torch, x):
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


# ------------------------------------------------------------- dequant unit
def _random_f16(seed, n, allow_subnormal=True):
    b = synth.rand_bytes(seed, (n, 2)).view(np.uint16).reshape(-1).copy()
    exp = (b >> 10) & 31
    b[exp == 31] &= 0x83FF  # no inf/nan: clear exponent
    if not allow_subnormal:
        b[exp == 0] |= 0x0400
    return b


def test_dequant_iq2_bitexact(torch_cuda):
    torch = torch_cuda
    nb = 100_003  # not a multiple of any tile
    codes = synth.rand_bytes(11, (nb, 64))
    d = _random_f16(12, nb)
    ref = oracle.dequant_iq2(codes, d)
    out = torch.full((nb * 256,), float("nan"), dtype=torch.float32, device="cuda")
    moe2bit.debug_dequant_iq2(_t(torch, codes), _t(torch, d), out)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_dequant_q2k_bitexact(torch_cuda):
    torch = torch_cuda
    nb = 100_003
    codes = synth.rand_bytes(13, (nb, 80))
    dd = (_random_f16(14, nb).astype(np.uint32) | (_random_f16(15, nb).astype(np.uint32) << 16))
    ref = oracle.dequant_q2k(codes, dd)
    out = torch.full((nb * 256,), float("nan"), dtype=torch.float32, device="cuda")
    moe2bit.debug_dequant_q2k(_t(torch, codes), _t(torch, dd), out)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_dequant_exhaustive_groups(torch_cuda):
    """Every (codebook row, sign field) pair for all 16 scales in one pass."""
    torch = torch_cuda
    rows = np.arange(256)
    sig = np.arange(128)
    pairs = np.array([(r, s) for r in rows for s in sig])  # 32768 groups
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
            v |= (s << (7 * j)) | (ls << 28)
            codes[b, 8 * sb + 4:8 * sb + 8] = np.frombuffer(np.uint32(v & 0xFFFFFFFF).tobytes(), np.uint8)
            g += 1
    d = np.full(nb, 0x3A21, np.uint16)
    ref = oracle.dequant_iq2(codes, d)
    out = torch.empty(nb * 256, dtype=torch.float32, device="cuda")
    moe2bit.debug_dequant_iq2(_t(torch, codes), _t(torch, d), out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


# ----------------------------------------------------------------- helpers
def _route_gpu(torch, dl, x, T, E, k):
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(max(T * k, 1), dtype=torch.int32, device="cuda")
    inv = torch.empty(max(T * k, 1), dtype=torch.int32, device="cuda")
    ws = moe2bit.alloc_workspace(dl.desc, T)
    moe2bit.route(dl.desc, dl.tensors["router_w"], dl.tensors["router_bias"], _x_dev(torch, x), idx, w, off, perm,
                  inv, ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy(), off.cpu().numpy(), perm.cpu().numpy()[:T * k], inv.cpu().numpy()[:T * k]


def _forward_gpu(torch, dl, x, residual=None, alias=False):
    T = x.shape[0]
    y = torch.full((T, dl.desc.hidden), float("nan"), dtype=torch.float32, device="cuda")
    res = None
    if residual is not None:
        res = torch.from_numpy(np.ascontiguousarray(residual)).cuda()
        if alias:
            y = res
    ws = moe2bit.alloc_workspace(dl.desc, T)
    moe2bit.layer_forward(dl, _x_dev(torch, x), res, y, ws)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def _check_route(torch, cfg, lw, dl, x):
    idx, w, off, perm, inv = _route_gpu(torch, dl, x, x.shape[0], cfg.E, cfg.k)
    ridx, rw = oracle.route(lw.router_w, lw.router_bias, x, cfg.k)
    assert np.array_equal(idx, ridx)
    assert np.max(np.abs(w - rw), initial=0.0) <= TOPK_W_TOL
    roff, rperm, rinv = oracle.permute(ridx, cfg.E)
    assert np.array_equal(off, roff)
    assert np.array_equal(perm, rperm)
    assert np.array_equal(inv, rinv)


# ---------------------------------------------------------------- configs
def _small(**kw):
    base = dict(name="small", T=37, H=512, I=256, E=16, k=4, Is=64, x_dtype="bf16", x_std=1.0, zipf=False,
                layers=1, seed=0x5A11)
    base.update(kw)
    return synth.Config(**base)


SMALL_CASES = {
    "tiny": synth.CONFIGS["tiny"],
    "small_bf16": _small(),
    "small_f32_zipf": _small(x_dtype="f32", zipf=True, T=29, seed=0x5A12),
    "ragged_many_tiles": _small(H=1280, I=768, E=24, k=6, Is=0, T=53, seed=0x5A13),
    "flat_blocks_k1": _small(H=256, I=64, E=4, k=1, Is=32, T=9, seed=0x5A14),
    "single_expert": _small(E=1, k=1, Is=0, T=5, seed=0x5A15),
    "k_eq_E": _small(E=4, k=4, T=7, seed=0x5A16),
    # shapes served by the TMA-fed GEMVs (H % 1024 == 0, I % 512 == 0, T <= 16; above 16 tokens the
    # tensor-core grouped GEMM takes over)
    "tma_t1": _small(H=1024, I=512, E=16, k=4, Is=64, T=1, seed=0x5A17),
    "tma_t5": _small(H=2048, I=1024, E=8, k=4, Is=128, T=5, seed=0x5A18),
    "tma_t16": _small(H=1024, I=512, E=8, k=4, Is=64, T=16, seed=0x5A19),
    "tma_t16_zipf_f32": _small(H=1024, I=1024, E=12, k=3, Is=0, T=16, x_dtype="f32", zipf=True, seed=0x5A1A),
    "tma_t3_shared_experts": _small(H=1024, I=512, E=4, k=4, Is=128, T=3, seed=0x5A20),
    # shapes served by the tensor-core grouped GEMM (T > 16, H, I multiples of 256, I_s of 128)
    "tc_t17": _small(H=512, I=256, E=4, k=2, Is=128, T=17, seed=0x5A1B),
    "tc_t64_f32": _small(H=1024, I=512, E=8, k=2, Is=256, T=64, x_dtype="f32", seed=0x5A1C),
    "tc_t200_zipf": _small(H=768, I=512, E=16, k=4, Is=0, T=200, zipf=True, seed=0x5A1D),
    "tc_t300_many_tiles": _small(H=1280, I=768, E=2, k=1, Is=384, T=300, seed=0x5A1E),
    # routing in one warp up to 32 assignments (here exactly 32), the block kernel above (here 40)
    "route_n32": _small(H=512, I=256, E=64, k=8, Is=64, T=4, seed=0x5A23),
    "route_n40": _small(H=512, I=256, E=64, k=8, Is=64, T=5, seed=0x5A24),
    # activations far from unit scale: the fp16 operands of the tensor-core path carry a
    # power-of-2 exponent per token, so neither overflow (g * u beyond 65504) nor underflow
    "tc_t40_large_x": _small(H=512, I=256, E=8, k=2, Is=128, T=40, x_std=300.0, seed=0x5A21),
    "tc_t40_small_x_f32": _small(H=512, I=256, E=8, k=2, Is=128, T=40, x_dtype="f32", x_std=1e-3, seed=0x5A22),
    # router logits on the tensor cores too (bf16 x, T > 64, E % 128 == 0)
    "tc_router_t130": _small(H=512, I=256, E=128, k=4, Is=128, T=130, seed=0x5A1F),
}


@pytest.mark.parametrize("name", list(SMALL_CASES))
def test_route_small(torch_cuda, name):
    cfg = SMALL_CASES[name]
    lw = synth.make_layer(cfg)
    x = screened_x(cfg, lw)
    _check_route(torch_cuda, cfg, lw, moe2bit.to_device(lw), x)


# Normwise and element-wise errors of every layer comparison, written out as a
# JSON report when MOE_PARITY_REPORT names a file (the element-wise figure uses a
# floor of 1e-3 * max |y_ref|; the bound asserted is the normwise one).
REPORT = {}


def _record(name, y, ref):
    REPORT[name] = {"normwise": normwise(y, ref), "elementwise_floor_1e-3": elementwise(y, ref)}
    return REPORT[name]["normwise"]


@pytest.mark.parametrize("name", list(SMALL_CASES))
def test_layer_forward_small(torch_cuda, name):
    cfg = SMALL_CASES[name]
    lw = synth.make_layer(cfg)
    x = screened_x(cfg, lw)
    res = synth.make_residual(cfg, cfg.T)
    dl = moe2bit.to_device(lw)
    y = _forward_gpu(torch_cuda, dl, x, res)
    ref, _, _ = oracle.layer_forward(lw, x, res)
    assert _record(name, y, ref) <= FFN_TOL
    # residual may alias the output
    y2 = _forward_gpu(torch_cuda, dl, x, res, alias=True)
    assert np.array_equal(y2, y)


def test_layer_forward_deterministic(torch_cuda):
    cfg = SMALL_CASES["small_bf16"]
    lw = synth.make_layer(cfg)
    x = screened_x(cfg, lw)
    dl = moe2bit.to_device(lw)
    y1 = _forward_gpu(torch_cuda, dl, x)
    y2 = _forward_gpu(torch_cuda, dl, x)
    assert np.array_equal(y1, y2)


def test_expert_ffn_caller_routing(torch_cuda):
    """Caller-made routing (weights not summing to one, repeated experts across
    tokens, some experts idle) through moe_expert_ffn."""
    torch = torch_cuda
    cfg = SMALL_CASES["small_bf16"]
    lw = synth.make_layer(cfg)
    x = synth.make_x(cfg)
    rng = np.random.default_rng(3)
    idx = np.stack([rng.choice(6, cfg.k, replace=False) for _ in range(cfg.T)]).astype(np.int32)
    w = rng.uniform(-1, 2, (cfg.T, cfg.k)).astype(np.float32)
    off, perm, inv = oracle.permute(idx, cfg.E)
    dl = moe2bit.to_device(lw)
    y = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device="cuda")
    ws = moe2bit.alloc_workspace(dl.desc, cfg.T)
    moe2bit.expert_ffn(dl, _x_dev(torch, x), _t(torch, w), _t(torch, off), _t(torch, perm), _t(torch, inv), None,
                       y, ws)
    torch.cuda.synchronize()
    ref = oracle.expert_ffn(lw, x, idx, w)
    assert normwise(y.cpu().numpy(), ref) <= FFN_TOL


def test_zero_tokens_is_noop(torch_cuda):
    torch = torch_cuda
    cfg = SMALL_CASES["small_bf16"]
    dl = moe2bit.to_device(synth.make_layer(cfg))
    x = torch.empty((0, cfg.H), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((0, cfg.H), dtype=torch.float32, device="cuda")
    ws = moe2bit.alloc_workspace(dl.desc, 0)
    moe2bit.layer_forward(dl, x, None, y, ws)
    torch.cuda.synchronize()


# ------------------------------------------------------- outlier activations
# One large element (+-64) per 256-element block among N(0,1) values: the
# decode GEMVs quantise x in 256-element blocks (the outlier sets the block's
# scale) and the grouped GEMM scales each token by one power of two.
OUTLIER_CASES = {
    "outlier_gemv_t1": _small(H=1024, I=512, E=16, k=4, Is=64, T=1, seed=0x5A40),
    "outlier_gemv_t6": _small(H=2048, I=1024, E=8, k=4, Is=128, T=6, seed=0x5A41),
    "outlier_gemm_t40": _small(H=1024, I=512, E=8, k=2, Is=128, T=40, seed=0x5A42),
    "outlier_gemm_t40_f32": _small(H=1024, I=512, E=8, k=2, Is=128, T=40, x_dtype="f32", seed=0x5A43),
}


@pytest.mark.parametrize("name", list(OUTLIER_CASES))
def test_layer_forward_outliers(torch_cuda, name):
    cfg = OUTLIER_CASES[name]
    lw = synth.make_layer(cfg)
    x = screened_x(cfg, lw, outliers=True)
    _check_route(torch_cuda, cfg, lw, moe2bit.to_device(lw), x)
    y = _forward_gpu(torch_cuda, moe2bit.to_device(lw), x)
    ref, _, _ = oracle.layer_forward(lw, x)
    assert _record(name, y, ref) <= FFN_TOL


# ------------------------------------------------------- full-size configs
def _full_case(torch, name):
    """The whole workload against the oracle: routing bit-exact for every token,
    every token's output within the normwise bound (the oracle runs on all host
    cores; each output is still one sequential double loop)."""
    cfg = synth.CONFIGS[name]
    lw = synth.make_layer(cfg)
    x = screened_x(cfg, lw)
    dl = moe2bit.to_device(lw)
    _check_route(torch, cfg, lw, dl, x)
    y = _forward_gpu(torch, dl, x)
    ref, _, _ = oracle.layer_forward(lw, x)
    _record(name, y, ref)
    per_token = [normwise(y[t:t + 1], ref[t:t + 1]) for t in range(cfg.T)]
    assert max(per_token) <= FFN_TOL, (name, int(np.argmax(per_token)), max(per_token))
    return y


@pytest.mark.slow
def test_full_decode1(torch_cuda):
    _full_case(torch_cuda, "decode1")


@pytest.mark.slow
def test_full_decode32(torch_cuda):
    _full_case(torch_cuda, "decode32")


@pytest.mark.slow
def test_full_prefill_every_token(torch_cuda):
    _full_case(torch_cuda, "prefill")


@pytest.mark.slow
def test_full_stack_two_layers_teacher_forced(torch_cuda):
    """The 8-layer stack's shapes (16 tokens, H=7168, E=256, Zipf routing): two
    chained layers, each checked against the oracle on the exact bf16 input and
    fp32 residual the GPU saw (teacher-forced), output written over the
    residual in place, as the stack step runs."""
    torch = torch_cuda
    cfg = synth.CONFIGS["stack"]
    layers = [synth.make_layer(cfg, layer=l) for l in range(2)]
    x = screened_x(cfg, layers[0])
    res = synth.make_residual(cfg, cfg.T)
    y = torch.from_numpy(np.ascontiguousarray(res)).cuda()
    ws = moe2bit.alloc_workspace(moe2bit.to_device(layers[0]).desc, cfg.T)
    for l, lw in enumerate(layers):
        dl = moe2bit.to_device(lw)
        res_in = y.cpu().numpy().copy()
        _, _, logits = oracle.route(lw.router_w, lw.router_bias, x, cfg.k, want_logits=True)
        srt = -np.sort(-logits, axis=1)
        keep = (srt[:, cfg.k - 1] - srt[:, cfg.k]) >= 1e-4  # tokens whose routing fp32 cannot flip
        idx, _, off, _, _ = _route_gpu(torch, dl, x, cfg.T, cfg.E, cfg.k)
        ridx, _ = oracle.route(lw.router_w, lw.router_bias, x, cfg.k)
        assert np.array_equal(idx[keep], ridx[keep]), l
        moe2bit.layer_forward(dl, _x_dev(torch, x), y, y, ws)
        torch.cuda.synchronize()
        out = y.cpu().numpy()
        ref, _, _ = oracle.layer_forward(lw, x, res_in)
        assert keep.sum() >= cfg.T // 2, l
        assert _record(f"stack_layer{l}", out[keep], ref[keep]) <= FFN_TOL, l
        b = out.view(np.uint32)
        x = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)  # next input: bf16 (RNE) of the stream


def test_layer_chain_teacher_forced(torch_cuda):
    """A residual stream through four chained layers (the 8-layer stack's
    structure at small shapes, Zipf-biased routing, 16 tokens): each layer's
    output is checked against the oracle given the same bf16 input and fp32
    residual the GPU saw, with the output written over the residual in place.
    Tokens whose oracle top-k gap is below 1e-4 (a routing decision fp32 may
    take differently) are left out of the output comparison."""
    torch = torch_cuda
    cfg = _small(H=1024, I=512, E=16, k=4, Is=128, T=16, zipf=True, seed=0x5A25)
    layers = [synth.make_layer(cfg, layer=l) for l in range(4)]
    x = screened_x(cfg, layers[0])
    res = synth.make_residual(cfg, cfg.T)
    y = torch.from_numpy(np.ascontiguousarray(res)).cuda()
    ws = moe2bit.alloc_workspace(moe2bit.to_device(layers[0]).desc, cfg.T)
    for l, lw in enumerate(layers):
        dl = moe2bit.to_device(lw)
        res_in = y.cpu().numpy().copy()
        moe2bit.layer_forward(dl, _x_dev(torch, x), y, y, ws)  # y += layer(x), in place
        torch.cuda.synchronize()
        out = y.cpu().numpy()
        assert np.isfinite(out).all(), l
        ref, _, _ = oracle.layer_forward(lw, x, res_in)
        _, _, logits = oracle.route(lw.router_w, lw.router_bias, x, cfg.k, want_logits=True)
        srt = -np.sort(-logits, axis=1)
        keep = (srt[:, cfg.k - 1] - srt[:, cfg.k]) >= 1e-4
        assert keep.sum() >= cfg.T // 2, l
        assert normwise(out[keep], ref[keep]) <= FFN_TOL, l
        # the next layer's input: the residual stream rounded to bf16 (round to nearest even)
        b = out.view(np.uint32)
        x = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)


def test_zz_write_parity_report():
    """Writes the collected error figures (only when MOE_PARITY_REPORT is set)."""
    import json
    import os

    path = os.environ.get("MOE_PARITY_REPORT")
    if path:
        with open(path, "w") as f:
            json.dump(REPORT, f, indent=1, sort_keys=True)
