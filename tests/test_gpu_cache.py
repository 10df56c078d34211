"""The expert cache: routed experts on the host, a few of them in GPU slots.

moe_layer_forward_cached must give the resident layer's output bit for bit
(the same kernels run over slots instead of experts) through sequences of calls
that hit and miss, evict least-recently-used slots, and serve both the decode
GEMVs and the grouped GEMM; its counters must add up; and a call that needs
more experts than there are slots must say so.
"""
import numpy as np
import pytest

import synth
from bit_quantized_routed_iq2_b200 import build as moebuild
from bit_quantized_routed_iq2_b200 import moe2bit
from helpers import screened_x

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


CASES = [
    # (name, T per call, slots, x dtype, zipf)
    ("decode_t1", 1, 6, "bf16", False),
    ("decode_t3_zipf", 3, 12, "bf16", True),
    ("decode_t2_f32", 2, 8, "f32", False),
    ("gemm_t40", 40, 16, "bf16", False),
]


@pytest.mark.parametrize("name,T,slots,xdt,zipf", CASES)
def test_cached_layer_matches_resident(torch_cuda, name, T, slots, xdt, zipf):
    torch = torch_cuda
    cfg = synth.Config(name, T, 1024, 512, 16, 4, 128, xdt, 1.0, zipf, 1, 0xCAC0 + T)
    lw = synth.make_layer(cfg)
    dl = moe2bit.to_device(lw)
    shared = moe2bit.to_device_shared_only(lw)
    cache = moe2bit.ExpertCache(lw, slots)
    ws = moe2bit.alloc_workspace(dl.desc, T)
    eb = sum(getattr(lw, n)[0].nbytes for n in moe2bit.ExpertCache.ROUTED)
    tot_active = 0
    for call in range(6):
        c = synth.Config(**{**cfg.__dict__, "seed": cfg.seed + 17 * call})
        x = screened_x(c, lw)
        xd = _x_dev(torch, x)
        y_ref = torch.empty((T, cfg.H), dtype=torch.float32, device="cuda")
        y = torch.full((T, cfg.H), float("nan"), dtype=torch.float32, device="cuda")
        res = torch.from_numpy(synth.make_residual(c, T)).cuda()
        moe2bit.layer_forward(dl, xd, res, y_ref, ws)
        # the routing's distinct experts, for the counters
        idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
        off = torch.empty(cfg.E + 1, dtype=torch.int32, device="cuda")
        perm = torch.empty(T * cfg.k, dtype=torch.int32, device="cuda")
        inv = torch.empty(T * cfg.k, dtype=torch.int32, device="cuda")
        moe2bit.route(dl.desc, dl.tensors["router_w"], dl.tensors["router_bias"], xd, idx, w, off, perm, inv, ws)
        tot_active += int(np.count_nonzero(np.diff(off.cpu().numpy())))
        cache.forward(shared, xd, res, y, ws)
        torch.cuda.synchronize()
        assert np.array_equal(y.cpu().numpy(), y_ref.cpu().numpy()), (name, call)
    st = cache.stats()
    assert st["calls"] == 6
    assert st["hits"] + st["misses"] == tot_active
    assert st["bytes_copied"] == st["misses"] * eb
    assert st["misses"] >= min(slots, cfg.E) // 2  # the cache started empty
    cache.close()


def test_too_few_slots_is_reported(torch_cuda):
    torch = torch_cuda
    cfg = synth.Config("few", 1, 1024, 512, 16, 4, 64, "bf16", 1.0, False, 1, 0xCAD0)
    lw = synth.make_layer(cfg)
    shared = moe2bit.to_device_shared_only(lw)
    cache = moe2bit.ExpertCache(lw, 2)  # one token needs k = 4 experts
    ws = moe2bit.alloc_workspace(shared.desc, 1)
    x = _x_dev(torch, screened_x(cfg, lw))
    y = torch.empty((1, cfg.H), dtype=torch.float32, device="cuda")
    with pytest.raises(moe2bit.MoeError) as ei:
        cache.forward(shared, x, None, y, ws)
    assert ei.value.status == 3  # MOE_ERR_WORKSPACE_TOO_SMALL
    cache.close()
