"""The small parity cases of the decode GEMVs under the bounds-checked build.

libmoe2bit_bc.so is the same library compiled with -DMOE_BOUNDS_CHECK: every
shared-memory load of the decode GEMVs checks its address and alignment, every
partial-sum store and TMA box its buffer, and violations are counted instead of
trapping (a stand-in for a memory checker). The cases run in a child process
that loads that build; they must give the oracle's results with no violation.
"""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import json, os, sys
import numpy as np
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, os.path.join(sys.argv[1], "tests"))
import torch
import oracle, synth
from bit_quantized_routed_iq2_b200 import moe2bit
from helpers import normwise, screened_x
assert moe2bit.load().moe_debug_bounds_check_build() == 1
out = {}
cases = [
    ("t1", dict(T=1, H=1024, I=512, E=16, k=4, Is=64, zipf=False)),
    ("t3", dict(T=3, H=1024, I=512, E=4, k=4, Is=128, zipf=False)),
    ("t16_zipf", dict(T=16, H=1024, I=1024, E=12, k=3, Is=64, zipf=True)),
    ("t5_wide", dict(T=5, H=2048, I=1024, E=8, k=4, Is=128, zipf=False)),
]
for name, sh in cases:
    cfg = synth.Config(name=name, x_dtype="bf16", x_std=1.0, layers=1, seed=0xBC00 + sh["T"], **sh)
    lw = synth.make_layer(cfg)
    x = screened_x(cfg, lw)
    dl = moe2bit.to_device(lw)
    y = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device="cuda")
    ws = moe2bit.alloc_workspace(dl.desc, cfg.T)
    xd = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
    moe2bit.layer_forward(dl, xd, None, y, ws)
    torch.cuda.synchronize()
    ref, _, _ = oracle.layer_forward(lw, x)
    out[name] = {"err": normwise(y.cpu().numpy(), ref), "violations": moe2bit.bounds_violations(),
                 "status": moe2bit.read_status(ws)}
print(json.dumps(out))
'''


def test_decode_gemvs_under_bounds_checks():
    from bit_quantized_routed_iq2_b200 import build as moebuild

    so = moebuild.build(bounds_check=True)
    env = dict(os.environ, MOE2BIT_SO=so)
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT], capture_output=True, text=True, env=env, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    for name, v in res.items():
        assert v["violations"] == 0, (name, v)
        assert v["status"] == 0, (name, v)
        assert v["err"] <= 2e-3, (name, v)
