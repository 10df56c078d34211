"""Host-side checks of the C ABI (no GPU): the library loads, exports every
symbol the header declares, computes workspace sizes, rejects bad arguments
before touching a device, and carries the same codebook as the oracle."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from bit_quantized_routed_iq2_b200 import build as moebuild
from bit_quantized_routed_iq2_b200 import moe2bit

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    moebuild.build()
    return moe2bit.load()


def _header_symbols():
    src = open(os.path.join(ROOT, "include", "moe2bit.h")).read()
    return set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src))


def test_header_declares_the_binding_exports():
    assert _header_symbols() == set(moe2bit.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    for name in _header_symbols():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in moe2bit.STATUS.items():
        assert moe2bit.status_string(code) == name


def test_codebook_matches_oracle(lib):
    # two independent implementations of the same generator definition
    assert moe2bit.debug_grid() == oracle.grid().tobytes()


DECODE = dict(H=7168, I=2048, E=256, k=8, Is=2048)


def test_workspace_size_monotone(lib):
    d = moe2bit.desc_of(**DECODE)
    sizes = [moe2bit.workspace_size(d, T) for T in (0, 1, 2, 16, 32, 2048)]
    assert all(a <= b for a, b in zip(sizes, sizes[1:]))
    assert sizes[1] > 0


@pytest.mark.parametrize(
    "shape",
    [dict(H=100, I=2048, E=256, k=8, Is=2048), dict(H=7168, I=300, E=256, k=8, Is=2048),
     dict(H=7168, I=2048, E=4, k=8, Is=2048), dict(H=7168, I=2048, E=256, k=17, Is=2048),
     dict(H=7168, I=2048, E=2048, k=8, Is=2048), dict(H=7168, I=2048, E=256, k=8, Is=4)],
)
def test_unsupported_shapes_rejected(lib, shape):
    d = moe2bit.desc_of(**shape)
    n = ctypes.c_size_t(0)
    assert lib.moe_workspace_size(ctypes.byref(d), 4, ctypes.byref(n)) == 2


def test_invalid_arguments_rejected_without_launch(lib):
    d = moe2bit.desc_of(**DECODE)
    w = moe2bit.Weights()
    # null weights / activations: MOE_ERR_INVALID_ARG before any CUDA call
    assert lib.moe_layer_forward(ctypes.byref(d), ctypes.byref(w), None, 1, 1, None, None, None, 0, None) == 1
    assert lib.moe_layer_forward(ctypes.byref(d), None, None, 1, 1, None, None, None, 0, None) == 1
    assert lib.moe_route(ctypes.byref(d), None, None, None, 1, 1, None, None, None, None, None, None, 0, None) == 1
    # bad dtype
    assert lib.moe_route(ctypes.byref(d), None, None, None, 7, 1, None, None, None, None, None, None, 0, None) == 1
    # negative T
    assert lib.moe_layer_forward(ctypes.byref(d), ctypes.byref(w), None, 1, -1, None, None, None, 0, None) == 1
    # T == 0 is a no-op
    assert lib.moe_layer_forward(ctypes.byref(d), ctypes.byref(w), None, 1, 0, None, None, None, 0, None) == 0
    assert lib.moe_debug_dequant_iq2(None, None, 4, None, None) == 1
    assert lib.moe_debug_dequant_q2k(None, None, -1, None, None) == 1


def test_misaligned_and_small_workspace_rejected(lib):
    d = moe2bit.desc_of(**DECODE)
    fake = 1 << 40  # never dereferenced: validation fails first
    w = moe2bit.Weights(*([fake] * 11))
    need = moe2bit.workspace_size(d, 1)
    # misaligned activation pointer
    assert lib.moe_layer_forward(ctypes.byref(d), ctypes.byref(w), fake + 2, 1, 1, None, fake, fake, need, None) == 1
    # workspace too small
    assert lib.moe_layer_forward(ctypes.byref(d), ctypes.byref(w), fake, 1, 1, None, fake, fake, need - 1, None) == 3


def test_next_layer_output_validated_on_host(lib):
    # moe_layer_forward_next: y_next is required, 16-byte aligned and disjoint from x, y, residual and the
    # workspace; every case below fails validation before anything is enqueued
    d = moe2bit.desc_of(**DECODE)
    base = 1 << 40
    w = moe2bit.Weights(*([base] * 11))
    need = moe2bit.workspace_size(d, 1)
    x, y, ws, res = base, base + (1 << 30), base + (1 << 31), base + (3 << 30)
    f = lib.moe_layer_forward_next

    def call(y_next, residual=None):
        return f(ctypes.byref(d), ctypes.byref(w), x, 1, 1, residual, y, y_next, ws, need, None)

    assert call(None) == 1
    assert call(x) == 1                                   # the input itself
    assert call(x + 2 * d.hidden - 16) == 1               # the input's last 16 bytes
    assert call(y + 16) == 1                              # inside y
    assert call(res, residual=res) == 1                   # the residual
    assert call(ws + 4096) == 1                           # inside the workspace
    assert call(base + (1 << 32) + 8) == 1                # misaligned
    # T = 0 is a no-op for every entry point, y_next included
    assert f(ctypes.byref(d), ctypes.byref(w), x, 1, 0, None, y, None, ws, need, None) == 0


def test_status_query_and_injection_validate_on_host(lib):
    """The status query and the fault-injection switch reject bad arguments
    without touching a device; injection mode 0 is plain host state."""
    v = ctypes.c_int32(0)
    assert lib.moe_read_status(None, ctypes.byref(v), None) == 1
    assert lib.moe_read_status((1 << 40) + 4, ctypes.byref(v), None) == 1  # misaligned workspace
    assert lib.moe_read_status(1 << 40, None, None) == 1
    assert lib.moe_read_status_noalloc(None, None) == 1
    assert lib.moe_debug_inject(2, 0) == 1
    assert lib.moe_debug_inject(1, -1) == 1
    assert lib.moe_debug_inject(0, 0) == 0


def test_cache_arguments_validate_on_host(lib):
    d = moe2bit.desc_of(**DECODE)
    n = ctypes.c_size_t(0)
    assert lib.moe_cache_bytes(ctypes.byref(d), 0, ctypes.byref(n)) == 1
    assert lib.moe_cache_bytes(ctypes.byref(d), 257, ctypes.byref(n)) == 1
    assert lib.moe_cache_bytes(ctypes.byref(d), 8, ctypes.byref(n)) == 0
    per_expert = 2 * 2048 * 7168 // 256 * (64 + 2) + 7168 * 2048 // 256 * (80 + 4)
    assert n.value >= 8 * per_expert
    h = ctypes.c_void_p()
    w = moe2bit.Weights()
    assert lib.moe_cache_create(ctypes.byref(d), ctypes.byref(w), 8, None, n.value, ctypes.byref(h)) == 1
    assert lib.moe_cache_create(ctypes.byref(d), None, 8, 1 << 40, n.value, ctypes.byref(h)) == 1
    assert lib.moe_cache_create(ctypes.byref(d), ctypes.byref(w), 8, 1 << 40, n.value - 1, ctypes.byref(h)) == 3
    assert lib.moe_layer_forward_cached(None, ctypes.byref(w), None, 1, 1, None, None, None, 0, None) == 1
    assert lib.moe_cache_read_stats(None, None) == 1
