"""Build libmoe2bit.so in-tree with nvcc for sm_100a (no GPU needed)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SO = os.path.join(HERE, "libmoe2bit.so")
# the bounds-checked build (-DMOE_BOUNDS_CHECK): a test aid, never the product path
SO_BC = os.path.join(HERE, "libmoe2bit_bc.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-v",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(so: str = SO) -> bool:
    if not os.path.exists(so):
        return True
    t = os.path.getmtime(so)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(ROOT, "include", "moe2bit.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, bounds_check: bool = False) -> str:
    so = SO_BC if bounds_check else SO
    if not force and not _stale(so):
        return so
    nvcc = os.environ.get("NVCC", "nvcc")
    extra = ["-DMOE_BOUNDS_CHECK"] if bounds_check else []
    cmd = [nvcc, *NVCC_FLAGS, *extra, "-shared", "-o", so + ".tmp", *sources(), "-lcudart"]
    res = subprocess.run(cmd, cwd=CSRC, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libmoe2bit.so")
    if verbose:
        sys.stderr.write(res.stderr)
    os.makedirs(os.path.join(HERE, "_build"), exist_ok=True)
    with open(os.path.join(HERE, "_build", "ptxas_report_bc.txt" if bounds_check else "ptxas_report.txt"), "w") as f:
        f.write(res.stderr)
    os.replace(so + ".tmp", so)
    return so


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=False, bounds_check="--bounds-check" in sys.argv))
