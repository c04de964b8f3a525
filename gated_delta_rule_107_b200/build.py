"""Build libdeltarule.so in-tree with nvcc for sm_100a."""
from __future__ import annotations

import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libdeltarule.so")
ROOT = os.path.dirname(HERE)

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-warn-spills",
    "-Xlinker", "-z,defs",  # an undefined symbol fails the build, not the first load
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(ROOT, "include", "*.h")))


def source_digest(files: list[str] | None = None) -> str:
    """sha256 over library sources (identifies the code a profile was taken on): every source,
    or only the named files of csrc/ (those that define one kernel and its launch)."""
    import hashlib
    h = hashlib.sha256()
    paths = sources() if files is None else [os.path.join(CSRC, f) for f in sorted(files)]
    for p in paths:
        h.update(os.path.basename(p).encode())
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# the files that define each profiled kernel and its launch
KERNEL_FILES = {
    "k_bwd_chunk_tc": ["tc_bwd.cu", "tc_ptx.cuh", "tc_tile.cuh", "tc_inverse.cuh", "tc_host.cuh", "dr_common.cuh"],
}


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    """Compile csrc/delta_rule_lib.cu (the unity translation unit) into libdeltarule.so."""
    newest = max(os.path.getmtime(p) for p in sources())
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, *(extra or []), "-o", tmp, os.path.join(CSRC, "delta_rule_lib.cu")]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    import sys
    print(build(force="--force" in sys.argv, verbose=True, extra=["-Xptxas", "-v"] if "-v" in sys.argv else None))
