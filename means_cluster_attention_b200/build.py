"""Build libclusterattn.so in-tree for sm_100a with nvcc.

Run ``python -m means_cluster_attention_b200.build`` (or call ``build()``).
The library is a single translation unit (csrc/api.cu includes the kernels).
"""

from __future__ import annotations

import glob
import hashlib
import re
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libclusterattn.so")
# The bounds-checked build (-DCA_CHECKED): every computed index that addresses
# memory is checked on the device; a bad one records CA_ERR_DEVICE (read by
# ca_sync_status) and is clamped, so nothing faults.  Selected at load time
# with the environment variable CA_CHECKED=1.
LIB_CHECKED = os.path.join(PKG, "libclusterattn_checked.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: set NVCC or install the CUDA toolkit")


def sources() -> list:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(INCLUDE, "clusterattn.h")])


# Source files each profiled kernel is built from (its own code and the
# headers it includes), for deciding whether recorded counters still apply.
_TILED = ["tiled.cuh", "fused.cuh", "kmeans_tile.cuh", "umma.cuh", "mma.cuh", "common.cuh"]
KERNEL_SOURCES = {
    "fused_forward": ["fused.cuh", "kmeans_tile.cuh", "mma.cuh", "common.cuh"],
    "tiled_assign": _TILED,
    "tiled_window": _TILED,
    "tiled_centroid": _TILED,
}


def _code_only(text: bytes) -> bytes:
    """Source text without comments and blank lines: edits to comments do not
    change the kernel a measurement was taken on."""
    t = re.sub(rb"/\*.*?\*/", b"", text, flags=re.S)
    t = re.sub(rb"//[^\n]*", b"", t)
    return b"\n".join(line.rstrip() for line in t.splitlines() if line.strip())


def source_hash(kernel: str = None) -> str:
    """Hash of the code (comments excluded) a kernel is built from (all
    sources if None)."""
    files = sources() if kernel is None else [os.path.join(CSRC, f) for f in KERNEL_SOURCES[kernel]]
    h = hashlib.sha256()
    for s in files:
        h.update(os.path.basename(s).encode())
        with open(s, "rb") as f:
            h.update(_code_only(f.read()))
    return h.hexdigest()[:16]


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False, extra_flags=None, checked: bool = False) -> str:
    lib = LIB_CHECKED if checked else LIB
    if not force and not needs_build(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
           "-I", INCLUDE, "-I", CSRC, "-o", tmp, os.path.join(CSRC, "api.cu"), "-cudart", "static"]
    if checked:
        cmd.insert(1, "-DCA_CHECKED")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    if extra_flags:
        cmd[1:1] = list(extra_flags)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    print(build(force="--force" in sys.argv, checked=True))
