"""Build libbitlinear.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m bit_ternary_b200.build            # build if sources changed
    python -m bit_ternary_b200.build --force -v # rebuild, print ptxas usage
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(HERE, "libbitlinear.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = [
    "-std=c++17",
    "-O3",
    "-lineinfo",
    "-Xcompiler", "-fPIC",
    "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-shared",
]


def _nvcc() -> str:
    cand = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError(f"nvcc not found (tried {cand})")
    return cand


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))) + [
        os.path.join(INCLUDE, "bitlinear.h")
    ]


def sources_sha() -> str:
    """Hash of the kernel sources and header (identifies the measured kernels)."""
    import hashlib

    h = hashlib.sha256()
    for f in _inputs():
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


KERNEL_SOURCES = {
    "bl_ternary_decode_kernel": ["bl_decode.cu", "bl_device.cuh"],
    "gemm_kernel": ["bl_gemm.cu", "bl_device.cuh"],
}


def kernel_sha(kernel: str) -> str:
    """Hash of the source file that defines `kernel` and the device helpers it
    uses: profiler counters taken for a kernel stay valid while this holds."""
    import hashlib

    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        h.update(name.encode())
        with open(os.path.join(CSRC, name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


ID_PATH = LIB_PATH + ".id"  # sources_sha() of the sources the library was built from


def up_to_date() -> bool:
    """True when the library exists and was built from the current sources
    (compared by content hash, not by file times)."""
    if not (os.path.exists(LIB_PATH) and os.path.exists(ID_PATH)):
        return False
    with open(ID_PATH) as f:
        return f.read().strip() == sources_sha()


def build_library(force: bool = False, verbose: bool = False) -> str:
    """Compile every .cu under csrc/ into libbitlinear.so. Returns the path.
    The sources' hash is compiled in (bitlinear_build_id) and recorded beside
    the library, so a library built from other sources is rebuilt here and
    refused by the loader."""
    if not force and up_to_date():
        return LIB_PATH
    sha = sources_sha()
    cmd = [_nvcc(), *ARCH_FLAGS, *NVCC_FLAGS, f"-I{INCLUDE}", f"-I{CSRC}", f'-DBL_BUILD_ID="{sha}"']
    if verbose:
        cmd += ["-Xptxas", "-v"]
    tmp = LIB_PATH + ".tmp"
    cmd += ["-o", tmp, *sources(), "-lcudart"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, LIB_PATH)
    with open(ID_PATH, "w") as f:
        f.write(sha + "\n")
    return LIB_PATH


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    a = ap.parse_args(argv)
    print(build_library(force=a.force, verbose=a.verbose))


if __name__ == "__main__":
    main()
