"""Build libva3d.so in-tree with nvcc for sm_100a (B200).

The library is rebuilt whenever the SHA-256 of its sources (the .cu file, the
kernel headers and include/va3d.h) and of the nvcc command line differs from
the one recorded next to it at its last build (``libva3d.so.stamp``), so a
library built from other sources is never reused, whatever the file times.
"""
import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libva3d.so")
STAMP = LIB + ".stamp"
SOURCES = [os.path.join(CSRC, "va3d_api.cu")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-v",
    "-I", os.path.join(ROOT, "include"), "-I", CSRC,
]


def deps():
    headers = sorted(f for f in os.listdir(CSRC) if f.endswith(".cuh"))
    return SOURCES + [os.path.join(CSRC, f) for f in headers] + [
        os.path.join(ROOT, "include", "va3d.h")]


def source_hash(flags=None):
    """SHA-256 over the nvcc flags and every source file (name and bytes)."""
    h = hashlib.sha256()
    h.update(" ".join(NVCC_FLAGS if flags is None else flags).encode())
    for d in deps():
        h.update(os.path.relpath(d, ROOT).encode() + b"\0")
        with open(d, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def nvcc():
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    path = os.path.join(cuda, "bin", "nvcc")
    return path if os.path.exists(path) else "nvcc"


def up_to_date():
    if not (os.path.exists(LIB) and os.path.exists(STAMP)):
        return False
    with open(STAMP) as f:
        return f.read().strip() == source_hash()


def build(force=False, verbose=False):
    if not force and up_to_date():
        return LIB
    digest = source_hash()
    cmd = [nvcc()] + NVCC_FLAGS + ["-o", LIB] + SOURCES
    res = subprocess.run(cmd, capture_output=True, text=True)
    log = os.path.join(HERE, "build.log")
    with open(log, "w") as f:
        f.write(" ".join(cmd) + "\n" + res.stdout + res.stderr)
    if res.returncode != 0:
        sys.stderr.write(res.stderr)
        raise RuntimeError(f"nvcc failed (see {log})")
    with open(STAMP, "w") as f:
        f.write(digest + "\n")
    if verbose:
        sys.stderr.write(res.stderr)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
