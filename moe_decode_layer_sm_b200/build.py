"""Build step of libmonoffn.so (nvcc, sm_100a only), in-tree next to the
package so that the library travels with the source tree.

The library is rebuilt unless a stamp file beside it records the SHA-256 of
every source it is built from and of the nvcc command: a binary that merely
has a later modification time than its sources is not trusted."""

import hashlib
import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "mono_ffn.cu")
DEPS = [SRC] + [os.path.join(PKG, "csrc", f) for f in ("common.cuh", "cc_kernel.cuh", "tc_kernel.cuh", "ptx.cuh",
                                                         "route_noalloc.cuh", "tq_kernel.cuh")] + \
       [os.path.join(ROOT, "include", "mono_ffn.h")]
SO = os.path.join(PKG, "libmonoffn.so")
STAMP = SO + ".sha256"

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17", "-maxrregcount=168",
              "-Xcompiler", "-fPIC",
              "-shared", "-Xptxas", "-v"]


def command():
    return ["nvcc", *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-o", SO, SRC]


def source_hash():
    """SHA-256 over the sources (name and bytes, in a fixed order) and the
    nvcc command line."""
    h = hashlib.sha256()
    for d in DEPS:
        h.update(os.path.basename(d).encode() + b"\0")
        with open(d, "rb") as f:
            h.update(f.read())
    h.update(" ".join(command()).encode())
    return h.hexdigest()


def up_to_date():
    if not (os.path.exists(SO) and os.path.exists(STAMP)):
        return False
    with open(STAMP) as f:
        return f.read().strip() == source_hash()


def build(force=False, verbose=False):
    if not force and up_to_date():
        return SO
    if os.path.exists(STAMP):
        os.unlink(STAMP)
    cmd = command()
    res = subprocess.run(cmd, capture_output=True, text=True)
    log = res.stdout + res.stderr
    with open(os.path.join(PKG, "build.log"), "w") as f:
        f.write(" ".join(cmd) + "\n" + log)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + log[-4000:])
    with open(STAMP, "w") as f:
        f.write(source_hash() + "\n")
    if verbose:
        print(log)
    return SO


if __name__ == "__main__":
    build(force=True, verbose=True)
