"""Build step of libmonoffn.so (nvcc, sm_100a only), in-tree next to the
package so that the library travels with the source tree."""

import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "mono_ffn.cu")
DEPS = [SRC, os.path.join(PKG, "csrc", "common.cuh"), os.path.join(PKG, "csrc", "cc_kernel.cuh"),
        os.path.join(PKG, "csrc", "tc_kernel.cuh"), os.path.join(PKG, "csrc", "ptx.cuh"),
        os.path.join(PKG, "csrc", "route_noalloc.cuh"), os.path.join(PKG, "csrc", "tq_kernel.cuh"),
        os.path.join(ROOT, "include", "mono_ffn.h")]
SO = os.path.join(PKG, "libmonoffn.so")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17", "-maxrregcount=168",
              "-Xcompiler", "-fPIC",
              "-shared", "-Xptxas", "-v"]


def build(force=False, verbose=False):
    if not force and os.path.exists(SO) and os.path.getmtime(SO) >= max(os.path.getmtime(d) for d in DEPS):
        return SO
    cmd = ["nvcc", *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-o", SO, SRC]
    res = subprocess.run(cmd, capture_output=True, text=True)
    log = res.stdout + res.stderr
    with open(os.path.join(PKG, "build.log"), "w") as f:
        f.write(" ".join(cmd) + "\n" + log)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + log[-4000:])
    if verbose:
        print(log)
    return SO


if __name__ == "__main__":
    build(force=True, verbose=True)
