"""Seeded synthetic inputs for the fused decode FFN half-layer.

One generator, two builds: ``libsynth_cpu.so`` (host arrays, for the oracle)
and ``libsynth_gpu.so`` (device tensors, for the CUDA path and the benchmark).
Both compute every element from (seed, tensor tag, index) with the same
integer and correctly rounded IEEE operations, so they write the same bytes.
Nothing here computes any step of the layer.
"""

import ctypes
import hashlib
import math
import os
import subprocess

import numpy as np

from .configs import Workload

HERE = os.path.dirname(os.path.abspath(__file__))
CPU_SO = os.path.join(HERE, "libsynth_cpu.so")
GPU_SO = os.path.join(HERE, "libsynth_gpu.so")

HC_IN, MIX_W, NORM_W, ROUTER_W, ROUTER_BIAS, GATE, UP, DOWN = range(1, 9)
ATTN_X, ATTN_POST, ATTN_COMB, ATTN_Y = range(9, 13)
_OUT = {"f32": 0, "bf16": 1, "f64": 2}


def build(gpu=True):
    """Compile the generator (CPU with gcc; device with nvcc for sm_100a).
    Each library is rebuilt unless its stamp file records the SHA-256 of its
    sources and compile command."""
    src = os.path.join(HERE, "synth_cpu.c")
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared", "-o", CPU_SO, src, "-lm"]
    _build_stamped(CPU_SO, [src, os.path.join(HERE, "synth_core.h")], cmd)
    if gpu:
        src = os.path.join(HERE, "synth_gpu.cu")
        cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-fmad=false", "-std=c++17",
               "-Xcompiler", "-fPIC", "-shared", "-o", GPU_SO, src]
        _build_stamped(GPU_SO, [src, os.path.join(HERE, "synth_core.h")], cmd)


def _build_stamped(out, srcs, cmd):
    h = hashlib.sha256()
    for s in srcs:
        with open(s, "rb") as f:
            h.update(f.read())
    h.update(" ".join(cmd).encode())
    stamp = out + ".sha256"
    if os.path.exists(out) and os.path.exists(stamp) and open(stamp).read().strip() == h.hexdigest():
        return
    if os.path.exists(stamp):
        os.unlink(stamp)
    subprocess.check_call(cmd)
    with open(stamp, "w") as f:
        f.write(h.hexdigest() + "\n")


_cpu = None
_gpu = None


def cpu_lib():
    global _cpu
    if _cpu is None:
        if not os.path.exists(CPU_SO):
            build(gpu=False)
        lib = ctypes.CDLL(CPU_SO)
        u64, u32, i32, f64, vp = (ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int, ctypes.c_double,
                                  ctypes.c_void_p)
        lib.synth_fill.argtypes = [u64, u32, u32, u32, i32, f64, f64, u64, u64, i32, vp]
        lib.synth_quant_fp8.argtypes = [vp, u64, u64, vp, vp]
        lib.synth_quant_mxfp4.argtypes = [vp, u64, u64, vp, vp]
        lib.synth_fill_fp8.argtypes = [u64, u32, u32, u32, f64, u64, u64, vp, vp]
        lib.synth_fill_mxfp4.argtypes = [u64, u32, u32, u32, f64, u64, u64, u32, vp, vp]
        lib.synth_ln_probe.argtypes = [f64]
        lib.synth_ln_probe.restype = f64
        _cpu = lib
    return _cpu


def gpu_lib():
    global _gpu
    if _gpu is None:
        if not os.path.exists(GPU_SO):
            raise RuntimeError(f"{GPU_SO} is not built; run __graft_entry__.build()")
        lib = ctypes.CDLL(GPU_SO)
        u64, u32, i32, f64, vp = (ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int, ctypes.c_double,
                                  ctypes.c_void_p)
        lib.synth_gpu_fill.argtypes = [u64, u32, u32, u32, i32, f64, f64, u64, u64, i32, vp, vp]
        lib.synth_gpu_fill_fp8.argtypes = [u64, u32, u32, u32, f64, u64, u64, vp, vp, vp]
        lib.synth_gpu_fill_mxfp4.argtypes = [u64, u32, u32, u32, f64, u64, u64, u32, vp, vp, vp]
        for f in (lib.synth_gpu_fill, lib.synth_gpu_fill_fp8, lib.synth_gpu_fill_mxfp4):
            f.restype = i32
        _gpu = lib
    return _gpu


# ------------------------------------------------------------ tensor recipe --

def tensor_specs(w: Workload, layer: int):
    """(kind, shape, dist, p0, p1, element type) of the dense per-layer tensors."""
    S, H, E = w.hc, w.hidden, w.n_routed
    return {
        "mix_w": (MIX_W, (S * H, w.mix_cols), 0, 0.0, 1.0 / math.sqrt(S * H), "f32"),
        "norm_w": (NORM_W, (H,), 0, 1.0, 0.1, w.norm_dtype),
        "router_w": (ROUTER_W, (H, E), 0, 0.0, 1.0 / math.sqrt(H), "f32"),
        "router_bias": (ROUTER_BIAS, (E,), 1, -0.1, 0.1, "f32"),
    }


def expert_specs(w: Workload):
    """(kind, rows=out, cols=in, std) of the three expert matrices."""
    H, I = w.hidden, w.inter
    return {
        "gate": (GATE, I, H, 1.0 / math.sqrt(H)),
        "up": (UP, I, H, 1.0 / math.sqrt(H)),
        "down": (DOWN, H, I, 1.0 / math.sqrt(I)),
    }


def _np_dtype(t):
    return {"f32": np.float32, "bf16": np.uint16, "f64": np.float64}[t]


def cpu_fill(seed, layer, kind, expert, shape, dist, p0, p1, out="f32", offset=0):
    n = int(np.prod(shape))
    a = np.empty(n, dtype=_np_dtype(out))
    cpu_lib().synth_fill(seed, layer, kind, expert, dist, p0, p1, offset, n, _OUT[out],
                         a.ctypes.data_as(ctypes.c_void_p))
    return a.reshape(shape)


def cpu_hc_in(w: Workload):
    return cpu_fill(w.seed, 0, HC_IN, 0, (w.rows, w.hc, w.hidden), 0, 0.0, 1.0, w.hc_dtype)


def attn_specs(w: Workload):
    """(kind, shape, dist, p0, p1, element type) of the attention sublayer's
    pending state that opens a layer at the within-layer boundary: the
    residual streams before attention N(0, 1), its post U(0, 2), its comb
    U(0, 0.5) (any matrix: the boundary does not assume a doubly stochastic
    one), its output N(0, 1)."""
    R, S, H = w.rows, w.hc, w.hidden
    return {
        "x": (ATTN_X, (R, S, H), 0, 0.0, 1.0, w.hc_dtype),
        "post": (ATTN_POST, (R, S), 1, 0.0, 2.0, "f32"),
        "comb": (ATTN_COMB, (R, S, S), 1, 0.0, 0.5, "f32"),
        "y": (ATTN_Y, (R, H), 0, 0.0, 1.0, w.hc_dtype),
    }


def cpu_attn_pending(w: Workload):
    return {k: cpu_fill(w.seed, 0, kind, 0, shape, dist, p0, p1, t)
            for k, (kind, shape, dist, p0, p1, t) in attn_specs(w).items()}


def cpu_dense(w: Workload, layer: int):
    out = {}
    for name, (kind, shape, dist, p0, p1, t) in tensor_specs(w, layer).items():
        out[name] = cpu_fill(w.seed, layer, kind, 0, shape, dist, p0, p1, t)
    return out


def cpu_expert(w: Workload, layer: int, slot: int):
    """One expert slot's three matrices in the workload's format:
    {name: (codes, scales or None)}, each [out][in] (MXFP4 codes [out][in/2])."""
    lib = cpu_lib()
    res = {}
    for name, (kind, rows, cols, std) in expert_specs(w).items():
        if w.w_dtype in ("f32", "bf16"):
            res[name] = (cpu_fill(w.seed, layer, kind, slot, (rows, cols), 0, 0.0, std, w.w_dtype), None)
        elif w.w_dtype == "fp8":
            q = np.empty((rows, cols), np.uint8)
            s = np.empty((rows, cols // 128), np.float32)
            lib.synth_fill_fp8(w.seed, layer, kind, slot, std, rows, cols,
                               q.ctypes.data_as(ctypes.c_void_p), s.ctypes.data_as(ctypes.c_void_p))
            res[name] = (q, s)
        else:
            q = np.empty((rows, cols // 2), np.uint8)
            e = np.empty((rows, cols // 32), np.uint8)
            lib.synth_fill_mxfp4(w.seed, layer, kind, slot, std, rows, cols, w.mx_spread,
                                 q.ctypes.data_as(ctypes.c_void_p), e.ctypes.data_as(ctypes.c_void_p))
            res[name] = (q, e)
    return res


def cpu_expert_f32(w: Workload, layer: int, slot: int):
    """The fp32 values a quantised expert was encoded from."""
    res = {}
    for name, (kind, rows, cols, std) in expert_specs(w).items():
        res[name] = cpu_fill(w.seed, layer, kind, slot, (rows, cols), 0, 0.0, std, "f32")
    return res


def quant_fp8(x: np.ndarray):
    x = np.ascontiguousarray(x, np.float32)
    rows, cols = x.shape
    q = np.empty((rows, cols), np.uint8)
    s = np.empty((rows, cols // 128), np.float32)
    cpu_lib().synth_quant_fp8(x.ctypes.data_as(ctypes.c_void_p), rows, cols,
                              q.ctypes.data_as(ctypes.c_void_p), s.ctypes.data_as(ctypes.c_void_p))
    return q, s


def quant_mxfp4(x: np.ndarray):
    x = np.ascontiguousarray(x, np.float32)
    rows, cols = x.shape
    q = np.empty((rows, cols // 2), np.uint8)
    e = np.empty((rows, cols // 32), np.uint8)
    cpu_lib().synth_quant_mxfp4(x.ctypes.data_as(ctypes.c_void_p), rows, cols,
                                q.ctypes.data_as(ctypes.c_void_p), e.ctypes.data_as(ctypes.c_void_p))
    return q, e


# --------------------------------------------------------------- device side --

def _torch_dtype(t):
    import torch
    return {"f32": torch.float32, "bf16": torch.bfloat16, "f64": torch.float64}[t]


def _stream():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"synth {what}: CUDA error {rc}")


def gpu_fill_(t, seed, layer, kind, expert, dist, p0, p1, out, offset=0):
    rc = gpu_lib().synth_gpu_fill(seed, layer, kind, expert, dist, p0, p1, offset, t.numel(), _OUT[out],
                                  ctypes.c_void_p(t.data_ptr()), _stream())
    _check(rc, "fill")
    return t


def gpu_hc_in(w: Workload, device="cuda"):
    import torch
    t = torch.empty((w.rows, w.hc, w.hidden), dtype=_torch_dtype(w.hc_dtype), device=device)
    return gpu_fill_(t, w.seed, 0, HC_IN, 0, 0, 0.0, 1.0, w.hc_dtype)


def gpu_attn_pending(w: Workload, device="cuda"):
    import torch
    out = {}
    for k, (kind, shape, dist, p0, p1, t) in attn_specs(w).items():
        x = torch.empty(shape, dtype=_torch_dtype(t), device=device)
        out[k] = gpu_fill_(x, w.seed, 0, kind, 0, dist, p0, p1, t)
    return out


def gpu_dense(w: Workload, layer: int, device="cuda"):
    import torch
    out = {}
    for name, (kind, shape, dist, p0, p1, t) in tensor_specs(w, layer).items():
        x = torch.empty(shape, dtype=_torch_dtype(t), device=device)
        out[name] = gpu_fill_(x, w.seed, layer, kind, 0, dist, p0, p1, t)
    return out


def gpu_experts(w: Workload, layer: int, device="cuda"):
    """All E+1 expert slots of one layer, stacked: {name: (codes, scales or
    None)} with codes [E+1][out][in] (MXFP4 [E+1][out][in/2])."""
    import torch
    lib = gpu_lib()
    E1 = w.n_routed + 1
    res = {}
    for name, (kind, rows, cols, std) in expert_specs(w).items():
        if w.w_dtype in ("f32", "bf16"):
            q = torch.empty((E1, rows, cols), dtype=_torch_dtype(w.w_dtype), device=device)
            for e in range(E1):
                gpu_fill_(q[e], w.seed, layer, kind, e, 0, 0.0, std, w.w_dtype)
            res[name] = (q, None)
        elif w.w_dtype == "fp8":
            q = torch.empty((E1, rows, cols), dtype=torch.uint8, device=device)
            s = torch.empty((E1, rows, cols // 128), dtype=torch.float32, device=device)
            for e in range(E1):
                _check(lib.synth_gpu_fill_fp8(w.seed, layer, kind, e, std, rows, cols,
                                              ctypes.c_void_p(q[e].data_ptr()),
                                              ctypes.c_void_p(s[e].data_ptr()), _stream()), "fp8")
            res[name] = (q, s)
        else:
            q = torch.empty((E1, rows, cols // 2), dtype=torch.uint8, device=device)
            s = torch.empty((E1, rows, cols // 32), dtype=torch.uint8, device=device)
            for e in range(E1):
                _check(lib.synth_gpu_fill_mxfp4(w.seed, layer, kind, e, std, rows, cols, w.mx_spread,
                                                ctypes.c_void_p(q[e].data_ptr()),
                                                ctypes.c_void_p(s[e].data_ptr()), _stream()), "mxfp4")
            res[name] = (q, s)
    return res
