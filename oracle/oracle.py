"""ctypes front end of the CPU oracle (``libmono_oracle.so``) — TEST
INFRASTRUCTURE ONLY.  Tests, the smoke check and the benchmark's CPU-baseline
leg are the only callers; the product path never imports this module.
"""

import ctypes
import hashlib
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(HERE, "libmono_oracle.so")
SRC = os.path.join(HERE, "mono_oracle.c")
HDR = os.path.join(HERE, "mono_oracle.h")

F32, BF16, FP8, MXFP4 = 0, 1, 2, 3
_DT = {"f32": F32, "bf16": BF16, "fp8": FP8, "mxfp4": MXFP4}


def build():
    """Compile the oracle unless its stamp file records the SHA-256 of the
    sources and the compile command."""
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared", "-o", SO, SRC, "-lm"]
    h = hashlib.sha256()
    for s in (SRC, HDR):
        with open(s, "rb") as f:
            h.update(f.read())
    h.update(" ".join(cmd).encode())
    stamp = SO + ".sha256"
    if os.path.exists(SO) and os.path.exists(stamp) and open(stamp).read().strip() == h.hexdigest():
        return
    if os.path.exists(stamp):
        os.unlink(stamp)
    subprocess.check_call(cmd)
    with open(stamp, "w") as f:
        f.write(h.hexdigest() + "\n")


class Cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("hidden", "hc", "n_routed", "top_k", "inter", "rows", "hc_dtype",
                                            "norm_dtype", "w_dtype", "round_bf16", "sinkhorn_iters")] + \
               [(n, ctypes.c_double) for n in ("rms_eps", "pre_eps", "post_mult", "route_scale", "denom_clamp")] + \
               [("dense", ctypes.c_int), ("act_mx8", ctypes.c_int)]


class Weights(ctypes.Structure):
    _fields_ = [("mix_w", ctypes.c_void_p), ("norm_w", ctypes.c_void_p), ("router_w", ctypes.c_void_p),
                ("router_bias", ctypes.c_void_p)] + \
               [(n, ctypes.POINTER(ctypes.c_void_p)) for n in ("w_gate", "w_up", "w_down", "s_gate", "s_up",
                                                                "s_down")]


class Taps(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("rho", "mix", "pre", "post", "comb", "a", "n", "logits", "score",
                                               "sel", "idx", "w", "y")]


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(SO)
        vp = ctypes.c_void_p
        L.orc_layer.argtypes = [ctypes.POINTER(Cfg), ctypes.POINTER(Weights), vp, vp, ctypes.POINTER(Taps)]
        L.orc_route.argtypes = [ctypes.POINTER(Cfg), ctypes.POINTER(Weights), vp, ctypes.POINTER(Taps)]
        L.orc_chain.argtypes = [ctypes.POINTER(Cfg), ctypes.c_int, ctypes.POINTER(Weights), vp, vp, ctypes.c_int]
        L.orc_layer_pending.argtypes = [ctypes.POINTER(Cfg), ctypes.POINTER(Weights), vp, vp, vp, vp, vp, vp,
                                        ctypes.POINTER(Taps)]
        L.orc_expand.argtypes = [ctypes.POINTER(Cfg), vp, vp, vp, vp, vp]
        L.orc_sinkhorn.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp]
        L.orc_topk.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp]
        L.orc_dec_bf16.argtypes = [ctypes.c_uint16]
        L.orc_dec_bf16.restype = ctypes.c_double
        L.orc_dec_e4m3.argtypes = [ctypes.c_uint8]
        L.orc_dec_e4m3.restype = ctypes.c_double
        L.orc_dec_e2m1.argtypes = [ctypes.c_uint8]
        L.orc_dec_e2m1.restype = ctypes.c_double
        L.orc_dec_e8m0.argtypes = [ctypes.c_uint8]
        L.orc_dec_e8m0.restype = ctypes.c_double
        L.orc_round_bf16.argtypes = [ctypes.c_double]
        L.orc_round_bf16.restype = ctypes.c_uint16
        L.orc_quant_fp8.argtypes = [vp, ctypes.c_int64, ctypes.c_int64, vp, vp]
        L.orc_quant_mxfp4.argtypes = [vp, ctypes.c_int64, ctypes.c_int64, vp, vp]
        L.orc_quant_mx8.argtypes = [vp, ctypes.c_int64, vp, vp, vp]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def make_cfg(wl, rows=None):
    return Cfg(hidden=wl.hidden, hc=wl.hc, n_routed=wl.n_routed, top_k=wl.top_k, inter=wl.inter,
               rows=wl.rows if rows is None else rows, hc_dtype=_DT[wl.hc_dtype], norm_dtype=_DT[wl.norm_dtype],
               w_dtype=_DT[wl.w_dtype], round_bf16=int(wl.round_bf16), sinkhorn_iters=wl.sinkhorn_iters,
               rms_eps=wl.rms_eps, pre_eps=wl.pre_eps, post_mult=wl.post_mult, route_scale=wl.route_scale,
               denom_clamp=wl.denom_clamp, dense=int(wl.dense), act_mx8=int(wl.act_mx8))


class LayerWeights:
    """Host arrays of one layer in the logical layouts of mono_oracle.h.
    ``experts`` maps slot -> {"gate"|"up"|"down": (codes, scales or None)};
    slots that are absent are passed as NULL."""

    def __init__(self, wl, dense, experts):
        self.wl = wl
        self.keep = []
        E1 = wl.n_routed + 1
        self.mix_w = np.ascontiguousarray(dense["mix_w"], np.float32)
        self.norm_w = np.ascontiguousarray(dense["norm_w"])
        self.router_w = np.ascontiguousarray(dense["router_w"], np.float32)
        self.router_bias = np.ascontiguousarray(dense["router_bias"], np.float32)
        arrs = {}
        for nm in ("gate", "up", "down"):
            codes = (ctypes.c_void_p * E1)()
            scales = (ctypes.c_void_p * E1)()
            for e, mats in experts.items():
                q, s = mats[nm]
                q = np.ascontiguousarray(q)
                self.keep.append(q)
                codes[e] = q.ctypes.data
                if s is not None:
                    s = np.ascontiguousarray(s)
                    self.keep.append(s)
                    scales[e] = s.ctypes.data
            arrs[nm] = (codes, scales)
        self.arrs = arrs
        self.struct = Weights(
            mix_w=self.mix_w.ctypes.data, norm_w=self.norm_w.ctypes.data, router_w=self.router_w.ctypes.data,
            router_bias=self.router_bias.ctypes.data,
            w_gate=ctypes.cast(arrs["gate"][0], ctypes.POINTER(ctypes.c_void_p)),
            w_up=ctypes.cast(arrs["up"][0], ctypes.POINTER(ctypes.c_void_p)),
            w_down=ctypes.cast(arrs["down"][0], ctypes.POINTER(ctypes.c_void_p)),
            s_gate=ctypes.cast(arrs["gate"][1], ctypes.POINTER(ctypes.c_void_p)),
            s_up=ctypes.cast(arrs["up"][1], ctypes.POINTER(ctypes.c_void_p)),
            s_down=ctypes.cast(arrs["down"][1], ctypes.POINTER(ctypes.c_void_p)))


class TapSet:
    def __init__(self, wl, rows):
        R, S, H, E, K, M = rows, wl.hc, wl.hidden, wl.n_routed, wl.top_k, wl.mix_cols
        self.rho = np.zeros(R)
        self.mix = np.zeros((R, M))
        self.pre = np.zeros((R, S))
        self.post = np.zeros((R, S))
        self.comb = np.zeros((R, S, S))
        self.a = np.zeros((R, H))
        self.n = np.zeros((R, H))
        self.logits = np.zeros((R, E), np.float32)
        self.score = np.zeros((R, E), np.float32)
        self.sel = np.zeros((R, E), np.float32)
        self.idx = np.zeros((R, K), np.int32)
        self.w = np.zeros((R, K), np.float32)
        self.y = np.zeros((R, H))
        self.struct = Taps(**{f: getattr(self, f).ctypes.data for f, _ in Taps._fields_})


def _hc_buf(wl, rows):
    dt = np.uint16 if wl.hc_dtype == "bf16" else np.float32
    return np.zeros((rows, wl.hc, wl.hidden), dt)


def route(wl, lw: LayerWeights, hc_in):
    """Steps up to the routing decision; returns the taps."""
    rows = hc_in.shape[0]
    cfg = make_cfg(wl, rows)
    taps = TapSet(wl, rows)
    hc_in = np.ascontiguousarray(hc_in)
    rc = lib().orc_route(ctypes.byref(cfg), ctypes.byref(lw.struct), _p(hc_in), ctypes.byref(taps.struct))
    if rc != 0:
        raise RuntimeError(f"orc_route failed: {rc}")
    return taps


def layer(wl, lw: LayerWeights, hc_in):
    """One layer: returns (hc_out raw array, taps)."""
    rows = hc_in.shape[0]
    cfg = make_cfg(wl, rows)
    taps = TapSet(wl, rows)
    hc_in = np.ascontiguousarray(hc_in)
    out = _hc_buf(wl, rows)
    rc = lib().orc_layer(ctypes.byref(cfg), ctypes.byref(lw.struct), _p(hc_in), _p(out), ctypes.byref(taps.struct))
    if rc != 0:
        raise RuntimeError(f"orc_layer failed: {rc}")
    return out, taps


def layer_pending(wl, lw: LayerWeights, x_attn, attn_post, attn_comb, y_attn):
    """One layer opened by the attention sublayer's pending expand: returns
    (hc_out raw array, materialised X raw array, taps)."""
    rows = x_attn.shape[0]
    cfg = make_cfg(wl, rows)
    taps = TapSet(wl, rows)
    x_attn = np.ascontiguousarray(x_attn)
    y_attn = np.ascontiguousarray(y_attn)
    post = np.ascontiguousarray(attn_post, np.float32)
    comb = np.ascontiguousarray(attn_comb, np.float32)
    out = _hc_buf(wl, rows)
    x = _hc_buf(wl, rows)
    rc = lib().orc_layer_pending(ctypes.byref(cfg), ctypes.byref(lw.struct), _p(x_attn), _p(post), _p(comb),
                                 _p(y_attn), _p(out), _p(x), ctypes.byref(taps.struct))
    if rc != 0:
        raise RuntimeError(f"orc_layer_pending failed: {rc}")
    return out, x, taps


def expand(wl, x_in, post, comb, y):
    """x_out_i = sum_j comb_ij x_in_j + post_i y per row, in the hc element type."""
    rows = x_in.shape[0]
    cfg = make_cfg(wl, rows)
    out = _hc_buf(wl, rows)
    rc = lib().orc_expand(ctypes.byref(cfg), _p(np.ascontiguousarray(x_in)), _p(np.ascontiguousarray(post, np.float32)),
                          _p(np.ascontiguousarray(comb, np.float32)), _p(np.ascontiguousarray(y)), _p(out))
    if rc != 0:
        raise RuntimeError(f"orc_expand failed: {rc}")
    return out


def chain(wl, lws, hc_in, deferred):
    rows = hc_in.shape[0]
    cfg = make_cfg(wl, rows)
    arr = (Weights * len(lws))(*[lw.struct for lw in lws])
    hc_in = np.ascontiguousarray(hc_in)
    out = _hc_buf(wl, rows)
    rc = lib().orc_chain(ctypes.byref(cfg), len(lws), arr, _p(hc_in), _p(out), int(deferred))
    if rc != 0:
        raise RuntimeError(f"orc_chain failed: {rc}")
    return out


def sinkhorn(logits, iters):
    L = np.ascontiguousarray(logits, np.float64)
    s = L.shape[0]
    C = np.zeros_like(L)
    lib().orc_sinkhorn(_p(L), s, iters, _p(C))
    return C


def topk(sel, k):
    sel = np.ascontiguousarray(sel, np.float32)
    idx = np.zeros(k, np.int32)
    lib().orc_topk(_p(sel), sel.shape[0], k, _p(idx))
    return idx


def quant_fp8(x):
    x = np.ascontiguousarray(x, np.float32)
    q = np.empty(x.shape, np.uint8)
    s = np.empty((x.shape[0], x.shape[1] // 128), np.float32)
    lib().orc_quant_fp8(_p(x), x.shape[0], x.shape[1], _p(q), _p(s))
    return q, s


def quant_mxfp4(x):
    x = np.ascontiguousarray(x, np.float32)
    q = np.empty((x.shape[0], x.shape[1] // 2), np.uint8)
    e = np.empty((x.shape[0], x.shape[1] // 32), np.uint8)
    lib().orc_quant_mxfp4(_p(x), x.shape[0], x.shape[1], _p(q), _p(e))
    return q, e


def quant_mx8(x):
    """MXFP8 (e4m3, e8m0 per 32) of a float64 vector: (values, codes, scales)."""
    x = np.ascontiguousarray(x, np.float64)
    out = np.empty_like(x)
    q = np.empty(x.shape, np.uint8)
    e = np.empty(x.size // 32, np.uint8)
    lib().orc_quant_mx8(_p(x), x.size, _p(out), _p(q), _p(e))
    return out, q, e


def decode_hc(wl, raw):
    """Raw hc buffer -> float64 values."""
    if wl.hc_dtype == "bf16":
        return (raw.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return raw.astype(np.float64)
