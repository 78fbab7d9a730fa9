"""Thin ctypes binding of libmonoffn (include/mono_ffn.h).

Argument marshalling only: device pointers and the current CUDA stream go in,
error codes come out.  Every step of the layer runs in the library's CUDA
kernels; there is no Python or CPU fallback — loading fails loudly when the
shared library is missing.
"""

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(PKG, "libmonoffn.so")

F32, BF16, FP8E4M3_B128, MXFP4 = 0, 1, 2, 3
DTYPE = {"f32": F32, "bf16": BF16, "fp8": FP8E4M3_B128, "mxfp4": MXFP4}

STAGE = {"MIX": 1, "LOGITS": 2, "LISTS": 3, "ACT": 4, "RING": 5, "Y": 6, "COLLAPSE": 7}

ERRORS = {0: "OK", -1: "INVALID_ARG", -2: "UNSUPPORTED_ARCH", -3: "NOT_CORESIDENT", -4: "OOM",
          -5: "NOT_PACKED", -6: "CUDA", -7: "DEVICE_TIMEOUT", -8: "DEVICE_ABORTED"}

SYMBOLS = ["mono_ffn_plan", "mono_ffn_pack_weights", "mono_ffn_step", "mono_ffn_step_host", "mono_ffn_set_taps",
           "mono_ffn_query_error", "mono_ffn_get_info", "mono_ffn_debug_skip_arrival", "mono_ffn_last_error",
           "mono_ffn_destroy", "mono_ffn_abi_version", "mono_ffn_set_trace", "mono_ffn_route_noalloc",
           "mono_ffn_debug_jitter", "mono_ffn_step_pending", "mono_ffn_step_padded"]


class Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("hidden", "hc", "n_routed", "top_k", "inter", "max_rows", "n_layers",
                                            "hc_dtype", "norm_dtype", "expert_dtype", "round_bf16")] + \
               [(n, ctypes.c_float) for n in ("rms_eps", "pre_eps", "post_mult", "route_scale", "denom_clamp")] + \
               [("sinkhorn_iters", ctypes.c_int), ("wait_timeout_us", ctypes.c_uint), ("device", ctypes.c_int),
                ("grid", ctypes.c_int), ("dense", ctypes.c_int), ("act_mx8", ctypes.c_int)]


class LayerWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("mix_w", "norm_w", "router_w", "router_bias", "w_gate", "w_up", "w_down",
                                               "s_gate", "s_up", "s_down")]


class TapsStruct(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("mix", "pre", "post", "comb", "n", "logits", "idx", "w", "y", "x")]


class Status(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("code", "stage", "cta", "layer")]


class Info(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("grid", "threads", "smem_bytes", "ring_stages", "ring_slot_bytes")] + \
               [(n, ctypes.c_int64) for n in ("expert_bytes", "dense_bytes", "packed_bytes", "scratch_bytes")]


class MonoError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(SO):
            raise RuntimeError(f"{SO} is missing: build it with __graft_entry__.build() (nvcc, sm_100a)")
        L = ctypes.CDLL(SO)
        vp, i32 = ctypes.c_void_p, ctypes.c_int
        L.mono_ffn_plan.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(vp)]
        L.mono_ffn_pack_weights.argtypes = [vp, i32, ctypes.POINTER(LayerWeights), vp]
        L.mono_ffn_step.argtypes = [vp, i32, vp, vp, vp]
        L.mono_ffn_step_host.argtypes = [vp, i32, vp, vp, vp]
        L.mono_ffn_step_pending.argtypes = [vp, i32, vp, vp, vp, vp, vp, vp]
        L.mono_ffn_step_padded.argtypes = [vp, i32, vp, vp, vp, vp]
        L.mono_ffn_set_taps.argtypes = [vp, i32, ctypes.POINTER(TapsStruct)]
        L.mono_ffn_query_error.argtypes = [vp, ctypes.POINTER(Status)]
        L.mono_ffn_get_info.argtypes = [vp, ctypes.POINTER(Info)]
        L.mono_ffn_debug_skip_arrival.argtypes = [vp, i32, i32]
        L.mono_ffn_debug_jitter.argtypes = [vp, ctypes.c_uint]
        L.mono_ffn_set_trace.argtypes = [vp, vp]
        L.mono_ffn_last_error.argtypes = [vp]
        L.mono_ffn_last_error.restype = ctypes.c_char_p
        L.mono_ffn_destroy.argtypes = [vp]
        L.mono_ffn_destroy.restype = None
        f32 = ctypes.c_float
        L.mono_ffn_route_noalloc.argtypes = [i32, i32, i32, i32, vp, i32, vp, vp, f32, f32, vp, vp, vp]
        for f in ("mono_ffn_plan", "mono_ffn_pack_weights", "mono_ffn_step", "mono_ffn_step_host", "mono_ffn_set_taps",
                  "mono_ffn_query_error", "mono_ffn_get_info", "mono_ffn_debug_skip_arrival", "mono_ffn_abi_version",
                  "mono_ffn_set_trace", "mono_ffn_route_noalloc", "mono_ffn_debug_jitter", "mono_ffn_step_pending",
                  "mono_ffn_step_padded"):
            getattr(L, f).restype = i32
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class Plan:
    """One plan: packed weights for n_layers layers plus scratch, on one device."""

    def __init__(self, hidden, n_routed, top_k, inter, max_rows, n_layers=1, hc_dtype="bf16", norm_dtype="bf16",
                 expert_dtype="bf16", round_bf16=True, rms_eps=1e-6, pre_eps=1e-6, post_mult=2.0, route_scale=2.5,
                 denom_clamp=1e-20, sinkhorn_iters=20, wait_timeout_us=0, device=0, grid=0, dense=False,
                 act_mx8=False):
        self._lib = lib()
        self.cfg = Config(hidden=hidden, hc=4, n_routed=n_routed, top_k=top_k, inter=inter, max_rows=max_rows,
                          n_layers=n_layers, hc_dtype=DTYPE[hc_dtype], norm_dtype=DTYPE[norm_dtype],
                          expert_dtype=DTYPE[expert_dtype], round_bf16=int(round_bf16), rms_eps=rms_eps,
                          pre_eps=pre_eps, post_mult=post_mult, route_scale=route_scale, denom_clamp=denom_clamp,
                          sinkhorn_iters=sinkhorn_iters, wait_timeout_us=wait_timeout_us, device=device, grid=grid,
                          dense=int(dense), act_mx8=int(act_mx8))
        h = ctypes.c_void_p()
        rc = self._lib.mono_ffn_plan(ctypes.byref(self.cfg), ctypes.byref(h))
        if rc != 0:
            raise MonoError(rc, self._lib.mono_ffn_last_error(None).decode())
        self.handle = h
        self._taps = {}

    @classmethod
    def for_workload(cls, wl, **kw):
        return cls(wl.hidden, wl.n_routed, wl.top_k, wl.inter, max_rows=wl.rows, n_layers=wl.n_layers,
                   hc_dtype=wl.hc_dtype, norm_dtype=wl.norm_dtype, expert_dtype=wl.w_dtype,
                   round_bf16=wl.round_bf16, rms_eps=wl.rms_eps, pre_eps=wl.pre_eps, post_mult=wl.post_mult,
                   route_scale=wl.route_scale, denom_clamp=wl.denom_clamp, sinkhorn_iters=wl.sinkhorn_iters,
                   dense=getattr(wl, "dense", False), act_mx8=getattr(wl, "act_mx8", False), **kw)

    def _check(self, rc):
        if rc != 0:
            raise MonoError(rc, self._lib.mono_ffn_last_error(self.handle).decode())

    def pack(self, layer, mix_w, norm_w, router_w, router_bias, gate, up, down, s_gate=None, s_up=None, s_down=None,
             stream=None):
        w = LayerWeights(*[_ptr(t) for t in (mix_w, norm_w, router_w, router_bias, gate, up, down, s_gate, s_up,
                                             s_down)])
        self._check(self._lib.mono_ffn_pack_weights(self.handle, layer, ctypes.byref(w), _stream(stream)))

    def step(self, rows, hc_in, hc_out, stream=None):
        self._check(self._lib.mono_ffn_step(self.handle, rows, _ptr(hc_in), _ptr(hc_out), _stream(stream)))

    def step_padded(self, width, row_slot, hc_in, hc_out, stream=None):
        """A step at a fixed width: row_slot int32 [width] CUDA tensor, rows
        with a slot below zero are padding (input ignored, output untouched)."""
        self._check(self._lib.mono_ffn_step_padded(self.handle, width, _ptr(row_slot), _ptr(hc_in), _ptr(hc_out),
                                                   _stream(stream)))

    def step_pending(self, rows, x_attn, attn_post, attn_comb, y_attn, hc_out, stream=None):
        """A step opened by the attention sublayer's pending expand: x_attn
        [rows][4][H] and y_attn [rows][H] in the hc dtype, attn_post [rows][4]
        and attn_comb [rows][4][4] fp32, all CUDA tensors."""
        self._check(self._lib.mono_ffn_step_pending(self.handle, rows, _ptr(x_attn), _ptr(attn_post), _ptr(attn_comb),
                                                    _ptr(y_attn), _ptr(hc_out), _stream(stream)))

    def step_host(self, rows, hc_in, hc_out, stream=None):
        """hc_in / hc_out are CPU tensors (pinned for asynchronous copies)."""
        self._check(self._lib.mono_ffn_step_host(self.handle, rows, _ptr(hc_in), _ptr(hc_out), _stream(stream)))

    def set_taps(self, layer, **taps):
        """Register device tensors for intermediate values (keys of TapsStruct)."""
        t = TapsStruct(**{k: (v.data_ptr() if v is not None else None) for k, v in taps.items()})
        self._taps[layer] = taps
        self._check(self._lib.mono_ffn_set_taps(self.handle, layer, ctypes.byref(t)))

    def clear_taps(self, layer):
        self._taps.pop(layer, None)
        self._check(self._lib.mono_ffn_set_taps(self.handle, layer, None))

    def query_error(self):
        st = Status()
        rc = self._lib.mono_ffn_query_error(self.handle, ctypes.byref(st))
        return rc, st

    def set_trace(self, buf):
        """buf: int64 device tensor of n_layers * grid * 32 entries, or None."""
        self._check(self._lib.mono_ffn_set_trace(self.handle, _ptr(buf)))

    def debug_skip_arrival(self, cta, stage=STAGE["LOGITS"]):
        """Tests: CTA `cta` (-1: none) withholds its arrival at `stage`."""
        self._check(self._lib.mono_ffn_debug_skip_arrival(self.handle, cta, stage))

    def debug_jitter(self, max_ns):
        """Tests: publishing threads sleep hash(CTA, epoch, point) % max_ns first."""
        self._check(self._lib.mono_ffn_debug_jitter(self.handle, max_ns))

    def info(self):
        inf = Info()
        self._check(self._lib.mono_ffn_get_info(self.handle, ctypes.byref(inf)))
        return {f: getattr(inf, f) for f, _ in Info._fields_}

    def close(self):
        if getattr(self, "handle", None):
            self._lib.mono_ffn_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def route_noalloc(n, router_w, router_bias, top_k, route_scale, denom_clamp, idx, w, stream=None):
    """mono_ffn_route_noalloc: router select with no plan and no allocation.
    n [rows][hidden] (bf16 or fp32), router_w [hidden][n_routed] fp32,
    router_bias [n_routed] fp32, idx [rows][top_k] int32 and w [rows][top_k]
    fp32 written in place; all CUDA tensors on the current device."""
    import torch
    if n.dim() != 2 or router_w.dim() != 2 or router_bias.dim() != 1:
        raise ValueError("route_noalloc: n [rows][hidden], router_w [hidden][n_routed], router_bias [n_routed]")
    rows, hidden = n.shape
    n_routed = router_w.shape[1]
    why = []
    if n.dtype not in (torch.bfloat16, torch.float32):
        why.append("n must be bf16 or fp32")
    if router_w.dtype != torch.float32 or router_bias.dtype != torch.float32 or w.dtype != torch.float32:
        why.append("router_w, router_bias and w must be fp32")
    if idx.dtype != torch.int32:
        why.append("idx must be int32")
    if router_w.shape[0] != hidden or router_bias.numel() != n_routed:
        why.append("router_w must be [hidden][n_routed] and router_bias [n_routed]")
    if tuple(idx.shape) != (rows, top_k) or tuple(w.shape) != (rows, top_k):
        why.append("idx and w must be [rows][top_k]")
    ts = (n, router_w, router_bias, idx, w)
    if not all(t.is_contiguous() for t in ts):
        why.append("every tensor must be contiguous")
    if not all(t.is_cuda for t in ts) or any(t.device.index != torch.cuda.current_device() for t in ts):
        why.append("every tensor must be on the current CUDA device")
    if why:
        raise ValueError("route_noalloc: " + "; ".join(why))
    rc = lib().mono_ffn_route_noalloc(rows, hidden, n_routed, top_k, _ptr(n), 1 if n.dtype == torch.bfloat16 else 0,
                                      _ptr(router_w), _ptr(router_bias), route_scale, denom_clamp, _ptr(idx), _ptr(w),
                                      _stream(stream))
    if rc != 0:
        msg = lib().mono_ffn_last_error(None)
        raise RuntimeError(f"mono_ffn_route_noalloc: {ERRORS.get(rc, rc)}: {msg.decode() if msg else ''}")
