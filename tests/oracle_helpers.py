"""Host-side helpers shared by the oracle pins and the GPU parity tests: build
oracle inputs from the seeded generator, with optional overrides."""

import numpy as np

from oracle import oracle as O
from synth import configs as C
from synth import synth as S


def tiny(**kw):
    """A tiny workload for brute force (H=32, E=6, k=2, I=16)."""
    base = C.TINY_FP32.with_(name="brute", hidden=32, n_routed=6, top_k=2, inter=16, rows=3, seed=11)
    return base.with_(**kw)


def all_experts(wl, layer=0):
    return {e: S.cpu_expert(wl, layer, e) for e in range(wl.n_routed + 1)}


def touched_experts(wl, dense, hc_in, layer=0):
    lw = O.LayerWeights(wl, dense, {})
    taps = O.route(wl, lw, hc_in)
    slots = sorted(set(int(x) for x in taps.idx.ravel()) | {wl.n_routed})
    return {e: S.cpu_expert(wl, layer, e) for e in slots}, taps


def layer_inputs(wl, layer=0, experts="touched", hc_in=None, dense=None):
    hc_in = S.cpu_hc_in(wl) if hc_in is None else hc_in
    dense = S.cpu_dense(wl, layer) if dense is None else dense
    if experts == "all":
        ex = all_experts(wl, layer)
    elif experts == "touched":
        ex, _ = touched_experts(wl, dense, hc_in, layer)
    else:
        ex = experts
    return hc_in, dense, ex


def zero_expert(wl):
    z = {}
    for nm, (_, rows, cols, _) in S.expert_specs(wl).items():
        assert wl.w_dtype == "f32"
        z[nm] = (np.zeros((rows, cols), np.float32), None)
    return z


def f32_of(wl, mats):
    """Decode one expert's {name: (codes, scales)} to float64 [out][in]."""
    import torch
    out = {}
    for nm, (q, s) in mats.items():
        if wl.w_dtype == "f32":
            out[nm] = q.astype(np.float64)
        elif wl.w_dtype == "bf16":
            out[nm] = (q.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        elif wl.w_dtype == "fp8":
            v = torch.from_numpy(q.copy()).view(torch.float8_e4m3fn).double().numpy()
            out[nm] = v * np.repeat(s.astype(np.float64), 128, axis=1)
        else:
            tab = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0])
            lo = tab[q & 15]
            hi = tab[q >> 4]
            v = np.stack([lo, hi], axis=-1).reshape(q.shape[0], q.shape[1] * 2)
            sc = torch.from_numpy(s.copy()).view(torch.float8_e8m0fnu).double().numpy()
            out[nm] = v * np.repeat(sc, 32, axis=1)
    return out
