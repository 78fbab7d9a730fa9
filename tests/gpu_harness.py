"""GPU-side helpers of the parity tests: inputs from the seeded generator's
device build, one plan per workload, taps for the intermediate values, and
the comparison rules (routing exemption at near ties, tolerances)."""

import numpy as np

from oracle import oracle as O
from synth import synth as S
from tests.oracle_helpers import layer_inputs

# tolerances of the target layer's numerics
FP32_MAX_ABS = 1e-4
BF16_REL_L2 = 2e-2
BF16_MAX_ABS = 5e-2
TIE_REL = 1e-5


class LayerRun:
    """Generate a workload's inputs on the device, pack, and run steps."""

    def __init__(self, wl, dense_override=None, hc_in=None, **plan_kw):
        import torch

        from moe_decode_layer_sm_b200 import Plan
        self.wl = wl
        self.plan = Plan.for_workload(wl, **plan_kw)
        for l in range(wl.n_layers):
            d = S.gpu_dense(wl, l)
            if dense_override:
                for k, v in dense_override(l).items():
                    d[k] = torch.from_numpy(np.ascontiguousarray(v)).cuda()
            ex = S.gpu_experts(wl, l)
            self.plan.pack(l, d["mix_w"], d["norm_w"], d["router_w"], d["router_bias"], ex["gate"][0], ex["up"][0],
                           ex["down"][0], ex["gate"][1], ex["up"][1], ex["down"][1])
            del ex
        torch.cuda.synchronize()
        self.hc = S.gpu_hc_in(wl) if hc_in is None else hc_in
        self.out = torch.empty_like(self.hc)
        self.taps = []
        R, H, E, K = wl.rows, wl.hidden, wl.n_routed, wl.top_k
        for l in range(wl.n_layers):
            t = dict(mix=torch.zeros(R, 24, device="cuda"), pre=torch.zeros(R, 4, device="cuda"),
                     post=torch.zeros(R, 4, device="cuda"), comb=torch.zeros(R, 16, device="cuda"),
                     n=torch.zeros(R, H, device="cuda"), logits=torch.zeros(R, E, device="cuda"),
                     idx=torch.full((R, K), -1, dtype=torch.int32, device="cuda"),
                     w=torch.zeros(R, K, device="cuda"), y=torch.zeros(R, H, device="cuda"),
                     x=torch.zeros(R, 4, H, device="cuda"))
            self.plan.set_taps(l, **t)
            self.taps.append(t)

    def step(self, rows=None):
        import torch
        rows = self.wl.rows if rows is None else rows
        self.plan.step(rows, self.hc, self.out)
        rc, st = self.plan.query_error()
        assert rc == 0, f"device error {rc} at stage {st.stage} cta {st.cta} layer {st.layer}"
        torch.cuda.synchronize()
        return self.out_host()

    def out_host(self):
        import torch
        if self.wl.hc_dtype == "bf16":
            return self.out.float().double().cpu().numpy()
        return self.out.double().cpu().numpy()

    def tap(self, l, name):
        return self.taps[l][name].cpu().numpy()

    def close(self):
        self.plan.close()


def raw_hc(wl, x):
    """fp32 values that are exact in the hc element type -> the raw host array."""
    x = np.ascontiguousarray(x, np.float32)
    if wl.hc_dtype == "bf16":
        return (x.view(np.uint32) >> 16).astype(np.uint16)
    return x


def oracle_rows(wl, rows_sel, layer=0, hc_in=None, dense=None):
    """Oracle for the selected rows of one layer (inputs from the host build)."""
    hc = S.cpu_hc_in(wl) if hc_in is None else hc_in
    hc = hc[rows_sel]
    hc, dense, ex = layer_inputs(wl.with_(rows=len(rows_sel)), layer=layer, hc_in=hc, dense=dense)
    out, taps = O.layer(wl.with_(rows=len(rows_sel)), O.LayerWeights(wl, dense, ex), hc)
    return O.decode_hc(wl, out), taps


def routing_ok(gpu_idx, orc_idx, orc_sel, k):
    """Expert indices and order bit-exact, except where the oracle's k-th and
    (k+1)-th (or two adjacent selected) selection scores differ by less than
    1e-5 relative.  Returns (ok, exempted)."""
    if np.array_equal(gpu_idx, orc_idx):
        return True, False
    order = np.argsort(-orc_sel.astype(np.float64), kind="stable")
    s = orc_sel.astype(np.float64)

    def near(a, b):
        return abs(s[a] - s[b]) <= TIE_REL * max(abs(s[a]), abs(s[b]))

    # boundary exemption: the (k+1)-th may replace the k-th
    if k < len(order) and near(order[k - 1], order[k]):
        alt = orc_idx.copy()
        alt[k - 1] = order[k]
        if np.array_equal(gpu_idx, alt):
            return True, True
    # adjacent swaps of near-equal selected entries
    g = list(gpu_idx)
    o = list(orc_idx)
    if sorted(g) == sorted(o):
        for j in range(k):
            if g[j] != o[j]:
                if not near(g[j], o[j]):
                    return False, False
        return True, True
    return False, False


def bf16_ulp(x):
    """Spacing of bf16 values at |x| (8 significant bits)."""
    a = np.maximum(np.abs(np.asarray(x, np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def compare_out(wl, got, want, what="hc_out"):
    """One layer's result against the oracle's on the same inputs.  fp32
    configurations: max-abs 1e-4.  bf16 / FP8 / MXFP4: rel-L2 2e-2 and max-abs
    5e-2, where an element may also differ by one bf16 spacing of the
    oracle's value: both sides round the same quantity to bf16 last, and at
    |x| >= 8 one spacing (0.0625) already exceeds 5e-2."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    err = np.abs(got - want)
    if err.size == 0:
        return 0.0
    if wl.hc_dtype == "f32" and not wl.round_bf16:
        assert err.max() <= FP32_MAX_ABS, f"{what}: max-abs {err.max():.3e}"
    else:
        rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
        assert rel <= BF16_REL_L2, f"{what}: rel-L2 {rel:.3e}"
        bad = err > np.maximum(BF16_MAX_ABS, bf16_ulp(want) * 1.0000001)
        assert not bad.any(), f"{what}: max-abs {err.max():.3e} at |x| = {np.abs(want[bad]).max():.3e}"
    return float(err.max())


def compare_rel_l2(got, want, what):
    """Relative L2 difference within 2e-2 (the bf16 configurations' bound)."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    assert rel <= BF16_REL_L2, f"{what}: rel-L2 {rel:.3e}"
    return float(rel)


def near_tie(sel, k):
    """Where the oracle's selection values of one row leave the canonical
    top-k open to rounding: the k-th and (k+1)-th, or two adjacent selected
    entries, within 1e-5 relative.  Returns a description, or None."""
    s = np.asarray(sel, np.float64)
    order = np.argsort(-s, kind="stable")
    for j in range(min(k, len(order) - 1)):
        a, b = order[j], order[j + 1]
        if abs(s[a] - s[b]) <= TIE_REL * max(abs(s[a]), abs(s[b])):
            return f"selection values of experts {a} and {b} (ranks {j + 1}, {j + 2}) within 1e-5 relative"
    return None


def select_weights(wl, logits, idx, bias):
    """Router weights recomputed in float64 from given fp32 logits and a
    given selection: score = sqrt(softplus), w = score / max(sum, clamp) * scale."""
    lg = np.asarray(logits, np.float64)
    sc = np.sqrt(np.logaddexp(0.0, lg))
    out = np.zeros(idx.shape)
    for r in range(idx.shape[0]):
        s = sc[r, idx[r]]
        out[r] = s / max(s.sum(), wl.denom_clamp) * wl.route_scale
    return out


LOGIT_TOL = 1e-5


def check_logits(run, layer, t, rows, what=""):
    """The router logits tap against the oracle's fp32 logits on the rows
    whose n (the matvec's input) equals the oracle's bit for bit: both sides
    then sum the same products, the kernel in fp32, the oracle in double,
    rounded once to fp32.  Returns the rows compared."""
    n_gpu = run.tap(layer, "n")[rows]
    lg = run.tap(layer, "logits")[rows].astype(np.float64)
    same = [i for i in range(len(rows)) if np.array_equal(n_gpu[i].astype(np.float64), t.n[i])]
    for i in same:
        want = t.logits[i].astype(np.float64)
        assert np.allclose(lg[i], want, rtol=LOGIT_TOL, atol=LOGIT_TOL), \
            f"{what} row {rows[i]}: logits max diff {np.abs(lg[i] - want).max():.3e}"
    return same


def check_chain_layer(wl, run, layer, lw, nxt):
    """Layer `layer` of a chain, every row, on the residual streams the
    kernel materialised for it (x tap): routing exact except at the oracle's
    near ties, the logits on rows with identical n, and y and the next
    streams `nxt` (the next layer's x tap, or the step's output) within the
    single-layer tolerance on the rows whose routing agreed.  Returns the
    rows whose oracle selection shows a near tie, with the cause."""
    x_gpu = raw_hc(wl, run.tap(layer, "x"))
    out, t = O.layer(wl, lw, x_gpu)
    rows = list(range(wl.rows))
    ties = {}
    keep = []
    gidx = run.tap(layer, "idx")
    for r in rows:
        ok, exempt = routing_ok(gidx[r], t.idx[r], t.sel[r], wl.top_k)
        assert ok, f"layer {layer} row {r}: gpu {gidx[r]} oracle {t.idx[r]}"
        cause = near_tie(t.sel[r], wl.top_k)
        if cause:
            ties[r] = f"layer {layer}: {cause}"
        if not exempt:
            keep.append(r)
    check_logits(run, layer, t, rows, f"layer {layer}")
    compare_out(wl, run.tap(layer, "n")[keep], t.n[keep], f"layer {layer} n")
    compare_out(wl, run.tap(layer, "y")[keep], t.y[keep], f"layer {layer} y")
    compare_out(wl, np.asarray(nxt)[keep], O.decode_hc(wl, out)[keep], f"layer {layer} expand")
    return ties


def routing_divergence(wl, run, oracle_taps):
    """Rows whose selected experts in the oracle's own chain (oracle_taps[l],
    run from hc_in) differ from the kernel's in some layer, with the cause.  The
    kernel's routing is checked against the oracle on the kernel's own
    streams layer by layer (check_chain_layer); the two chains' residual
    streams drift apart by rounding differences (a one-spacing change grows
    through the layers), so where a selection margin is small they can pick
    different experts, after which the rows are no longer comparable."""
    out = {}
    for l, t in enumerate(oracle_taps):
        gidx = run.tap(l, "idx")
        for r in range(wl.rows):
            # the same experts in another order give the same routed sum (only
            # the fp32 rounding of the weights' denominator can differ)
            if r in out or np.array_equal(np.sort(gidx[r]), np.sort(t.idx[r])):
                continue
            s = t.sel[r].astype(np.float64)
            order = np.argsort(-s, kind="stable")
            k = wl.top_k
            gap = abs(s[order[k - 1]] - s[order[k]]) / max(abs(s[order[k - 1]]), 1e-30)
            out[r] = (f"layer {l}: the oracle's chain selects {t.idx[r].tolist()}, the kernel {gidx[r].tolist()} "
                      f"(oracle's k-th / (k+1)-th selection margin {gap:.2e} relative)")
    return out
