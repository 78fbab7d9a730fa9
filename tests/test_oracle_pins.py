"""Pins of the CPU oracle to facts outside itself: closed forms, invariants,
library routines and brute force on tiny shapes.  CPU only."""

import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import oracle as O
from synth import configs as C
from synth import synth as S
from tests.oracle_helpers import all_experts, f32_of, layer_inputs, tiny, zero_expert

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    vals = {}
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, v = line.split()
        vals[k] = float(v)
    return vals


# ------------------------------------------------------------------ codecs --

def test_bf16_round_matches_torch_on_fp32_patterns():
    rng = np.random.default_rng(0)
    bits = np.concatenate([rng.integers(0, 2**32, 200000, dtype=np.uint64).astype(np.uint32),
                           np.arange(0, 2**16, dtype=np.uint32) << 16 | 0x8000,  # exact ties
                           np.arange(0, 2**16, dtype=np.uint32) << 16 | 0x7FFF,
                           np.arange(0, 2**16, dtype=np.uint32) << 16 | 0x8001])
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    L = O.lib()
    got = np.array([L.orc_round_bf16(float(x)) for x in f[:20000]], np.uint16)
    assert np.array_equal(got, want[:20000])
    # the tie patterns all
    sel = np.arange(200000, f.shape[0])[:: 7]
    got = np.array([L.orc_round_bf16(float(f[i])) for i in sel], np.uint16)
    assert np.array_equal(got, want[sel])


def test_bf16_round_double_is_single_rounding():
    L = O.lib()
    # 1 + 2^-8 is the midpoint of 1 and 1 + 2^-7: ties to even -> 1.0
    assert L.orc_round_bf16(1.0 + 2**-8) == 0x3F80
    # just above the midpoint (not representable in fp32): rounds up once
    assert L.orc_round_bf16(1.0 + 2**-8 + 2**-40) == 0x3F81
    # 1 + 3 * 2^-8 ties to even upward -> 1 + 2^-6
    assert L.orc_round_bf16(1.0 + 3 * 2**-8) == 0x3F82
    assert L.orc_round_bf16(-2.5) == 0xC020
    assert L.orc_round_bf16(0.0) == 0 and L.orc_round_bf16(-0.0) == 0x8000


def test_e4m3_decode_all_codes_vs_torch():
    L = O.lib()
    want = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([L.orc_dec_e4m3(c) for c in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(want))
    m = ~np.isnan(want)
    assert np.array_equal(got[m], want[m])
    assert np.array_equal(np.signbit(got[m]), np.signbit(want[m]))


def test_e8m0_decode_all_codes_vs_torch():
    L = O.lib()
    want = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).double().numpy()
    got = np.array([L.orc_dec_e8m0(c) for c in range(256)])
    assert np.isnan(got[255]) and np.isnan(want[255])
    assert np.array_equal(got[:255], want[:255])


def test_e2m1_decode_vs_ocp_table():
    L = O.lib()
    tab = {}
    for line in open(os.path.join(GOLD, "e2m1_codes.txt")):
        if line.strip() and not line.startswith("#"):
            c, v = line.split()
            tab[int(c)] = float(v)
    for c in range(16):
        got = L.orc_dec_e2m1(c)
        assert got == tab[c] and math.copysign(1, got) == math.copysign(1, tab[c]), c


def _fp8_inputs(rows=64, cols=512, seed=0):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    x[0] = 0.0                       # zero block rows
    x[1, :128] = 448.0 * 3.0         # saturating scale path
    x[2, :128] = rng.standard_normal(128).astype(np.float32) * 1e-30   # tiny
    x[3, 5] = -0.0
    return x


def test_oracle_fp8_quantiser_vs_torch():
    x = _fp8_inputs()
    q, s = O.quant_fp8(x)
    sref = np.maximum(np.abs(x).reshape(x.shape[0], -1, 128).max(-1), 0)
    sref = np.where(sref > 0, (sref / np.float32(448.0)).astype(np.float32), np.float32(1.0))
    assert np.array_equal(s, sref)
    v = (x / np.repeat(s, 128, axis=1)).astype(np.float32)    # fp32 quotient
    assert np.abs(v).max() < 464.0   # amax / (amax / 448) may land an ulp above 448
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, want)


def _brute_e2m1(v):
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    a = min(abs(float(v)), 6.0)
    d = np.abs(mags - a)
    best = np.flatnonzero(d == d.min())
    code = int(best[0]) if len(best) == 1 else int(best[best % 2 == 0][0])
    return code | (8 if np.signbit(v) else 0)


def test_oracle_mxfp4_quantiser_vs_brute_force():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((8, 256)) * 0.05).astype(np.float32)
    x[0, :32] = 0.0
    # exact ties after scaling: amax 4 -> X = 0, elements on the e2m1 midpoints
    x[1, :32] = np.array([4.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0] * 4, np.float32) * np.array(
        [1, 1, 1, 1, -1, -1, -1, -1] * 4, np.float32)
    q, e = O.quant_mxfp4(x)
    for r in range(x.shape[0]):
        for b in range(x.shape[1] // 32):
            blk = x[r, b * 32:(b + 1) * 32]
            amax = float(np.abs(blk).max())
            X = -127 if amax == 0 else math.floor(math.log2(amax)) - 2
            assert e[r, b] == max(0, min(254, X + 127))
            Xs = int(e[r, b]) - 127
            for i in range(32):
                v = np.float32(math.ldexp(float(blk[i]), -Xs))
                byte = q[r, b * 16 + i // 2]
                code = (byte >> 4) if i % 2 else (byte & 15)
                assert code == _brute_e2m1(v), (r, b, i, blk[i])


def test_synth_encoders_equal_oracle_quantisers():
    """The generator's encoders write the bytes the oracle's rule gives."""
    x = _fp8_inputs(rows=96, cols=1024, seed=5)
    assert all(np.array_equal(a, b) for a, b in zip(O.quant_fp8(x), S.quant_fp8(x)))
    x = (np.random.default_rng(6).standard_normal((96, 1024)) * 0.03).astype(np.float32)
    x[0, :32] = 0.0
    x[1, :64] = 1e-41   # subnormal block amax
    assert all(np.array_equal(a, b) for a, b in zip(O.quant_mxfp4(x), S.quant_mxfp4(x)))


def test_synth_fused_quant_fill_equals_quantised_fill():
    wl = tiny(w_dtype="fp8", hidden=256, inter=128)
    f = S.cpu_expert_f32(wl, 0, 3)
    q = S.cpu_expert(wl, 0, 3)
    for nm in ("gate", "up", "down"):
        assert all(np.array_equal(a, b) for a, b in zip(q[nm], O.quant_fp8(f[nm])))
    wl = wl.with_(w_dtype="mxfp4")
    q = S.cpu_expert(wl, 0, 3)
    for nm in ("gate", "up", "down"):
        assert all(np.array_equal(a, b) for a, b in zip(q[nm], O.quant_mxfp4(f[nm])))


# ---------------------------------------------------------------- Sinkhorn --

def test_sinkhorn_doubly_stochastic_invariant():
    rng = np.random.default_rng(2)
    for _ in range(50):
        L = rng.standard_normal((4, 4))      # the mix logits are O(1)
        Cm = O.sinkhorn(L, 20)
        assert (Cm > 0).all()
        assert np.abs(Cm.sum(0) - 1).max() < 1e-6
        assert np.abs(Cm.sum(1) - 1).max() < 1e-4
        # wider logits converge slower, but more iterations bring the rows closer
        e20 = np.abs(O.sinkhorn(L * 3, 20).sum(1) - 1).max()
        e400 = np.abs(O.sinkhorn(L * 3, 400).sum(1) - 1).max()
        assert e400 <= e20


def test_sinkhorn_fixed_point_and_constant():
    P = 0.6 * np.roll(np.eye(4), 1, axis=1) + 0.1 * np.ones((4, 4))   # doubly stochastic, not symmetric
    assert np.allclose(O.sinkhorn(np.log(P), 20), P, atol=1e-12, rtol=0)
    assert np.allclose(O.sinkhorn(np.full((4, 4), 3.7), 20), 0.25, atol=1e-15, rtol=0)


# ------------------------------------------------------------------- top-k --

def test_topk_brute_force_rank_with_ties():
    rng = np.random.default_rng(3)
    for trial in range(200):
        E = int(rng.integers(2, 40))
        k = int(rng.integers(1, E + 1))
        sel = rng.integers(0, 5, E).astype(np.float32) if trial % 2 else rng.standard_normal(E).astype(np.float32)
        # rank of expert x = number of experts that beat it under (sel desc, idx asc)
        rank = [sum(1 for y in range(E) if sel[y] > sel[x] or (sel[y] == sel[x] and y < x)) for x in range(E)]
        want = [x for r in range(k) for x in range(E) if rank[x] == r]
        assert O.topk(sel, k).tolist() == want


def test_topk_all_tie_is_ascending_and_library_on_distinct():
    assert O.topk(np.zeros(256, np.float32), 8).tolist() == list(range(8))
    sel = np.random.default_rng(4).permutation(256).astype(np.float32)
    assert O.topk(sel, 8).tolist() == torch.topk(torch.from_numpy(sel), 8).indices.tolist()


# ------------------------------------------------------------ closed forms --

@pytest.mark.parametrize("base", [C.TINY_FP32, C.scaled(C.FLASH_BF16_R1, hidden=256, n_routed=16, top_k=8, inter=128)])
def test_zero_input_closed_form(base):
    gold = _golden("zero_input_closed_form.txt")
    wl = base.with_(rows=2)
    hc = np.zeros((2, 4, wl.hidden), np.uint16 if wl.hc_dtype == "bf16" else np.float32)
    dense = S.cpu_dense(wl, 0)
    dense["router_bias"] = np.zeros_like(dense["router_bias"])
    ex = {e: S.cpu_expert(wl, 0, e) for e in list(range(wl.top_k)) + [wl.n_routed]}
    out, t = O.layer(wl, O.LayerWeights(wl, dense, ex), hc)
    assert np.all(t.pre == gold["pre"]) or np.allclose(t.pre, gold["pre"], rtol=1e-15)
    assert np.allclose(t.post, gold["post"], rtol=1e-15, atol=0)
    assert np.allclose(t.comb, gold["comb"], rtol=1e-15, atol=0)
    assert np.all(t.a == gold["a"]) and np.all(t.n == gold["n"]) and np.all(t.logits == gold["logit"])
    assert np.all(t.score == np.float32(math.sqrt(gold["score_sq"])))
    assert t.idx.tolist() == [list(range(wl.top_k))] * 2
    assert np.all(t.w == np.float32(2.5 / wl.top_k))
    assert np.all(t.y == gold["y"])
    assert np.all(O.decode_hc(wl, out) == gold["out"])


def test_zero_input_ties_within_bias_groups():
    """All scores tie; the bias has 4 levels, so the order inside a level is
    the ascending expert index."""
    wl = C.TINY_FP32
    hc = np.zeros((1, 4, wl.hidden), np.float32)
    dense = S.cpu_dense(wl, 0)
    levels = np.array([-0.075, -0.025, 0.025, 0.075], np.float32)
    b = dense["router_bias"]
    dense["router_bias"] = levels[np.minimum(3, np.floor((b + 0.1) / 0.05).astype(int))]
    t = O.route(wl, O.LayerWeights(wl, dense, {}), hc)
    order = sorted(range(wl.n_routed), key=lambda e: (-dense["router_bias"][e], e))
    assert t.idx[0].tolist() == order[:wl.top_k]


def test_zero_mix_weights_closed_form():
    """mix_w = 0: pre = 0.5 + 1e-6, post = 1, comb = 1/4, so
    a = (0.5 + 1e-6) sum_s X_s and out_i = mean_s X_s + y."""
    wl = tiny()
    hc, dense, ex = layer_inputs(wl, experts="all")
    dense["mix_w"] = np.zeros_like(dense["mix_w"])
    out, t = O.layer(wl, O.LayerWeights(wl, dense, ex), hc)
    X = hc.astype(np.float64)
    assert np.allclose(t.a, (0.5 + 1e-6) * X.sum(1), rtol=1e-14, atol=1e-15)
    want = X.mean(1, keepdims=True) + t.y[:, None, :]
    assert np.allclose(O.decode_hc(wl, out), want, rtol=1e-6, atol=1e-6)   # fp32 output rounding


def test_planted_comb_orientation_and_layout():
    """Mix weights chosen so the 16 comb logits are log P for a doubly
    stochastic, non-symmetric P (its own Sinkhorn fixed point) and experts
    are zero: out_i = sum_j P_ij X_j exactly (comb row-major at 2S + S i + j,
    out_i = sum_j comb_ij X_j)."""
    wl = tiny(n_routed=2, top_k=1, rows=1)
    H, S_ = wl.hidden, wl.hc
    X = np.zeros((1, S_, H), np.float32)
    X[0, 0, 0] = 1.0                                 # flattened row = e_0
    P = 0.6 * np.roll(np.eye(4), 1, axis=1) + 0.1 * np.ones((4, 4))
    W = np.zeros((S_ * H, wl.mix_cols), np.float32)
    rho = 1.0 / math.sqrt(1.0 / (S_ * H) + wl.rms_eps)
    W[0, 8:] = (np.log(P).ravel() / rho).astype(np.float32)
    X[0, :, 1:] = np.random.default_rng(7).standard_normal((S_, H - 1)).astype(np.float32) * 1e-3
    X[0, 0, 0] = 1.0
    dense = S.cpu_dense(wl, 0)
    dense["mix_w"] = W
    ex = {e: zero_expert(wl) for e in range(wl.n_routed + 1)}
    out, t = O.layer(wl, O.LayerWeights(wl, dense, ex), X)
    Xd = X[0].astype(np.float64)
    # rho uses the true square sum; the planted logits are scaled for e_0 alone
    Lr = np.log(P) * (t.rho[0] / rho)
    Pd = O.sinkhorn(Lr, 20)
    assert np.allclose(t.comb[0], Pd, atol=1e-12)
    assert np.abs(t.comb[0] - P).max() < 1e-3
    assert not np.allclose(t.comb[0], t.comb[0].T)
    assert np.allclose(O.decode_hc(wl, out)[0], Pd @ Xd, rtol=1e-6, atol=1e-7)


def test_constant_row_mix_closed_form():
    """X = c everywhere: rho = 1/sqrt(c^2 + eps), mix = c rho colsum(mix_w)."""
    wl = tiny(rows=1)
    c = 0.75
    X = np.full((1, wl.hc, wl.hidden), c, np.float32)
    dense = S.cpu_dense(wl, 0)
    t = O.route(wl, O.LayerWeights(wl, dense, {}), X)
    want = c / math.sqrt(c * c + wl.rms_eps) * dense["mix_w"].astype(np.float64).sum(0)
    assert np.allclose(t.mix[0], want, rtol=1e-13, atol=1e-15)
    sig = 1 / (1 + np.exp(-want))
    assert np.allclose(t.pre[0], sig[:4] + 1e-6, rtol=1e-14)
    assert np.allclose(t.post[0], 2 * sig[4:8], rtol=1e-14)
    # collapse of a constant row: a = c sum(pre)
    assert np.allclose(t.a[0], c * t.pre[0].sum(), rtol=1e-14)


def test_weighted_rmsnorm_and_router_scores_vs_library():
    wl = tiny(rows=3)
    hc, dense, ex = layer_inputs(wl)
    t = O.route(wl, O.LayerWeights(wl, dense, {}), hc)
    a = torch.from_numpy(t.a)
    wn = torch.from_numpy(dense["norm_w"].astype(np.float64))
    n = F.rms_norm(a, (wl.hidden,), weight=wn, eps=wl.rms_eps)
    assert torch.allclose(torch.from_numpy(t.n), n, rtol=1e-13, atol=1e-15)
    logits = torch.from_numpy(t.n) @ torch.from_numpy(dense["router_w"].astype(np.float64))
    assert torch.allclose(torch.from_numpy(t.logits.astype(np.float64)), logits, rtol=1e-6, atol=1e-7)
    score = torch.sqrt(F.softplus(torch.from_numpy(t.logits.astype(np.float64)))).float()
    assert torch.equal(torch.from_numpy(t.score), score)


def test_single_expert_reduces_to_swiglu_mlp():
    """E = k = 1 and a zero shared expert: y = 2.5 * down(silu(gate n) * up n)."""
    wl = tiny(n_routed=1, top_k=1, rows=2)
    hc, dense, ex = layer_inputs(wl, experts="all")
    ex[wl.n_routed] = zero_expert(wl)
    out, t = O.layer(wl, O.LayerWeights(wl, dense, ex), hc)
    n = torch.from_numpy(t.n)
    g, u, d = (torch.from_numpy(ex[0][k][0].astype(np.float64)) for k in ("gate", "up", "down"))
    y = 2.5 * F.linear(F.silu(F.linear(n, g)) * F.linear(n, u), d)
    assert t.w.ravel().tolist() == [2.5, 2.5]
    assert torch.allclose(torch.from_numpy(t.y), y, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("wdt", ["fp8", "mxfp4"])
def test_quantised_expert_equals_library_dequantised_f32(wdt):
    """The oracle's FP8 / MXFP4 path equals its fp32 path fed with the weights
    decoded by torch's float8_e4m3fn / float8_e8m0fnu (and the OCP e2m1 table)."""
    wl = tiny(hidden=256, inter=128, n_routed=4, top_k=2, w_dtype=wdt)
    hc, dense, ex = layer_inputs(wl, experts="all")
    out_q, tq = O.layer(wl, O.LayerWeights(wl, dense, ex), hc)
    wf = wl.with_(w_dtype="f32")
    exf = {e: {k: (v.astype(np.float32), None) for k, v in f32_of(wl, m).items()} for e, m in ex.items()}
    # every dequantised value is exact in fp32 (e4m3 x fp32 scale may not be:
    # keep the comparison at the rounding of that product)
    out_f, tf = O.layer(wf, O.LayerWeights(wf, dense, exf), hc)
    assert np.array_equal(tq.idx, tf.idx)
    tol = 0 if wdt == "mxfp4" else 1e-6
    assert np.allclose(tq.y, tf.y, rtol=tol, atol=tol)


# ----------------------------------------------------------- brute force --

def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float64)).float().bfloat16().double().numpy()


def brute_layer(wl, hc, dense, ex):
    """Dense-MoE statement of the layer in numpy float64: every expert is
    evaluated and mixed through a gate vector that is zero off the top-k."""
    R, S_, H, E, K = hc.shape[0], wl.hc, wl.hidden, wl.n_routed, wl.top_k
    rb = _bf16 if wl.round_bf16 else (lambda v: v)
    X = O.decode_hc(wl, hc)
    nw = O.decode_hc(wl.with_(hc_dtype=wl.norm_dtype), dense["norm_w"][None])[0]
    experts = {e: f32_of(wl, m) for e, m in ex.items()}
    outs = []
    for r in range(R):
        xf = X[r].ravel()
        rho = 1 / np.sqrt(np.mean(xf ** 2) + wl.rms_eps)
        mix = rho * (xf @ dense["mix_w"].astype(np.float64))
        sg = 1 / (1 + np.exp(-mix))
        pre, post = sg[:S_] + wl.pre_eps, wl.post_mult * sg[S_:2 * S_]
        M = np.exp(mix[2 * S_:].reshape(S_, S_) - mix[2 * S_:].max())
        for _ in range(wl.sinkhorn_iters):
            M = M / M.sum(1, keepdims=True)
            M = M / M.sum(0, keepdims=True)
        a = rb(pre @ X[r])
        n = rb(a / np.sqrt(np.mean(a ** 2) + wl.rms_eps) * nw)
        logit = (n @ dense["router_w"].astype(np.float64)).astype(np.float32)
        score = np.sqrt(np.logaddexp(0.0, logit.astype(np.float64))).astype(np.float32)
        sel = (score.astype(np.float64) + dense["router_bias"].astype(np.float64)).astype(np.float32)
        rank = np.array([np.sum((sel > sel[x]) | ((sel == sel[x]) & (np.arange(E) < x))) for x in range(E)])
        gate = np.zeros(E)
        chosen = [int(np.flatnonzero(rank == j)[0]) for j in range(K)]
        den = max(np.float32(score[chosen].astype(np.float64).sum()), np.float32(wl.denom_clamp))
        for e in chosen:
            gate[e] = np.float32(np.float32(score[e] / den) * np.float32(wl.route_scale))
        y = np.zeros(H)
        for e in range(E + 1):
            g = rb(experts[e]["gate"] @ n)
            u = rb(experts[e]["up"] @ n)
            d = experts[e]["down"] @ (g / (1 + np.exp(-g)) * u)
            y = y + (gate[e] if e < E else 1.0) * d
        y = rb(y)
        out = M @ X[r] + post[:, None] * y[None, :]
        outs.append(_bf16(out) if wl.hc_dtype == "bf16" else out.astype(np.float32).astype(np.float64))
    return np.stack(outs)


@pytest.mark.parametrize("kw", [dict(), dict(hc_dtype="bf16", norm_dtype="bf16", round_bf16=True),
                                dict(hc_dtype="bf16", norm_dtype="bf16", round_bf16=True, w_dtype="bf16"),
                                dict(hidden=256, inter=128, w_dtype="fp8", hc_dtype="bf16", norm_dtype="bf16",
                                     round_bf16=True),
                                dict(hidden=64, inter=32, w_dtype="mxfp4", hc_dtype="bf16", norm_dtype="bf16",
                                     round_bf16=True)])
def test_whole_layer_brute_force(kw):
    wl = tiny(**kw)
    hc, dense, ex = layer_inputs(wl, experts="all")
    out, _ = O.layer(wl, O.LayerWeights(wl, dense, ex), hc)
    want = brute_layer(wl, hc, dense, ex)
    got = O.decode_hc(wl, out)
    if wl.hc_dtype == "f32":
        assert np.allclose(got, want, rtol=1e-6, atol=1e-7)   # both round once to fp32
        assert np.mean(got == want) > 0.99
    else:
        assert np.mean(got == want) > 0.999                   # same bf16 value almost everywhere
        assert np.allclose(got, want, rtol=2 ** -7, atol=1e-6)


# ------------------------------------------------------------------ chains --

@pytest.mark.parametrize("wdt", ["bf16", "mxfp4"])
def test_deferred_post_chain_is_bit_identical(wdt):
    wl = C.scaled(C.FLASH_MXFP4_CHAIN4_R8, hidden=128, n_routed=8, top_k=2, inter=64, rows=3, w_dtype=wdt)
    hc = S.cpu_hc_in(wl)
    lws = [O.LayerWeights(wl, S.cpu_dense(wl, l), all_experts(wl, l)) for l in range(wl.n_layers)]
    a = O.chain(wl, lws, hc, deferred=False)
    b = O.chain(wl, lws, hc, deferred=True)
    assert np.array_equal(a, b)
    # and the chain equals layer after layer through the public one-layer call
    x = hc
    for lw in lws:
        x, _ = O.layer(wl, lw, x)
    assert np.array_equal(a, x)


# ------------------------------------------------- within-layer boundary --

def _pending_case(wdt, hc="bf16"):
    wl = C.scaled(C.FLASH_BF16_R8, hidden=128, n_routed=8, top_k=2, inter=64, rows=3, w_dtype=wdt, seed=77)
    if hc == "f32":
        wl = wl.with_(hc_dtype="f32", norm_dtype="f32", round_bf16=False)
    lw = O.LayerWeights(wl, S.cpu_dense(wl, 0), all_experts(wl, 0))
    return wl, lw, S.cpu_attn_pending(wl)


@pytest.mark.parametrize("wdt, hc", [("bf16", "bf16"), ("mxfp4", "bf16"), ("f32", "f32")])
def test_pending_boundary_equals_expand_then_layer(wdt, hc):
    """The attention sublayer's expand closed in the FFN's opening pass (mix
    products and square sum taken in the same pass) equals closing it first
    and running the layer on the result, bit for bit."""
    wl, lw, a = _pending_case(wdt, hc)
    out, x, t = O.layer_pending(wl, lw, a["x"], a["post"], a["comb"], a["y"])
    x_ref = O.expand(wl, a["x"], a["post"], a["comb"], a["y"])
    assert np.array_equal(x, x_ref)
    out_ref, t_ref = O.layer(wl, lw, x_ref)
    assert np.array_equal(out, out_ref)
    assert np.array_equal(t.mix, t_ref.mix) and np.array_equal(t.idx, t_ref.idx) and np.array_equal(t.y, t_ref.y)


def test_pending_boundary_special_cases():
    """comb = identity and post = 0 leave the streams as they are (the layer
    then sees x_attn itself); comb = 0 and post = 1 give every stream the
    attention output y (rounded to the stream type)."""
    wl, lw, a = _pending_case("bf16")
    R, S_ = wl.rows, wl.hc
    eye = np.broadcast_to(np.eye(S_, dtype=np.float32), (R, S_, S_)).copy()
    out, x, _ = O.layer_pending(wl, lw, a["x"], np.zeros((R, S_), np.float32), eye, a["y"])
    assert np.array_equal(x, a["x"])
    assert np.array_equal(out, O.layer(wl, lw, a["x"])[0])
    x2 = O.expand(wl, a["x"], np.ones((R, S_), np.float32), np.zeros((R, S_, S_), np.float32), a["y"])
    assert np.array_equal(x2, np.broadcast_to(a["y"][:, None, :], x2.shape))


# ------------------------------------------------------------- dense layer --

def test_dense_layer_is_one_swiglu_mlp_over_every_slot():
    """A dense layer (no router): y = down(silu(gate n) * up n) with the
    E + 1 slots' gate / up rows stacked and their down rows side by side,
    one MLP of width (E + 1) I, against torch.nn.functional in float64; the
    taps show every slice with weight 1."""
    wl = tiny(n_routed=5, top_k=5, rows=2, dense=True)
    hc, dense, ex = layer_inputs(wl, experts="all")
    out, t = O.layer(wl, O.LayerWeights(wl, dense, ex), hc)
    n = torch.from_numpy(t.n)
    slots = range(wl.n_routed + 1)
    g = torch.cat([torch.from_numpy(ex[e]["gate"][0].astype(np.float64)) for e in slots], 0)
    u = torch.cat([torch.from_numpy(ex[e]["up"][0].astype(np.float64)) for e in slots], 0)
    d = torch.cat([torch.from_numpy(ex[e]["down"][0].astype(np.float64)) for e in slots], 1)
    y = F.linear(F.silu(F.linear(n, g)) * F.linear(n, u), d)
    assert torch.allclose(torch.from_numpy(t.y), y, rtol=1e-12, atol=1e-14)
    assert t.idx.tolist() == [list(range(5))] * 2 and np.all(t.w == 1.0)


def test_dense_layer_with_bf16_rounding_equals_routed_slices_of_weight_one():
    """With the bf16 roundings, the dense MLP equals the same slots taken as
    experts with weight 1 (the routed + shared sum of the MoE step written
    out by hand): bf16 round of g and u is per element, so splitting the
    width changes only the order of the double-precision sum."""
    wl = tiny(n_routed=5, top_k=5, rows=2, dense=True, hc_dtype="bf16", norm_dtype="bf16", w_dtype="bf16",
              round_bf16=True)
    hc, dense, ex = layer_inputs(wl, experts="all")
    _, t = O.layer(wl, O.LayerWeights(wl, dense, ex), hc)
    n = t.n
    y = np.zeros_like(t.y)
    for e in range(wl.n_routed + 1):
        m = f32_of(wl, ex[e])
        rb = lambda v: torch.from_numpy(v).to(torch.float32).to(torch.bfloat16).double().numpy()
        gg, uu = rb(n @ m["gate"].T), rb(n @ m["up"].T)
        y += (gg / (1 + np.exp(-gg)) * uu) @ m["down"].T
    yb = torch.from_numpy(y).to(torch.float32).to(torch.bfloat16).double().numpy()
    assert np.mean(yb == t.y) > 0.99
    assert np.allclose(yb, t.y, rtol=2 ** -7, atol=1e-6)


# ------------------------------------------------------ MXFP8 activations --

def _e4m3_table():
    return np.array([O.lib().orc_dec_e4m3(c) for c in range(127)], np.float64)   # code 127 is NaN


def test_mx8_quantiser_vs_brute_force():
    """OCP MX rule for e4m3 blocks: scale 2^(floor(log2 amax) - 8); each value
    the nearest of the 127 e4m3 magnitudes times the scale (ties to the even
    code), saturating at 448; brute force over every code, on blocks spanning
    normal, subnormal, saturating and zero values."""
    mag = _e4m3_table()
    rng = np.random.default_rng(8)
    x = np.concatenate([rng.standard_normal(32 * 40) * 10.0 ** rng.integers(-6, 6, 32 * 40),
                        np.zeros(32), np.full(32, 448.0 * 2 ** -3), rng.standard_normal(32) * 1e-30])
    got, codes, scales = O.quant_mx8(x)
    for b in range(x.size // 32):
        blk = x[b * 32:(b + 1) * 32]
        amax = np.abs(blk).max()
        if amax == 0:
            assert scales[b] == 0 and np.all(got[b * 32:(b + 1) * 32] == 0)
            continue
        X = max(-127, min(127, int(np.floor(np.log2(amax))) - 8))
        assert scales[b] == X + 127
        for i, v in enumerate(blk):
            a = abs(v) / 2.0 ** X
            d = np.abs(mag - a)
            best = np.flatnonzero(d == d.min())
            code = best[0] if len(best) == 1 else (best[0] if best[0] % 2 == 0 else best[1])
            want = np.copysign(mag[code] * 2.0 ** X, v) if code else 0.0
            assert got[b * 32 + i] == want, (b, i, v, got[b * 32 + i], want)


def test_mx8_quantiser_matches_torch_float8_in_range():
    """Within the e4m3 range the element codes equal torch's float8_e4m3fn
    rounding of x / 2^X (RNE)."""
    rng = np.random.default_rng(9)
    x = rng.standard_normal(32 * 64) * 3.0
    _, codes, scales = O.quant_mx8(x)
    X = scales.astype(np.int64) - 127
    v = torch.from_numpy(x / np.repeat(2.0 ** X, 32))
    t = v.to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    keep = np.abs(v.numpy()) <= 448.0
    assert np.array_equal(t[keep], codes[keep])


def test_mx8_single_expert_reduces_to_swiglu_mlp_on_quantised_activations():
    """E = k = 1, zero shared expert, MXFP4 weights, act_mx8: y = 2.5 down(q(
    silu(gate q(n)) up q(n))) with q the MXFP8 quantiser, evaluated with
    torch.nn.functional in float64 on the dequantised weights."""
    wl = tiny(n_routed=1, top_k=1, rows=2, hidden=64, inter=32, w_dtype="mxfp4", act_mx8=True)
    hc, dense, ex = layer_inputs(wl, experts="all")
    zq, zs = (np.zeros_like(a) for a in ex[0]["gate"])
    ex[1] = {"gate": (zq, zs), "up": (zq.copy(), zs.copy()),
             "down": (np.zeros_like(ex[0]["down"][0]), np.zeros_like(ex[0]["down"][1]))}
    _, t = O.layer(wl, O.LayerWeights(wl, dense, ex), hc)
    m = f32_of(wl, ex[0])
    for r in range(wl.rows):
        nq = torch.from_numpy(O.quant_mx8(t.n[r])[0])
        g = F.linear(nq, torch.from_numpy(m["gate"]))
        u = F.linear(nq, torch.from_numpy(m["up"]))
        act = torch.from_numpy(O.quant_mx8((F.silu(g) * u).numpy())[0])
        y = 2.5 * F.linear(act, torch.from_numpy(m["down"]))
        assert torch.allclose(torch.from_numpy(t.y[r]), y, rtol=1e-12, atol=1e-14)
    # and the quantisation is really applied: without it the result differs
    _, t2 = O.layer(wl.with_(act_mx8=False), O.LayerWeights(wl, dense, ex), hc)
    assert not np.allclose(t.y, t2.y, rtol=1e-9)
