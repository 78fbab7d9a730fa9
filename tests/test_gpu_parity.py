"""Parity of the CUDA path (through the C ABI) with the CPU oracle on the same
seeded inputs, at sizes the oracle finishes in seconds: several weight-ring
tiles per CTA, a ragged tail of items, every rows count 1..8, the all-zero
tie rounds, FP8 and MXFP4 experts, and a 4-layer chain."""

import numpy as np
import pytest

from oracle import oracle as O
from synth import configs as C
from synth import synth as S
from tests.gpu_harness import (LayerRun, check_chain_layer, check_logits, compare_out, compare_rel_l2, oracle_rows,
                               routing_divergence, routing_ok, select_weights)
from tests.oracle_helpers import all_experts

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__
    __graft_entry__.build()


def _check_layer(wl, run, rows, layer=0, hc_in=None, dense=None):
    """Compare every tap and the output of `rows` with the oracle."""
    want, t = oracle_rows(wl, rows, layer=layer, hc_in=hc_in, dense=dense)
    got = run.out_host()[rows]
    idx = run.tap(layer, "idx")[rows]
    exempt = []
    for i in range(len(rows)):
        ok, ex = routing_ok(idx[i], t.idx[i], t.sel[i], wl.top_k)
        assert ok, f"row {rows[i]}: gpu {idx[i]} oracle {t.idx[i]}"
        if ex:
            exempt.append(i)
    keep = [i for i in range(len(rows)) if i not in exempt]
    tol_mix = 1e-4
    assert np.allclose(run.tap(layer, "mix")[rows], t.mix, rtol=tol_mix, atol=tol_mix)
    assert np.allclose(run.tap(layer, "pre")[rows], t.pre, rtol=1e-5, atol=1e-6)
    assert np.allclose(run.tap(layer, "comb")[rows], t.comb.reshape(len(rows), 16), rtol=1e-4, atol=1e-5)
    # the router matvec: on the kernel's own n for every row (a bf16 rounding
    # flip in n moves a logit by ~1e-4), and against the oracle's fp32 logits
    # on the rows whose n equals the oracle's bit for bit
    d = S.cpu_dense(wl, layer) if dense is None else dense
    n_gpu = run.tap(layer, "n")[rows].astype(np.float64)
    lg_want = n_gpu @ d["router_w"].astype(np.float64)
    assert np.allclose(run.tap(layer, "logits")[rows], lg_want, rtol=1e-4, atol=1e-5)
    check_logits(run, layer, t, rows)
    # the select math on the kernel's own logits and selection, then the
    # weights against the oracle's (which see the oracle's n)
    w = run.tap(layer, "w")[rows]
    w_own = select_weights(wl, run.tap(layer, "logits")[rows], idx, None)
    assert np.allclose(w, w_own, rtol=2e-6, atol=1e-7)
    wtol = 1e-5 if not wl.round_bf16 else 1e-3
    assert np.allclose(w[keep], t.w[keep], rtol=wtol, atol=wtol * 1e-1)
    if keep:
        compare_out(wl, run.tap(layer, "n")[rows][keep], t.n[keep], "n")
        compare_out(wl, run.tap(layer, "y")[rows][keep], t.y[keep], "y")
        if wl.n_layers == 1:
            compare_out(wl, got[keep], want[keep], "hc_out")
    return t


def test_tiny_fp32_all_rows():
    wl = C.TINY_FP32
    run = LayerRun(wl)
    run.step()
    _check_layer(wl, run, [0])
    run.close()


@pytest.mark.parametrize("rows", [1, 2, 3, 4, 5, 6, 7, 8])
def test_tiny_fp32_rows_sweep(rows):
    wl = C.TINY_FP32.with_(rows=rows, seed=100 + rows)
    run = LayerRun(wl)
    run.step()
    _check_layer(wl, run, list(range(rows)))
    run.close()


def test_rows_zero_is_noop_and_rows_above_max_refused():
    import torch

    from moe_decode_layer_sm_b200 import MonoError
    wl = C.TINY_FP32.with_(rows=2)
    run = LayerRun(wl)
    run.out.fill_(7.0)
    run.plan.step(0, run.hc, run.out)
    torch.cuda.synchronize()
    assert bool((run.out == 7.0).all())
    with pytest.raises(MonoError):
        run.plan.step(3, run.hc, run.out)
    run.close()


@pytest.mark.parametrize("bias", ["zero", "four-levels"])
def test_zero_input_tie_rounds(bias):
    import torch
    wl = C.TINY_FP32.with_(rows=2)
    d = S.cpu_dense(wl, 0)
    if bias == "zero":
        b = np.zeros_like(d["router_bias"])
    else:
        levels = np.array([-0.075, -0.025, 0.025, 0.075], np.float32)
        b = levels[np.minimum(3, np.floor((d["router_bias"] + 0.1) / 0.05).astype(int))]
    hc = torch.zeros((2, 4, wl.hidden), dtype=torch.float32, device="cuda")
    run = LayerRun(wl, dense_override=lambda l: {"router_bias": b}, hc_in=hc)
    run.step()
    d["router_bias"] = b
    t = _check_layer(wl, run, [0, 1], hc_in=np.zeros((2, 4, wl.hidden), np.float32), dense=d)
    order = sorted(range(wl.n_routed), key=lambda e: (-b[e], e))
    assert run.tap(0, "idx").tolist() == [order[:wl.top_k]] * 2 == t.idx.tolist()
    assert np.all(run.out_host() == 0.0)
    run.close()


@pytest.mark.parametrize("rows", [1, 3, 8])
def test_scaled_bf16(rows):
    wl = C.scaled(C.FLASH_BF16_R8, rows=rows, seed=200 + rows)
    run = LayerRun(wl)
    run.step()
    _check_layer(wl, run, list(range(rows)))
    # a second step on the same plan (epoch-tagged counters, no reset) gives the same bytes
    first = run.out_host().copy()
    run.step()
    assert np.array_equal(first, run.out_host())
    run.close()


@pytest.mark.parametrize("case", ["tiny-fp32", "scaled-bf16", "scaled-fp8"])
def test_rows_vary_across_steps_on_one_plan(case):
    """One plan stepped with row counts on both sides of the mix reduction's
    one-level / two-level switch (3 | 4 rows): every grid counter must stay in
    step with the others whatever path a step took, so no wait times out and
    every step matches the oracle on its rows."""
    wl, seq = {"tiny-fp32": (C.TINY_FP32.with_(rows=8, seed=120), [2, 8, 3, 5, 1]),
               "scaled-bf16": (C.scaled(C.FLASH_BF16_R8, seed=121), [2, 8, 3, 5, 1]),
               "scaled-fp8": (C.scaled(C.FLASH_FP8_R4, seed=122), [2, 4, 3, 4, 1])}[case]
    run = LayerRun(wl)
    for n in seq:
        run.step(n)   # asserts that the device reported no error
        _check_layer(wl, run, list(range(n)))
    run.close()


def test_scaled_fp8_rows4():
    wl = C.scaled(C.FLASH_FP8_R4, seed=301)
    run = LayerRun(wl)
    run.step()
    _check_layer(wl, run, list(range(wl.rows)))
    run.close()


def test_cuda_core_bf16_hidden_not_multiple_of_128():
    """bf16 experts with hidden 1056 and inter 544: not whole 128-row blocks,
    so the CUDA-core kernel."""
    wl = C.scaled(C.FLASH_BF16_R8, seed=221, hidden=1056, inter=544, rows=5)
    run = LayerRun(wl)
    assert run.plan.info()["ring_slot_bytes"] != 16384   # not the tensor-core layout
    run.step()
    _check_layer(wl, run, list(range(wl.rows)))
    run.close()


def test_cuda_core_fp8_fp32_streams():
    """FP8 experts with fp32 residual streams and no bf16 rounding: the
    CUDA-core kernel (the tensor-core kernels take only the rounded layer);
    compared at the fp32 tolerance."""
    wl = C.scaled(C.FLASH_FP8_R4, seed=311, hc_dtype="f32", norm_dtype="f32", round_bf16=False)
    run = LayerRun(wl)
    assert run.plan.info()["ring_slot_bytes"] != 2 * 16384   # not the tensor-core layout
    run.step()
    _check_layer(wl, run, list(range(wl.rows)))
    run.close()


def test_cuda_core_mxfp4_hidden_not_multiple_of_128():
    """MXFP4 with hidden 1056 and inter 544 (multiples of 32, not of 128): the
    CUDA-core kernel."""
    wl = C.scaled(C.FLASH_MXFP4_CHAIN4_R8, n_layers=1, seed=411, hidden=1056, inter=544, rows=3)
    run = LayerRun(wl)
    assert run.plan.info()["ring_slot_bytes"] != 2 * 16384 + 2 * 512   # not the tensor-core layout
    run.step()
    _check_layer(wl, run, list(range(wl.rows)))
    run.close()


def test_scaled_mxfp4_wide_block_spread():
    """MXFP4 rows whose block scales span up to 2^20: the tensor-core path
    applies each 32-element block's e8m0 scale inside the block-scaled MMA,
    so every block keeps its own exponent, however far from its row's
    largest."""
    wl = C.scaled(C.FLASH_MXFP4_CHAIN4_R8, n_layers=1, seed=431, mx_spread=20)
    run = LayerRun(wl)
    run.step()
    _check_layer(wl, run, list(range(wl.rows)))
    run.close()


def test_mxfp4_nan_scale_refused_at_packing():
    """e8m0 code 255 is NaN: the tensor-core path's packing refuses it with
    INVALID_ARG before any step, instead of expanding a NaN scale."""
    import torch
    from moe_decode_layer_sm_b200 import Plan
    from moe_decode_layer_sm_b200.binding import MonoError
    wl = C.scaled(C.FLASH_MXFP4_CHAIN4_R8, n_layers=1, seed=451)
    plan = Plan.for_workload(wl)
    d = S.gpu_dense(wl, 0)
    ex = S.gpu_experts(wl, 0)
    ex["up"][1][3, 17, 2] = 255
    torch.cuda.synchronize()
    with pytest.raises(MonoError) as err:
        plan.pack(0, d["mix_w"], d["norm_w"], d["router_w"], d["router_bias"], ex["gate"][0], ex["up"][0],
                  ex["down"][0], ex["gate"][1], ex["up"][1], ex["down"][1])
    assert "NaN" in str(err.value) and "INVALID_ARG" in str(err.value)
    plan.close()


def test_scaled_mxfp4_single_layer():
    wl = C.scaled(C.FLASH_MXFP4_CHAIN4_R8, n_layers=1, seed=401)
    run = LayerRun(wl)
    run.step()
    _check_layer(wl, run, list(range(wl.rows)))
    run.close()


@pytest.mark.parametrize("rows", [8, 3])
def test_scaled_mxfp4_mxfp8_activations(rows):
    """MXFP4 experts with MXFP8 activations (one e4m3 term per row under an
    e8m0 scale per 32 values, block-scaled MMAs with N = 8) against the
    oracle's act_mx8 numerics."""
    wl = C.scaled(C.FLASH_MXFP4_CHAIN4_R8, n_layers=1, seed=461 + rows, rows=rows, act_mx8=True)
    run = LayerRun(wl)
    run.step()
    _check_layer(wl, run, list(range(wl.rows)))
    run.close()


def test_scaled_mxfp4_mxfp8_activations_chain():
    wl = C.scaled(C.FLASH_MXFP4_CHAIN4_R8, seed=471, act_mx8=True)
    run = LayerRun(wl)
    got = run.step()
    lws = [O.LayerWeights(wl, S.cpu_dense(wl, l), all_experts(wl, l)) for l in range(wl.n_layers)]
    for l, lw in enumerate(lws):
        nxt = run.tap(l + 1, "x") if l + 1 < wl.n_layers else got
        check_chain_layer(wl, run, l, lw, nxt)
    run.close()


@pytest.mark.parametrize("wdt, rows", [("bf16", 8), ("mxfp4", 8), ("bf16", 2), ("mxfp4", 1)])
def test_scaled_chain_four_layers(wdt, rows):
    """Every layer of the chain, every row, checked on the residual streams
    the kernel materialised for it (x tap): routing exact (near-tie
    exemption), logits, n, y and the next layer's streams within the
    single-layer tolerance.  Then the whole chain against the oracle's own
    chain in relative L2, on every row whose routing met no near tie along
    the way; the end-to-end max-abs is printed, not bounded by one layer's
    tolerance: the oracle's own chain moves by more than that under a
    one-spacing change of one value after its first layer
    (tests/test_chain_conditioning.py).  At 8, 2 and 1 rows (R <= 4 also
    moves the top-k to warps 4-7 on the bf16 path)."""
    wl = C.scaled(C.FLASH_MXFP4_CHAIN4_R8, w_dtype=wdt, seed=402, rows=rows)
    run = LayerRun(wl)
    got = run.step()
    lws = [O.LayerWeights(wl, S.cpu_dense(wl, l), all_experts(wl, l)) for l in range(wl.n_layers)]
    assert np.array_equal(run.tap(0, "x"), O.decode_hc(wl, S.cpu_hc_in(wl)))
    ties = {}
    for l, lw in enumerate(lws):
        nxt = run.tap(l + 1, "x") if l + 1 < wl.n_layers else got
        for r, cause in check_chain_layer(wl, run, l, lw, nxt).items():
            ties.setdefault(r, cause)
    # the oracle's own chain from hc_in, layer by layer (equal bit for bit to
    # its deferred-post form: tests/test_oracle_pins.py)
    x, otaps = S.cpu_hc_in(wl), []
    for lw in lws:
        x, t = O.layer(wl, lw, x)
        otaps.append(t)
    want = O.decode_hc(wl, x)
    assert np.array_equal(want, O.decode_hc(wl, O.chain(wl, lws, S.cpu_hc_in(wl), deferred=True)))
    for r, cause in routing_divergence(wl, run, otaps).items():
        ties.setdefault(r, cause)
    keep = [r for r in range(wl.rows) if r not in ties]
    assert 2 * len(keep) >= wl.rows, f"rows left out: {ties}"
    for r in keep:
        compare_rel_l2(got[r], want[r], f"chain hc_out row {r}")
    print(f"chain end to end: max-abs {np.abs(got[keep] - want[keep]).max():.4e}; rows left out: {ties}")
    run.close()


_TIMEOUT_CASES = [("tiny-fp32", st) for st in ("MIX", "COLLAPSE", "LOGITS", "ACT")] + \
                 [("scaled-bf16", st) for st in ("MIX", "COLLAPSE", "LOGITS", "ACT", "Y")] + \
                 [("scaled-fp8", st) for st in ("ACT", "Y")]


def _timeout_workload(case):
    if case == "tiny-fp32":
        return C.TINY_FP32.with_(rows=1)
    if case == "scaled-bf16":
        return C.scaled(C.FLASH_BF16_R8, rows=2, seed=231)
    return C.scaled(C.FLASH_FP8_R4, rows=2, seed=331)


@pytest.mark.parametrize("case, stage", _TIMEOUT_CASES)
def test_device_timeout_is_reported_and_recovers(case, stage):
    """One CTA withholds its arrival at one grid stage (at the activation
    stage of the tensor-core kernels: the count of the shared expert's first
    gate/up block): the waits there expire after the plan's 20 ms bound, the
    step reports DEVICE_TIMEOUT at that stage, and the next step on the same
    plan is correct again.  No GPU fault: every wait is bounded."""
    from moe_decode_layer_sm_b200.binding import STAGE
    wl = _timeout_workload(case)
    run = LayerRun(wl, wait_timeout_us=20000)
    run.plan.debug_skip_arrival(3, STAGE[stage])
    run.plan.step(wl.rows, run.hc, run.out)
    rc, st = run.plan.query_error()
    assert rc == -7 and st.stage == STAGE[stage], (rc, st.stage, st.cta, st.layer)
    run.plan.debug_skip_arrival(-1)
    run.step()
    _check_layer(wl, run, list(range(wl.rows)))
    run.close()


@pytest.mark.parametrize("case", ["tiny-fp32", "scaled-bf16-r8", "scaled-fp8-r4", "scaled-mxfp4-r8"])
def test_arrival_jitter_keeps_results_bitwise(case):
    """Race detection: every thread that publishes a grid-visible arrival
    first sleeps hash(CTA, step, point) % 2 us, so the order in which CTAs
    arrive, and which CTA completes each split block, changes from step to
    step.  1000 such steps give the bytes of the first, unjittered step."""
    import torch
    wl = {"tiny-fp32": C.TINY_FP32.with_(rows=3),
          "scaled-bf16-r8": C.scaled(C.FLASH_BF16_R8, seed=241),
          "scaled-fp8-r4": C.scaled(C.FLASH_FP8_R4, seed=341),
          "scaled-mxfp4-r8": C.scaled(C.FLASH_MXFP4_CHAIN4_R8, n_layers=1, seed=441)}[case]
    run = LayerRun(wl)
    run.step()
    ref = run.out.clone()
    run.plan.debug_jitter(2000)
    bad = torch.zeros((), dtype=torch.int64, device="cuda")
    for _ in range(1000):
        run.plan.step(wl.rows, run.hc, run.out)
        bad += (run.out.view(torch.int16 if wl.hc_dtype == "bf16" else torch.int32)
                != ref.view(torch.int16 if wl.hc_dtype == "bf16" else torch.int32)).sum()
    rc, st = run.plan.query_error()
    assert rc == 0, (rc, st.stage)
    assert int(bad) == 0
    run.plan.debug_jitter(0)
    run.close()
