"""Parity of mono_ffn_step_pending (the within-layer boundary: the attention
sublayer's pending post / expand closed in the FFN's opening pass) with the
oracle's orc_layer_pending, through the C ABI, on the same seeded inputs:
the materialised residual streams, every layer on the kernel's own streams,
and the output."""

import numpy as np
import pytest

from oracle import oracle as O
from synth import configs as C
from synth import synth as S
from tests.gpu_harness import (FP32_MAX_ABS, LayerRun, bf16_ulp, check_chain_layer, compare_out, compare_rel_l2,
                               raw_hc, routing_divergence)
from tests.oracle_helpers import all_experts, touched_experts

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__
    __graft_entry__.build()


def _run_pending(wl):
    run = LayerRun(wl)
    a = S.gpu_attn_pending(wl)
    run.plan.step_pending(wl.rows, a["x"], a["post"], a["comb"], a["y"], run.out)
    rc, st = run.plan.query_error()
    assert rc == 0, (rc, st.stage)
    return run, S.cpu_attn_pending(wl)


def _check_streams(wl, x_gpu, x_want):
    """The materialised streams: both sides round sum_j comb_ij x_j + post_i y
    (fp32 on the device, double in the oracle) to the stream type once, so
    they agree except where the sum lies within rounding of a bf16 midpoint:
    then by one spacing."""
    x_gpu = np.asarray(x_gpu, np.float64)
    x_want = O.decode_hc(wl, x_want)
    d = np.abs(x_gpu - x_want)
    if wl.hc_dtype == "f32":
        assert d.max() <= FP32_MAX_ABS
    else:
        assert np.all(d <= bf16_ulp(x_want) * 1.0000001)
        assert np.mean(d > 0) < 1e-3, np.mean(d > 0)


@pytest.mark.parametrize("case", ["tiny-fp32-r3", "scaled-bf16-r1", "scaled-bf16-r8", "scaled-fp8-r4",
                                  "scaled-mxfp4-r8"])
def test_step_pending_single_layer(case):
    wl = {"tiny-fp32-r3": C.TINY_FP32.with_(rows=3, seed=501),
          "scaled-bf16-r1": C.scaled(C.FLASH_BF16_R1, seed=502),
          "scaled-bf16-r8": C.scaled(C.FLASH_BF16_R8, seed=503),
          "scaled-fp8-r4": C.scaled(C.FLASH_FP8_R4, seed=504),
          "scaled-mxfp4-r8": C.scaled(C.FLASH_MXFP4_CHAIN4_R8, n_layers=1, seed=505)}[case]
    run, a = _run_pending(wl)
    lw = O.LayerWeights(wl, S.cpu_dense(wl, 0), all_experts(wl, 0))
    out, x, _ = O.layer_pending(wl, lw, a["x"], a["post"], a["comb"], a["y"])
    _check_streams(wl, run.tap(0, "x"), x)
    # the layer on the streams the kernel materialised, at one layer's tolerance
    check_chain_layer(wl, run, 0, lw, run.out_host())
    # and the whole boundary + layer against the oracle's
    compare_out(wl, run.out_host(), O.decode_hc(wl, out), "hc_out")
    run.close()


def test_step_pending_opens_a_chain():
    """A 4-layer chain opened by the attention sublayer's expand: every layer
    on the kernel's own streams, then end to end in relative L2 on the rows
    whose routing agrees with the oracle's own chain."""
    wl = C.scaled(C.FLASH_MXFP4_CHAIN4_R8, w_dtype="bf16", seed=506, rows=4)
    run, a = _run_pending(wl)
    got = run.out_host()
    lws = [O.LayerWeights(wl, S.cpu_dense(wl, l), all_experts(wl, l)) for l in range(wl.n_layers)]
    out0, x0, t0 = O.layer_pending(wl, lws[0], a["x"], a["post"], a["comb"], a["y"])
    _check_streams(wl, run.tap(0, "x"), x0)
    ties = {}
    for l, lw in enumerate(lws):
        nxt = run.tap(l + 1, "x") if l + 1 < wl.n_layers else got
        for r, cause in check_chain_layer(wl, run, l, lw, nxt).items():
            ties.setdefault(r, cause)
    x, otaps = out0, [t0]
    for lw in lws[1:]:
        x, t = O.layer(wl, lw, x)
        otaps.append(t)
    for r, cause in routing_divergence(wl, run, otaps).items():
        ties.setdefault(r, cause)
    keep = [r for r in range(wl.rows) if r not in ties]
    assert 2 * len(keep) >= wl.rows, f"rows left out: {ties}"
    want = O.decode_hc(wl, x)
    for r in keep:
        compare_rel_l2(got[r], want[r], f"chain hc_out row {r}")
    run.close()


def test_step_pending_full_size_bf16_r1():
    """The bf16 layer at one row, full size, opened by the pending expand."""
    wl = C.FLASH_BF16_R1
    run, a = _run_pending(wl)
    dense = S.cpu_dense(wl, 0)
    x_ref = O.expand(wl, a["x"], a["post"], a["comb"], a["y"])
    ex, _ = touched_experts(wl, dense, x_ref, 0)
    ex2, _ = touched_experts(wl, dense, raw_hc(wl, run.tap(0, "x")), 0)
    ex.update(ex2)
    lw = O.LayerWeights(wl, dense, ex)
    out, x, _ = O.layer_pending(wl, lw, a["x"], a["post"], a["comb"], a["y"])
    _check_streams(wl, run.tap(0, "x"), x)
    check_chain_layer(wl, run, 0, lw, run.out_host())
    compare_out(wl, run.out_host(), O.decode_hc(wl, out), "hc_out")
    run.close()


def test_step_pending_refusals():
    """Overlapping buffers and rows above the plan's maximum are refused on
    the host before any launch."""
    import torch

    from moe_decode_layer_sm_b200 import MonoError
    wl = C.TINY_FP32.with_(rows=2, seed=507)
    run = LayerRun(wl)
    a = S.gpu_attn_pending(wl)
    with pytest.raises(MonoError, match="overlap"):
        run.plan.step_pending(2, a["x"], a["post"], a["comb"], a["y"], a["x"])
    with pytest.raises(MonoError, match="rows 3"):
        run.plan.step_pending(3, a["x"], a["post"], a["comb"], a["y"], run.out)
    run.out.fill_(7.0)
    run.plan.step_pending(0, a["x"], a["post"], a["comb"], a["y"], run.out)
    torch.cuda.synchronize()
    assert bool((run.out == 7.0).all())
    run.close()
