"""mono_ffn_step_padded: a fixed launch width with padding rows (slot < 0).
Padding rows hold NaN inputs; their outputs must stay as they were, and the
live rows must match the oracle on those rows alone."""

import numpy as np
import pytest

from oracle import oracle as O
from synth import configs as C
from synth import synth as S
from tests.gpu_harness import LayerRun, compare_out, routing_ok
from tests.oracle_helpers import all_experts

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__
    __graft_entry__.build()


CASES = {
    "tiny-fp32-w4": (C.TINY_FP32.with_(rows=4, seed=601), [1, 2]),
    "scaled-bf16-w8": (C.scaled(C.FLASH_BF16_R8, seed=602), [0, 3, 5]),
    "scaled-bf16-w2": (C.scaled(C.FLASH_BF16_R8, rows=2, seed=603), [1]),
    "scaled-fp8-w4": (C.scaled(C.FLASH_FP8_R4, seed=604), [0, 2, 3]),
    "scaled-mxfp4-w8": (C.scaled(C.FLASH_MXFP4_CHAIN4_R8, n_layers=1, seed=605), [0, 1, 2, 4, 7]),
    "scaled-bf16-chain4-w8": (C.scaled(C.FLASH_MXFP4_CHAIN4_R8, w_dtype="bf16", seed=606), [2, 3, 4, 5, 6, 7]),
}


@pytest.mark.parametrize("case", list(CASES))
def test_step_padded(case):
    import torch
    wl, live = CASES[case]
    W = wl.rows
    run = LayerRun(wl)
    hc = run.hc.clone()
    pad = [r for r in range(W) if r not in live]
    hc[pad] = float("nan")
    slot = torch.tensor([r if r in live else -1 for r in range(W)], dtype=torch.int32, device="cuda")
    run.out.fill_(7.0)
    run.plan.step_padded(W, slot, hc, run.out)
    rc, st = run.plan.query_error()
    assert rc == 0, (rc, st.stage)
    got = run.out_host()
    assert np.all(got[pad] == 7.0)
    # the live rows alone, through the oracle, each layer on the streams the
    # kernel materialised for them (layer 0: hc_in itself)
    wl_l = wl.with_(rows=len(live))
    assert np.array_equal(run.tap(0, "x")[live], O.decode_hc(wl, S.cpu_hc_in(wl)[live]))
    for l in range(wl.n_layers):
        lw = O.LayerWeights(wl_l, S.cpu_dense(wl, l), all_experts(wl, l))
        xg = np.ascontiguousarray(run.tap(l, "x")[live], np.float32)
        if wl.hc_dtype == "bf16":
            xg = (xg.view(np.uint32) >> 16).astype(np.uint16)
        out_k, t = O.layer(wl_l, lw, xg)
        gidx = run.tap(l, "idx")[live]
        for i in range(len(live)):
            assert routing_ok(gidx[i], t.idx[i], t.sel[i], wl.top_k)[0], (l, live[i])
        nxt = run.tap(l + 1, "x")[live] if l + 1 < wl.n_layers else got[live]
        compare_out(wl, nxt, O.decode_hc(wl, out_k), f"layer {l} expand")
    run.close()


def test_step_padded_refusals():
    import torch

    from moe_decode_layer_sm_b200 import MonoError
    wl = C.TINY_FP32.with_(rows=2, seed=607)
    run = LayerRun(wl)
    slot = torch.zeros(3, dtype=torch.int32, device="cuda")
    with pytest.raises(MonoError, match="width 3"):
        run.plan.step_padded(3, slot, run.hc, run.out)
    with pytest.raises(MonoError, match="overlap"):
        run.plan.step_padded(2, slot, run.hc, run.hc)
    run.close()
