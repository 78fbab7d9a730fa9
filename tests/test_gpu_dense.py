"""Dense layers (no router): the SwiGLU MLP of width (E + 1) x inter over
every slot, run by the same kernels as expert-shaped slices taken with
weight 1, against the oracle's dense MLP evaluated as one matrix."""

import numpy as np
import pytest

from oracle import oracle as O
from synth import configs as C
from synth import synth as S
from tests.gpu_harness import LayerRun, compare_out
from tests.oracle_helpers import all_experts

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__
    __graft_entry__.build()


def _dense(base, **kw):
    return C.scaled(base, n_routed=5, top_k=5, dense=True, **kw)


CASES = {
    "tiny-fp32-r2": C.TINY_FP32.with_(rows=2, n_routed=5, top_k=5, dense=True, seed=701),
    "scaled-bf16-r1": _dense(C.FLASH_BF16_R1, seed=702),
    "scaled-bf16-r8": _dense(C.FLASH_BF16_R8, seed=703),
    "scaled-fp8-r4": _dense(C.FLASH_FP8_R4, seed=704),
    "scaled-mxfp4-r3": _dense(C.FLASH_MXFP4_CHAIN4_R8, n_layers=1, rows=3, seed=705),
    "full-bf16-r1": C.DENSE6_BF16_R1,
}


@pytest.mark.parametrize("case", list(CASES))
def test_dense_layer(case):
    wl = CASES[case]
    run = LayerRun(wl)
    got = run.step()
    lw = O.LayerWeights(wl, S.cpu_dense(wl, 0), all_experts(wl, 0))
    out, t = O.layer(wl, lw, S.cpu_hc_in(wl))
    assert run.tap(0, "idx").tolist() == [list(range(wl.top_k))] * wl.rows
    assert np.all(run.tap(0, "w") == 1.0)
    compare_out(wl, run.tap(0, "n"), t.n, "n")
    compare_out(wl, run.tap(0, "y"), t.y, "y")
    compare_out(wl, got, O.decode_hc(wl, out), "hc_out")
    run.close()
