"""Conditioning of a chain of layers, measured with the oracle alone (CPU).

A layer's output is rounded to bf16 at several points (collapse, norm,
gate/up, the routed+shared sum, the expand).  When two correct computations
of a layer round one value to neighbouring bf16 numbers, the next layer sees
inputs one spacing apart.  These tests measure what such a one-spacing
difference does to the rest of a chain, using nothing but the oracle: it is
the reason a chain is compared layer by layer, on the residual streams the
computation under test produced, at the single-layer tolerance, and end to
end only in relative L2.

The layer's definition (ds4 "v41: fuse the single-box decode glue", HC and
MoE fusion commits; SGLang "[DeepSeek-V4] Add mhc_fused_post_pre kernel",
Modifications: the deferred post equals the op-by-op result) fixes the
roundings; the 5e-2 max-abs and 2e-2 relative-L2 bounds are the tolerances
of one layer's bf16 result."""

import numpy as np
import pytest

from oracle import oracle as O
from synth import configs as C
from synth import synth as S
from tests.oracle_helpers import all_experts

BF16_MAX_ABS = 5e-2
BF16_REL_L2 = 2e-2


def _bump(x, flat_index, step):
    """x: raw bf16 codes.  Move one element to its neighbour (one spacing)."""
    y = x.copy()
    y.flat[flat_index] = np.uint16(int(y.flat[flat_index]) + step)
    return y


@pytest.fixture(scope="module")
def chain_case():
    wl = C.scaled(C.FLASH_MXFP4_CHAIN4_R8, w_dtype="bf16", seed=402, rows=8)
    lws = [O.LayerWeights(wl, S.cpu_dense(wl, l), all_experts(wl, l)) for l in range(wl.n_layers)]
    return wl, lws


def _run(wl, lws, x, first=0):
    for l in range(first, wl.n_layers):
        x, _ = O.layer(wl, lws[l], x)
    return x


def test_one_spacing_after_layer_0_moves_the_chain_beyond_one_layer_tolerance(chain_case):
    """Change ONE of the 8 x 4 x 1024 residual values after layer 0 by one
    bf16 spacing and run layers 1-3 with the oracle: in at least one of four
    seeded trials the end result moves by more than the single-layer max-abs
    bound, while staying far inside the relative-L2 bound.  So an end-to-end
    max-abs comparison of a chain at one layer's tolerance demands that every
    bf16 rounding of the three later layers agrees bit for bit."""
    wl, lws = chain_case
    x1, _ = O.layer(wl, lws[0], S.cpu_hc_in(wl))
    ref = O.decode_hc(wl, _run(wl, lws, x1, first=1))
    rng = np.random.default_rng(7)
    worst, rels = 0.0, []
    for _ in range(4):
        i = int(rng.integers(x1.size))
        got = O.decode_hc(wl, _run(wl, lws, _bump(x1, i, 1), first=1))
        d = np.abs(got - ref)
        worst = max(worst, float(d.max()))
        rels.append(float(np.linalg.norm(got - ref) / np.linalg.norm(ref)))
    assert worst > BF16_MAX_ABS, worst
    assert max(rels) < BF16_REL_L2 / 4, rels


def test_one_spacing_before_the_last_layer_stays_inside_one_layer_tolerance(chain_case):
    """The same one-spacing change in front of the LAST layer only: the
    output moves by at most a few spacings, inside the single-layer bound.
    The growth above comes from the layers the difference travels through."""
    wl, lws = chain_case
    x = S.cpu_hc_in(wl)
    for l in range(wl.n_layers - 1):
        x, _ = O.layer(wl, lws[l], x)
    ref = O.decode_hc(wl, _run(wl, lws, x, first=wl.n_layers - 1))
    rng = np.random.default_rng(7)
    for _ in range(4):
        i = int(rng.integers(x.size))
        got = O.decode_hc(wl, _run(wl, lws, _bump(x, i, 1), first=wl.n_layers - 1))
        assert np.abs(got - ref).max() <= BF16_MAX_ABS
