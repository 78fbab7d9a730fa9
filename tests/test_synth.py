"""The seeded input generator: distributions, determinism, and (on a GPU) that
its device build writes the same bytes as its host build."""

import math

import numpy as np
import pytest

from synth import configs as C
from synth import synth as S


def test_normal_moments_and_ln():
    a = S.cpu_fill(9, 0, S.GATE, 0, (400000,), 0, 0.0, 1.0, "f64")
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1) < 0.01
    assert abs(((a - a.mean()) ** 4).mean() / a.var() ** 2 - 3) < 0.05
    lib = S.cpu_lib()
    for x in (1e-30, 0.001, 0.3, 0.5, 0.70710678, 0.999999, 1.7):
        assert abs(lib.synth_ln_probe(x) - math.log(x)) <= 4e-16 * max(1.0, abs(math.log(x)))


def test_uniform_bias_range():
    b = S.cpu_fill(1, 0, S.ROUTER_BIAS, 0, (100000,), 1, -0.1, 0.1, "f32")
    assert b.min() >= -0.1 and b.max() < 0.1 and abs(b.mean()) < 1e-3


def test_offsets_and_tags_are_counter_based():
    full = S.cpu_fill(3, 2, S.DOWN, 5, (10000,), 0, 0.0, 0.5, "f32")
    part = S.cpu_fill(3, 2, S.DOWN, 5, (1000,), 0, 0.0, 0.5, "f32", offset=4000)
    assert np.array_equal(full[4000:5000], part)
    other = S.cpu_fill(3, 2, S.DOWN, 6, (1000,), 0, 0.0, 0.5, "f32", offset=4000)
    assert not np.array_equal(part, other)
    bf = S.cpu_fill(3, 2, S.DOWN, 5, (10000,), 0, 0.0, 0.5, "bf16")
    import torch
    assert np.array_equal(bf, torch.from_numpy(full).bfloat16().view(torch.int16).numpy().view(np.uint16))


def test_recipe_scales():
    wl = C.scaled(C.FLASH_BF16_R1, hidden=512, n_routed=8, top_k=2, inter=256)
    d = S.cpu_dense(wl, 0)
    assert abs(d["mix_w"].std() * math.sqrt(4 * 512) - 1) < 0.02
    assert abs(d["router_w"].std() * math.sqrt(512) - 1) < 0.03
    nw = (d["norm_w"].astype(np.uint32) << 16).view(np.float32)
    assert abs(nw.mean() - 1) < 0.02 and abs(nw.std() - 0.1) < 0.01


def test_mxfp4_block_spread():
    """mx_spread widens the block scales of a row; spread 0 is the default
    generator, byte for byte."""
    wl = C.scaled(C.FLASH_BF16_R1, hidden=512, n_routed=4, top_k=2, inter=256, w_dtype="mxfp4")
    base = S.cpu_expert(wl, 0, 1)
    same = S.cpu_expert(wl.with_(mx_spread=0), 0, 1)
    wide = S.cpu_expert(wl.with_(mx_spread=20), 0, 1)
    for nm in ("gate", "up", "down"):
        assert np.array_equal(base[nm][0], same[nm][0]) and np.array_equal(base[nm][1], same[nm][1])
        e0, e1 = base[nm][1].astype(int), wide[nm][1].astype(int)
        span0 = (e0.max(axis=1) - e0.min(axis=1)).max()
        span1 = (e1.max(axis=1) - e1.min(axis=1))
        assert span0 <= 4
        # most rows now span more than 2^14, and each block moved down by 0..20
        assert (span1 > 14).mean() > 0.9 and span1.max() <= 20 + span0
        assert ((e0 - e1) >= -1).all() and ((e0 - e1) <= 21).all()


@pytest.mark.gpu
@pytest.mark.parametrize("wdt", ["bf16", "fp8", "mxfp4", "mxfp4-spread"])
def test_device_build_writes_host_bytes(wdt):
    import torch
    S.build(gpu=True)
    spread = 20 if wdt == "mxfp4-spread" else 0
    wdt = wdt.split("-")[0]
    wl = C.scaled(C.FLASH_BF16_R1, hidden=512, n_routed=4, top_k=2, inter=256, w_dtype=wdt, mx_spread=spread)
    dev = S.gpu_experts(wl, 1)
    torch.cuda.synchronize()
    for slot in (0, 4):
        host = S.cpu_expert(wl, 1, slot)
        for nm in ("gate", "up", "down"):
            q, s = dev[nm]
            if wdt == "bf16":
                qh = q[slot].view(torch.int16).cpu().numpy().view(np.uint16)
            else:
                qh = q[slot].cpu().numpy().view(host[nm][0].dtype)
            assert np.array_equal(qh, host[nm][0])
            if s is not None:
                assert np.array_equal(s[slot].cpu().numpy(), host[nm][1])
    dd = S.gpu_dense(wl, 1)
    hd = S.cpu_dense(wl, 1)
    assert np.array_equal(dd["mix_w"].cpu().numpy(), hd["mix_w"])
    assert np.array_equal(dd["router_bias"].cpu().numpy(), hd["router_bias"])
    assert np.array_equal(dd["norm_w"].view(torch.int16).cpu().numpy().view(np.uint16), hd["norm_w"])
    assert np.array_equal(S.gpu_hc_in(wl).view(torch.int16).cpu().numpy().view(np.uint16), S.cpu_hc_in(wl))
