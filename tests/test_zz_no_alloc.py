"""mono_ffn_route_noalloc (router select with no plan and no allocation)
against the fused step's own routing: same normed rows n, same router
weights and bias, two calls in a row; at its size limits against a
float64 restatement of the select; and captured in a CUDA graph.  The file name puts it last in
collection, so that a run stopping at the first failure has run every other
test first; it passes alone in a fresh process and after the others."""

import numpy as np
import pytest

from moe_decode_layer_sm_b200 import binding
from synth import configs as C
from synth import synth as S
from tests.gpu_harness import FP32_MAX_ABS, LayerRun, routing_ok


def _sel(wl, logits, bias):
    lg = np.asarray(logits, np.float64)
    sp = np.maximum(lg, 0.0) + np.log1p(np.exp(-np.abs(lg)))
    return np.sqrt(sp) + np.asarray(bias, np.float64)[None, :]


CASES = {
    "tiny-fp32-r3": lambda: C.TINY_FP32.with_(rows=3),
    "scaled-bf16-r8": lambda: C.scaled(C.FLASH_BF16_R8, seed=611),
    "v41flash-bf16-r8": lambda: C.FLASH_BF16_R8,
}


@pytest.mark.gpu
@pytest.mark.parametrize("case", list(CASES))
def test_route_noalloc_matches_fused_step(case):
    import torch
    wl = CASES[case]()
    run = LayerRun(wl)
    run.step()
    R, K = wl.rows, wl.top_k
    d = S.gpu_dense(wl, 0)
    n = run.taps[0]["n"]
    if wl.round_bf16:
        n = n.to(torch.bfloat16)   # the fused step's n is bf16-valued; exact
    want_idx, want_w = run.tap(0, "idx"), run.tap(0, "w")
    sel = _sel(wl, run.tap(0, "logits"), d["router_bias"].cpu().numpy())
    got = []
    for _ in range(2):   # two calls in a row on one stream
        idx = torch.full((R, K), -1, dtype=torch.int32, device="cuda")
        w = torch.full((R, K), -1.0, dtype=torch.float32, device="cuda")
        binding.route_noalloc(n, d["router_w"], d["router_bias"], K, wl.route_scale, wl.denom_clamp, idx, w)
        torch.cuda.synchronize()
        got.append((idx.cpu().numpy(), w.cpu().numpy()))
    for idx, w in got:
        for r in range(R):
            ok, exempt = routing_ok(idx[r], want_idx[r], sel[r], K)
            assert ok, f"row {r}: noalloc {idx[r]} fused {want_idx[r]}"
            if not exempt:
                assert np.abs(w[r] - want_w[r]).max() <= FP32_MAX_ABS, f"row {r}: w {w[r]} vs {want_w[r]}"
    # the same inputs give the same bytes on the second call
    assert np.array_equal(got[0][0], got[1][0]) and np.array_equal(got[0][1], got[1][1])
    run.close()


def test_route_noalloc_refuses_sizes_beyond_its_scratch():
    """Refusals happen on the host, before any CUDA call."""
    import ctypes
    L = binding.lib()
    null = ctypes.c_void_p(0)
    for rows, E, k, what in [(9, 256, 8, b"rows 9 above the scratch limit 8"),
                             (1, 2048, 8, b"n_routed 2048 outside 1..1024"),
                             (1, 256, 17, b"top_k 17 outside")]:
        rc = L.mono_ffn_route_noalloc(rows, 5120, E, k, null, 1, null, null, 2.5, 1e-20, null, null, null)
        assert rc == -1
        assert what in L.mono_ffn_last_error(None)
    assert L.mono_ffn_route_noalloc(0, 5120, 256, 8, null, 1, null, null, 2.5, 1e-20, null, null, null) == 0


@pytest.mark.gpu
def test_route_noalloc_at_its_limits_against_float64():
    """n_routed 1000 (not a multiple of 32: a partial last lane block, 32 keys
    a lane), top_k 16 and 8 rows, the largest sizes the static scratch takes,
    against the select restated in float64: logits, sqrt(softplus) scores,
    canonical (selection desc, index asc) top-k, weights.  The device
    allocator's free memory is the same before and after the calls."""
    import torch
    g = torch.Generator().manual_seed(1000)
    R, H, E, K = 8, 512, 1000, 16
    n = torch.randn(R, H, generator=g).to(torch.bfloat16)
    rw = (torch.randn(H, E, generator=g) / H ** 0.5).float()
    rb = (torch.rand(E, generator=g) * 0.2 - 0.1).float()
    lg = n.double() @ rw.double()
    sc = torch.sqrt(torch.nn.functional.softplus(lg))
    sel = (sc + rb.double()).numpy()
    want_idx = np.stack([sorted(range(E), key=lambda e: (-sel[r, e], e))[:K] for r in range(R)])
    want_w = np.stack([sc[r, want_idx[r]].numpy() / sc[r, want_idx[r]].numpy().sum() * 2.5 for r in range(R)])
    nd, rwd, rbd = n.cuda(), rw.cuda(), rb.cuda()
    idx = torch.full((R, K), -1, dtype=torch.int32, device="cuda")
    w = torch.zeros((R, K), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(2):
        binding.route_noalloc(nd, rwd, rbd, K, 2.5, 1e-20, idx, w)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    gi, gw = idx.cpu().numpy(), w.cpu().numpy()
    for r in range(R):
        ok, exempt = routing_ok(gi[r], want_idx[r], sel[r].astype(np.float32), K)
        assert ok, f"row {r}: {gi[r]} vs {want_idx[r]}"
        if not exempt:
            assert np.allclose(gw[r], want_w[r], rtol=1e-5, atol=1e-6), (gw[r], want_w[r])


def test_route_noalloc_binding_checks_its_arguments():
    """Wrong dtypes or shapes are refused in Python before any pointer goes
    to the library (no device needed: the checks come first)."""
    import torch
    n = torch.zeros(2, 64, dtype=torch.bfloat16)
    rw = torch.zeros(64, 32)
    rb = torch.zeros(32)
    with pytest.raises(ValueError, match="idx must be int32"):
        binding.route_noalloc(n, rw, rb, 4, 2.5, 1e-20, torch.zeros(2, 4), torch.zeros(2, 4))
    with pytest.raises(ValueError, match=r"\[rows\]\[top_k\]"):
        binding.route_noalloc(n, rw, rb, 4, 2.5, 1e-20, torch.zeros(2, 3, dtype=torch.int32), torch.zeros(2, 3))


@pytest.mark.gpu
def test_route_noalloc_inside_a_captured_graph():
    """The call between captured graph segments, the case it exists for: after
    one eager call (which looks up the scratch), one call is captured into a
    CUDA graph; replaying the graph gives the eager call's bytes, and the
    replays allocate no device memory."""
    import torch
    g = torch.Generator().manual_seed(1001)
    R, H, E, K = 4, 1024, 256, 8
    n = torch.randn(R, H, generator=g).to(torch.bfloat16).cuda()
    rw = (torch.randn(H, E, generator=g) / H ** 0.5).float().cuda()
    rb = (torch.rand(E, generator=g) * 0.2 - 0.1).float().cuda()
    idx0 = torch.full((R, K), -1, dtype=torch.int32, device="cuda")
    w0 = torch.zeros((R, K), dtype=torch.float32, device="cuda")
    binding.route_noalloc(n, rw, rb, K, 2.5, 1e-20, idx0, w0)
    torch.cuda.synchronize()
    idx = torch.full((R, K), -1, dtype=torch.int32, device="cuda")
    w = torch.zeros((R, K), dtype=torch.float32, device="cuda")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        binding.route_noalloc(n, rw, rb, K, 2.5, 1e-20, idx, w)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        idx.fill_(-1)
        w.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(idx, idx0) and torch.equal(w, w0)
    assert torch.cuda.mem_get_info()[0] == free0
    del graph
