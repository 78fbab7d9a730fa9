"""The C-ABI library loads and exports every entry point include/mono_ffn.h
declares (no GPU needed: nothing is called that touches a device)."""

import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "mono_ffn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mono_ffn_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    import __graft_entry__
    from moe_decode_layer_sm_b200 import binding
    from moe_decode_layer_sm_b200 import build as b
    b.build()
    L = binding.lib()
    names = _declared()
    assert "mono_ffn_plan" in names and "mono_ffn_step" in names
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing
    assert set(names) == set(binding.SYMBOLS)
    assert L.mono_ffn_abi_version() == 2
    assert __graft_entry__.ROOT == ROOT


def test_plan_refusal_lists_every_reason_without_a_gpu():
    """With bad arguments the plan refuses before touching the device."""
    from moe_decode_layer_sm_b200 import binding
    L = binding.lib()
    import ctypes
    cfg = binding.Config(hidden=100, hc=3, n_routed=0, top_k=0, inter=0, max_rows=9, n_layers=0, hc_dtype=5,
                         norm_dtype=0, expert_dtype=1, round_bf16=0, sinkhorn_iters=20, device=0)
    h = ctypes.c_void_p()
    rc = L.mono_ffn_plan(ctypes.byref(cfg), ctypes.byref(h))
    assert rc == -1
    msg = L.mono_ffn_last_error(None).decode()
    for frag in ("hc must be 4", "n_routed", "top_k", "max_rows", "n_layers", "hc_dtype"):
        assert frag in msg, (frag, msg)


def test_plan_refuses_sizes_beyond_the_32_bit_work_partition():
    """The kernels partition each work list in 32-bit arithmetic (units x
    grid < 2^31); the plan refuses larger hidden x inter before any device
    call, and takes the largest workload of the pages."""
    from moe_decode_layer_sm_b200 import binding
    L = binding.lib()
    import ctypes

    def reasons(hidden, inter):
        cfg = binding.Config(hidden=hidden, hc=4, n_routed=256, top_k=16, inter=inter, max_rows=8, n_layers=1,
                             hc_dtype=1, norm_dtype=1, expert_dtype=1, round_bf16=1, sinkhorn_iters=20, device=0)
        h = ctypes.c_void_p()
        if L.mono_ffn_plan(ctypes.byref(cfg), ctypes.byref(h)) == 0:   # a GPU machine: the plan is made
            L.mono_ffn_destroy(h)
            return ""
        return L.mono_ffn_last_error(None).decode()

    assert "work partition" in reasons(65536, 65536)
    assert "work partition" not in reasons(5120, 2048)


def test_build_is_keyed_on_the_source_hash(tmp_path, monkeypatch):
    """build() trusts the library only when the stamp beside it holds the
    hash of the current sources and nvcc command; a later modification time
    alone does not count."""
    from moe_decode_layer_sm_b200 import build as b
    b.build()
    assert b.up_to_date()
    stamp = tmp_path / "stamp"
    stamp.write_text("0" * 64 + "\n")
    monkeypatch.setattr(b, "STAMP", str(stamp))
    os.utime(b.SO, None)   # the binary is newer than every source
    assert not b.up_to_date()
    stamp.write_text(b.source_hash() + "\n")
    assert b.up_to_date()
