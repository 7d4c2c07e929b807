"""Host-only checks of the C ABI (no GPU needed, no kernel launched).

The library loads, exports every function include/coli.h declares, and rejects
bad arguments on the host before touching CUDA.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def coli():
    from int4_routed_expert_bias_b200 import _build
    _build.build()
    import int4_routed_expert_bias_b200 as m
    return m


def declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"COLI_API\s+[\w\s\*]+?\b(coli_\w+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ("coli_router_topk", "coli_expert_union", "coli_moe_workspace_size", "coli_moe_forward",
              "coli_status_string", "coli_last_error", "coli_moe_profile_next", "coli_moe_path"):
        assert n in names


def test_library_exports_every_declared_symbol(coli):
    lib = coli.lib()
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_status_strings(coli):
    assert coli.status_string(0) == "COLI_OK"
    assert coli.status_string(3) == "COLI_ERR_WORKSPACE"
    assert coli.status_string(99) == "COLI_ERR_UNKNOWN"


def _layer(coli, **over):
    fake = 1 << 20  # non-null, aligned host integers: never dereferenced by argument checks
    kw = dict(hidden=6144, ffn=2048, n_experts=256, top_k=8, group=64, routed_scale=2.5,
              w_router=fake, sel_bias=fake, gate_q=fake, up_q=fake, down_q=fake,
              gate_s=fake, up_s=fake, down_s=fake)
    kw.update(over)
    s = coli._LayerStruct()
    for k, v in kw.items():
        setattr(s, k, v)
    return s


def _fwd(coli, s, T=1, x=1 << 20, out=1 << 20, ws=1 << 20, ws_bytes=1 << 40, xt=0, ot=0):
    return coli.lib().coli_moe_forward(ctypes.byref(s), x, xt, T, out, ot, ws, ws_bytes, None, None, None)


def test_workspace_size_is_positive_and_grows(coli):
    s = _layer(coli)
    w1 = coli.lib().coli_moe_workspace_size(ctypes.byref(s), 1)
    w64 = coli.lib().coli_moe_workspace_size(ctypes.byref(s), 64)
    assert 0 < w1 < w64
    assert coli.lib().coli_moe_workspace_size(None, 1) == 0
    assert coli.lib().coli_moe_workspace_size(ctypes.byref(_layer(coli, hidden=100)), 1) == 0


def test_status_word_offset(coli):
    """The device status word sits inside the workspace of the call it belongs
    to, 4-byte aligned; calls that do not write it (empty batches, invalid
    layers) report none."""
    none = ctypes.c_size_t(-1).value
    lib = coli.lib()
    s = _layer(coli)
    for T in (1, 2, 4, 64, 65, 4096):
        off = lib.coli_moe_status_word_offset(ctypes.byref(s), T)
        assert off != none and off % 4 == 0
        assert off + 4 <= lib.coli_moe_workspace_size(ctypes.byref(s), T)
    assert lib.coli_moe_status_word_offset(ctypes.byref(s), 0) == none
    assert lib.coli_moe_status_word_offset(None, 4) == none
    assert lib.coli_moe_status_word_offset(ctypes.byref(_layer(coli, hidden=100)), 4) == none
    small = _layer(coli, hidden=1024, ffn=512, n_experts=64)
    assert lib.coli_moe_status_word_offset(ctypes.byref(small), 1) != none
    # the Python binding maps "none" to None
    L = coli.Layer.__new__(coli.Layer)
    L.struct = s
    assert coli.moe_status_word_offset(L, 0) is None
    assert coli.moe_status_word_offset(L, 4) == lib.coli_moe_status_word_offset(ctypes.byref(s), 4)


@pytest.mark.parametrize("over,status", [
    (dict(hidden=100), 1), (dict(hidden=0), 1), (dict(ffn=96), 1), (dict(top_k=0), 1),
    (dict(top_k=33), 1), (dict(n_experts=4, top_k=8), 1), (dict(n_experts=2000), 1),
    (dict(group=128), 2), (dict(hidden=32768), 2), (dict(w_router=0), 1), (dict(gate_q=(1 << 20) + 8), 1),
    (dict(routed_scale=float("inf")), 1), (dict(top_p=-0.5), 1), (dict(top_p=float("nan")), 1),
    (dict(act_int8=2), 1), (dict(act_int8=-1), 1),
])
def test_forward_rejects_bad_layers(coli, over, status):
    assert _fwd(coli, _layer(coli, **over)) == status
    assert coli.last_error() != ""


def test_int8_activations_only_in_the_decode_kernel(coli):
    """The integer-activation variant runs in the fused decode kernel; a batch
    that goes to another chain is refused before anything is launched."""
    s = _layer(coli, act_int8=1)
    assert _fwd(coli, s, T=65) == 2
    assert "act_int8" in coli.last_error()
    assert _fwd(coli, s, T=4096) == 2


def test_forward_rejects_bad_calls(coli):
    s = _layer(coli)
    assert _fwd(coli, s, T=-1) == 1
    assert _fwd(coli, s, T=70000) == 1
    assert _fwd(coli, s, xt=7) == 1
    assert _fwd(coli, s, ot=7) == 1
    assert _fwd(coli, s, x=0) == 1
    assert _fwd(coli, s, x=(1 << 20) + 4) == 1
    assert _fwd(coli, s, ws=(1 << 20) + 16) == 1
    need = coli.lib().coli_moe_workspace_size(ctypes.byref(s), 1)
    assert _fwd(coli, s, ws_bytes=need - 1) == 3
    assert "workspace" in coli.last_error()


def _fwd_host(coli, s, T=1, xh=1 << 21, xd=1 << 20, oh=1 << 21, od=1 << 20, ws=1 << 20, ws_bytes=1 << 30):
    L = coli.lib()
    return L.coli_moe_forward_host(ctypes.byref(s), xh, xd, 0, T, oh, od, 0, ws, ws_bytes, None)


def test_forward_host_rejects_bad_calls(coli):
    # every argument is checked before anything is enqueued (no CUDA call is made for these)
    s = _layer(coli)
    assert _fwd_host(coli, s, xh=0) == 1
    assert _fwd_host(coli, s, oh=0) == 1
    assert _fwd_host(coli, s, xd=0) == 1
    assert _fwd_host(coli, s, od=(1 << 20) + 4) == 1
    assert _fwd_host(coli, s, ws=(1 << 20) + 16) == 1
    assert _fwd_host(coli, s, T=-1) == 1
    need = coli.lib().coli_moe_workspace_size(ctypes.byref(s), 1)
    assert _fwd_host(coli, s, ws_bytes=need - 1) == 3
    assert _fwd_host(coli, s, T=0, xh=0, oh=0, xd=0, od=0, ws=0, ws_bytes=0) == 0


def test_forward_checks_the_lookahead_layer(coli):
    s, n = _layer(coli), _layer(coli, gate_q=0)
    s.prefetch_next = ctypes.addressof(n)
    assert _fwd(coli, s) == 1
    assert "prefetch_next" in coli.last_error()
    n2 = _layer(coli, group=32)
    s.prefetch_next = ctypes.addressof(n2)
    assert _fwd(coli, s) == 2
    s.prefetch_next = ctypes.addressof(s)  # a layer may name itself: the check does not follow the chain
    assert _fwd(coli, s, ws_bytes=1) == 3


def test_empty_forward_is_ok_without_launching(coli):
    assert _fwd(coli, _layer(coli), T=0, x=0, out=0, ws=0, ws_bytes=0) == 0


def test_router_rejects_bad_calls(coli):
    L = coli.lib()
    fake = 1 << 20
    assert L.coli_router_topk(fake, 0, 1, 100, fake, fake, 256, 8, 2.5, fake, fake, None) == 1
    assert L.coli_router_topk(fake, 0, 1, 6144, fake, fake, 4, 8, 2.5, fake, fake, None) == 1
    assert L.coli_router_topk(fake, 3, 1, 6144, fake, fake, 256, 8, 2.5, fake, fake, None) == 1
    assert L.coli_router_topk(None, 0, 1, 6144, fake, fake, 256, 8, 2.5, fake, fake, None) == 1
    assert L.coli_router_topk(fake + 4, 0, 1, 6144, fake, fake, 256, 8, 2.5, fake, fake, None) == 1
    assert L.coli_router_topk(fake, 0, 1, 6144, fake, fake, 256, 8, float("nan"), fake, fake, None) == 1
    assert L.coli_router_topk(None, 0, 0, 6144, None, None, 256, 8, 2.5, None, None, None) == 0


def test_union_rejects_bad_calls(coli):
    L = coli.lib()
    fake = 1 << 20
    assert L.coli_expert_union(fake, -1, 8, 256, fake, fake, fake, fake, fake, fake, None) == 1
    assert L.coli_expert_union(fake, 1, 0, 256, fake, fake, fake, fake, fake, fake, None) == 1
    assert L.coli_expert_union(fake, 1, 8, 4, fake, fake, fake, fake, fake, fake, None) == 1
    assert L.coli_expert_union(fake, 1, 8, 256, None, fake, fake, fake, fake, fake, None) == 1
    assert L.coli_expert_union(None, 1, 8, 256, fake, fake, fake, fake, fake, fake, None) == 1


def test_path_choice(coli):
    """The kernel chain is chosen from the shapes alone, the same way the
    forward call and the status-word query see it."""
    L = coli.Layer.__new__(coli.Layer)
    L.struct = _layer(coli)
    assert [coli.moe_path(L, T) for T in (0, 1, 2, 64, 65, 4096)] == \
        ["none", "single", "decode", "decode", "prefill", "prefill"]
    L.struct = _layer(coli, hidden=256, ffn=128, n_experts=16, top_k=4)
    assert coli.moe_path(L, 130) == "wide"    # ffn not a multiple of 256: CUDA-core expert phases
    assert coli.moe_path(L, 1) == "single"
    assert coli.moe_path(L, 64) == "decode"
    # the decode kernel's shared memory (activations, union tables) does not fit: expert phases
    L.struct = _layer(coli, hidden=16384, ffn=16384, n_experts=1024, top_k=32)
    assert coli.moe_path(L, 64) == "wide"
    L.struct = _layer(coli, hidden=256, ffn=256, n_experts=16, top_k=4)
    assert coli.moe_path(L, 130) == "prefill"
    L.struct = _layer(coli, hidden=100)
    assert coli.moe_path(L, 4) == "none"


def test_wait_limit_hook_takes_any_value(coli):
    coli.debug_set_wait_ns(1000)
    coli.debug_set_wait_ns(0)  # the built-in limit again


def test_profile_hook_arms_and_disarms(coli):
    L = coli.lib()
    assert L.coli_moe_profile_next(None, 0) == 0
    assert L.coli_moe_profile_next(1 << 20, -1) == 1
