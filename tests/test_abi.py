"""The C ABI: library loads, exports every declared symbol, and rejects bad arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

import bit_dequant_expert_router_b200 as fmoe
from bit_dequant_expert_router_b200 import _abi
import gen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(fmoe_[a-z0-9_]+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported_and_bound():
    names = _declared()
    assert len(names) >= 14
    lib = ctypes.CDLL(_abi.SO_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert names == {s[0] for s in _abi.SIGNATURES}


def test_version_and_status_strings():
    L = fmoe.lib()
    assert L.fmoe_version() >= 100
    assert L.fmoe_status_string(0) == b"FMOE_OK"
    assert L.fmoe_status_string(6) == b"FMOE_ERR_DEVICE_TIMEOUT"


@pytest.mark.parametrize("bits,H,I,group", [(4, 4096, 1024, 64), (2, 4096, 1024, 64), (4, 256, 128, 64),
                                             (2, 256, 128, 64), (8, 4096, 1024, 64), (4, 4096, 1024, 128),
                                             (8, 1024, 2048, 128)])
def test_bank_layout_matches_generator_layout(bits, H, I, group):
    assert fmoe.bank_layout(bits, H, I, group) == gen.record_layout(bits, H, I, group)


def _fake_bank(bits=4, H=4096, I=1024, E=512, base=0x10000000, stride=None, off=None, group=64):
    nb, o = gen.record_layout(bits, H, I, group)
    b = _abi.FmoeBank(bits, group, H, I, E, 0, base, nb if stride is None else stride,
                      (ctypes.c_int64 * 9)(*(o if off is None else off)))
    return b


def _fake_layer(**kw):
    k = kw.pop("top_k", 4)
    routed = _fake_bank(**kw)
    shared = _fake_bank(**dict(kw, E=1))
    return _abi.FmoeLayer(routed, shared, 0x20000000, None, 0x30000000, 0x40000000, 1e-6, k)


def _call_layer(layer, T=1, ws=0x50000000, ws_bytes=1 << 30, h=0x60000000, out=0x60000000):
    return fmoe.lib().fmoe_moe_layer(ctypes.byref(layer), h, T, out, None, None, ws, ws_bytes, None)


def test_layer_validation_errors_are_reported_before_any_launch():
    L = fmoe.lib()
    assert L.fmoe_moe_layer(None, 0x1000, 1, 0x1000, None, None, 0x1000, 1 << 20, None) == 1
    assert b"NULL" in L.fmoe_last_error()
    assert _call_layer(_fake_layer(bits=3)) == 3
    assert _call_layer(_fake_layer(top_k=0)) == 1
    assert _call_layer(_fake_layer(top_k=513)) == 1
    assert _call_layer(_fake_layer(top_k=33)) == 1
    assert _call_layer(_fake_layer(H=4000)) == 3
    assert _call_layer(_fake_layer(H=384)) == 3       # H*bits/128 not a power of two
    assert _call_layer(_fake_layer(base=0x10000008)) == 2
    assert _call_layer(_fake_layer(stride=7077888 + 8)) == 2
    off = list(gen.record_layout(4, 4096, 1024)[1])
    off[4] += 4
    assert _call_layer(_fake_layer(off=off)) == 2
    assert _call_layer(_fake_layer(), ws=0x50000010) == 2   # not 256-byte aligned
    assert _call_layer(_fake_layer(), ws_bytes=1024) == 4
    assert _call_layer(_fake_layer(), ws=None) == 4
    assert _call_layer(_fake_layer(), h=0x60000004) == 2
    assert _call_layer(_fake_layer(), T=-1) == 1
    assert _call_layer(_fake_layer(), T=0) == 0            # empty batch: nothing enqueued
    # (top_k + 1) * inter*bits/128 must fit one 512-thread CTA
    assert _call_layer(_fake_layer(top_k=16)) == 3
    # code widths 2, 4, 8 and groups of 64 or 128 pass the format checks (the misaligned
    # base is then what fails); other widths and group sizes do not
    assert _call_layer(_fake_layer(bits=8, base=0x10000008)) == 2
    assert _call_layer(_fake_layer(group=128, base=0x10000008)) == 2
    assert _call_layer(_fake_layer(bits=8, group=128, base=0x10000008)) == 2
    assert _call_layer(_fake_layer(group=96)) == 3
    assert _call_layer(_fake_layer(group=128, H=512, I=512)) == 3   # groups of 128 from hidden 1024 up
    assert _call_layer(_fake_layer(bits=6)) == 3


def test_workspace_size_query_is_positive_and_monotone():
    L = fmoe.lib()
    lay = _fake_layer()
    n4 = L.fmoe_moe_layer_workspace_size(ctypes.byref(lay), 1)
    lay8 = _fake_layer(top_k=8)
    assert n4 > 0 and L.fmoe_moe_layer_workspace_size(ctypes.byref(lay8), 1) >= n4
    assert L.fmoe_router_topk_workspace_size(64, 512) > L.fmoe_router_topk_workspace_size(1, 512)


def test_workspace_sizes_at_the_qwen_shapes():
    """The per-token workspace covers every T below the grouped threshold (8 tokens); from
    there the grouped layout is added.  The figures are the ones the design notes state.
    The query never shrinks as T grows, although the grouped layout alone does (its router
    split shrinks once a batch needs a second tile of 64 tokens): a workspace sized for T
    holds the grouped layout of every smaller batch."""
    L = fmoe.lib()
    for kw in ({}, {"bits": 2}, {"H": 1024, "I": 512, "E": 8}, {"E": 64, "top_k": 8}):
        lay = _fake_layer(**kw)
        size = lambda T: L.fmoe_moe_layer_workspace_size(ctypes.byref(lay), T)
        sizes = [size(T) for T in range(1, 600)]
        assert all(b >= a for a, b in zip(sizes, sizes[1:])), kw
    lay = _fake_layer()
    size = lambda T: L.fmoe_moe_layer_workspace_size(ctypes.byref(lay), T)
    assert [size(T) for T in (1, 2, 7)] == [214016] * 3
    assert size(8) == 1686272 and size(64) == 11982848
    assert size(65) == size(64)          # the T = 65 layout alone needs 11,101,440 bytes
    assert size(1 << 20) > size(600)     # large T: no stall in the query, the size keeps growing
    # FMOE_STATIC_SCRATCH_BYTES holds the per-token layout but not the grouped one at these
    # shapes, so the static entry point runs batches of 8 or more token by token here
    assert size(1) <= 524288 < size(8)


def test_last_error_is_per_host_thread():
    """fmoe_last_error reports the last failure of the calling thread: two threads that fail
    with different messages at the same time each read back their own."""
    import threading
    L = fmoe.lib()
    bad = {"rmsnorm": lambda: L.fmoe_rmsnorm(None, None, 1e-6, 1, 4096, 0x1000, None),
           "layer": lambda: L.fmoe_moe_layer(None, 0x1000, 1, 0x1000, None, None, 0x1000, 1 << 20, None)}
    seen = {}
    for name, call in bad.items():
        assert call() == 1
        seen[name] = L.fmoe_last_error()
    assert seen["rmsnorm"] != seen["layer"]
    start = threading.Barrier(2)
    wrong = []

    def worker(name):
        start.wait()
        for _ in range(2000):
            bad[name]()
            if L.fmoe_last_error() != seen[name]:
                wrong.append(name)
                return

    ts = [threading.Thread(target=worker, args=(n,)) for n in bad]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert not wrong


def test_other_entry_points_validate():
    L = fmoe.lib()
    assert L.fmoe_rmsnorm(0x1000, None, 1e-6, 0, 4096, 0x1000, None) == 0
    assert L.fmoe_rmsnorm(None, None, 1e-6, 1, 4096, 0x1000, None) == 1
    assert L.fmoe_router_topk(0x1000, 0x2000, None, 1, 4096, 512, 0, 0x3000, 0x4000, None, 0x5000, 1 << 20,
                              None) == 1
    assert L.fmoe_router_topk(0x1000, 0x2000, None, 1, 100, 512, 4, 0x3000, 0x4000, None, 0x5000, 1 << 20,
                              None) == 3
    b = _fake_bank()
    assert L.fmoe_expert_ffn(ctypes.byref(b), 512, 0x1000, 0x2000, 0x5000, 1 << 20, None) == 1
    assert L.fmoe_expert_ffn(ctypes.byref(b), -1, 0x1000, 0x2000, 0x5000, 1 << 20, None) == 1
    assert L.fmoe_moe_stack(None, 1, 0x1000, 1, 0x1000, 0x5000, 1 << 20, None) == 1
    assert L.fmoe_workspace_init(None, 100, None) == 4


def test_routed_layer_and_wait_flag_reject_bad_arguments_before_any_launch():
    L = fmoe.lib()
    lay = _fake_layer()
    ok = (ctypes.byref(lay), 0x60000000, 1, 0x70000000, 0x70001000, 0x60000000, 0x50000000, 1 << 30, None)
    # NULL routing, misaligned routing, misaligned h, workspace too small
    assert L.fmoe_moe_layer_routed(ctypes.byref(lay), 0x60000000, 1, None, 0x70001000, 0x60000000, 0x50000000,
                                   1 << 30, None) == 1
    assert L.fmoe_moe_layer_routed(ctypes.byref(lay), 0x60000000, 1, 0x70000002, 0x70001000, 0x60000000, 0x50000000,
                                   1 << 30, None) == 2
    assert L.fmoe_moe_layer_routed(ctypes.byref(lay), 0x60000008, 1, 0x70000000, 0x70001000, 0x60000000, 0x50000000,
                                   1 << 30, None) == 2
    assert L.fmoe_moe_layer_routed(ctypes.byref(lay), 0x60000000, 1, 0x70000000, 0x70001000, 0x60000000, 0x50000000,
                                   1024, None) == 4
    assert L.fmoe_moe_layer_routed(ctypes.byref(lay), 0x60000000, 0, *ok[3:]) == 0
    # the bounded wait: limits outside 1 ns .. 60 s, NULL or misaligned flag or workspace
    assert L.fmoe_wait_flag(0x70000000, 1, 0, 0x50000000, None) == 1
    assert L.fmoe_wait_flag(0x70000000, 1, 61 * 10 ** 9, 0x50000000, None) == 1
    assert L.fmoe_wait_flag(None, 1, 1000, 0x50000000, None) == 1
    assert L.fmoe_wait_flag(0x70000002, 1, 1000, 0x50000000, None) == 2
    assert L.fmoe_wait_flag(0x70000000, 1, 1000, 0x50000010, None) == 2


def test_gdn_step_rejects_bad_arguments_before_any_launch():
    L = fmoe.lib()
    S, q, k, v, a, b, o = 0x60000000, 0x61000000, 0x62000000, 0x63000000, 0x64000000, 0x65000000, 0x66000000
    good = (S, q, k, v, a, b, o)
    assert L.fmoe_gdn_step(*good, 0, 128, 128, 0, None) == 0          # n = 0: nothing enqueued
    assert L.fmoe_gdn_step(*good, -1, 128, 128, 0, None) == 1         # negative n
    assert L.fmoe_gdn_step(*good, 64, 128, 0, 0, None) == 1           # dv < 1
    assert L.fmoe_gdn_step(*good, 64, 128, 128, 2, None) == 1         # unknown flag
    assert L.fmoe_gdn_step(None, *good[1:], 64, 128, 128, 0, None) == 1
    assert L.fmoe_gdn_step(*good[:6], None, 64, 128, 128, 1, None) == 1
    for dk in (64, 96, 200, 640):
        assert L.fmoe_gdn_step(*good, 64, dk, 128, 0, None) == 3      # unsupported key width
    assert L.fmoe_gdn_step(*good, 1 << 20, 128, 4096, 0, None) == 3   # rows beyond 2^31
    assert L.fmoe_gdn_step(S + 8, *good[1:], 64, 128, 128, 0, None) == 2
    assert L.fmoe_gdn_step(S, q + 4, *good[2:], 64, 128, 128, 0, None) == 2
    assert L.fmoe_gdn_step(*good[:3], v + 2, *good[4:], 64, 128, 128, 0, None) == 2
    assert L.fmoe_gdn_step(*good[:6], o + 1, 64, 128, 128, 0, None) == 2


def test_expert_cache_rejects_bad_arguments_before_any_launch():
    L = fmoe.lib()
    assert L.fmoe_expert_cache_state_size(0, 4) == 0
    # header 64 B, three lists of 32 ints, slot_of [512], expert_of [64], last_use [64]
    assert L.fmoe_expert_cache_state_size(512, 64) == 64 + 384 + 2048 + 256 + 256
    C = fmoe.FmoeExpertCache
    ok = dict(host_base=0x7000000000, host_stride=4096, slots=0x60000000, slot_stride=4096, record_bytes=4096,
              num_experts=16, num_slots=4, state=0x61000000)
    assert L.fmoe_expert_cache_reset(None, None) == 1
    assert L.fmoe_expert_cache_reset(ctypes.byref(C(**dict(ok, state=None))), None) == 1
    assert L.fmoe_expert_cache_reset(ctypes.byref(C(**dict(ok, num_slots=0))), None) == 1
    assert L.fmoe_expert_cache_reset(ctypes.byref(C(**dict(ok, record_bytes=4008))), None) == 2
    assert L.fmoe_expert_cache_reset(ctypes.byref(C(**dict(ok, slots=0x60000008))), None) == 2
    assert L.fmoe_expert_cache_reset(ctypes.byref(C(**dict(ok, host_stride=2048))), None) == 1
    # host_base that is not pinned, mapped host memory (here: no device at all)
    assert L.fmoe_expert_cache_reset(ctypes.byref(C(**ok)), None) == 1
    assert L.fmoe_expert_cache_fetch(ctypes.byref(C(**ok)), 0x62000000, 4, None, None) == 1
    assert L.fmoe_moe_layer_cached(None, ctypes.byref(C(**ok)), 0x60000000, 1, 0x60000000, None, None, 0x50000000,
                                   1 << 20, None) == 1


def test_debug_build_exports_the_same_entry_points():
    """libfmoe_debug.so (the bounds-checking build) carries every declared entry point and
    says it is the debug build; libfmoe.so says it is not."""
    import os
    dbg = os.path.join(os.path.dirname(_abi.SO_PATH), "libfmoe_debug.so")
    if not os.path.exists(dbg):
        pytest.skip("libfmoe_debug.so not built")
    L = ctypes.CDLL(dbg)
    for name in _declared():
        assert hasattr(L, name), name
    L.fmoe_debug_bounds.restype = ctypes.c_int
    assert L.fmoe_debug_bounds() == 1
    assert fmoe.lib().fmoe_debug_bounds() == 0
    L.fmoe_status_string.restype = ctypes.c_char_p
    assert L.fmoe_status_string(7) == b"FMOE_ERR_DEVICE_BOUNDS"


def test_binding_refuses_host_tensors_for_the_new_entry_points():
    """The binding only marshals device tensors: host tensors are refused before the library
    is called (no CPU fallback)."""
    t = __import__("torch")
    S = t.zeros((2, 4, 128))
    q = t.zeros((2, 128))
    with pytest.raises(ValueError):
        fmoe.gdn_step(S, q, q, t.zeros((2, 4)), t.zeros(2), t.zeros(2), o=t.zeros((2, 4)))
    with pytest.raises(ValueError):
        fmoe.ExpertCache(t.zeros(1024, dtype=t.uint8), 4, 256, 256, 2)   # not pinned
