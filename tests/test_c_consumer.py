"""A plain C11 program built against include/*.h and linked with libfmoe.so (no GPU needed).

The headers must serve a C caller with no CUDA or C++ headers around it, and the structs
must have one layout for that caller, for the library (built as C++ by nvcc) and for the
Python binding (ctypes).  tests/c_consumer.c makes the host-only calls and prints what it
sees; this test builds it with gcc (warnings as errors), runs it, and compares.
"""
import ctypes
import os
import shutil
import subprocess

import pytest

import bit_dequant_expert_router_b200 as fmoe
from bit_dequant_expert_router_b200 import _abi
import gen

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
INC = os.path.join(ROOT, "include")


def _run_consumer(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(_abi.SO_PATH)
    exe = tmp_path / "c_consumer"
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Wextra", "-Wpedantic", "-Werror", "-I", INC,
                           os.path.join(HERE, "c_consumer.c"), "-o", str(exe), "-L", libdir, "-lfmoe",
                           f"-Wl,-rpath,{libdir}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    vals = {}
    for line in out.stdout.splitlines():
        key, _, rest = line.partition(" ")
        vals[key] = rest
    return vals


def test_c_caller_sees_the_binding_layout_and_results(tmp_path):
    v = _run_consumer(tmp_path)
    L = fmoe.lib()
    assert int(v["version"]) == L.fmoe_version()
    # one struct layout for C, for the library and for ctypes
    assert int(v["sizeof_bank"]) == ctypes.sizeof(_abi.FmoeBank)
    assert int(v["sizeof_layer"]) == ctypes.sizeof(_abi.FmoeLayer)
    assert int(v["sizeof_cache"]) == ctypes.sizeof(_abi.FmoeExpertCache)
    assert int(v["offsetof_bank_base"]) == _abi.FmoeBank.base.offset
    assert int(v["offsetof_bank_off"]) == _abi.FmoeBank.off.offset
    assert int(v["offsetof_layer_shared"]) == _abi.FmoeLayer.shared.offset
    assert int(v["offsetof_layer_eps"]) == _abi.FmoeLayer.eps.offset
    assert int(v["offsetof_layer_top_k"]) == _abi.FmoeLayer.top_k.offset
    assert int(v["offsetof_cache_num_experts"]) == _abi.FmoeExpertCache.num_experts.offset
    assert int(v["offsetof_cache_state"]) == _abi.FmoeExpertCache.state.offset
    # status names, constants
    for k in range(8):
        assert v[f"status_{k}"] == _abi.STATUS_NAMES[k]
    assert int(v["static_scratch_bytes"]) == 524288 and int(v["gdn_state_early"]) == 1
    # layout and size queries agree with the binding and the generator
    nb, off = gen.record_layout(4, 4096, 1024)
    assert int(v["record_bytes_4bit"]) == nb
    assert [int(x) for x in v["record_off_4bit"].split()] == list(off)
    assert int(v["record_bytes_2bit"]) == gen.record_layout(2, 4096, 1024)[0] == 3932160
    nb4 = gen.record_layout(4, 4096, 1024)
    bank = lambda E: _abi.FmoeBank(4, 64, 4096, 1024, E, 0, 0x10000000, nb4[0], (ctypes.c_int64 * 9)(*nb4[1]))
    lay = _abi.FmoeLayer(bank(512), bank(1), 0x20000000, None, 0x30000000, 0x40000000, 1e-6, 4)
    assert int(v["layer_ws_1"]) == L.fmoe_moe_layer_workspace_size(ctypes.byref(lay), 1)
    assert int(v["layer_ws_64"]) == L.fmoe_moe_layer_workspace_size(ctypes.byref(lay), 64)
    assert int(v["router_ws_1_512"]) == L.fmoe_router_topk_workspace_size(1, 512)
    assert int(v["ffn_ws"]) == L.fmoe_expert_ffn_workspace_size(ctypes.byref(lay.routed))
    assert int(v["cache_state_512_64"]) == L.fmoe_expert_cache_state_size(512, 64)
    # argument errors: status codes and a message, nothing enqueued
    assert int(v["null_layer"]) == 1 and v["null_layer_message"] == "set"
    assert int(v["empty_batch"]) == 0
    assert int(v["short_workspace"]) == 4
    assert int(v["bad_top_k"]) == 1
    assert int(v["gdn_null_state"]) == 1


def test_headers_compile_as_c_and_as_cxx(tmp_path):
    """Every header stands alone, in C (c99 and c11) and in C++, with warnings as errors."""
    for cc, std in (("gcc", "c99"), ("gcc", "c11"), ("g++", "c++17")):
        if shutil.which(cc) is None:
            pytest.skip(f"no {cc}")
        for h in sorted(os.listdir(INC)):
            if not h.endswith(".h"):
                continue
            src = tmp_path / f"only_{h}.{'cc' if cc == 'g++' else 'c'}"
            src.write_text(f'#include "{h}"\nint fmoe_header_probe(void) {{ return 0; }}\n')
            subprocess.check_call([cc, f"-std={std}", "-Wall", "-Wextra", "-Wpedantic", "-Werror", "-I", INC,
                                   "-fsyntax-only", str(src)])
