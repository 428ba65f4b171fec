"""The debug build (libfmoe_debug.so: the kernels with device-side bounds checks) on the
GPU (needs a B200): the per-token layer, the expert cache and the static scratch run
with every check on, match the normal build bit for bit, and report no failed check.
It runs in a child process, which loads the debug library through FMOE_SO."""
import os
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import numpy as np, torch, gen
import bit_dequant_expert_router_b200 as fmoe
assert fmoe.lib().fmoe_debug_bounds() == 1
for bits, spec in ((4, gen.tiny_layer(4)), (2, gen.small_layer(2)), (8, gen.tiny_layer(8))):
    hl = gen.host_layer(spec, seed=90 + bits)
    dl = gen.upload_layer(hl)
    lay = gen.binding_layer(dl)
    h = torch.from_numpy(gen.host_tokens(9000, 5, spec.hidden)).cuda()
    ws = fmoe.workspace(fmoe.moe_layer_workspace_size(lay, 5))
    out = fmoe.moe_layer(lay, h, ws=ws)
    fmoe.workspace_check(ws)           # raises FMOE_ERR_DEVICE_BOUNDS on a failed check
    np.save(f"{OUT}/out{bits}.npy", out.cpu().numpy())
# expert cache on the small layer
spec = gen.small_layer(4)
hl = gen.host_layer(spec, seed=97)
dl = gen.upload_layer(hl)
nbytes, off = gen.record_layout(spec.bits, spec.hidden, spec.inter)
routed = fmoe.Bank(None, spec.bits, spec.hidden, spec.inter, spec.experts, nbytes, off)
shared = fmoe.Bank(dl.shared, spec.bits, spec.hidden, spec.inter, 1, nbytes, off)
lay = fmoe.Layer(routed, shared, dl.w_router, dl.w_shared_gate, dl.gamma, None, spec.eps, spec.top_k)
cache = fmoe.ExpertCache(dl.bank.cpu().pin_memory(), spec.experts, nbytes, nbytes, 5)
h = torch.from_numpy(gen.host_tokens(9100, 6, spec.hidden)).cuda()
ws = fmoe.workspace(fmoe.moe_layer_workspace_size(lay, 1))
out = fmoe.moe_layer_cached(lay, cache, h, ws=ws)
fmoe.workspace_check(ws)
cache.stats()
np.save(f"{OUT}/cached.npy", out.cpu().numpy())
print("debug build ok")
'''


def _run(tmp_path, so):
    env = dict(os.environ, FMOE_SO=so, PYTHONPATH=ROOT)
    code = f"OUT = {str(tmp_path)!r}\n" + CHILD
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    return r


def test_debug_build_reports_no_failed_check_and_matches_the_normal_build(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import numpy as np
    import bit_dequant_expert_router_b200.build as pkg_build
    dbg = pkg_build.DEBUG_SO
    if not os.path.exists(dbg):  # built in-tree beside libfmoe.so by __graft_entry__.build()
        dbg = pkg_build.build(debug_bounds=True)
    (tmp_path / "d").mkdir()
    (tmp_path / "n").mkdir()
    _run(tmp_path / "d", dbg)
    # the normal build on the same inputs (its flag query says 0)
    code_n = CHILD.replace("assert fmoe.lib().fmoe_debug_bounds() == 1", "assert fmoe.lib().fmoe_debug_bounds() == 0")
    env = dict(os.environ, PYTHONPATH=ROOT)
    env.pop("FMOE_SO", None)
    r = subprocess.run([sys.executable, "-c", f"OUT = {str(tmp_path / 'n')!r}\n" + code_n], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    for name in ("out4", "out2", "out8", "cached"):
        assert np.array_equal(np.load(tmp_path / "d" / f"{name}.npy"), np.load(tmp_path / "n" / f"{name}.npy")), name
