"""fmoe_moe_layer_static (library-owned static scratch) against fmoe_moe_layer (caller workspace).

Named to be collected last, so it runs both alone and after every other test
has used the device.
"""
import ctypes

import numpy as np
import pytest

import gen
from tests.helpers import max_rel_err, ulp32

torch = pytest.importorskip("torch")

TOL = 2e-3


def _fake_layer(bits, H, I, E, K):
    import bit_dequant_expert_router_b200 as m
    nb, off = gen.record_layout(bits, H, I)
    bank = lambda e: m.FmoeBank(bits, 64, H, I, e, 0, 0x10000000, nb, (ctypes.c_int64 * 9)(*off))
    return m.FmoeLayer(bank(E), bank(1), 0x20000000, None, 0x30000000, 0x40000000, 1e-6, K)


STATIC_BYTES = 524288   # FMOE_STATIC_SCRATCH_BYTES


def test_static_scratch_covers_every_admitted_shape():
    """No shape that passes the layer checks is turned away for scratch size; bad arguments still fail first."""
    import bit_dequant_expert_router_b200 as m
    L = m.lib()
    admitted = 0
    for bits in (2, 4):
        for H in (128, 512, 2048, 8192):
            for I in (128, 1024, 4096, 8192):
                for K in (1, 4, 9, 16, 32):
                    lay = _fake_layer(bits, H, I, 4096, K)
                    # misaligned h: every layer check runs, then the alignment check stops the call
                    st = L.fmoe_moe_layer_static(ctypes.byref(lay), 0x60000008, 1, 0x60000000, None, None, None, None)
                    assert st in (2, 3), (bits, H, I, K, st)
                    if st == 2:
                        admitted += 1
                        assert L.fmoe_moe_layer_workspace_size(ctypes.byref(lay), 1) <= STATIC_BYTES
    assert admitted > 40
    qwen = _fake_layer(4, 4096, 1024, 512, 4)
    assert L.fmoe_moe_layer_workspace_size(ctypes.byref(qwen), 1) == 214016
    assert L.fmoe_moe_layer_static(None, 0x60000000, 1, 0x60000000, None, None, None, None) == 1
    assert L.fmoe_moe_layer_static(ctypes.byref(qwen), 0x60000000, 1, 0x60000000, None, None, 0x70000002, None) == 2
    assert L.fmoe_moe_layer_static(ctypes.byref(qwen), 0x60000000, 0, 0x60000000, None, None, None, None) == 0


def _both(m, lay, h, K):
    T = h.shape[0]
    ref = torch.empty_like(h)
    ref_idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    ref_w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    ws = m.workspace(m.moe_layer_workspace_size(lay, T))
    m.moe_layer(lay, h, out=ref, topk_idx=ref_idx, topk_w=ref_w, ws=ws)
    m.workspace_check(ws)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    runs = []
    for _ in range(2):   # two calls in a row on the same static scratch
        out = torch.empty_like(h)
        idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
        w = torch.empty((T, K), dtype=torch.float32, device="cuda")
        m.moe_layer_static(lay, h, out=out, topk_idx=idx, topk_w=w, dev_err=err)
        runs.append((out, idx, w))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    h64 = h.cpu().numpy().astype(np.float64)
    r = ref.cpu().numpy().astype(np.float64)
    for out, idx, w in runs:
        o = out.cpu().numpy().astype(np.float64)
        assert torch.equal(idx, ref_idx)
        assert max_rel_err(o, r) <= TOL
        assert max_rel_err(o - h64, r - h64, slack=ulp32(o)) <= TOL
        assert np.allclose(w.cpu().numpy(), ref_w.cpu().numpy(), rtol=1e-6, atol=0)


@pytest.mark.gpu
@pytest.mark.parametrize("bits", [4, 2])
def test_static_scratch_matches_workspace_entry_point_tiny(bits):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_dequant_expert_router_b200 as m
    spec = gen.tiny_layer(bits)
    dl = gen.upload_layer(gen.host_layer(spec, seed=11))
    lay = gen.binding_layer(dl)
    h = torch.from_numpy(gen.host_tokens(40, 6, spec.hidden)).cuda()
    _both(m, lay, h, lay.top_k)


@pytest.mark.gpu
def test_static_scratch_matches_workspace_entry_point_full_size():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_dequant_expert_router_b200 as m
    spec = gen.qwen397_layer(4)
    dl = gen.device_layer(spec)
    lay = gen.binding_layer(dl)
    h = gen.device_tokens(3, 2, spec.hidden)
    _both(m, lay, h, lay.top_k)
    del dl
    torch.cuda.empty_cache()


@pytest.mark.gpu
def test_static_scratch_grouped_and_token_by_token_batches():
    """hidden 512: a T = 8 batch's grouped layout fits the static scratch, so it runs
    expert-grouped there; T = 16 does not fit and runs token by token.  Two static calls
    in a row with different T share the scratch.  Both against fmoe_moe_layer."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_dequant_expert_router_b200 as m
    L = m.lib()
    spec = gen.small_layer(4)
    dl = gen.upload_layer(gen.host_layer(spec, seed=41))
    lay = gen.binding_layer(dl)
    assert L.fmoe_moe_layer_workspace_size(ctypes.byref(lay.s), 8) <= STATIC_BYTES
    assert L.fmoe_moe_layer_workspace_size(ctypes.byref(lay.s), 16) > STATIC_BYTES
    _both(m, lay, torch.from_numpy(gen.host_tokens(4100, 8, spec.hidden)).cuda(), lay.top_k)
    _both(m, lay, torch.from_numpy(gen.host_tokens(4200, 16, spec.hidden)).cuda(), lay.top_k)


@pytest.mark.gpu
def test_static_scratch_full_size_batch_runs_token_by_token():
    """The Qwen3.5-397B-A17B-shaped layer with T = 8: the grouped layout exceeds the static
    scratch, so the batch runs token by token, with the results of fmoe_moe_layer."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_dequant_expert_router_b200 as m
    spec = gen.qwen397_layer(4)
    dl = gen.device_layer(spec)
    lay = gen.binding_layer(dl)
    h = gen.device_tokens(4300, 8, spec.hidden)
    # the caller workspace holds only the per-token layout, so both calls run token by token
    T, K = 8, lay.top_k
    ref = torch.empty_like(h)
    ref_idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    ws = m.workspace(m.moe_layer_workspace_size(lay, 1))
    m.moe_layer(lay, h, out=ref, topk_idx=ref_idx, ws=ws)
    m.workspace_check(ws)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(h)
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    m.moe_layer_static(lay, h, out=out, topk_idx=idx, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(idx, ref_idx) and torch.equal(out, ref)
    del dl
    torch.cuda.empty_cache()
