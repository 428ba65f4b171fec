"""The single-kernel path (FMOE_FUSED=1) against the CPU oracle and against the three-kernel path (needs a B200)."""
import numpy as np
import pytest

import gen
import oracle
from tests.helpers import max_rel_err, oracle_layer, oracle_layer_sparse, routing_margin
from tests.test_parity_gpu import TOL, _compare_layer, _run_layer

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fmoe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_dequant_expert_router_b200 as m
    m.lib()
    return m


@pytest.fixture
def fused(monkeypatch):
    monkeypatch.setenv("FMOE_FUSED", "1")


@pytest.mark.parametrize("bits", [4, 2])
def test_fused_tiny_layer_matches_oracle(fmoe, fused, bits):
    spec = gen.LayerSpec(**{**gen.tiny_layer(bits).__dict__, "random_gamma": True})
    hl = gen.host_layer(spec, seed=4)
    dl = gen.upload_layer(hl)
    h = gen.host_tokens(300, 24, spec.hidden)
    out, idx, w = _run_layer(fmoe, dl, h)
    exact, _ = _compare_layer(hl, h, out, idx, w)
    assert exact >= 22


@pytest.mark.parametrize("top_k", [1, 8])
def test_fused_tiny_top1_and_all_experts(fmoe, fused, top_k):
    spec = gen.tiny_layer(4)
    hl = gen.host_layer(spec, seed=6)
    dl = gen.upload_layer(hl)
    h = gen.host_tokens(50, 8, spec.hidden)
    out, idx, w = _run_layer(fmoe, dl, h, top_k=top_k)
    _compare_layer(hl, h, out, idx, w, L=oracle_layer(hl, top_k=top_k))


def test_fused_tiny_stack_matches_oracle(fmoe, fused):
    spec = gen.tiny_layer(4)
    hls = [gen.host_layer(spec, seed=1, layer=l) for l in range(5)]
    lays = [gen.binding_layer(gen.upload_layer(hl)) for hl in hls]
    h_np = gen.host_tokens(20, 3, spec.hidden)
    out = fmoe.moe_stack(lays, torch.from_numpy(h_np).cuda()).cpu().numpy().astype(np.float64)
    ref = h_np.astype(np.float64)
    for hl in hls:
        ref = oracle_layer(hl).forward(ref.astype(np.float32))["out"]
    assert max_rel_err(out, ref) <= TOL


def test_fused_full_size_layer_matches_oracle(fmoe, fused):
    spec = gen.qwen397_layer(4)
    dl = gen.device_layer(spec, seed=0, layer=0)
    T = 2
    h = gen.host_tokens(800, T, spec.hidden)
    out, idx, w = _run_layer(fmoe, dl, h)
    hl0 = gen.host_layer(spec, seed=0, layer=0, experts=[])
    need = set(idx.reshape(-1).tolist())
    for t in range(T):
        x = oracle.rmsnorm(h[t], hl0.gamma, spec.eps)
        logits, _ = routing_margin(hl0.w_router, x, hl0.logit_bias)
        need |= set(np.argsort(-logits, kind="stable")[:spec.top_k].tolist())
    hl = gen.host_layer(spec, seed=0, layer=0, experts=sorted(need))
    _compare_layer(hl, h, out, idx, w, L=oracle_layer_sparse(hl))
    del dl
    torch.cuda.empty_cache()


def test_fused_and_three_kernel_paths_agree_on_a_full_size_stack(fmoe, monkeypatch):
    spec = gen.qwen397_layer(2, zipf=1.1)
    lays = [gen.binding_layer(gen.device_layer(spec, seed=0, layer=l)) for l in range(3)]
    h = gen.device_tokens(900, 2, spec.hidden)
    monkeypatch.setenv("FMOE_FUSED", "1")
    a = fmoe.moe_stack(lays, h)
    b = fmoe.moe_stack(lays, h)  # same workspace epoch logic, a second launch
    monkeypatch.setenv("FMOE_FUSED", "0")
    c = fmoe.moe_stack(lays, h)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    h64 = h.cpu().numpy().astype(np.float64)
    ra, rc = a.cpu().numpy().astype(np.float64), c.cpu().numpy().astype(np.float64)
    assert max_rel_err(ra - h64, rc - h64) <= TOL
    del lays
    torch.cuda.empty_cache()
