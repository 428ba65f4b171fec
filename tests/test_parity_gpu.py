"""GPU path against the CPU oracle, through the C ABI (needs a B200)."""
import numpy as np
import pytest

import gen
import oracle
from tests.helpers import (check_routing, max_rel_err, oracle_layer, oracle_layer_sparse, routing_margin,
                           ulp32)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module")
def fmoe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_dequant_expert_router_b200 as m
    m.lib()
    return m


def _compare_layer(hl, h, gpu_out, gpu_idx, gpu_w, L=None, use_gamma=True):
    """Checks GPU routing (exact unless near-tied) and outputs (out and out - h) against the oracle."""
    spec = hl.spec
    L = L or oracle_layer(hl, gamma=use_gamma)
    free = L.forward(h)
    T, K = gpu_idx.shape
    exact = 0
    for t in range(T):
        x = oracle.rmsnorm(h[t], hl.gamma, spec.eps) if use_gamma else h[t].astype(np.float64)
        logits, delta = routing_margin(hl.w_router, x, hl.logit_bias)
        exact += check_routing(gpu_idx[t], logits, K, delta)
    ref = L.forward(h, force_idx=gpu_idx)  # same experts as the GPU took (identical where not near-tied)
    assert max_rel_err(gpu_out, ref["out"]) <= TOL
    # the MoE part alone; out is stored in fp32, so out - h carries one fp32 ulp of out
    assert max_rel_err(gpu_out - h, ref["out"] - h, slack=ulp32(gpu_out)) <= TOL
    assert np.allclose(gpu_w, ref["w"], rtol=1e-4, atol=1e-6)
    return exact, free


def _run_layer(fmoe, dl, h_np, top_k=None, use_gamma=True, T_per_call=None):
    lay = gen.binding_layer(dl, top_k=top_k, use_gamma=use_gamma)
    h = torch.from_numpy(h_np).cuda()
    T = h.shape[0]
    K = lay.top_k
    out = torch.empty_like(h)
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    ws = fmoe.workspace(fmoe.moe_layer_workspace_size(lay, T))
    fmoe.moe_layer(lay, h, out=out, topk_idx=idx, topk_w=w, ws=ws)
    fmoe.workspace_check(ws)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), idx.cpu().numpy(), w.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("bits", [4, 2, 8])
@pytest.mark.parametrize("random_gamma", [False, True])
def test_tiny_layer_matches_oracle(fmoe, bits, random_gamma):
    spec = gen.LayerSpec(**{**gen.tiny_layer(bits).__dict__, "random_gamma": random_gamma})
    hl = gen.host_layer(spec, seed=0)
    dl = gen.upload_layer(hl)
    h = gen.host_tokens(0, 64, spec.hidden)
    out, idx, w = _run_layer(fmoe, dl, h)
    exact, _ = _compare_layer(hl, h, out, idx, w)
    assert exact >= 60


@pytest.mark.parametrize("top_k", [1, 8])
def test_tiny_layer_top1_and_all_experts(fmoe, top_k):
    spec = gen.tiny_layer(4)
    hl = gen.host_layer(spec, seed=3)
    dl = gen.upload_layer(hl)
    h = gen.host_tokens(100, 16, spec.hidden)
    out, idx, w = _run_layer(fmoe, dl, h, top_k=top_k)
    _compare_layer(hl, h, out, idx, w, L=oracle_layer(hl, top_k=top_k))
    if top_k == 1:
        assert np.all(w == 1.0)


def test_tiny_layer_without_norm_and_with_logit_bias(fmoe):
    spec = gen.LayerSpec(**{**gen.tiny_layer(2).__dict__, "zipf": 1.1})
    hl = gen.host_layer(spec, seed=5)
    dl = gen.upload_layer(hl)
    h = gen.host_tokens(7, 32, spec.hidden)
    out, idx, w = _run_layer(fmoe, dl, h, use_gamma=False)
    _compare_layer(hl, h, out, idx, w, use_gamma=False)


def test_in_place_residual_and_empty_batch(fmoe):
    spec = gen.tiny_layer(4)
    hl = gen.host_layer(spec, seed=1)
    dl = gen.upload_layer(hl)
    lay = gen.binding_layer(dl)
    h_np = gen.host_tokens(0, 8, spec.hidden)
    h = torch.from_numpy(h_np).cuda()
    ref = fmoe.moe_layer(lay, h)
    h2 = h.clone()
    fmoe.moe_layer(lay, h2, out=h2)
    torch.cuda.synchronize()
    assert torch.equal(ref, h2)
    empty = torch.empty((0, spec.hidden), dtype=torch.float32, device="cuda")
    assert fmoe.moe_layer(lay, empty).shape == (0, spec.hidden)


def test_results_are_deterministic(fmoe):
    spec = gen.tiny_layer(2)
    dl = gen.upload_layer(gen.host_layer(spec, seed=2))
    lay = gen.binding_layer(dl)
    h = torch.from_numpy(gen.host_tokens(0, 16, spec.hidden)).cuda()
    a = fmoe.moe_layer(lay, h)
    b = fmoe.moe_layer(lay, h)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("bits", [4, 2, 8])
def test_expert_ffn_matches_oracle(fmoe, bits):
    spec = gen.tiny_layer(bits)
    hl = gen.host_layer(spec, seed=4)
    dl = gen.upload_layer(hl)
    lay = gen.binding_layer(dl)
    L = oracle_layer(hl)
    rng = np.random.default_rng(0)
    for e in (0, 5, 7):
        x = rng.standard_normal(spec.hidden).astype(np.float32)
        y = fmoe.expert_ffn(lay.routed, e, torch.from_numpy(x).cuda()).cpu().numpy()
        ref = oracle.expert_ffn(L.routed, e, x)
        assert max_rel_err(y, ref) <= TOL


def test_rmsnorm_matches_oracle(fmoe):
    rng = np.random.default_rng(1)
    h = rng.standard_normal((5, 4096)).astype(np.float32) * 3
    gamma = (1 + 0.1 * rng.standard_normal(4096)).astype(np.float32)
    y = fmoe.rmsnorm(torch.from_numpy(h).cuda(), torch.from_numpy(gamma).cuda(), 1e-6).cpu().numpy()
    for t in range(5):
        ref = oracle.rmsnorm(h[t], gamma, 1e-6)
        assert np.max(np.abs(y[t] - ref) / np.abs(ref).max()) < 1e-6


@pytest.mark.parametrize("zipf", [0.0, 1.1])
def test_router_topk_matches_oracle(fmoe, zipf):
    spec = gen.qwen397_layer(4, zipf=zipf)
    wr = gen.host_normal_bf16(gen.key(0, 0, gen.EXPERT_LAYER, gen.KIND_ROUTER), 0.02, 512 * 4096).reshape(512, 4096)
    bias = gen.zipf_logit_bias(spec, 0, 0) if zipf else None
    x = np.random.default_rng(2).standard_normal((64, 4096)).astype(np.float32)
    probs = torch.empty((64, 512), dtype=torch.float32, device="cuda")
    idx, w = fmoe.router_topk(torch.from_numpy(x).cuda(), torch.from_numpy(wr.view(np.int16)).cuda(), 4,
                              logit_bias=None if bias is None else torch.from_numpy(bias).cuda(), probs=probs)
    idx, w, probs = idx.cpu().numpy(), w.cpu().numpy(), probs.cpu().numpy()
    exact = 0
    for t in range(64):
        logits, delta = routing_margin(wr, x[t].astype(np.float64), bias)
        exact += check_routing(idx[t], logits, 4, delta)
        p = oracle.softmax(logits)
        assert np.allclose(probs[t], p, rtol=1e-4, atol=1e-7)
        sel = p[idx[t]]
        assert np.allclose(w[t], sel / sel.sum(), rtol=1e-4, atol=1e-6)
    assert exact >= 56


# --------------------------------------------------------------------------- full Qwen3.5-397B-A17B shapes


@pytest.fixture(scope="module", params=[4, 2])
def big(fmoe, request):
    spec = gen.qwen397_layer(request.param, zipf=1.1 if request.param == 2 else 0.0)
    dl = gen.device_layer(spec, seed=0, layer=0)
    torch.cuda.synchronize()
    yield spec, dl
    del dl
    torch.cuda.empty_cache()


def full_size_oracle_layer(spec, h, gpu_idx, seed=0, layer=0):
    """Oracle layer of a full-size spec holding only the records the comparison needs.

    Draws the router and the shared expert, then every expert that either the GPU
    or the exact (fp64) routing of a token selects; the other records stay absent
    (the oracle is never asked for them)."""
    hl0 = gen.host_layer(spec, seed=seed, layer=layer, experts=[])
    need = set(np.asarray(gpu_idx).reshape(-1).tolist())
    for t in range(h.shape[0]):
        x = oracle.rmsnorm(h[t], hl0.gamma, spec.eps)
        logits, _ = routing_margin(hl0.w_router, x, hl0.logit_bias)
        need |= set(np.argsort(-logits, kind="stable")[:spec.top_k].tolist())
    hl = gen.host_layer(spec, seed=seed, layer=layer, experts=sorted(need))
    return hl, oracle_layer_sparse(hl)


def test_full_size_layer_matches_oracle(fmoe, big):
    """32 fresh tokens of the Qwen3.5-397B-A17B-shaped layer (4-bit; 2-bit with Zipf
    routing), every token against the oracle: routing exact wherever the top K+1
    logits are separated (at least 30 of 32 tokens), outputs within 2e-3."""
    spec, dl = big
    T = 32
    h = gen.host_tokens(500, T, spec.hidden)
    out, idx, w = _run_layer(fmoe, dl, h)
    hl, L = full_size_oracle_layer(spec, h, idx)
    # the device-drawn bytes of the experts compared equal the host-drawn ones
    nbytes = gen.record_bytes(spec)
    for e in sorted(hl.routed):
        dev = dl.bank[e * nbytes:(e + 1) * nbytes].cpu().numpy()
        assert np.array_equal(dev, hl.routed[e]), e
    assert np.array_equal(dl.shared.cpu().numpy(), hl.shared)
    assert np.array_equal(dl.w_router.cpu().numpy().view(np.uint16), hl.w_router)
    exact, _ = _compare_layer(hl, h, out, idx, w, L=L)
    assert exact >= 30, exact


def test_full_size_expert_ffn_matches_oracle(fmoe, big):
    spec, dl = big
    lay = gen.binding_layer(dl)
    hl = gen.host_layer(spec, seed=0, layer=0, experts=[17])
    L = oracle_layer_sparse(hl)
    x = np.random.default_rng(9).standard_normal(spec.hidden).astype(np.float32)
    y = fmoe.expert_ffn(lay.routed, 17, torch.from_numpy(x).cuda()).cpu().numpy()
    assert max_rel_err(y, oracle.expert_ffn(L.routed, 17, x)) <= TOL


def test_stack_of_layers_matches_oracle(fmoe):
    spec = gen.tiny_layer(2)
    hls = [gen.host_layer(spec, seed=0, layer=l) for l in range(4)]
    lays = [gen.binding_layer(gen.upload_layer(hl)) for hl in hls]
    h_np = gen.host_tokens(0, 4, spec.hidden)
    out = fmoe.moe_stack(lays, torch.from_numpy(h_np).cuda()).cpu().numpy().astype(np.float64)
    ref = h_np.astype(np.float64)
    for hl in hls:
        ref = oracle_layer(hl).forward(ref.astype(np.float32))["out"]
    # fp32 inputs between layers on the oracle side; routing of this seed has no near-ties
    assert max_rel_err(out, ref) <= TOL


# --------------------------------------------------------------------------- the two-kernel per-token path


@pytest.fixture
def two_kernels(monkeypatch):
    monkeypatch.setenv("FMOE_TOKEN_KERNELS", "2")


@pytest.mark.parametrize("bits", [4, 2])
def test_two_kernel_path_small_layer(fmoe, two_kernels, bits):
    """hidden 512, intermediate 512 (the smallest rows the two-kernel path stages), 16
    experts, top-4, random gamma: 32 tokens against the oracle."""
    spec = gen.LayerSpec(**{**gen.small_layer(bits).__dict__, "random_gamma": True})
    hl = gen.host_layer(spec, seed=21)
    dl = gen.upload_layer(hl)
    h = gen.host_tokens(2100, 32, spec.hidden)
    out, idx, w = _run_layer(fmoe, dl, h)
    exact, _ = _compare_layer(hl, h, out, idx, w)
    assert exact >= 30


@pytest.mark.parametrize("top_k", [1, 15])
def test_two_kernel_path_top1_and_nearly_all_experts(fmoe, two_kernels, top_k):
    spec = gen.small_layer(4)
    hl = gen.host_layer(spec, seed=22)
    dl = gen.upload_layer(hl)
    h = gen.host_tokens(2200, 6, spec.hidden)
    out, idx, w = _run_layer(fmoe, dl, h, top_k=top_k)
    _compare_layer(hl, h, out, idx, w, L=oracle_layer(hl, top_k=top_k))


@pytest.mark.parametrize("bits", [4, 2])
def test_two_kernel_path_expert_ffn(fmoe, two_kernels, bits):
    spec = gen.small_layer(bits)
    hl = gen.host_layer(spec, seed=23)
    dl = gen.upload_layer(hl)
    lay = gen.binding_layer(dl)
    L = oracle_layer(hl)
    rng = np.random.default_rng(23)
    for e in (0, 15):
        x = rng.standard_normal(spec.hidden).astype(np.float32)
        y = fmoe.expert_ffn(lay.routed, e, torch.from_numpy(x).cuda()).cpu().numpy()
        assert max_rel_err(y, oracle.expert_ffn(L.routed, e, x)) <= TOL


def test_two_kernel_path_full_size(fmoe, big, two_kernels):
    """The Qwen3.5-397B-A17B-shaped layer (4-bit; 2-bit with Zipf routing), 16 fresh
    tokens against the oracle."""
    spec, dl = big
    T = 16
    h = gen.host_tokens(2500, T, spec.hidden)
    out, idx, w = _run_layer(fmoe, dl, h)
    hl, L = full_size_oracle_layer(spec, h, idx)
    exact, _ = _compare_layer(hl, h, out, idx, w, L=L)
    assert exact >= 14, exact


def test_eight_bit_small_layer_batch_runs_token_by_token(fmoe):
    """8-bit codes (one of the formats the gillilab page lists): a 16-token batch of the
    hidden-512 layer, which the grouped path does not take at 8 bits, against the oracle."""
    spec = gen.LayerSpec(**{**gen.small_layer(8).__dict__, "random_gamma": True})
    hl = gen.host_layer(spec, seed=81)
    dl = gen.upload_layer(hl)
    h = gen.host_tokens(8100, 16, spec.hidden)
    out, idx, w = _run_layer(fmoe, dl, h)
    exact, _ = _compare_layer(hl, h, out, idx, w)
    assert exact >= 15


def test_eight_bit_full_size_layer(fmoe):
    """The Qwen3.5-397B-A17B-shaped layer with 8-bit codes: 16 fresh tokens against the oracle."""
    spec = gen.qwen397_layer(8)
    dl = gen.device_layer(spec, seed=0, layer=0)
    T = 16
    h = gen.host_tokens(8200, T, spec.hidden)
    out, idx, w = _run_layer(fmoe, dl, h)
    hl, L = full_size_oracle_layer(spec, h, idx)
    nbytes = gen.record_bytes(spec)
    e = int(idx[0, 0])
    assert np.array_equal(dl.bank[e * nbytes:(e + 1) * nbytes].cpu().numpy(), hl.routed[e])
    exact, _ = _compare_layer(hl, h, out, idx, w, L=L)
    assert exact >= 14
    del dl
    torch.cuda.empty_cache()


@pytest.mark.parametrize("bits", [4, 2, 8])
def test_group_128_layer_matches_oracle(fmoe, bits):
    """Weights grouped by 128 columns (the gillilab page gives groups of 128 or 64): hidden
    and intermediate 1024, 8 experts, top-2, 16 tokens against the oracle."""
    spec = gen.LayerSpec(hidden=1024, experts=8, inter=1024, top_k=2, bits=bits, group=128,
                         router_std=1.0 / 32.0, random_gamma=True)
    hl = gen.host_layer(spec, seed=128 + bits)
    dl = gen.upload_layer(hl)
    h = gen.host_tokens(12800, 16, spec.hidden)
    out, idx, w = _run_layer(fmoe, dl, h)
    exact, _ = _compare_layer(hl, h, out, idx, w)
    assert exact >= 15
    lay = gen.binding_layer(dl)
    L = oracle_layer(hl)
    x = np.random.default_rng(bits).standard_normal(spec.hidden).astype(np.float32)
    y = fmoe.expert_ffn(lay.routed, 3, torch.from_numpy(x).cuda()).cpu().numpy()
    assert max_rel_err(y, oracle.expert_ffn(L.routed, 3, x)) <= TOL


def test_group_128_full_size_layer(fmoe):
    """The Qwen3.5-397B-A17B-shaped 4-bit layer with groups of 128: 16 fresh tokens."""
    spec = gen.LayerSpec(**{**gen.qwen397_layer(4).__dict__, "group": 128})
    dl = gen.device_layer(spec, seed=0, layer=0)
    T = 16
    h = gen.host_tokens(12900, T, spec.hidden)
    out, idx, w = _run_layer(fmoe, dl, h)
    hl, L = full_size_oracle_layer(spec, h, idx)
    exact, _ = _compare_layer(hl, h, out, idx, w, L=L)
    assert exact >= 14
    del dl
    torch.cuda.empty_cache()
