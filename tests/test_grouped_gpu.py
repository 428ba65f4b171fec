"""The expert-grouped batched path (T >= 8 tokens of one layer) against the CPU oracle and the per-token path."""
import numpy as np
import pytest

import gen
import oracle
from tests.helpers import max_rel_err, oracle_layer, oracle_layer_sparse, routing_margin, check_routing, ulp32
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


@pytest.mark.parametrize("bits", [4, 2])
def test_grouped_small_batch_matches_oracle(fmoe, bits):
    # 64 tokens over 16 experts: every expert's group spans many work units
    spec = gen.LayerSpec(**{**gen.small_layer(bits).__dict__, "random_gamma": True})
    hl = gen.host_layer(spec, seed=12)
    dl = gen.upload_layer(hl)
    h = gen.host_tokens(700, 64, spec.hidden)
    out, idx, w = _run_layer(fmoe, dl, h)
    exact, _ = _compare_layer(hl, h, out, idx, w)
    assert exact >= 60


@pytest.mark.parametrize("bits", [4, 2])
def test_grouped_longer_rows(fmoe, monkeypatch, bits):
    """hidden 1024 and intermediate 2048: other staged-row widths, items and K slices than
    the 512-wide layer (gate/up 16 groups per row, down 32).  The per-token path gives the
    same routing and, summing in another order, not the same bits: the batch ran grouped."""
    # (top-2: the per-token down kernel holds (K + 1) * 32 groups of digits, at most 128)
    spec = gen.LayerSpec(hidden=1024, experts=16, inter=2048, top_k=2, bits=bits, router_std=1.0 / 32.0,
                         random_gamma=True)
    hl = gen.host_layer(spec, seed=17)
    dl = gen.upload_layer(hl)
    h = gen.host_tokens(1700, 24, spec.hidden)
    out, idx, w = _run_layer(fmoe, dl, h)
    _compare_layer(hl, h, out, idx, w)
    monkeypatch.setenv("FMOE_GROUPED", "0")
    out1, idx1, _ = _run_layer(fmoe, dl, h)
    assert np.array_equal(idx, idx1) and not np.array_equal(out, out1)


def test_grouped_small_batch_top1_all_experts_and_odd_size(fmoe):
    spec = gen.small_layer(4, experts=8, top_k=2)
    hl = gen.host_layer(spec, seed=13)
    dl = gen.upload_layer(hl)
    for top_k, T in ((1, 9), (8, 23)):
        h = gen.host_tokens(900 + T, T, spec.hidden)
        out, idx, w = _run_layer(fmoe, dl, h, top_k=top_k)
        _compare_layer(hl, h, out, idx, w, L=oracle_layer(hl, top_k=top_k))


def test_grouped_many_token_tiles_and_repeated_calls(fmoe):
    """200 tokens: the router's grid spans four token tiles, the sort 800 pairs; a second
    call on the same workspace (tickets, counters and slots reused) gives the same bytes."""
    spec = gen.LayerSpec(**{**gen.small_layer(4, experts=16, top_k=4).__dict__, "random_gamma": True})
    hl = gen.host_layer(spec, seed=16)
    dl = gen.upload_layer(hl)
    lay = gen.binding_layer(dl)
    T, K = 200, spec.top_k
    h_np = gen.host_tokens(1300, T, spec.hidden)
    h = torch.from_numpy(h_np).cuda()
    ws = fmoe.workspace(fmoe.moe_layer_workspace_size(lay, T))
    outs = []
    for _ in range(2):
        out = torch.empty_like(h)
        idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
        w = torch.empty((T, K), dtype=torch.float32, device="cuda")
        fmoe.moe_layer(lay, h, out=out, topk_idx=idx, topk_w=w, ws=ws)
        outs.append((out, idx, w))
    fmoe.workspace_check(ws)
    torch.cuda.synchronize()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    out, idx, w = (x.cpu().numpy() for x in outs[0])
    _compare_layer(hl, h_np, out.astype(np.float64), idx, w.astype(np.float64))


def test_small_workspace_falls_back_to_the_per_token_path(fmoe):
    """A workspace sized for one token cannot hold the grouped path's regions: a 16-token
    call then runs token by token and must give the oracle's results."""
    spec = gen.small_layer(2)
    hl = gen.host_layer(spec, seed=17)
    dl = gen.upload_layer(hl)
    lay = gen.binding_layer(dl)
    T, K = 16, spec.top_k
    h_np = gen.host_tokens(1500, T, spec.hidden)
    h = torch.from_numpy(h_np).cuda()
    small = fmoe.moe_layer_workspace_size(lay, 1)
    assert small < fmoe.moe_layer_workspace_size(lay, T)
    ws = fmoe.workspace(small)
    out = torch.empty_like(h)
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    fmoe.moe_layer(lay, h, out=out, topk_idx=idx, topk_w=w, ws=ws)
    fmoe.workspace_check(ws)
    torch.cuda.synchronize()
    _compare_layer(hl, h_np, out.cpu().numpy().astype(np.float64), idx.cpu().numpy(),
                   w.cpu().numpy().astype(np.float64))


def test_tiny_layer_batch_takes_the_per_token_path(fmoe):
    # hidden 256: scale rows of 8 bytes are below the batched path's staging line, so the
    # call falls back to the per-token kernels; the result must not change
    spec = gen.tiny_layer(4)
    hl = gen.host_layer(spec, seed=15)
    dl = gen.upload_layer(hl)
    h = gen.host_tokens(1100, 12, spec.hidden)
    out, idx, w = _run_layer(fmoe, dl, h)
    _compare_layer(hl, h, out, idx, w)


def test_per_token_path_still_matches_oracle(fmoe, monkeypatch):
    monkeypatch.setenv("FMOE_GROUPED", "0")
    spec = gen.tiny_layer(2)
    hl = gen.host_layer(spec, seed=14)
    dl = gen.upload_layer(hl)
    h = gen.host_tokens(1000, 16, spec.hidden)
    out, idx, w = _run_layer(fmoe, dl, h)
    _compare_layer(hl, h, out, idx, w)


@pytest.mark.parametrize("bits,zipf", [(4, 0.0), (2, 1.1)])
def test_grouped_full_size_batch(fmoe, monkeypatch, bits, zipf):
    """64 tokens of the Qwen3.5-397B-A17B-shaped layer on the grouped path, every token
    against the oracle: routing exact wherever the top K+1 logits are separated (at
    least 60 of 64), outputs and out - h within 2e-3.  The oracle holds every record
    that the GPU or the exact routing selects (about 200 at 4-bit), so each active
    expert's work units, row items and K slices are compared."""
    from tests.test_parity_gpu import full_size_oracle_layer
    spec = gen.qwen397_layer(bits, zipf=zipf)
    dl = gen.device_layer(spec, seed=0, layer=0)
    lay = gen.binding_layer(dl)
    T, K = 64, spec.top_k
    h_np = gen.host_tokens(2000, T, spec.hidden)
    h = torch.from_numpy(h_np).cuda()
    out = torch.empty_like(h)
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    ws = fmoe.workspace(fmoe.moe_layer_workspace_size(lay, T))
    fmoe.moe_layer(lay, h, out=out, topk_idx=idx, topk_w=w, ws=ws)
    fmoe.workspace_check(ws)
    torch.cuda.synchronize()
    o = out.cpu().numpy().astype(np.float64)
    gi = idx.cpu().numpy()
    hl, L = full_size_oracle_layer(spec, h_np, gi)
    exact, _ = _compare_layer(hl, h_np, o, gi, w.cpu().numpy().astype(np.float64), L=L)
    assert exact >= 60, exact
    # the per-token path on the same batch: same routing where not near-tied (an extra check)
    monkeypatch.setenv("FMOE_GROUPED", "0")
    ref_idx = torch.empty_like(idx)
    fmoe.moe_layer(lay, h, topk_idx=ref_idx, ws=ws)
    torch.cuda.synchronize()
    assert np.sum(np.all(gi == ref_idx.cpu().numpy(), axis=1)) >= T - 2
    del dl, lay
    torch.cuda.empty_cache()
