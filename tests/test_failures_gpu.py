"""Failure detection on the device, in the forms that leave the GPU usable: a bounded wait
that runs out, an expert index outside the bank, and guard bands around every buffer the
kernels write (needs a B200).  Nothing here faults, traps or hangs the GPU: the waits
return after their limit with an error status that the host reads."""
import numpy as np
import pytest

import gen
import oracle
from tests.helpers import max_rel_err, oracle_layer
from tests.test_parity_gpu import TOL

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fmoe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_dequant_expert_router_b200 as m
    m.lib()
    return m


def test_bounded_wait_on_a_flag_that_is_never_set_reports_a_timeout(fmoe):
    spec = gen.tiny_layer(4)
    hl = gen.host_layer(spec, seed=31)
    lay = gen.binding_layer(gen.upload_layer(hl))
    ws = fmoe.workspace(fmoe.moe_layer_workspace_size(lay, 1))
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    fmoe.wait_flag(flag, 1, 5_000_000, ws)   # 5 ms, nothing sets the flag
    with pytest.raises(fmoe.FmoeError) as e:
        fmoe.workspace_check(ws)
    assert e.value.status == 6                  # FMOE_ERR_DEVICE_TIMEOUT
    fmoe.workspace_check(ws)                    # the check cleared the error word
    flag.fill_(1)
    fmoe.wait_flag(flag, 1, 5_000_000, ws)   # already set: returns at once, no error
    fmoe.workspace_check(ws)
    # the context is still usable: a layer call after the timeout gives the oracle's result
    h = gen.host_tokens(3100, 2, spec.hidden)
    out = fmoe.moe_layer(lay, torch.from_numpy(h).cuda(), ws=ws).cpu().numpy()
    fmoe.workspace_check(ws)
    assert max_rel_err(out, oracle_layer(hl).forward(h)["out"]) <= TOL


def test_routed_layer_matches_the_oracle_and_reports_a_bad_index(fmoe):
    spec = gen.small_layer(4)
    hl = gen.host_layer(spec, seed=32)
    lay = gen.binding_layer(gen.upload_layer(hl))
    T, K = 6, spec.top_k
    h = gen.host_tokens(3200, T, spec.hidden)
    rng = np.random.default_rng(32)
    idx = np.stack([rng.choice(spec.experts, K, replace=False) for _ in range(T)]).astype(np.int32)
    w = rng.random((T, K)).astype(np.float32)
    ws = fmoe.workspace(fmoe.moe_layer_workspace_size(lay, 1))
    out = fmoe.moe_layer_routed(lay, torch.from_numpy(h).cuda(), torch.from_numpy(idx).cuda(),
                                torch.from_numpy(w).cuda(), ws=ws)
    fmoe.workspace_check(ws)
    # the oracle with the same experts; its weights are the renormalised softmax ones, so
    # compare sum_k w_k y_k + sigma y_s term by term from the oracle's expert outputs
    L = oracle_layer(hl)
    got = out.cpu().numpy().astype(np.float64)
    for t in range(T):
        x = oracle.rmsnorm(h[t], hl.gamma, spec.eps)
        ref = h[t].astype(np.float64).copy()
        for k in range(K):
            ref += float(w[t, k]) * oracle.expert_ffn(L.routed, int(idx[t, k]), x)
        z = float(np.dot((hl.w_shared_gate.astype(np.uint32) << 16).view(np.float32).astype(np.float64), x))
        ref += 1.0 / (1.0 + np.exp(-z)) * oracle.expert_ffn(L.shared, 0, x)
        assert max_rel_err(got[t], ref) <= TOL, t
    # an index outside the bank: the kernels take expert 0 instead and record it
    bad = idx.copy()
    bad[2, 1] = spec.experts + 5
    fmoe.moe_layer_routed(lay, torch.from_numpy(h).cuda(), torch.from_numpy(bad).cuda(), torch.from_numpy(w).cuda(),
                          ws=ws)
    with pytest.raises(fmoe.FmoeError) as e:
        fmoe.workspace_check(ws)
    assert e.value.status == 1                  # FMOE_ERR_INVALID_ARG
    fmoe.workspace_check(ws)


@pytest.mark.parametrize("shape", ["tiny", "small", "small_two_kernels"])
def test_guard_bands_around_outputs_and_workspace_stay_untouched(fmoe, monkeypatch, shape):
    """Every buffer the kernels write (out, the routing outputs, the workspace) sits between
    guard bands of a fixed pattern; a call must leave the bands as they were."""
    if shape == "small_two_kernels":
        monkeypatch.setenv("FMOE_TOKEN_KERNELS", "2")
    spec = gen.tiny_layer(4) if shape == "tiny" else gen.small_layer(4)
    hl = gen.host_layer(spec, seed=33)
    lay = gen.binding_layer(gen.upload_layer(hl))
    T, K, H = 5, spec.top_k, spec.hidden
    G = 4096                                    # guard elements (16 KiB) on each side
    h = torch.from_numpy(gen.host_tokens(3300, T, H)).cuda()

    def banded(n, dtype):
        buf = torch.empty(n + 2 * G, dtype=dtype, device="cuda")
        buf.view(torch.uint8).fill_(0xA5)
        return buf, buf[G:G + n]

    outb, out = banded(T * H, torch.float32)
    idxb, idx = banded(T * K, torch.int32)
    wb, w = banded(T * K, torch.float32)
    nws = fmoe.moe_layer_workspace_size(lay, T)
    wsb = torch.empty(nws + 2 * 4 * G, dtype=torch.uint8, device="cuda")
    wsb.fill_(0xA5)
    ws = wsb[4 * G:4 * G + nws]
    fmoe.workspace_init(ws)
    fmoe.moe_layer(lay, h, out=out.view(T, H), topk_idx=idx.view(T, K), topk_w=w.view(T, K), ws=ws)
    fmoe.workspace_check(ws)
    torch.cuda.synchronize()
    for buf, n, unit in ((outb, T * H, 4), (idxb, T * K, 4), (wb, T * K, 4), (wsb, nws, 1)):
        raw = buf.view(torch.uint8).cpu().numpy()
        g = G * unit if buf is not wsb else 4 * G
        assert np.all(raw[:g] == 0xA5), "guard band before the buffer was written"
        assert np.all(raw[g + n * unit if buf is not wsb else g + n:] == 0xA5), "guard band after the buffer was written"
    ref = oracle_layer(hl).forward(h.cpu().numpy(), force_idx=idx.view(T, K).cpu().numpy())["out"]
    assert max_rel_err(out.view(T, H).cpu().numpy(), ref) <= TOL
