"""The 60-layer stack of Qwen3.5-397B-A17B-shaped 2-bit MoE blocks against the CPU oracle (needs a B200).

Two fresh tokens go through all 60 full-size layers with fmoe_moe_stack (the
default path).  The same tokens are run layer by layer through fmoe_moe_layer,
which must give the stack's bytes and exposes every layer's input and routing.
Each layer is then compared with the oracle on the GPU's own input of that
layer: routing exact wherever the top K+1 logits are separated, outputs within
2e-3.  Finally a chain computed by the oracle alone, from the first input, must
end within 2e-3 of the stack's output whenever no layer of it is near-tied.
The oracle draws only the router, the shared expert and the selected records
of each layer.
"""
import numpy as np
import pytest

import gen
import oracle
from tests.helpers import check_routing, max_rel_err, routing_margin, ulp32
from tests.test_parity_gpu import TOL, full_size_oracle_layer

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

NL = 60


@pytest.fixture(scope="module")
def fmoe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_dequant_expert_router_b200 as m
    m.lib()
    return m


def test_stack60_full_size_matches_oracle(fmoe):
    spec = gen.qwen397_layer(2)
    dls = [gen.device_layer(spec, seed=0, layer=l) for l in range(NL)]
    lays = [gen.binding_layer(dl) for dl in dls]
    T, K = 2, spec.top_k
    h0 = gen.host_tokens(3000, T, spec.hidden)
    h = torch.from_numpy(h0).cuda()
    out = fmoe.moe_stack(lays, h)
    # layer by layer: the inputs and routings of every layer
    states, idxs, ws_ = [h0], [], []
    cur = h
    for lay in lays:
        idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
        w = torch.empty((T, K), dtype=torch.float32, device="cuda")
        cur = fmoe.moe_layer(lay, cur, topk_idx=idx, topk_w=w)
        states.append(cur.cpu().numpy())
        idxs.append(idx.cpu().numpy())
        ws_.append(w.cpu().numpy().astype(np.float64))
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    assert np.array_equal(out, states[-1])   # the stack is the layers in order
    del dls, lays
    torch.cuda.empty_cache()

    exact = 0
    chain = h0.astype(np.float32)
    chain_tied = False
    for l in range(NL):
        hin, hout = states[l], states[l + 1].astype(np.float64)
        hl, L = full_size_oracle_layer(spec, np.concatenate([hin, chain]), idxs[l], layer=l)
        for t in range(T):
            x = oracle.rmsnorm(hin[t], hl.gamma, spec.eps)
            logits, delta = routing_margin(hl.w_router, x, hl.logit_bias)
            exact += check_routing(idxs[l][t], logits, K, delta)
        ref = L.forward(hin, force_idx=idxs[l])
        assert max_rel_err(hout, ref["out"]) <= TOL, l
        hin64 = hin.astype(np.float64)
        assert max_rel_err(hout - hin64, ref["out"] - hin64, slack=ulp32(hout)) <= TOL, l
        assert np.allclose(ws_[l], ref["w"], rtol=1e-4, atol=1e-6), l
        # the oracle's own chain: its routing must be clear of near-ties for the end-to-end check
        for t in range(T):
            x = oracle.rmsnorm(chain[t], hl.gamma, spec.eps)
            logits, delta = routing_margin(hl.w_router, x, hl.logit_bias)
            top = np.sort(logits)[::-1][:K + 1]
            chain_tied |= bool(np.any(top[:-1] - top[1:] <= delta))
        chain = L.forward(chain)["out"].astype(np.float32)
    assert exact >= 2 * NL - 6, exact
    if not chain_tied:
        assert max_rel_err(out.astype(np.float64), chain.astype(np.float64)) <= TOL
