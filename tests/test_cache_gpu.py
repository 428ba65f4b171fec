"""Expert cache in HBM in front of host-resident experts (needs a B200).

The replacement policy is checked against a plain Python model of it (least recently used
slot among those the lookup has not used, empty slots first, lowest index among equals),
the slot contents against the host records byte for byte, and the cached layer against
the oracle and, bit for bit, against the same routing run on a device-resident bank."""
import ctypes

import numpy as np
import pytest

import gen
from tests.helpers import check_routing, max_rel_err, oracle_layer, routing_margin
from tests.test_parity_gpu import TOL, full_size_oracle_layer

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fmoe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_dequant_expert_router_b200 as m
    m.lib()
    return m


class LruModel:
    def __init__(self, C):
        self.C = C
        self.slot_of, self.expert_of, self.last = {}, [-1] * C, [0] * C
        self.clock = self.hits = self.misses = 0

    def lookup(self, idx):
        self.clock += 1
        out = []
        for e in idx:
            s = self.slot_of.get(e)
            if s is None:
                s = min((self.last[c], c) for c in range(self.C) if self.last[c] != self.clock)[1]
                if self.expert_of[s] >= 0:
                    del self.slot_of[self.expert_of[s]]
                self.expert_of[s] = e
                self.slot_of[e] = s
                self.misses += 1
            else:
                self.hits += 1
            self.last[s] = self.clock
            out.append(s)
        return out


def test_lookups_follow_the_replacement_policy_and_copy_the_records(fmoe):
    E, C, stride, rec = 40, 6, 4096, 4000
    rng = np.random.default_rng(1)
    host = torch.from_numpy(rng.integers(0, 256, E * stride, dtype=np.uint8)).pin_memory()
    cache = fmoe.ExpertCache(host, E, stride, rec, C)
    model = LruModel(C)
    for step in range(60):
        K = int(rng.integers(1, 5))
        idx = rng.integers(0, 12 if step < 30 else E, K).astype(np.int32)   # a hot set, then everything
        slot = cache.fetch(torch.from_numpy(idx).cuda())
        want = model.lookup(idx.tolist())
        assert slot.cpu().numpy().tolist() == want, step
        slots = cache.slots.cpu().numpy().reshape(C, stride)
        hostv = host.numpy().reshape(E, stride)
        for e, s in model.slot_of.items():
            assert np.array_equal(slots[s, :rec], hostv[e, :rec]), (step, e, s)
    hits, misses, nbytes = cache.stats()
    assert (hits, misses, nbytes) == (model.hits, model.misses, model.misses * rec)
    cache.reset()
    assert cache.stats() == (0, 0, 0)
    assert cache.fetch(torch.tensor([3, 3, 5], dtype=torch.int32, device="cuda")).cpu().tolist() == [0, 0, 1]


def test_an_index_outside_the_bank_is_reported(fmoe):
    E, C, stride = 8, 4, 256
    host = torch.zeros(E * stride, dtype=torch.uint8).pin_memory()
    cache = fmoe.ExpertCache(host, E, stride, stride, C)
    cache.fetch(torch.tensor([1, 99], dtype=torch.int32, device="cuda"))
    with pytest.raises(fmoe.FmoeError) as e:
        cache.stats()
    assert e.value.status == 1
    cache.stats()   # the record was cleared


def test_pageable_host_memory_is_refused_before_any_launch(fmoe):
    E, stride = 4, 256
    pageable = np.zeros(E * stride, dtype=np.uint8)
    slots = torch.empty(2 * stride, dtype=torch.uint8, device="cuda")
    state = torch.empty(fmoe.lib().fmoe_expert_cache_state_size(E, 2), dtype=torch.uint8, device="cuda")
    c = fmoe.FmoeExpertCache(pageable.ctypes.data, stride, slots.data_ptr(), stride, stride, E, 2, state.data_ptr())
    assert fmoe.lib().fmoe_expert_cache_reset(ctypes.byref(c), None) == 1


def _cached_binding(fmoe, dl, host_bank, C):
    spec = dl.spec
    nbytes, off = gen.record_layout(spec.bits, spec.hidden, spec.inter, spec.group)
    routed = fmoe.Bank(None, spec.bits, spec.hidden, spec.inter, spec.experts, nbytes, off, spec.group)
    shared = fmoe.Bank(dl.shared, spec.bits, spec.hidden, spec.inter, 1, nbytes, off, spec.group)
    lay = fmoe.Layer(routed, shared, dl.w_router, dl.w_shared_gate, dl.gamma, dl.logit_bias, spec.eps, spec.top_k)
    cache = fmoe.ExpertCache(host_bank, spec.experts, nbytes, nbytes, C)
    return lay, cache


def _run_cached(fmoe, lay, cache, h_np, K):
    T = h_np.shape[0]
    h = torch.from_numpy(h_np).cuda()
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    ws = fmoe.workspace(fmoe.moe_layer_workspace_size(lay, 1))
    out = fmoe.moe_layer_cached(lay, cache, h, topk_idx=idx, topk_w=w, ws=ws)
    fmoe.workspace_check(ws)
    return out, idx, w, h


def test_cached_layer_matches_the_oracle_and_the_resident_bank(fmoe):
    spec = gen.small_layer(4)
    hl = gen.host_layer(spec, seed=41)
    dl = gen.upload_layer(hl)
    host_bank = dl.bank.cpu().pin_memory()
    lay, cache = _cached_binding(fmoe, dl, host_bank, C=6)
    T, K = 16, spec.top_k
    h_np = gen.host_tokens(4100, T, spec.hidden)
    out, idx, w, h = _run_cached(fmoe, lay, cache, h_np, K)
    got = out.cpu().numpy().astype(np.float64)
    gi = idx.cpu().numpy()
    # routing: exact wherever the top K+1 logits are separated; output against the oracle
    L = oracle_layer(hl)
    import oracle
    exact = 0
    for t in range(T):
        x = oracle.rmsnorm(h_np[t], hl.gamma, spec.eps)
        logits, delta = routing_margin(hl.w_router, x, hl.logit_bias)
        exact += check_routing(gi[t], logits, K, delta)
    assert exact >= 14
    ref = L.forward(h_np, force_idx=gi)
    assert max_rel_err(got, ref["out"]) <= TOL
    assert np.allclose(w.cpu().numpy(), ref["w"], rtol=1e-4, atol=1e-6)
    # the same routing on the device-resident bank gives the same bits
    res = gen.binding_layer(dl)
    same = fmoe.moe_layer_routed(res, h, idx, w)
    assert torch.equal(same, out)
    # the cache's counters follow the policy on this routing
    model = LruModel(6)
    for t in range(T):
        model.lookup(gi[t].tolist())
    assert cache.stats() == (model.hits, model.misses, model.misses * gen.record_bytes(spec))


def test_cached_layer_full_size(fmoe):
    """Qwen3.5-397B-A17B-shaped 4-bit layer, all 512 experts in pinned host memory, 8 slots."""
    spec = gen.qwen397_layer(4)
    dl = gen.device_layer(spec, seed=0, layer=0)
    host_bank = torch.empty(dl.bank.numel(), dtype=torch.uint8, pin_memory=True)
    host_bank.copy_(dl.bank)
    lay, cache = _cached_binding(fmoe, dl, host_bank, C=8)
    T, K = 6, spec.top_k
    h_np = gen.host_tokens(7000, T, spec.hidden)
    out, idx, w, h = _run_cached(fmoe, lay, cache, h_np, K)
    same = fmoe.moe_layer_routed(gen.binding_layer(dl), h, idx, w)
    assert torch.equal(same, out)
    gi = idx.cpu().numpy()
    hl, L = full_size_oracle_layer(spec, h_np, gi)
    ref = L.forward(h_np, force_idx=gi)
    assert max_rel_err(out.cpu().numpy().astype(np.float64), ref["out"]) <= TOL
    hits, misses, nbytes = cache.stats()
    assert hits + misses == T * K and nbytes == misses * gen.record_bytes(spec)
    del dl, host_bank
    torch.cuda.empty_cache()
