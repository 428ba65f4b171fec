"""Gated DeltaNet state update on the GPU against the oracle (needs a B200).

The kernel computes in fp32, as the pages' single-precision BLAS calls do; the oracle in
fp64 on the same fp32 inputs.  The tolerance is derived per element from the arithmetic
(unit roundoff eps = 2^-24, lane sums of 4 dk/128 terms then a 5-level tree):
  u_i:   (4 dk/128 + 6) eps sum_j |alpha s_ij k_j|
  d_i:   beta |du_i| + 2 eps beta (|v_i| + |u_i|)
  s'_ij: eps (|s'_ij| + |alpha s_ij|) + |k_j| |dd_i|
  o_i:   (4 dk/128 + 5) eps sum_j |s'_ij q_j| + sum_j |q_j| |ds'_ij|
and the test allows twice that.
"""
import numpy as np
import pytest

import gen
import oracle

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

EPS = 2.0 ** -24


@pytest.fixture(scope="module")
def fmoe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_dequant_expert_router_b200 as m
    m.lib()
    return m


def bounds(S, t):
    """Per-element error bounds (state, o) of one fp32 step from state S (fp64 copy of the fp32
    input) with inputs t, following the derivation in the module docstring."""
    n, dv, dk = S.shape
    m = 4 * (dk // 128)
    a = t["alpha"].astype(np.float64)[:, None, None]
    b = t["beta"].astype(np.float64)[:, None]
    k = t["k"].astype(np.float64)
    q = t["q"].astype(np.float64)
    v = t["v"].astype(np.float64)
    aS = a * S
    u = np.einsum("hij,hj->hi", aS, k)
    du = (m + 6) * EPS * np.einsum("hij,hj->hi", np.abs(aS), np.abs(k))
    dd = b * du + 2 * EPS * b * (np.abs(v) + np.abs(u))
    S2 = aS + (b * (v - u))[:, :, None] * k[:, None, :]
    dS = EPS * (np.abs(S2) + np.abs(aS)) + np.abs(k)[:, None, :] * dd[:, :, None]
    do = (m + 5) * EPS * np.einsum("hij,hj->hi", np.abs(S2), np.abs(q)) + np.einsum("hij,hj->hi", dS, np.abs(q))
    return 2 * dS, 2 * do


def to_dev(t):
    return {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in t.items()}


def step_and_check(fmoe, S_dev, t, early=False):
    """One kernel step from the device state S_dev, checked element by element against the
    oracle's step from the same fp32 state."""
    S0 = S_dev.cpu().numpy().astype(np.float64)
    d = to_dev(t)
    o = fmoe.gdn_step(S_dev, d["q"], d["k"], d["v"], d["alpha"], d["beta"], early=early)
    torch.cuda.synchronize()
    S_ref, o_ref = oracle.gdn_step(S0, t["q"], t["k"], t["v"], t["alpha"], t["beta"])
    bS, bo = bounds(S0, t)
    S_got = S_dev.cpu().numpy().astype(np.float64)
    o_got = o.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(S_got - S_ref) <= bS), float(np.max(np.abs(S_got - S_ref) / bS))
    assert np.all(np.abs(o_got - o_ref) <= bo), float(np.max(np.abs(o_got - o_ref) / bo))
    return o


@pytest.mark.parametrize("n,dk,dv", [(64, 128, 128), (3, 128, 5), (2, 128, 1), (5, 256, 7), (2, 384, 33),
                                     (1, 512, 1), (7, 128, 129)])
def test_gdn_step_matches_the_oracle(fmoe, n, dk, dv):
    spec = gen.GdnSpec(heads=n, dk=dk, dv=dv)
    S = torch.from_numpy(gen.host_gdn_state(spec, layer=3)).cuda()
    step_and_check(fmoe, S, gen.host_gdn_token(spec, 3, 0))


def test_gdn_sixteen_steps_full_size(fmoe):
    """64 heads x 128 x 128, 16 tokens: every step within its bound from the kernel's own state,
    and the 16-step fp32 chain within 16 single-step bounds of the fp64 chain."""
    spec = gen.gdn_qwen397()
    S0 = gen.host_gdn_state(spec, layer=0)
    S = torch.from_numpy(S0).cuda()
    chain = S0.astype(np.float64)
    total = np.zeros_like(chain)
    for t in range(16):
        tk = gen.host_gdn_token(spec, 0, t)
        bS, _ = bounds(S.cpu().numpy().astype(np.float64), tk)
        total = total + bS
        step_and_check(fmoe, S, tk)
        chain, _ = oracle.gdn_step(chain, tk["q"], tk["k"], tk["v"], tk["alpha"], tk["beta"])
    assert np.all(np.abs(S.cpu().numpy() - chain) <= total)


def test_gdn_early_state_read_gives_the_same_bits(fmoe):
    """Two layers' states stepped alternately, with and without the early-read flag: identical."""
    spec = gen.gdn_qwen397()
    runs = []
    for early in (False, True):
        Ss = [torch.from_numpy(gen.host_gdn_state(spec, layer=l)).cuda() for l in range(2)]
        outs = []
        for t in range(4):
            for l in range(2):
                d = to_dev(gen.host_gdn_token(spec, l, t))
                outs.append(fmoe.gdn_step(Ss[l], d["q"], d["k"], d["v"], d["alpha"], d["beta"], early=early))
        torch.cuda.synchronize()
        runs.append(([s.cpu() for s in Ss], [o.cpu() for o in outs]))
    for a, b in zip(runs[0][0] + runs[0][1], runs[1][0] + runs[1][1]):
        assert torch.equal(a, b)


def test_gdn_batch_of_sequences_equals_separate_calls(fmoe):
    spec1 = gen.gdn_qwen397()
    spec8 = gen.gdn_qwen397(batch=8)
    S8 = torch.from_numpy(gen.host_gdn_state(spec8, layer=5)).cuda()
    t8 = gen.host_gdn_token(spec8, 5, 0)
    parts = [S8[64 * b:64 * (b + 1)].clone() for b in range(8)]
    d8 = to_dev(t8)
    o8 = fmoe.gdn_step(S8, d8["q"], d8["k"], d8["v"], d8["alpha"], d8["beta"])
    for b in range(8):
        sl = slice(64 * b, 64 * (b + 1))
        d = {k: v[sl].contiguous() for k, v in d8.items()}
        o = fmoe.gdn_step(parts[b], d["q"], d["k"], d["v"], d["alpha"], d["beta"])
        assert torch.equal(o, o8[sl]) and torch.equal(parts[b], S8[sl])
    del spec1


def test_gdn_degenerate_gates(fmoe):
    spec = gen.GdnSpec(heads=8, dk=128, dv=16)
    S0 = gen.host_gdn_state(spec, layer=7)
    t = gen.host_gdn_token(spec, 7, 0)
    # alpha = 1, beta = 0: the state keeps its bits, the read-out is S q
    t1 = dict(t, alpha=np.ones(8, np.float32), beta=np.zeros(8, np.float32))
    S = torch.from_numpy(S0).cuda()
    step_and_check(fmoe, S, t1)
    assert np.array_equal(S.cpu().numpy(), S0)
    # alpha = 0: the memory is replaced by one write, beta v k^T
    t0 = dict(t, alpha=np.zeros(8, np.float32))
    S = torch.from_numpy(S0).cuda()
    step_and_check(fmoe, S, t0)
    # beta = 1 at a unit key with q = k: the read-out is v (delta rule), to the bound
    tq = dict(t, q=t["k"].copy(), beta=np.ones(8, np.float32))
    S = torch.from_numpy(S0).cuda()
    o = step_and_check(fmoe, S, tq)
    assert np.allclose(o.cpu().numpy(), t["v"], rtol=0, atol=1e-5)


def test_gdn_largest_batch_sampled(fmoe):
    """64 sequences x 64 heads (256 MiB of state, above L2), 8 heads checked in full."""
    spec = gen.gdn_qwen397(batch=64)
    S = gen.device_gdn_state(spec, layer=9)
    t = gen.host_gdn_token(spec, 9, 0)
    heads = [0, 1, 777, 2048, 3000, 4094, 4095, 1234]
    S0 = S[heads].cpu().numpy().astype(np.float64)
    d = to_dev(t)
    o = fmoe.gdn_step(S, d["q"], d["k"], d["v"], d["alpha"], d["beta"])
    torch.cuda.synchronize()
    sub = {k: v[heads] for k, v in t.items()}
    S_ref, o_ref = oracle.gdn_step(S0, sub["q"], sub["k"], sub["v"], sub["alpha"], sub["beta"])
    bS, bo = bounds(S0, sub)
    assert np.all(np.abs(S[heads].cpu().numpy() - S_ref) <= bS)
    assert np.all(np.abs(o[heads].cpu().numpy() - o_ref) <= bo)


def test_gdn_zero_heads_and_guard_bands(fmoe):
    spec = gen.GdnSpec(heads=3, dk=128, dv=5)
    G = 4096
    Sb = torch.full((G * 2 + 3 * 5 * 128,), -7.0, device="cuda")
    ob = torch.full((G * 2 + 15,), -7.0, device="cuda")
    S = Sb[G:G + 3 * 5 * 128].view(3, 5, 128)
    S.copy_(torch.from_numpy(gen.host_gdn_state(spec)))
    o = ob[G:G + 15].view(3, 5)
    d = to_dev(gen.host_gdn_token(spec, 0, 0))
    fmoe.gdn_step(S[:0], d["q"][:0], d["k"][:0], d["v"][:0], d["alpha"][:0], d["beta"][:0], o=o[:0])
    fmoe.gdn_step(S, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o=o)
    torch.cuda.synchronize()
    for buf, n in ((Sb, 3 * 5 * 128), (ob, 15)):
        assert torch.all(buf[:G] == -7.0) and torch.all(buf[G + n:] == -7.0)
