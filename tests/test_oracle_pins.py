"""Pins the CPU oracle to facts other than itself (no GPU needed).

Each test is chosen so that a plausible slip in the oracle fails it: a wrong
code order or field width (worked examples), a dropped or mis-signed bias term
(worked examples, closed forms), a wrong group index or a transposed operand
(brute force on non-square shapes with distinct per-group scales), a missing
renormalisation or wrong sort order (top-K/softmax), a dropped router bias
(one-hot router rows), swapped SwiGLU operands or
sigmoid sign (closed-form constant experts), and a missing residual or shared
term (K = E invariant and closed-form combine).
"""
import json
import math
import os

import numpy as np
import pytest

import gen
import oracle
from tests.helpers import (bf16_to_f64, dense_from_record, f32_to_bf16_exact, np_pack, np_unpack, oracle_layer,
                           silu)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _one_group_matrix(case):
    bits = case["bits"]
    words = np.array([int(w, 16) for w in case["group_words"]], dtype=np.uint32).reshape(1, -1)
    s = f32_to_bf16_exact([case["scale"]]).reshape(1, 1)
    b = f32_to_bf16_exact([case["bias"]]).reshape(1, 1)
    return oracle.matrix(words, s, b, bits, 1, 64)


@pytest.mark.parametrize("name", ["nibbles_0_to_15", "two_bit_0123_repeating", "all_fifteen"])
def test_worked_examples(name):
    case = [c for c in _golden()["cases"] if c["name"] == name][0]
    m = _one_group_matrix(case)
    got = np.array([oracle.weight(m, 0, c) for c in range(64)])
    exp = case["expect"]
    assert got[:len(exp)].tolist() == exp
    if "expect_rest" in case:
        assert np.all(got[len(exp):] == case["expect_rest"])
    if "expect_rest_period" in case:
        per = case["expect_rest_period"]
        assert got.tolist() == per * (64 // len(per))


def test_code_fields_lsb_first():
    # Word 0x76543210: field j holds j (4-bit); 0xE4 = 0b11100100 holds 0,1,2,3 (2-bit).
    assert [oracle.code([0x76543210], 4, c) for c in range(8)] == list(range(8))
    assert [oracle.code([0xE4E4E4E4], 2, c) for c in range(16)] == [0, 1, 2, 3] * 4
    # 8-bit: one code per byte, byte 0 first; 0xFF is 255 (codes are unsigned)
    assert [oracle.code([0xFF80_0100], 8, c) for c in range(4)] == [0, 1, 128, 255]


def test_record_sizes_match_pages():
    rs = _golden()["record_sizes"]
    b4 = gen.record_bytes(gen.qwen397_layer(4))
    b2 = gen.record_bytes(gen.qwen397_layer(2))
    assert b4 == rs["four_bit_bytes"] and b4 == rs["four_bit_mib"] * 2 ** 20
    assert b2 == rs["two_bit_bytes"] and round(b2 / 1e6, 1) == rs["two_bit_mb_approx"]


def _random_packed(rng, bits, rows, cols, group=64):
    codes = rng.integers(0, 1 << bits, size=(rows, cols))
    # distinct, bf16-exact scales and biases per (row, group)
    s = (rng.integers(1, 64, size=(rows, cols // group)) / 256.0).astype(np.float32)
    b = (rng.integers(-64, 64, size=(rows, cols // group)) / 128.0).astype(np.float32)
    dense = codes * np.repeat(s.astype(np.float64), group, axis=1) + np.repeat(b.astype(np.float64), group, axis=1)
    return codes, np_pack(codes, bits), f32_to_bf16_exact(s), f32_to_bf16_exact(b), dense


@pytest.mark.parametrize("bits,rows,cols,group", [(4, 3, 192, 64), (2, 5, 128, 64), (4, 7, 64, 64), (2, 2, 320, 64),
                                                  (8, 3, 128, 64), (8, 2, 192, 64), (4, 3, 256, 128),
                                                  (2, 2, 384, 128), (8, 3, 256, 128)])
def test_onegrid_roundtrip_and_dense_bruteforce(bits, rows, cols, group):
    rng = np.random.default_rng(bits * 1000 + rows + group)
    codes, qw, s, b, dense = _random_packed(rng, bits, rows, cols, group)
    assert np.array_equal(np_unpack(qw, bits, cols), codes)
    m = oracle.matrix(qw, s, b, bits, rows, cols, group=group)
    got = np.array([[oracle.weight(m, r, c) for c in range(cols)] for r in range(rows)])
    assert np.array_equal(got, dense)  # on-grid weights are exact in fp64
    x = rng.standard_normal(cols)
    y = oracle.matvec(m, x)
    ref = dense @ x
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(dense) @ np.abs(x))


def test_four_bit_codes_below_four_equal_two_bit():
    rng = np.random.default_rng(7)
    rows, cols = 4, 128
    codes = rng.integers(0, 4, size=(rows, cols))
    s = f32_to_bf16_exact(np.full((rows, cols // 64), 0.375, np.float32))
    b = f32_to_bf16_exact(np.full((rows, cols // 64), -0.5, np.float32))
    m4 = oracle.matrix(np_pack(codes, 4), s, b, 4, rows, cols)
    m2 = oracle.matrix(np_pack(codes, 2), s, b, 2, rows, cols)
    x = rng.standard_normal(cols)
    assert np.array_equal(oracle.matvec(m4, x), oracle.matvec(m2, x))


def test_topk_is_full_sort_with_ties_to_lower_index():
    rng = np.random.default_rng(3)
    p = rng.random(512)
    for k in (1, 4, 17, 512):
        assert oracle.topk(p, k).tolist() == np.argsort(-p, kind="stable")[:k].tolist()
    tied = np.array([0.1, 0.3, 0.3, 0.2, 0.3, 0.05])
    assert oracle.topk(tied, 4).tolist() == [1, 2, 4, 3]


def test_router_logits_closed_forms():
    # one-hot bf16 rows (W[e, i] = 1 if i == e): l_e = x_e + bias_e exactly; zero rows: l = bias
    E, H = 8, 64
    x = np.random.default_rng(6).standard_normal(H)
    bias = (np.arange(E, dtype=np.float32) - 3.5) / 4.0
    one = f32_to_bf16_exact([1.0])[0]
    w = np.zeros((E, H), np.uint16)
    w[np.arange(E), np.arange(E)] = one
    assert oracle.router_logits(w, bias, x).tolist() == (x[:E] + bias.astype(np.float64)).tolist()
    assert oracle.router_logits(w, None, x).tolist() == x[:E].tolist()
    assert oracle.router_logits(np.zeros((E, H), np.uint16), bias, x).tolist() == bias.astype(np.float64).tolist()


def test_softmax_closed_form_and_sum():
    p = oracle.softmax(np.array([0.0, math.log(2.0), math.log(3.0)]))
    assert np.allclose(p, [1 / 6, 2 / 6, 3 / 6], rtol=0, atol=1e-15)
    rng = np.random.default_rng(5)
    for _ in range(5):
        q = oracle.softmax(rng.standard_normal(512) * 3)
        assert abs(q.sum() - 1.0) <= 1e-12
        assert np.all(q > 0)


def test_rmsnorm_closed_forms():
    H = 256
    gamma = (1.0 + 0.1 * np.random.default_rng(1).standard_normal(H)).astype(np.float32)
    for c in (2.5, -0.75, 1e-4):
        h = np.full(H, c, np.float32)
        x = oracle.rmsnorm(h, gamma, 1e-6)
        cc = float(np.float32(c))
        assert np.allclose(x, gamma.astype(np.float64) * cc / math.sqrt(cc * cc + 1e-6), rtol=1e-14, atol=0)
    # gamma = None is unit weight; a one-hot h normalises to sqrt(H/(1+H eps))
    h = np.zeros(H, np.float32)
    h[17] = 3.0
    x = oracle.rmsnorm(h, None, 1e-6)
    assert abs(x[17] - 3.0 / math.sqrt(9.0 / H + 1e-6)) < 1e-12 and np.count_nonzero(x) == 1


def _constant_record(spec, bg, bu, bd, scale=0.5):
    """A record whose codes are all 0 (so scale must not matter) and biases are constants per matrix."""
    nbytes, off = gen.record_layout(spec.bits, spec.hidden, spec.inter, spec.group)
    rec = np.zeros(nbytes, np.uint8)
    for m, (rows, cols) in enumerate(gen.matrix_shapes(spec)):
        ng = rows * cols // spec.group
        rec[off[3 * m + 1]:off[3 * m + 1] + 2 * ng].view(np.uint16)[:] = f32_to_bf16_exact([scale])[0]
        rec[off[3 * m + 2]:off[3 * m + 2] + 2 * ng].view(np.uint16)[:] = f32_to_bf16_exact([(bg, bu, bd)[m]])[0]
    return rec


def test_constant_expert_closed_form_swiglu_order():
    # codes 0, biases b_g, b_u, b_d: g = b_g S, u = b_u S, a = silu(g) u, y_j = I a (S = sum x).
    spec = gen.LayerSpec(hidden=128, experts=1, inter=64, top_k=1, bits=4)
    nbytes, off = gen.record_layout(4, 128, 64)
    rec = _constant_record(spec, 2.0, -1.0, 0.25)
    bk = oracle.bank(rec, 4, 128, 64, 1, nbytes, off)
    x = np.zeros(128)
    x[:3] = [0.5, 0.25, 0.25]  # S = 1
    y, a = oracle.expert_ffn(bk, 0, x, want_act=True)
    a_exp = silu(2.0) * -1.0
    assert np.allclose(a, a_exp, rtol=1e-15) and abs(a_exp - silu(-1.0) * 2.0) > 1.0  # swapped order would differ
    assert np.allclose(y, 64 * 0.25 * a_exp, rtol=1e-14)


def test_layer_combine_closed_form():
    # Four constant experts with distinct biases, a router built to rank them, and a known shared gate.
    H, I, E, K = 128, 64, 4, 2
    spec = gen.LayerSpec(hidden=H, experts=E, inter=I, top_k=K, bits=2)
    nbytes, off = gen.record_layout(2, H, I)
    bdown = [0.5, -0.25, 1.0, 0.125]
    bank = np.stack([_constant_record(spec, 1.0, 0.5, bdown[e]) for e in range(E)])
    shared = _constant_record(spec, -0.5, 1.0, 2.0)
    # router: row e = c_e * ones, so l_e = c_e * sum(x)
    c = np.array([0.25, 1.0, -0.5, 0.5], np.float32)
    wr = np.repeat(f32_to_bf16_exact(c)[:, None], H, axis=1)
    wsg = f32_to_bf16_exact(np.full(H, 0.0078125, np.float32))
    L = oracle.Layer(bank, shared, wr, wsg, None, None, 2, H, I, K, nbytes, off)
    h = np.zeros((1, H), np.float32)
    h[0, :4] = [1.0, 0.5, 0.5, 0.0]  # gamma None: x = h, S = 2
    r = L.forward(h)
    S = 2.0
    logits = c.astype(np.float64) * S
    p = np.exp(logits - logits.max())
    p /= p.sum()
    assert r["idx"][0].tolist() == [1, 3]
    w = p[[1, 3]] / p[[1, 3]].sum()
    assert np.allclose(r["w"][0], w, rtol=1e-14)
    a_r = silu(1.0 * S) * 0.5 * S
    y = lambda bd: I * bd * a_r
    a_s = silu(-0.5 * S) * 1.0 * S
    sigma = 1.0 / (1.0 + math.exp(-0.0078125 * S))
    assert abs(r["sigma"][0] - sigma) < 1e-15
    exp = h[0].astype(np.float64) + w[0] * y(bdown[1]) + w[1] * y(bdown[3]) + sigma * I * 2.0 * a_s
    assert np.allclose(r["out"][0], exp, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("bits", [4, 2, 8])
def test_all_experts_identical_equals_dense_ffn(bits):
    # K = E with byte-identical experts: sum_k w_k y = y (weights sum to 1), so out = h + FFN(x) + sigma FFN_s(x),
    # checked against a dense numpy FFN built by whole-array unpacking.
    spec = gen.LayerSpec(hidden=128, experts=4, inter=64, top_k=4, bits=bits, router_std=0.1, random_gamma=True)
    hl = gen.host_layer(spec, seed=11)
    one = hl.routed[2]
    for e in range(spec.experts):
        hl.routed[e] = one.copy()
    L = oracle_layer(hl)
    h = gen.host_tokens(0, 3, spec.hidden)
    r = L.forward(h)
    Wg, Wu, Wd = dense_from_record(one, bits, 128, 64)
    Sg, Su, Sd = dense_from_record(hl.shared, bits, 128, 64)
    wsg = bf16_to_f64(hl.w_shared_gate)
    for t in range(3):
        ht = h[t].astype(np.float64)
        x = ht / np.sqrt(np.mean(ht * ht) + 1e-6) * hl.gamma.astype(np.float64)
        y = Wd @ (silu(Wg @ x) * (Wu @ x))
        ys = Sd @ (silu(Sg @ x) * (Su @ x))
        sig = 1.0 / (1.0 + np.exp(-(wsg @ x)))
        ref = ht + y + sig * ys
        assert np.allclose(r["w"][t].sum(), 1.0, rtol=0, atol=1e-14)
        assert np.max(np.abs(r["out"][t] - ref)) <= 1e-12 * np.max(np.abs(ref))
        assert sorted(r["idx"][t].tolist()) == [0, 1, 2, 3]


def test_top1_weight_is_one_and_zero_gate_is_half():
    spec = gen.LayerSpec(hidden=128, experts=8, inter=64, top_k=1, bits=4, router_std=0.1)
    hl = gen.host_layer(spec, seed=4)
    hl.w_shared_gate[:] = 0
    r = oracle_layer(hl).forward(gen.host_tokens(5, 4, 128))
    assert np.all(r["w"] == 1.0)
    assert np.all(r["sigma"] == 0.5)


def test_renormalised_weights_equal_softmax_over_selected_logits():
    spec = gen.tiny_layer()
    hl = gen.host_layer(spec, seed=2)
    r = oracle_layer(hl).forward(gen.host_tokens(0, 8, spec.hidden))
    for t in range(8):
        sel = r["logits"][t][r["idx"][t]]
        q = np.exp(sel - sel.max())
        assert np.allclose(r["w"][t], q / q.sum(), rtol=1e-13)
        assert abs(r["probs"][t].sum() - 1.0) < 1e-12
        assert r["idx"][t].tolist() == np.argsort(-r["probs"][t], kind="stable")[:spec.top_k].tolist()


def test_forced_routing_matches_free_routing_when_equal():
    spec = gen.tiny_layer()
    hl = gen.host_layer(spec, seed=9)
    L = oracle_layer(hl)
    h = gen.host_tokens(3, 4, spec.hidden)
    free = L.forward(h)
    forced = L.forward(h, force_idx=free["idx"])
    assert np.array_equal(free["out"], forced["out"])
    swapped = L.forward(h, force_idx=free["idx"][:, ::-1].copy())  # same set, other order: same sum up to rounding
    assert np.allclose(swapped["out"], free["out"], rtol=1e-13, atol=1e-13)


def test_sparse_record_table_equals_full_bank():
    spec = gen.tiny_layer(bits=2)
    hl = gen.host_layer(spec, seed=6)
    h = gen.host_tokens(0, 2, spec.hidden)
    full = oracle_layer(hl).forward(h)
    keep = set(full["idx"].reshape(-1).tolist())
    sub = gen.HostLayer(spec, {e: hl.routed[e] for e in keep}, hl.shared, hl.w_router, hl.w_shared_gate, hl.gamma,
                        hl.logit_bias)
    from tests.helpers import oracle_layer_sparse
    part = oracle_layer_sparse(sub).forward(h, force_idx=full["idx"])
    assert np.array_equal(full["out"], part["out"])


# ----------------------------------------------------------------------------------------------- Gated DeltaNet
# The state update of the linear-attention layers ("What is Flash-MoE", section 4; "Flash-MoE"
# wiki summary, key technique 4).  The oracle takes the three BLAS steps one by one; the pins
# below fix it by the gated delta rule's product form, by what the delta rule guarantees
# (writing v at a unit key k and reading k back returns v; directions orthogonal to k only
# decay), and by its special cases.  Shapes are non-square (dv != dk) so that a transposed
# operand cannot pass.

def _gdn_case(seed, n=3, dk=8, dv=5):
    rng = np.random.default_rng(seed)
    S = rng.standard_normal((n, dv, dk))
    q = rng.standard_normal((n, dk))
    k = rng.standard_normal((n, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((n, dv))
    alpha = rng.uniform(0.5, 1.0, n)
    beta = rng.uniform(0.1, 1.0, n)
    return S, q, k, v, alpha, beta


def test_gdn_equals_the_gated_delta_rule_product_form():
    # S' = alpha S (I - beta k k^T) + beta v k^T and o = S' q, for keys of any norm
    S, q, k, v, alpha, beta = _gdn_case(0)
    k = k * np.array([[0.5], [1.0], [2.0]])
    S2, o = oracle.gdn_step(S, q, k, v, alpha, beta)
    for h in range(S.shape[0]):
        P = alpha[h] * S[h] @ (np.eye(S.shape[2]) - beta[h] * np.outer(k[h], k[h])) + beta[h] * np.outer(v[h], k[h])
        assert np.allclose(S2[h], P, rtol=0, atol=1e-13)
        assert np.allclose(o[h], P @ q[h], rtol=0, atol=1e-13)


def test_gdn_full_write_at_a_unit_key_reads_back_the_value():
    S, q, k, v, alpha, _ = _gdn_case(1)
    S2, o = oracle.gdn_step(S, k, k, v, alpha, np.ones(3))   # query = key
    for h in range(3):
        assert np.allclose(S2[h] @ k[h], v[h], rtol=0, atol=1e-13)
        assert np.allclose(o[h], v[h], rtol=0, atol=1e-13)


def test_gdn_directions_orthogonal_to_the_key_only_decay():
    S, q, k, v, alpha, beta = _gdn_case(2)
    S2, _ = oracle.gdn_step(S, q, k, v, alpha, beta)
    rng = np.random.default_rng(3)
    for h in range(3):
        w = rng.standard_normal(S.shape[2])
        w -= np.dot(w, k[h]) * k[h]
        assert np.allclose(S2[h] @ w, alpha[h] * (S[h] @ w), rtol=0, atol=1e-13)
        # and along k: S' k = alpha (1 - beta) S k + beta v
        assert np.allclose(S2[h] @ k[h], alpha[h] * (1 - beta[h]) * (S[h] @ k[h]) + beta[h] * v[h], rtol=0,
                           atol=1e-13)


def test_gdn_special_cases():
    S, q, k, v, alpha, beta = _gdn_case(4)
    zero, one = np.zeros(3), np.ones(3)
    S2, o = oracle.gdn_step(S, q, k, v, zero, beta)          # no memory left: a single write
    for h in range(3):
        assert np.allclose(S2[h], beta[h] * np.outer(v[h], k[h]), rtol=0, atol=1e-14)
        assert np.allclose(o[h], beta[h] * np.dot(k[h], q[h]) * v[h], rtol=0, atol=1e-14)
    S2, o = oracle.gdn_step(S, q, k, v, one, zero)           # no decay, no write
    assert np.array_equal(S2, S)
    assert np.allclose(o, np.einsum("hij,hj->hi", S, q), rtol=0, atol=1e-13)
    S2, _ = oracle.gdn_step(S, q, k, v, alpha, zero)         # decay only
    assert np.allclose(S2, alpha[:, None, None] * S, rtol=0, atol=1e-15)


def test_gdn_orthonormal_keys_form_an_associative_memory_with_overwrite():
    # from an empty state, full writes at orthonormal keys store every value; writing a new
    # value at an old key replaces it and leaves the others alone (plain linear attention,
    # without the delta term, would add the two values instead)
    dk, dv, m = 6, 4, 5
    rng = np.random.default_rng(5)
    keys = np.linalg.qr(rng.standard_normal((dk, dk)))[0][:, :m].T
    vals = rng.standard_normal((m, dv))
    S = np.zeros((1, dv, dk))
    for i in range(m):
        S, _ = oracle.gdn_step(S, keys[i:i + 1], keys[i:i + 1], vals[i:i + 1], np.ones(1), np.ones(1))
    for i in range(m):
        assert np.allclose(S[0] @ keys[i], vals[i], rtol=0, atol=1e-13)
    new = rng.standard_normal((1, dv))
    S, o = oracle.gdn_step(S, keys[1:2], keys[1:2], new, np.ones(1), np.ones(1))
    assert np.allclose(o[0], new[0], rtol=0, atol=1e-13)
    for i in range(m):
        assert np.allclose(S[0] @ keys[i], new[0] if i == 1 else vals[i], rtol=0, atol=1e-13)


def test_gdn_heads_are_independent():
    S, q, k, v, alpha, beta = _gdn_case(6)
    S2, o = oracle.gdn_step(S, q, k, v, alpha, beta)
    for h in range(3):
        Sh, oh = oracle.gdn_step(S[h:h + 1], q[h:h + 1], k[h:h + 1], v[h:h + 1], alpha[h:h + 1], beta[h:h + 1])
        assert np.array_equal(Sh[0], S2[h]) and np.array_equal(oh[0], o[h])


def test_results_do_not_depend_on_the_thread_count():
    """Threads split only independent output rows and heads, so one thread and many give
    the same bits (the bench times the oracle on all host cores, the tests on few)."""
    before = oracle.lib().or_get_threads()
    try:
        hl = gen.host_layer(gen.tiny_layer(4), seed=3)
        L = oracle_layer(hl)
        h = gen.host_tokens(77, 3, hl.spec.hidden)
        S, q, k, v, alpha, beta = _gdn_case(9, n=8, dk=16, dv=16)
        runs = []
        for n in (1, 4):
            oracle.set_threads(n)
            r = L.forward(h)
            runs.append((r["out"], r["idx"], r["w"], *oracle.gdn_step(S, q, k, v, alpha, beta)))
        for a, b in zip(*runs):
            assert np.array_equal(a, b)
    finally:
        oracle.set_threads(before)
