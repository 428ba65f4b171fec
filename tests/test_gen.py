"""Seeded input generator: determinism, distributions and layout (no GPU needed)."""
import numpy as np

import gen
from tests.helpers import bf16_to_f64, dense_from_record


def test_normal_draws_are_deterministic_and_standard():
    a = gen.host_normal_f32(gen.token_key(0), 1.0, 1 << 18)
    b = gen.host_normal_f32(gen.token_key(0), 1.0, 1 << 18)
    c = gen.host_normal_f32(gen.token_key(1), 1.0, 1 << 18)
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1.0) < 0.01
    assert abs(np.corrcoef(a, c)[0, 1]) < 0.01
    # Irwin-Hall(12) is bounded by 6 and exactly a multiple of 2^-16
    assert np.all(np.abs(a) <= 6.0) and np.all(a * 65536 == np.round(a * 65536))


def test_bf16_rounding_is_nearest_even():
    x = gen.host_normal_f32(gen.token_key(7), 0.02, 4096)
    b = gen.host_normal_bf16(gen.token_key(7), 0.02, 4096)
    back = bf16_to_f64(b)
    ulp = np.abs(back) * 2.0 ** -7
    assert np.all(np.abs(back - x) <= ulp / 2 * (1 + 1e-6))


def test_quantiser_codes_span_range_and_error_bound():
    spec = gen.tiny_layer(bits=4)
    rec = gen.host_record(spec, 0, 0, 3)
    Wg, Wu, Wd = dense_from_record(rec, 4, spec.hidden, spec.inter)
    # the dequantised weights approximate N(0, 0.02) draws
    assert abs(Wg.std() - 0.02) < 0.002 and abs(Wd.mean()) < 0.002
    rec2 = gen.host_record(gen.tiny_layer(bits=2), 0, 0, 3)
    Wg2, _, _ = dense_from_record(rec2, 2, spec.hidden, spec.inter)
    # same underlying draws: the 2-bit approximation is coarser but correlated
    assert np.corrcoef(Wg.ravel(), Wg2.ravel())[0, 1] > 0.85


def test_layer_draw_is_reproducible_and_layers_differ():
    spec = gen.tiny_layer()
    a = gen.host_layer(spec, layer=0)
    b = gen.host_layer(spec, layer=0)
    c = gen.host_layer(spec, layer=1)
    assert np.array_equal(gen.bank_array(a), gen.bank_array(b))
    assert not np.array_equal(gen.bank_array(a), gen.bank_array(c))
    assert not np.array_equal(a.routed[0], a.routed[1])
    assert not np.array_equal(a.shared, a.routed[0])


def test_zipf_bias_is_a_permuted_zipf_distribution():
    spec = gen.qwen397_layer(2, zipf=1.1)
    beta = gen.zipf_logit_bias(spec, 0, 0)
    p = np.exp(beta.astype(np.float64))
    assert abs(p.sum() - 1.0) < 1e-5
    ranks = np.arange(1, 513, dtype=np.float64) ** -1.1
    assert np.allclose(np.sort(p)[::-1], ranks / ranks.sum(), rtol=1e-5)
    assert np.argmax(p) != 0 or np.argmax(gen.zipf_logit_bias(spec, 0, 1)) != 0


def test_record_layout_offsets_are_aligned_and_ordered():
    for bits in (2, 4, 8):
        for H, I in ((256, 128), (4096, 1024)):
            n, off = gen.record_layout(bits, H, I)
            assert all(o % 16 == 0 for o in off) and off == sorted(off) and n % 16 == 0
    # groups of 128: the scale and bias arrays are half as long
    n64, _ = gen.record_layout(4, 4096, 1024)
    n128, _ = gen.record_layout(4, 4096, 1024, group=128)
    assert n64 - n128 == 3 * 2 * 1024 * (4096 // 128) * 2
    assert gen.algorithmic_bytes_per_token(gen.qwen397_layer(4)) == 39583744
    assert gen.algorithmic_bytes_per_token(gen.qwen397_layer(2)) == 23855104
    assert gen.algorithmic_bytes_per_token(gen.tiny_layer()) == 169984


def test_gdn_inputs_follow_the_recipe():
    """Gated DeltaNet inputs: unit keys, queries of norm dk^-1/2, gates in their ranges on a
    2^-24 grid, a seeded state with the stated spread; fresh draws per token and layer."""
    spec = gen.GdnSpec(heads=16, dk=128, dv=64)
    t0 = gen.host_gdn_token(spec, 2, 0)
    assert np.allclose(np.linalg.norm(t0["k"].astype(np.float64), axis=1), 1.0, atol=1e-6)
    assert np.allclose(np.linalg.norm(t0["q"].astype(np.float64), axis=1), 128 ** -0.5, atol=1e-6)
    assert np.all((t0["alpha"] >= 0.8) & (t0["alpha"] < 1.0)) and np.all((t0["beta"] >= 0) & (t0["beta"] < 1))
    assert np.all(t0["beta"] * 2.0 ** 24 == np.round(t0["beta"] * 2.0 ** 24))
    assert t0["v"].shape == (16, 64) and t0["q"].shape == (16, 128)
    t1 = gen.host_gdn_token(spec, 2, 1)
    u = gen.host_gdn_token(spec, 3, 0)
    assert not np.array_equal(t0["k"], t1["k"]) and not np.array_equal(t0["k"], u["k"])
    assert np.array_equal(t0["k"], gen.host_gdn_token(spec, 2, 0)["k"])
    S = gen.host_gdn_state(spec, layer=2)
    assert S.shape == (16, 64, 128) and abs(float(S.std()) - 0.1) < 0.005
