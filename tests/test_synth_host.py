"""The seeded input generator on the host (CPU only)."""
import numpy as np
import torch

from synth import gen


def test_splitmix64_published_test_vector():
    # first five outputs of SplitMix64 seeded with 1234567 (the published reference values)
    got = [int(x) for x in gen.raw_u64(1234567, 0, 5)]
    assert got == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                   4593380528125082431, 16408922859458223821]


def test_streams_are_addressable_and_distinct():
    k = gen.stream_key(7, gen.KIND_K, 3, 1, 2)
    a = gen.raw_u64(k, 0, 1000)
    b = gen.raw_u64(k, 600, 400)
    assert np.array_equal(a[600:], b)
    k2 = gen.stream_key(7, gen.KIND_K, 3, 1, 3)
    assert not np.array_equal(gen.raw_u64(k2, 0, 16), a[:16])


def test_normal_moments():
    x = gen.normal_f64(gen.stream_key(1, gen.KIND_V, 0, 0, 0), 0, 1 << 20)
    assert abs(x.mean()) < 5e-3
    assert abs(x.std() - 1.0) < 5e-3
    assert np.max(np.abs(x)) <= 2 * 3 ** 0.5
    # excess kurtosis of the Irwin-Hall(4) law is -6/20
    k = np.mean(x ** 4) / np.mean(x ** 2) ** 2 - 3
    assert abs(k + 0.3) < 0.02


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-6, 6, 100000),
                        np.array([0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1 + 2 ** -8)])])
    ours = gen.f64_to_bf16_bits(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(ours.view(np.int16), ref)


def test_key_offset_has_variance_two():
    offs = np.concatenate([gen.key_offset(3, 0, 0, g, 128) for g in range(256)])
    assert abs(offs.var() - 2.0) < 0.1


def test_needles_distinct_in_candidate_range():
    q = gen.gen_q(5, 1, 32, 128)
    nd = gen.gen_needles(5, 0, q, 8, 64, 131072, 128, 512)
    for g in range(8):
        p = nd.pos[0, g]
        assert len(set(p.tolist())) == 64
        assert p.min() >= 128 and p.max() < 131072 - 512
        assert set(nd.head[0, g].tolist()) == set(range(g * 4, g * 4 + 4))


def test_budgets_as_fractions():
    assert gen.workload("l8b_128k_k1pct").k == 1310
    assert gen.workload("l8b_1m_32layer").k == 20971
    assert gen.workload("l8b_b16_256k").k == 2621
    assert gen.workload("sweep_k1pct_g4_d128").k == 5242
    assert gen.workload("sweep_k5pct_g8_d64").k == 26214
    assert len(gen.sweep_names()) == 18
