"""Pins for the float acceptance rule and the seeded input generator."""

import numpy as np

import oracle as O
from synthetic import gen, WORKLOADS, layer_inputs


def _scalar_splitmix(seed, n):
    out, s = [], seed
    for _ in range(n):
        s = (s + 0x9E3779B97F4A7C15) & 0xFFFFFFFFFFFFFFFF
        z = s
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & 0xFFFFFFFFFFFFFFFF
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & 0xFFFFFFFFFFFFFFFF
        out.append(z ^ (z >> 31))
    return out


def test_splitmix_matches_scalar_definition():
    for seed in (0, 1, 12345, 2 ** 63 + 7):
        assert gen.splitmix64(seed, 50).tolist() == _scalar_splitmix(seed, 50)
    assert gen.splitmix64(9, 5, offset=20).tolist() == _scalar_splitmix(9, 25)[20:]


def test_normal_draws_are_deterministic_and_standard():
    a = gen.normal(42, 200000, 1.0)
    assert np.array_equal(a, gen.normal(42, 200000, 1.0))
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1.0) < 0.01
    assert abs(gen.normal(43, 100000, 0.02).std() - 0.02) < 0.0005


def test_normal_draws_do_not_depend_on_the_thread_split():
    count = 2 * gen._BLOCK_PAIRS * 2 + 3  # two full blocks of pairs and a ragged third
    blocked = gen.normal(44, count, 1.0)
    whole = np.empty(2 * ((count + 1) // 2))
    gen._box_muller(44, 0, (count + 1) // 2, whole)
    assert np.array_equal(blocked.view(np.uint64), whole[:count].view(np.uint64))
    # each draw depends only on its index: a block starting mid-stream agrees
    part = np.empty_like(whole)
    gen._box_muller(44, 12345, 12345 + 64, part)
    assert np.array_equal(part[2 * 12345:2 * 12345 + 128].view(np.uint64),
                          whole[2 * 12345:2 * 12345 + 128].view(np.uint64))


def test_bf16_rounding_of_inputs():
    f = np.float32([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, np.inf])
    assert gen.f32_to_bf16_bits(f).tolist() == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x7F80]


def test_workload_shapes():
    wl = WORKLOADS["tiny_256x512x512_r16"]
    d = layer_inputs(wl, wl.layers[0])
    assert d["X"].shape == (256, 512) and d["X"].dtype == np.uint16
    assert d["W"].shape == (512, 512) and d["W"].dtype == np.float32
    assert d["A"].shape == (16, 512) and d["B"].shape == (512, 16) and not d["B"].any()
    assert d["dY"].shape == (256, 512)


def test_tolerance_accepts_rounded_and_rejects_two_ulps():
    rng = np.random.default_rng(5)
    R = rng.standard_normal((64, 64))
    Rb = O.bf16_round(R)
    assert O.within_tolerance(Rb, R)
    bad = Rb.copy()
    bad[3, 4] = bad[3, 4] + 2 if (bad[3, 4] & 0x7F) < 0x7D else bad[3, 4] - 2
    assert not O.within_tolerance(bad, R)


def test_tolerance_floor_near_zero_and_all_zero():
    R = np.array([1.0, 1e-6, -1e-7, 0.0])
    G = np.array([1.0, 1e-3 * 2 ** -8, 0.0, 2 ** -9 * 2 ** -8])  # below tau-scaled ulp
    assert O.within_tolerance(G, R)
    assert not O.within_tolerance(np.array([1.0, 0.01, 0.0, 0.0]), R)
    assert O.within_tolerance(np.zeros(4), np.zeros(4))
    assert not O.within_tolerance(np.array([0, 0, 1e-30, 0.0]), np.zeros(4))
