"""The seeded input generator: determinism, sub-range draws, distributions, rank rule."""
import numpy as np

from synth import gen


def test_counter_based_subranges():
    k = gen.stream_key(3, gen.T_X, 2, 5)
    full = gen.normals(k, 1000)
    np.testing.assert_array_equal(full[200:300], gen.normals(k, 100, offset=200))
    np.testing.assert_array_equal(full[201:260], gen.normals(k, 59, offset=201))
    np.testing.assert_array_equal(gen.uniforms(k, 10), gen.uniforms(k, 10))
    assert gen.stream_key(3, 1) != gen.stream_key(3, 2)
    # SplitMix64 reference values: mix64(0x9E3779B97F4A7C15) for seed 0, first output
    z = gen.raw64(np.uint64(0), 1)[0]
    assert int(z) == 0xE220A8397B1DCDAF


def test_normal_moments():
    x = gen.normals(gen.stream_key(1, 0), 200000)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01


def test_haar_frame_orthonormal():
    U = gen.haar_frame(gen.stream_key(2, 0), 300, 64)
    assert np.abs(U.T @ U - np.eye(64)).max() < 1e-12


def test_ragged_ranks_rule():
    for seed in range(6):
        r = gen.ragged_ranks(seed, 0, 32)
        assert sum(r) == 32 * 32 and all(16 <= x <= 64 and x % 8 == 0 for x in r)
        r = gen.ragged_ranks(seed, 0, 8)
        assert sum(r) == 8 * 32 and all(16 <= x <= 64 and x % 8 == 0 for x in r)
    assert gen.config_spec(1).key_ranks == gen.config_spec(2).key_ranks


def test_page_tables_cover_pool():
    pt, n = gen.page_tables(0, [33, 16, 1], 16, extra_pages=3)
    used = pt[pt >= 0]
    assert len(set(used.tolist())) == len(used) == 3 + 1 + 1 and n == 8 and used.max() < n
