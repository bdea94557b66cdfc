"""The seeded input generators: parameter draws match the pages' statement
(odd multipliers below 2^31, one distinct prime per head, a surjective
compressed-ID lookup) and the workload sizes match the stated shapes."""
import numpy as np

from hashed_gram_conditional_hash_b200 import workloads as W


def _fermat_probable_prime(n):
    return all(pow(a, n - 1, n) == 1 for a in (2, 3, 5, 7, 11, 13) if a < n)


def test_primes_are_distinct_primes_from_base():
    for w in W.CONFIGS.values():
        p = W.head_primes(w)
        assert len(p) == w.nh and len(set(p.tolist())) == w.nh
        assert p[0] >= w.prime_base and np.all(np.diff(p) > 0)
        assert all(_fermat_probable_prime(int(v)) for v in p)
    # the tiny workload's first primes from 1009
    assert W.head_primes(W.CONFIGS["tiny_f32"]).tolist() == [1009, 1013, 1019, 1021, 1031, 1033, 1039, 1049]


def test_multipliers_odd_and_seeded_per_layer():
    w = W.CONFIGS["large_table_bf16"]
    m = W.multipliers(w)
    assert len(m) == w.max_n and np.all(m % 2 == 1) and np.all(m < 2 ** 31)
    assert not np.array_equal(m, W.multipliers(w.replace(layer_id=1)))
    np.testing.assert_array_equal(m, W.multipliers(w))


def test_lookup_is_surjective_and_ids_in_range():
    w = W.CONFIGS["tiny_f32"]
    lut = W.compress_lookup(w)
    assert lut.shape == (2048,) and set(lut.tolist()) == set(range(1580))
    ids = W.token_ids(w)
    assert ids.shape == (1, 128) and ids.min() >= 0 and ids.max() < 2048
    for name in ("model_bf16", "hbm_table_bf16"):
        w = W.CONFIGS[name]
        ids = W.token_ids(w)
        assert ids.shape == (w.B, w.T) and ids.min() >= 0 and ids.max() < w.vocab


def test_decode_stream_shape():
    w = W.CONFIGS["decode_bf16"]
    assert W.token_ids(w).shape == (1024, 256)


def test_table_sizes():
    gb = lambda n: W.table_bytes(W.CONFIGS[n]) / 1e9
    assert 0.12 < gb("model_bf16") < 0.15
    assert 3.1 < gb("large_table_bf16") < 3.3
    assert 17.0 < gb("hbm_table_bf16") < 17.4
