"""The top-k kernels compare raw fp32 scores with a threshold's float value in
their streaming passes instead of turning every score into its order-preserving
32-bit key first.  That is exact only if, for every non-NaN score f and every
key value th, key(f) >= th exactly when f >= score(th), and key(f) > th / == th
exactly when f > score(th) / f == score(th), where -0.0 and +0.0 map to the same
key (the selection treats them as equal, as the oracle's float comparison does).

This restates the two maps from their definition (sign bit flipped for
non-negative floats, all bits complemented for negative ones, -0.0 folded onto
+0.0) and checks the equivalences over float landmarks, random scores and random
thresholds, including thresholds that are keys of no score in the row."""
import numpy as np


def _key(f):
    u = np.asarray(f, np.float32).view(np.uint32).copy()
    u[(u << np.uint32(1)) == 0] = 0                      # -0.0 -> +0.0
    neg = (u & np.uint32(0x80000000)) != 0
    return np.where(neg, ~u, u | np.uint32(0x80000000)).astype(np.uint32)


def _score(k):
    k = np.asarray(k, np.uint32)
    pos = (k & np.uint32(0x80000000)) != 0
    return np.where(pos, k & np.uint32(0x7FFFFFFF), ~k).astype(np.uint32).view(np.float32)


def _scores():
    rng = np.random.default_rng(7)
    landmarks = np.array([0.0, -0.0, 1.0, -1.0, 1e-45, -1e-45, 1.17549435e-38, -1.17549435e-38,
                          3.4028235e38, -3.4028235e38, np.inf, -np.inf, 0.5, -0.5], np.float32)
    return np.concatenate([landmarks, rng.standard_normal(4000).astype(np.float32),
                           (rng.integers(-16, 16, 2000) / 8).astype(np.float32),
                           rng.standard_normal(500).astype(np.float32) * np.float32(1e-38)])


def test_key_order_is_float_order_with_signed_zeros_equal():
    f = _scores()
    k = _key(f)
    i, j = np.random.default_rng(1).integers(0, f.size, (2, 20000))
    assert np.array_equal(k[i] > k[j], f[i] > f[j])
    assert np.array_equal(k[i] == k[j], f[i] == f[j])
    assert _key(np.float32(-0.0)) == _key(np.float32(0.0))


def test_threshold_compares_match_on_keys_and_on_floats():
    f = _scores()
    k = _key(f)
    rng = np.random.default_rng(2)
    own = np.concatenate([k[rng.integers(0, f.size, 300)], _key(np.array([0.0, -0.0], np.float32))])
    # A sampled threshold (the single passes, ">=") can be any key, also one that
    # is the key of no score -- 0x7fffffff lies between the key of the largest
    # negative float and that of zero; the exact threshold of the output passes
    # (">", "==") is always the key of a score of the row.
    anyk = np.concatenate([own, rng.integers(0, 2**32, 300, dtype=np.uint64).astype(np.uint32),
                           np.array([0x7FFFFFFF, 0x80000000, 0x7FFFFFFE], np.uint32)])
    anyk = anyk[~np.isnan(_score(anyk))]                                 # keys of NaN are no threshold
    for th in anyk:
        assert np.array_equal(k >= th, f >= _score(np.array([th]))[0])
    for th in own:
        tf = _score(np.array([th]))[0]
        assert np.array_equal(k > th, f > tf)
        assert np.array_equal(k == th, f == tf)


def test_score_of_key_round_trips():
    f = _scores()
    back = _score(_key(f))
    assert np.array_equal(back.view(np.uint32), np.where(f == 0, np.float32(0.0), f).view(np.uint32))
