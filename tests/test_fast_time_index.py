"""Host-side checks of the float time-bucket index the tensor-core kernels use.

When a sequence's timestamps span less than 2^24 s the kernels take
dt = float(t_i - t_min) - float(t_j - t_min) and index a small per-CTA table by
the float's exponent and top sub_bits mantissa bits:
    idx(dt) = max(bits(dt) >> (23 - s), R0) - R0,   R0 = (127 << s) - 1.
(The GPU test test_buckets_bit_exact checks that the table maps idx to the
oracle's bucket.)  Two shortcuts rest on properties of idx that these tests
pin down on the CPU:

* chunk classification: for sorted timestamps idx is monotone in dt, so a
  chunk whose two ends share an index holds one bucket, and ends one apart
  hold at most two;
* the two-bucket split: for b >= 0 and dt >= 0,
      idx(dt) >= b + 1  <=>  dt >= float_from_bits((b + 1 + R0) << (23 - s)),
  so one float compare picks the bucket of a pair.
"""
import numpy as np
import pytest


def idx(dt: np.ndarray, s: int) -> np.ndarray:
    bits = np.asarray(dt, np.float32).view(np.int32).astype(np.int64)
    r0 = (127 << s) - 1
    return np.maximum(bits >> (23 - s), r0) - r0


def thr(b: int, s: int) -> np.float32:
    r0 = (127 << s) - 1
    return np.array([(b + 1 + r0) << (23 - s)], np.int32).view(np.float32)[0]


def table_size(s: int) -> int:
    return (24 << s) + 1


def samples(rng) -> np.ndarray:
    # The float path is taken only when a sequence spans less than 2^24 s, so
    # dt lies in [0, 2^24 - 1]: exact integers, powers of two and their
    # neighbours, the top of the range, and random integers over all of it.
    ints = np.arange(0, 4097, dtype=np.float32)
    p2 = 2.0 ** np.arange(0, 24)
    near = np.concatenate([p2 - 1, p2, p2 + 1, [2.0 ** 24 - 1]]).astype(np.float32)
    rnd = rng.integers(0, 2 ** 24, size=20000).astype(np.float32)
    return np.unique(np.concatenate([ints, near, rnd]))


@pytest.mark.parametrize("s", [0, 1, 2, 3, 4])
def test_index_is_monotone_and_within_the_table(s):
    dt = samples(np.random.default_rng(s))
    i = idx(dt, s)
    assert np.all(np.diff(i) >= 0)
    assert i.min() == 0 and i.max() < table_size(s)
    # negative deltas (masked pairs) fall to index 0
    assert np.all(idx(-dt[dt > 0], s) == 0)


@pytest.mark.parametrize("s", [0, 1, 2, 3, 4])
def test_two_bucket_threshold_is_exact(s):
    rng = np.random.default_rng(10 + s)
    base = samples(rng)
    for b in range(table_size(s) - 1):
        t = thr(b, s)
        # the threshold itself and its float neighbours on both sides
        edge = np.array([np.nextafter(t, np.float32(0)), t, np.nextafter(t, np.float32(np.inf))],
                        np.float32)
        dt = np.concatenate([base, edge])
        want = idx(dt, s) >= b + 1
        got = dt >= t
        assert np.array_equal(want, got), (s, b)


def test_threshold_lands_on_bucket_boundaries():
    # s = 0: the index is the float exponent, so the thresholds are 2^b
    for b in range(0, 24):
        assert thr(b, 0) == np.float32(2.0 ** b)
    # s = 2: four sub-buckets per octave, boundaries at 1, 1.25, 1.5, 1.75, 2, 2.5 ...
    want = [1.0, 1.25, 1.5, 1.75, 2.0, 2.5, 3.0, 3.5, 4.0]
    assert [float(thr(b, 2)) for b in range(9)] == want
