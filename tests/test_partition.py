"""hstu_partition_batch (the data-parallel split of a jagged batch) on the
CPU: every sequence goes to one rank, the reported loads are the visible-pair
counts, the split is deterministic, and its largest load stays within the
longest-processing-time bound 4/3 - 1/(3 world) of the best split, which brute
force finds on small batches."""
import itertools

import numpy as np
import pytest

from hstu_pointwise_attention_b200 import ops


def pairs(L, nc):
    nh = L - nc
    return nh * (nh + 1) // 2 + nc * (nh + 1)


def offsets(lengths):
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)


@pytest.mark.parametrize("seed, world", [(0, 2), (1, 3), (2, 2), (3, 4)])
def test_split_is_within_the_lpt_bound_of_brute_force(seed, world):
    rng = np.random.default_rng(seed)
    B = 7
    lengths = rng.integers(0, 300, size=B)
    nc = np.minimum(rng.integers(0, 40, size=B), lengths).astype(np.int32)
    rank_of, load = ops.partition_batch(offsets(lengths), world, nc)
    cost = [pairs(int(L), int(c)) for L, c in zip(lengths, nc)]
    assert rank_of.shape == (B,) and np.all((rank_of >= 0) & (rank_of < world))
    for r in range(world):
        assert load[r] == sum(c for c, rr in zip(cost, rank_of) if rr == r)
    best = min(max(sum(c for c, rr in zip(cost, a) if rr == r) for r in range(world))
               for a in itertools.product(range(world), repeat=B))
    assert load.max() <= (4 / 3 - 1 / (3 * world)) * best + 1e-9


def test_equal_sequences_split_evenly_and_deterministically():
    off = offsets([8192] * 8)
    a, la = ops.partition_batch(off, 4)
    b, lb = ops.partition_batch(off, 4)
    assert np.array_equal(a, b) and np.array_equal(la, lb)
    assert np.bincount(a, minlength=4).tolist() == [2, 2, 2, 2]
    assert len(set(la.tolist())) == 1


def test_more_ranks_than_sequences_and_empty_batch():
    rank_of, load = ops.partition_batch(offsets([5, 3]), 4)
    assert sorted(rank_of.tolist()) == [0, 1] and load.tolist() == [15, 6, 0, 0]
    rank_of, load = ops.partition_batch(np.zeros(1, np.int64), 3)
    assert rank_of.size == 0 and load.tolist() == [0, 0, 0]


@pytest.mark.parametrize("off, nc, world", [
    ([1, 5], None, 2),          # offsets[0] != 0
    ([0, 5, 3], None, 2),       # decreasing
    ([0, 5], [6], 2),           # more candidates than tokens
    ([0, 5], None, 0),          # no ranks
])
def test_bad_arguments_are_rejected(off, nc, world):
    with pytest.raises(ops.HstuError):
        ops.partition_batch(np.array(off, np.int64), world,
                            None if nc is None else np.array(nc, np.int32))
