"""Pins for the oracle's split-KV work partition (no GPU): a hand-worked fixture,
and structural invariants checked by brute force over every (sequence, block)."""
import numpy as np
import pytest

import oracle
from tests import meta_util


def test_hand_worked_fixture():
    seqlens, C, cases = meta_util.load_golden()
    assert cases
    for P, T, meta, cum in cases:
        tm, ns = oracle.metadata(seqlens, P, C)
        assert np.array_equal(tm, meta), (P, tm, meta)
        assert np.array_equal(ns, cum), (P, ns, cum)


def test_all_empty_sequences():
    tm, ns = oracle.metadata([0, 0, 0], 4, 5)
    assert np.all(ns == 0)
    assert np.all(tm[:, 2] == -1)


@pytest.mark.parametrize("seed", range(12))
def test_random_partitions_are_valid(seed):
    rng = np.random.default_rng(seed)
    b = int(rng.integers(1, 200))
    kind = seed % 3
    if kind == 0:
        sl = rng.integers(0, 9000, size=b)
    elif kind == 1:
        sl = np.clip(np.rint(rng.lognormal(np.log(2048), 1.5, size=b)), 1, 65536)
    else:
        sl = rng.choice([1, 63, 64, 65, 65536, 0, 128, 4096], size=b)
    sl = sl.astype(np.int32)
    P = int(rng.integers(1, 160))
    C = int(rng.integers(0, 9))
    tm, ns = oracle.metadata(sl, P, C)
    meta_util.check_partition(sl, tm, ns, P, C)


def test_single_part_takes_everything_unsplit():
    sl = np.array([5, 700, 64], dtype=np.int32)
    tm, ns = oracle.metadata(sl, 1, 3)
    assert list(tm[0, :5]) == [0, 0, 2, 1, 0]
    assert list(ns) == [0, 1, 2, 3]


def test_one_long_sequence_splits_evenly():
    # 1024 blocks, C = 4, P = 8 -> U = 1028, T = 129: part p holds units [129p, 129p+129)
    tm, ns = oracle.metadata([65536], 8, 4)
    assert ns[1] == 8
    sizes = tm[:, 3] - tm[:, 1]
    assert sizes[0] == 125 and np.all(sizes[1:7] == 129) and sizes[7] == 1024 - 125 - 6 * 129
    assert list(tm[:, 4]) == list(range(8))
