"""Host-side helpers of the sparse decode's inputs (no GPU): the seeded index lists and the
algorithmic byte/flop counts bench.py divides by."""
import numpy as np
import pytest

from mla_decode_attention_14_b200 import workloads as W


@pytest.mark.parametrize("order", ["sorted", "shuffled"])
def test_sparse_indices_are_distinct_positions_of_their_sequence(order):
    sl = np.array([0, 5, 64, 1000], dtype=np.int32)
    ix = W.sparse_indices(sl, 3, 100, seed=7, order=order)
    assert ix.shape == (4, 3, 100) and ix.dtype == np.int32
    for b, n in enumerate(sl):
        for t in range(3):
            row = ix[b, t]
            k = min(100, int(n))
            assert np.all(row[k:] == -1)  # padding past the sequence's own positions
            keys = row[:k]
            assert len(set(keys.tolist())) == k and np.all((keys >= 0) & (keys < n))
            if order == "sorted":
                assert np.all(np.diff(keys) > 0)
    # a sequence shorter than the list lists every position
    assert sorted(ix[1, 0, :5].tolist()) == [0, 1, 2, 3, 4]


def test_sparse_indices_are_seeded():
    sl = np.array([300, 700], dtype=np.int32)
    a = W.sparse_indices(sl, 2, 64, seed=3, order="shuffled")
    assert np.array_equal(a, W.sparse_indices(sl, 2, 64, seed=3, order="shuffled"))
    assert not np.array_equal(a, W.sparse_indices(sl, 2, 64, seed=4, order="shuffled"))


def test_sparse_counts_count_keys_not_list_entries():
    wl = W.custom(2, 16, 2, [10, 100])
    ix = np.full((2, 2, 8), -1, dtype=np.int32)
    ix[0, 0, :3] = [0, 9, 10]      # 10 is past sequence 0's end: 2 keys
    ix[1, 1, :] = [5] * 8          # a position listed 8 times counts 8 times
    c = W.sparse_counts(wl, ix)
    keys = 2 + 8
    assert c["kv_bytes"] == keys * 1152
    assert c["q_bytes"] == 2 * 2 * 16 * 1152
    assert c["flops"] == keys * 16 * 2 * (576 + 512)
    assert c["bytes"] == c["kv_bytes"] + c["q_bytes"]
