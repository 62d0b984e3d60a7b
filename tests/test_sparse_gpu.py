"""GPU parity of the sparse decode (mla_decode_sparse) against the CPU oracle (needs a B200).

Row (b, t, h) attends to the cache positions indices[b, t, :] only (entries outside
[0, seqlens[b]) are no key, duplicates count twice, order does not matter). The oracle is
oracle.decode_sparse; tolerances are those of the dense decode.
"""
import numpy as np
import pytest
import torch

import mla_decode_attention_14_b200 as mla
import oracle
from mla_decode_attention_14_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu

MLA_ERR_BOUNDS = 6


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def run_sparse(inp, indices, num_parts=None):
    q, kv, bt, sl = parity.to_device(inp)
    b, s_q, h_q, _ = q.shape
    ix = torch.from_numpy(np.ascontiguousarray(indices, dtype=np.int32)).cuda()
    meta = mla.get_metadata_sparse(b, s_q, h_q, ix.shape[2], num_parts=num_parts)
    out, lse = mla.decode_sparse(q, kv, bt, sl, ix, inp["scale"], meta)
    return out, lse, mla.check_status()


def sparse_parity(inp, indices, num_parts=None, what=""):
    out, lse, status = run_sparse(inp, indices, num_parts)
    assert status == 0, "%s: device error status %d" % (what, status)
    ref_o, ref_l = oracle.decode_sparse(inp["q"], inp["kv"], inp["block_table"], inp["seqlens"], indices,
                                        inp["scale"])
    parity.compare(parity.bf16_to_f64(out), lse.cpu().numpy().astype(np.float64), ref_o, ref_l, what)
    return out, lse


CASES = [
    # seqlens, h_q, s_q, topk, order, num_parts
    ([1000, 64, 333], 16, 1, 100, "sorted", None),
    ([1000, 64, 333], 16, 1, 100, "shuffled", 5),
    ([1000, 64, 333], 128, 1, 256, "shuffled", None),
    ([700, 90], 128, 2, 37, "sorted", 3),      # two 128-row groups with different lists
    ([700, 90, 5], 64, 4, 130, "shuffled", None),  # lists longer than a sequence: -1 padding
    ([3000], 16, 2, 1000, "sorted", 1),       # one part walks every block
]


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_sparse_parity(case):
    seqlens, h_q, s_q, topk, order, parts = case
    wl = W.custom(len(seqlens), h_q, s_q, seqlens)
    inp = W.make_inputs(wl, seed=21, tail="nan", spare_blocks=2)
    ix = W.sparse_indices(wl.seqlens, s_q, topk, seed=3, order=order)
    sparse_parity(inp, ix, parts, "sparse %s" % (case,))


def test_invalid_and_duplicate_entries():
    """-1, negative and past-the-end entries are no key; a duplicated position counts twice."""
    wl = W.custom(2, 16, 1, [500, 200])
    inp = W.make_inputs(wl, seed=4, tail="nan")
    ix = W.sparse_indices(wl.seqlens, 1, 150, seed=9, order="shuffled")
    ix[0, 0, ::7] = -1
    ix[0, 0, 3::11] = 500          # == seqlen: no key
    ix[1, 0, 5::13] = -12345
    ix[1, 0, 100:110] = ix[1, 0, 0]  # ten copies of one key
    sparse_parity(inp, ix, what="invalid and duplicate entries")


def test_full_list_in_order_equals_dense():
    """Listing every position of each sequence in order reproduces the dense decode."""
    wl = W.custom(3, 64, 1, [300, 64, 129])
    inp = W.make_inputs(wl, seed=8, tail="nan")
    ix = np.full((3, 1, 300), -1, dtype=np.int32)
    for b, n in enumerate(wl.seqlens):
        ix[b, 0, :n] = np.arange(n)
    out, lse = sparse_parity(inp, ix, what="full list")
    ref_o, ref_l = oracle.decode(inp["q"], inp["kv"], inp["block_table"], inp["seqlens"], inp["scale"], False)
    parity.compare(parity.bf16_to_f64(out), lse.cpu().numpy().astype(np.float64), ref_o, ref_l, "full list = dense")


def test_rows_without_keys_give_zero_and_neg_inf():
    wl = W.custom(3, 16, 2, [100, 0, 64])
    inp = W.make_inputs(wl, seed=2, tail="nan")
    ix = W.sparse_indices(wl.seqlens, 2, 64, seed=1)
    ix[2, 1, :] = -1  # one query token of a non-empty sequence with no valid entry
    out, lse, status = run_sparse(inp, ix)
    assert status == 0
    o, l = out.float().cpu(), lse.cpu()
    assert torch.all(o[1] == 0) and torch.all(torch.isneginf(l[1]))
    assert torch.all(o[2, 1] == 0) and torch.all(torch.isneginf(l[2, :, 1]))
    sparse_parity(inp, ix, what="rows without keys")


def test_bad_block_table_entry_is_reported_not_read():
    """A listed position whose block-table entry is outside [0, num_blocks) is skipped and reported."""
    wl = W.custom(2, 16, 1, [256, 128])
    inp = W.make_inputs(wl, seed=6, tail="nan")
    ix = W.sparse_indices(wl.seqlens, 1, 64, seed=2)
    inp["block_table"] = inp["block_table"].copy()
    inp["block_table"][0, 1] = inp["num_blocks"] + 7  # positions 64..127 of sequence 0
    _, _, status = run_sparse(inp, ix)
    assert status == MLA_ERR_BOUNDS


def test_sparse_metadata_is_the_partition_of_uniform_lengths():
    """mla_get_metadata_sparse equals the oracle partition of batch * s_q units of topk keys, bit for bit."""
    for b, s_q, h_q, topk, parts in [(128, 1, 128, 2048, 74), (3, 4, 64, 130, 7), (1, 1, 16, 1, 148)]:
        meta = mla.get_metadata_sparse(b, s_q, h_q, topk, num_parts=parts, fixed_cost=10)
        otm, ons = oracle.metadata(np.full(b * s_q, topk, dtype=np.int32), parts, 10)
        assert np.array_equal(meta.tile_meta.cpu().numpy(), otm)
        assert np.array_equal(meta.num_splits.cpu().numpy(), ons)


def test_full_size_v3_topk2048_every_row():
    """The v3 workload's sequences with 2048-key lists per query token (uniform, sorted), every row
    against the oracle, in the launch configuration bench.py times."""
    wl = W.workload("v3")
    inp = W.make_inputs(wl, seed=0, tail="nan")
    ix = W.sparse_indices(wl.seqlens, wl.s_q, 2048, seed=0)
    out, _ = sparse_parity(inp, ix, what="v3 top-2048")
    assert torch.isfinite(out.float()).all()
