"""Pins for the CPU oracle's sparse mode (no GPU): query token t of sequence b attends only to the
keys at the listed positions, shared by all its heads; entries outside the sequence are no key.

Tied to the pinned dense oracle (the full list in order is dense decode, bit for bit), to
invariants (list order, invalid entries), closed forms (one key, no key) and a float64 torch SDPA
over the gathered keys."""
import numpy as np
import pytest
import torch

import oracle
from mla_decode_attention_14_b200 import workloads as W

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")
BLK, DQK, DV = 64, 576, 512


def _inputs(seqlens, h_q, s_q, seed=0):
    wl = W.custom(len(seqlens), h_q, s_q, seqlens)
    return wl, W.make_inputs(wl, seed=seed, tail="nan", spare_blocks=2)


def test_full_list_in_order_is_dense_decode():
    wl, inp = _inputs([1, 70, 130], 8, 1)
    topk = 160
    ix = np.full((3, 1, topk), -1, np.int32)
    for b, n in enumerate(wl.seqlens):
        ix[b, 0, :n] = np.arange(n)
    so, sl = oracle.decode_sparse(inp["q"], inp["kv"], inp["block_table"], inp["seqlens"], ix, wl.scale)
    do, dl = oracle.decode(inp["q"], inp["kv"], inp["block_table"], inp["seqlens"], wl.scale, False)
    assert np.array_equal(so, do) and np.array_equal(sl, dl)


def test_list_order_and_invalid_entries_do_not_matter():
    wl, inp = _inputs([200, 90], 4, 2, seed=3)
    rng = np.random.default_rng(1)
    base = np.stack([np.stack([rng.choice(int(n), 40, replace=False) for _ in range(2)]) for n in wl.seqlens]).astype(np.int32)
    perm = base[..., rng.permutation(40)]
    padded = np.concatenate([base, np.full((2, 2, 5), -1, np.int32), np.full((2, 2, 3), 10 ** 6, np.int32)], axis=2)
    o1, l1 = oracle.decode_sparse(inp["q"], inp["kv"], inp["block_table"], inp["seqlens"], base, wl.scale)
    o2, l2 = oracle.decode_sparse(inp["q"], inp["kv"], inp["block_table"], inp["seqlens"], perm, wl.scale)
    o3, l3 = oracle.decode_sparse(inp["q"], inp["kv"], inp["block_table"], inp["seqlens"], padded, wl.scale)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(l2, l1, rtol=1e-13)
    assert np.array_equal(o3, o1) and np.array_equal(l3, l1)


def test_one_key_and_no_key():
    wl, inp = _inputs([100], 3, 2, seed=4)
    ix = np.array([[[-1, 37, -1], [-1, -1, 500]]], np.int32)  # token 0: key 37 only; token 1: none
    o, l = oracle.decode_sparse(inp["q"], inp["kv"], inp["block_table"], inp["seqlens"], ix, wl.scale)
    row = inp["kv"][inp["block_table"][0, 0], 37, 0]
    v = W.bf16_bits_to_f32(row).astype(np.float64)
    for h in range(3):
        assert np.array_equal(o[0, 0, h], v[:DV])
        qv = W.bf16_bits_to_f32(inp["q"][0, 0, h]).astype(np.float64)
        assert abs(l[0, h, 0] - wl.scale * (qv @ v)) < 1e-12 * max(1.0, abs(l[0, h, 0]))
    assert np.all(o[0, 1] == 0) and np.all(np.isneginf(l[0, :, 1]))


def test_matches_library_sdpa_on_gathered_keys():
    wl, inp = _inputs([300, 65], 4, 2, seed=5)
    rng = np.random.default_rng(2)
    ix = np.stack([np.stack([rng.choice(int(n), 50, replace=False) for _ in range(2)]) for n in wl.seqlens]).astype(np.int32)
    o, l = oracle.decode_sparse(inp["q"], inp["kv"], inp["block_table"], inp["seqlens"], ix, wl.scale, nthreads=4)
    for b in range(2):
        for t in range(2):
            rows = [inp["kv"][inp["block_table"][b, p // BLK], p % BLK, 0] for p in ix[b, t]]
            k = torch.from_numpy(W.bf16_bits_to_f32(np.stack(rows)).astype(np.float64))
            q = torch.from_numpy(W.bf16_bits_to_f32(inp["q"][b, t]).astype(np.float64))
            ref = torch.nn.functional.scaled_dot_product_attention(q[None, None], k[None, None], k[None, None, :, :DV],
                                                                   scale=wl.scale)[0, 0].numpy()
            np.testing.assert_allclose(o[b, t], ref, rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(l[b, :, t], torch.logsumexp(wl.scale * (q @ k.T), dim=-1).numpy(), rtol=1e-12)
