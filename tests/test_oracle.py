"""Pins for the CPU oracle's attention (no GPU).

Each test ties the oracle to something other than its own formula: a library
softmax-attention routine on dense, non-paged tensors; closed forms (one key, two
keys, q = 0); invariants (block relabelling, NaN tails past the sequence end);
and the causal reading reduced to shorter non-causal sequences.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from mla_decode_attention_14_b200 import workloads as W

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

BLK, DQK, DV = 64, 576, 512


def _bits(x):
    """bf16 bit pattern of one float (round to nearest even)."""
    return int(W.f32_to_bf16_bits(np.array([x], dtype=np.float32))[0])


def _dense_case(seqlens, h_q, s_q, seed, spare=3):
    """Dense per-sequence K (and q) first, then scattered into a paged cache."""
    rng = np.random.default_rng(seed)
    b = len(seqlens)
    q = W.f32_to_bf16_bits(rng.standard_normal((b, s_q, h_q, DQK), dtype=np.float32))
    dense = [W.f32_to_bf16_bits(rng.standard_normal((n, DQK), dtype=np.float32)) for n in seqlens]
    w = [(n + BLK - 1) // BLK for n in seqlens]
    nblk = sum(w) + spare
    perm = rng.permutation(nblk)
    kv = W.f32_to_bf16_bits(rng.standard_normal((nblk, BLK, 1, DQK), dtype=np.float32))
    bt = np.full((b, max(1, max(w))), -1, dtype=np.int32)
    off = 0
    for i, n in enumerate(seqlens):
        for k in range(w[i]):
            phys = perm[off]
            off += 1
            bt[i, k] = phys
            rows = dense[i][k * BLK:(k + 1) * BLK]
            kv[phys, :rows.shape[0], 0, :] = rows
            kv[phys, rows.shape[0]:, 0, :] = W.BF16_NAN   # poisoned tail
    return q, kv, bt, np.array(seqlens, dtype=np.int32), dense


def _torch_attention(q_bits, k_bits, scale):
    """float64 torch SDPA on dense tensors: q [rows, 576], k [n, 576] -> out, lse."""
    q = torch.from_numpy(W.bf16_bits_to_f32(q_bits).astype(np.float64))
    k = torch.from_numpy(W.bf16_bits_to_f32(k_bits).astype(np.float64))
    v = k[:, :DV]
    out = torch.nn.functional.scaled_dot_product_attention(
        q[None, None], k[None, None], v[None, None], scale=scale)[0, 0]
    lse = torch.logsumexp(scale * (q @ k.T), dim=-1)
    return out.numpy(), lse.numpy()


@pytest.mark.parametrize("seqlens,h_q", [([1, 63, 64, 65, 130], 4), ([257, 100], 16), ([200], 3)])
def test_dense_bruteforce_matches_library_sdpa(seqlens, h_q):
    scale = W.SCALE
    q, kv, bt, sl, dense = _dense_case(seqlens, h_q, 1, seed=len(seqlens) * 7 + h_q)
    out, lse = oracle.decode(q, kv, bt, sl, scale, causal=False, nthreads=4)
    for i, n in enumerate(seqlens):
        ref_o, ref_l = _torch_attention(q[i, 0], dense[i], scale)
        np.testing.assert_allclose(out[i, 0], ref_o, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(lse[i, :, 0], ref_l, rtol=1e-12, atol=1e-12)


def test_causal_reduces_to_shorter_noncausal():
    # s_q = 2: query 1 sees all n keys, query 0 sees the first n - 1.
    seqlens = [65, 129, 2, 64]
    h_q = 5
    q, kv, bt, sl, dense = _dense_case(seqlens, h_q, 2, seed=11)
    out_c, lse_c = oracle.decode(q, kv, bt, sl, 0.07, causal=True, nthreads=4)
    for i, n in enumerate(seqlens):
        for t, vis in ((0, n - 1), (1, n)):
            ref_o, ref_l = _torch_attention(q[i, t], dense[i][:vis], 0.07)
            np.testing.assert_allclose(out_c[i, t], ref_o, rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(lse_c[i, :, t], ref_l, rtol=1e-12, atol=1e-12)
    # non-causal with s_q = 2: both queries see every key
    out_n, _ = oracle.decode(q, kv, bt, sl, 0.07, causal=False, nthreads=4)
    for i, n in enumerate(seqlens):
        ref_o, _ = _torch_attention(q[i, 0], dense[i], 0.07)
        np.testing.assert_allclose(out_n[i, 0], ref_o, rtol=1e-10, atol=1e-12)


def test_fully_masked_rows_are_zero_and_neg_inf():
    # seqlen 1 with s_q = 2 causal: query 0 sees nothing; seqlen 0: nothing at all.
    q, kv, bt, sl, _ = _dense_case([1, 3], 2, 2, seed=3)
    sl = np.array([1, 0], dtype=np.int32)
    out, lse = oracle.decode(q, kv, bt, sl, 0.1, causal=True, nthreads=2)
    assert np.all(out[0, 0] == 0.0) and np.all(np.isneginf(lse[0, :, 0]))
    assert np.all(out[1] == 0.0) and np.all(np.isneginf(lse[1]))
    assert np.all(np.isfinite(out[0, 1])) and np.all(np.isfinite(lse[0, :, 1]))


def test_single_token_returns_its_value_row_exactly():
    q, kv, bt, sl, dense = _dense_case([1, 1], 7, 1, seed=5)
    out, lse = oracle.decode(q, kv, bt, sl, W.SCALE, causal=False, nthreads=2)
    for i in range(2):
        v = W.bf16_bits_to_f32(dense[i][0, :DV]).astype(np.float64)
        for h in range(7):
            assert np.array_equal(out[i, 0, h], v)
        # lse of one score is the score itself
        qf = W.bf16_bits_to_f32(q[i, 0]).astype(np.float64)
        kf = W.bf16_bits_to_f32(dense[i][0]).astype(np.float64)
        np.testing.assert_allclose(lse[i, :, 0], W.SCALE * (qf @ kf), rtol=1e-13)


def test_two_key_closed_form():
    # q = a e_0 + e_520, k_0 = x0 e_0 (+ value dim 7), k_1 = x1 e_0 + 0.5 e_520 (+ value
    # dim 7). Dim 520 is a rotary (key-only) dim. s_0 = scale a x0, s_1 = scale (a x1 + 0.5);
    # softmax over two scores is a logistic function, so out_d = sig v0_d + (1 - sig) v1_d.
    q = np.zeros((1, 1, 1, DQK), dtype=np.uint16)
    kv = np.zeros((1, BLK, 1, DQK), dtype=np.uint16)
    a, x0, x1 = 2.0, 1.5, -0.75
    q[0, 0, 0, 0] = _bits(a)
    q[0, 0, 0, 520] = _bits(1.0)     # rope dim
    kv[0, 0, 0, 0] = _bits(x0)
    kv[0, 1, 0, 0] = _bits(x1)
    kv[0, 1, 0, 520] = _bits(0.5)    # only key 1 has rope
    kv[0, 0, 0, 7] = _bits(3.0)      # value dims
    kv[0, 1, 0, 7] = _bits(-1.0)
    kv[0, 2:, 0, :] = W.BF16_NAN
    bt = np.zeros((1, 1), dtype=np.int32)
    sl = np.array([2], dtype=np.int32)
    scale = 0.25
    out, lse = oracle.decode(q, kv, bt, sl, scale, causal=False, nthreads=1)
    s0, s1 = scale * a * x0, scale * (a * x1 + 1.0 * 0.5)
    sig = 1.0 / (1.0 + math.exp(s1 - s0))
    assert out[0, 0, 0, 0] == pytest.approx(sig * x0 + (1 - sig) * x1, rel=1e-14)
    assert out[0, 0, 0, 7] == pytest.approx(sig * 3.0 + (1 - sig) * -1.0, rel=1e-14)
    assert out[0, 0, 0, 1] == 0.0
    assert lse[0, 0, 0] == pytest.approx(math.log(math.exp(s0) + math.exp(s1)), rel=1e-14)
    # dims 512..575 are key-only: they never show up in out (out has 512 dims)
    assert out.shape[-1] == DV


def test_zero_query_gives_mean_of_values():
    q, kv, bt, sl, dense = _dense_case([77, 128], 3, 1, seed=9)
    q[:] = 0
    out, lse = oracle.decode(q, kv, bt, sl, W.SCALE, causal=False, nthreads=2)
    for i, n in enumerate([77, 128]):
        v = W.bf16_bits_to_f32(dense[i][:, :DV]).astype(np.float64)
        np.testing.assert_allclose(out[i, 0], np.broadcast_to(v.mean(0), (3, DV)), rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lse[i, :, 0], math.log(n), rtol=1e-14)


def test_block_relabelling_is_invisible():
    wl = W.custom(3, 4, 1, [130, 64, 1])
    inp = W.make_inputs(wl, seed=1, spare_blocks=4)
    out0, lse0 = oracle.decode(inp["q"], inp["kv"], inp["block_table"], inp["seqlens"],
                               wl.scale, False, nthreads=3)
    rng = np.random.default_rng(42)
    nblk = inp["kv"].shape[0]
    perm = rng.permutation(nblk)              # new physical id of old block j is perm[j]
    kv2 = np.empty_like(inp["kv"])
    kv2[perm] = inp["kv"]
    bt2 = np.where(inp["block_table"] >= 0, perm[np.maximum(inp["block_table"], 0)], -1).astype(np.int32)
    out1, lse1 = oracle.decode(inp["q"], kv2, bt2, inp["seqlens"], wl.scale, False, nthreads=3)
    assert np.array_equal(out0, out1) and np.array_equal(lse0, lse1)


def test_nan_tail_and_pad_entries_are_never_read():
    wl = W.custom(2, 2, 1, [100, 257])
    a = W.make_inputs(wl, seed=4, tail="nan")
    b = W.make_inputs(wl, seed=4, tail="normal")
    oa, la = oracle.decode(a["q"], a["kv"], a["block_table"], a["seqlens"], wl.scale, False)
    ob, lb = oracle.decode(b["q"], b["kv"], b["block_table"], b["seqlens"], wl.scale, False)
    assert np.all(np.isfinite(oa)) and np.array_equal(oa, ob) and np.array_equal(la, lb)
    # pad entries (-1) past ceil(n/64) are never dereferenced
    assert (a["block_table"] == -1).any()


def test_task_subset_equals_full_run():
    wl = W.custom(2, 3, 2, [70, 5], causal=True)
    inp = W.make_inputs(wl, seed=8)
    full_o, full_l = oracle.decode(inp["q"], inp["kv"], inp["block_table"], inp["seqlens"],
                                   wl.scale, True)
    tasks = np.array([[1, 0, 2], [0, 1, 0]], dtype=np.int32)
    o, l = oracle.decode(inp["q"], inp["kv"], inp["block_table"], inp["seqlens"], wl.scale, True,
                         tasks=tasks)
    for b, t, h in tasks:
        assert np.array_equal(o[b, t, h], full_o[b, t, h]) and l[b, h, t] == full_l[b, h, t]
    assert np.isnan(o[0, 0, 0, 0])


def test_bad_block_id_is_an_error():
    wl = W.custom(1, 1, 1, [10])
    inp = W.make_inputs(wl)
    bt = inp["block_table"].copy()
    bt[0, 0] = 99
    with pytest.raises(ValueError):
        oracle.decode(inp["q"], inp["kv"], bt, inp["seqlens"], wl.scale, False)


def test_head_gemm_matches_brute_force():
    """The per-head projection oracle against explicit loops (a transposed operand or a wrong head
    index would show)."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((5, 3, 4))
    w = rng.standard_normal((3, 4, 6))
    y = oracle.head_gemm(x, w)
    for r in range(5):
        for h in range(3):
            for n in range(6):
                assert abs(y[r, h, n] - sum(x[r, h, kk] * w[h, kk, n] for kk in range(4))) < 1e-12
