"""Pins for the CPU oracle over the fp8 (E4M3) latent cache (no GPU).

The E4M3 decoding is tied to hand-worked values of the OCP OFP8 definition
(tests/golden/e4m3_values.txt) and to torch's own float8_e4m3fn type over all 256
codes. The attention over the fp8 cache is tied to the already-pinned bf16 oracle
(a power-of-two latent scale makes every dequantized value a bf16 number, so both
must agree bit for bit), to a dense float64 torch SDPA on keys dequantized by torch,
and to closed forms (one token, q = 0) and the NaN-tail invariant.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from mla_decode_attention_14_b200 import workloads as W

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

BLK, DQK, DV, REC = 64, 576, 512, 640
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_values.txt")


def _golden():
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        code, val = line.split()
        yield int(code, 16), val


def test_e4m3_decoding_matches_hand_worked_values():
    for code, val in _golden():
        got = oracle.e4m3_decode(np.array([code], dtype=np.uint8))[0]
        if val == "nan":
            assert np.isnan(got), hex(code)
        else:
            neg = val.startswith("-")
            want = float(Fraction(val.lstrip("-")))
            assert got == (-want if neg else want), (hex(code), got, val)
            assert np.signbit(got) == neg, hex(code)


def test_e4m3_decoding_matches_torch_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.array_equal(np.signbit(got[fin]), np.signbit(ref[fin]))


def _torch_dequant(kv8_rows, kv_scale):
    """[n, 640] fp8 records -> float64 [n, 576] through torch's float8 type (not the oracle's)."""
    lat = torch.from_numpy(np.ascontiguousarray(kv8_rows[:, :DV])).view(torch.float8_e4m3fn).to(torch.float64)
    rope_bits = np.ascontiguousarray(kv8_rows[:, DV:]).view("<u2")
    rope = torch.from_numpy(W.bf16_bits_to_f32(rope_bits).astype(np.float64))
    return torch.cat([lat * kv_scale, rope], dim=1)


def _dense_keys(inp, i):
    n = int(inp["seqlens"][i])
    rows = [inp["kv8"][inp["block_table"][i, j // BLK], j % BLK, 0] for j in range(n)]
    return np.stack(rows)


@pytest.mark.parametrize("kv_scale", [2.0 ** -6, 0.0123])
def test_dense_bruteforce_matches_library_sdpa(kv_scale):
    wl = W.custom(3, 8, 1, [1, 70, 130])
    inp = W.make_inputs_fp8(wl, seed=4, spare_blocks=2, kv_scale=kv_scale)
    out, lse = oracle.decode_fp8(inp["q"], inp["kv8"], kv_scale, inp["block_table"], inp["seqlens"],
                                 wl.scale, False, nthreads=4)
    for i in range(3):
        k = _torch_dequant(_dense_keys(inp, i), kv_scale)
        q = torch.from_numpy(W.bf16_bits_to_f32(inp["q"][i, 0]).astype(np.float64))
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[None, None], k[None, None], k[None, None, :, :DV], scale=wl.scale)[0, 0].numpy()
        ref_l = torch.logsumexp(wl.scale * (q @ k.T), dim=-1).numpy()
        np.testing.assert_allclose(out[i, 0], ref, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(lse[i, :, 0], ref_l, rtol=1e-12, atol=1e-12)


def test_power_of_two_scale_reduces_to_the_bf16_oracle():
    """With kv_scale = 2^-6 every dequantized latent value is a bf16 number: rewriting the
    cache as bf16 must give the same doubles in the same order, i.e. identical results."""
    wl = W.custom(4, 16, 2, [1, 64, 65, 200], causal=True)
    inp = W.make_inputs_fp8(wl, seed=11, tail="normal", spare_blocks=1)
    nb = inp["kv8"].shape[0]
    rec = inp["kv8"].reshape(nb * BLK, REC)
    lat = torch.from_numpy(np.ascontiguousarray(rec[:, :DV])).view(torch.float8_e4m3fn).to(torch.float32)
    lat = (lat * inp["kv_scale"]).numpy()
    lat_bits = W.f32_to_bf16_bits(lat)
    assert np.array_equal(W.bf16_bits_to_f32(lat_bits), lat), "scale must keep the values exact in bf16"
    kv16 = np.concatenate([lat_bits, np.ascontiguousarray(rec[:, DV:]).view("<u2")], axis=1)
    kv16 = kv16.reshape(nb, BLK, 1, DQK)
    o8, l8 = oracle.decode_fp8(inp["q"], inp["kv8"], inp["kv_scale"], inp["block_table"], inp["seqlens"],
                               wl.scale, True, nthreads=4)
    o16, l16 = oracle.decode(inp["q"], kv16, inp["block_table"], inp["seqlens"], wl.scale, True, nthreads=4)
    assert np.array_equal(o8, o16)
    assert np.array_equal(l8, l16)


def test_single_token_returns_its_dequantized_value_row():
    wl = W.custom(2, 5, 1, [1, 1])
    inp = W.make_inputs_fp8(wl, seed=2, kv_scale=0.0123)
    out, lse = oracle.decode_fp8(inp["q"], inp["kv8"], inp["kv_scale"], inp["block_table"], inp["seqlens"],
                                 wl.scale, False, nthreads=2)
    for i in range(2):
        k = _torch_dequant(_dense_keys(inp, i), inp["kv_scale"]).numpy()[0]
        for h in range(5):
            assert np.array_equal(out[i, 0, h], k[:DV])
        q = W.bf16_bits_to_f32(inp["q"][i, 0]).astype(np.float64)
        np.testing.assert_allclose(lse[i, :, 0], wl.scale * (q @ k), rtol=1e-12)


def test_zero_query_gives_mean_of_dequantized_values():
    wl = W.custom(2, 3, 1, [37, 150])
    inp = W.make_inputs_fp8(wl, seed=8, kv_scale=0.05)
    inp["q"][:] = 0
    out, lse = oracle.decode_fp8(inp["q"], inp["kv8"], inp["kv_scale"], inp["block_table"], inp["seqlens"],
                                 wl.scale, False, nthreads=2)
    for i, n in enumerate([37, 150]):
        k = _torch_dequant(_dense_keys(inp, i), inp["kv_scale"]).numpy()
        for h in range(3):
            np.testing.assert_allclose(out[i, 0, h], k[:, :DV].mean(axis=0), rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lse[i, :, 0], np.log(n), rtol=1e-14)


def test_nan_tail_is_never_read():
    wl = W.custom(3, 4, 1, [5, 64, 100])
    a = W.make_inputs_fp8(wl, seed=6, tail="nan")
    b = W.make_inputs_fp8(wl, seed=6, tail="normal")
    ra = oracle.decode_fp8(a["q"], a["kv8"], a["kv_scale"], a["block_table"], a["seqlens"], wl.scale, False)
    rb = oracle.decode_fp8(b["q"], b["kv8"], b["kv_scale"], b["block_table"], b["seqlens"], wl.scale, False)
    assert np.all(np.isfinite(ra[0]))
    assert np.array_equal(ra[0], rb[0]) and np.array_equal(ra[1], rb[1])


# ---------------------------------------------------------------- E4M3 encoding and appends
def test_e4m3_encoding_round_trips_every_finite_code():
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.e4m3_decode(codes).astype(np.float32)
    fin = ~np.isnan(vals)
    assert np.array_equal(oracle.e4m3_encode(vals)[fin], codes[fin])


@pytest.mark.parametrize("x,code", [
    (1.0625, 0x38),        # tie between 1 (mantissa 0) and 1.125 (1): to even, 1
    (1.1875, 0x3A),        # tie between 1.125 (1) and 1.25 (2): to even, 1.25
    (2.0 ** -10, 0x00),    # tie between 0 and the smallest subnormal 2^-9: to even, 0
    (3 * 2.0 ** -10, 0x02),  # tie between 2^-9 (1) and 2^-8 (2): to even, 2
    (-3 * 2.0 ** -10, 0x82),
    (0.9999, 0x38),        # rounds up into the next binade
    (460.0, 0x7E), (500.0, 0x7E), (float("inf"), 0x7E), (-1000.0, 0xFE),  # saturation to +-448
    (float("nan"), 0x7F),
])
def test_e4m3_encoding_hand_worked_cases(x, code):
    assert int(oracle.e4m3_encode(np.array([x], dtype=np.float32))[0]) == code


def test_e4m3_encoding_matches_torch_in_range():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 60
    x = np.clip(x, -448, 448)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(x), ref)


def _append_case(kv="bf16"):
    wl = W.custom(3, 4, 1, [5, 64, 130])
    gen = W.make_inputs_fp8 if kv == "fp8" else W.make_inputs
    inp = gen(wl, seed=13, tail="normal", spare_blocks=2)
    # the table must hold the new positions: lengths 5 + 3 stay in block 0, 64 + 3 spills into a new
    # block, 130 + 3 stays in block 2; give sequence 1 a spare physical block for its second entry
    bt = inp["block_table"].copy()
    if bt.shape[1] < 3:
        bt = np.concatenate([bt, np.full((3, 3 - bt.shape[1]), -1, np.int32)], axis=1)
    free = sorted(set(range(inp["num_blocks"])) - set(int(v) for v in bt[bt >= 0]))
    bt[1, 1] = free[0]
    new = W.f32_to_bf16_bits(np.random.default_rng(1).standard_normal((3, 3, DQK), dtype=np.float32))
    return inp, bt, new


def test_append_writes_rows_at_the_sequence_ends_only():
    inp, bt, new = _append_case()
    kv = oracle.append(new, inp["kv"], bt, inp["seqlens"])
    flat, old = kv.reshape(-1, DQK), inp["kv"].reshape(-1, DQK)
    touched = set()
    for b, n in enumerate(inp["seqlens"]):
        for t in range(3):
            pos = int(n) + t
            row = bt[b, pos // BLK] * BLK + pos % BLK
            assert np.array_equal(flat[row], new[b, t])
            touched.add(int(row))
    rest = np.array([r for r in range(flat.shape[0]) if r not in touched])
    assert np.array_equal(flat[rest], old[rest])


def test_fp8_append_decodes_back_within_e4m3_rounding():
    inp, bt, new = _append_case("fp8")
    sc = inp["kv_scale"]
    kv8 = oracle.append_fp8(new, inp["kv8"], np.float32(1.0 / sc), bt, inp["seqlens"])
    flat = kv8.reshape(-1, REC)
    for b, n in enumerate(inp["seqlens"]):
        for t in range(3):
            pos = int(n) + t
            rec = flat[bt[b, pos // BLK] * BLK + pos % BLK]
            x = W.bf16_bits_to_f32(new[b, t]).astype(np.float64)
            lat = oracle.e4m3_decode(rec[:DV]) * sc
            # E4M3 keeps 4 significant bits: relative error <= 2^-4 (normal range), absolute <= 2^-10 sc
            err = np.abs(lat - x[:DV])
            assert np.all(err <= np.maximum(np.abs(x[:DV]) * 2.0 ** -4, 2.0 ** -10 * sc) + 1e-12)
            assert np.array_equal(np.ascontiguousarray(rec[DV:]).view("<u2"), new[b, t, DV:])
