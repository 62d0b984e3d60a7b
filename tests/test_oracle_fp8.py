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
