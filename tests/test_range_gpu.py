"""Range of the pair's factor exchange (needs a B200).

The two SMs that share a row exchange, per token, R = 2^((s - m)/2 + 15) in fp16, where s is the
token's partial score over that SM's half of the 576 dims and m that SM's partial maximum over 32
tokens. R is exact to 2^-10 (once squared) while s - m >= -58 octaves; below that it is an fp16
subnormal and then 0. A row whose two partial maxima come from different keys and overstate its
true maximum by ~58 octaves or more can therefore lose the keys that dominate its softmax. The
decode must then report MLA_ERR_RANGE instead of returning a wrong row with MLA_OK.
"""
import numpy as np
import pytest
import torch

import mla_decode_attention_14_b200 as mla
import oracle
from mla_decode_attention_14_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu

MLA_ERR_RANGE = 7

# CTA h of a pair holds latent dims [256h, 256h+256) and rotary dims [512+32h, 512+32h+32)
HALF0 = np.r_[0:256, 512:544]
HALF1 = np.r_[256:512, 544:576]


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _opposed_keys(a: float):
    """One 64-token block with every query dim 1. All keys are 0 (score 0) except key 1 (+a on half
    0, -1.5a on half 1) and key 2 (the mirror). At a = 6 and scale 192^-0.5 each half of keys 1-2
    scores +-180 / -+270 octaves, so both partial maxima (+180 each) overstate the true maximum
    (0, on the 62 zero keys) by 360 octaves: far past the exchange's range."""
    k = np.zeros((64, 576), dtype=np.float32)
    k[1, HALF0], k[1, HALF1] = a, -1.5 * a
    k[2, HALF0], k[2, HALF1] = -1.5 * a, a
    return k


def _run_bf16(inp):
    q, kv, bt, sl = parity.to_device(inp)
    b, s_q, h_q, _ = q.shape
    meta = mla.get_metadata(sl, h_q, s_q)
    out, lse = mla.decode(q, kv, bt, sl, inp["scale"], inp["causal"], meta)
    return out, lse, mla.check_status()


def _run_fp8(inp):
    q = torch.from_numpy(inp["q"]).view(torch.bfloat16).cuda()
    kv8 = torch.from_numpy(inp["kv8"]).cuda()
    bt = torch.from_numpy(inp["block_table"]).cuda()
    sl = torch.from_numpy(inp["seqlens"]).cuda()
    meta = mla.get_metadata(sl, q.shape[2], q.shape[1])
    out, lse = mla.decode_fp8(q, kv8, bt, sl, inp["scale"], inp["kv_scale"], inp["causal"], meta)
    return out, lse, mla.check_status()


def test_bf16_row_past_the_exchange_range_is_reported():
    h_q = 16
    q = W.f32_to_bf16_bits(np.ones((1, 1, h_q, 576), dtype=np.float32))
    kv = W.f32_to_bf16_bits(_opposed_keys(6.0)).reshape(1, 64, 1, 576)
    inp = {"q": q, "kv": kv, "block_table": np.zeros((1, 1), np.int32), "seqlens": np.array([64], np.int32),
           "scale": W.SCALE, "causal": False}
    _, ref_lse = oracle.decode(inp["q"], inp["kv"], inp["block_table"], inp["seqlens"], inp["scale"], False)
    assert np.allclose(ref_lse, np.log(62.0))  # 62 keys at score 0, two at -90 octaves
    _, _, status = _run_bf16(inp)
    assert status == MLA_ERR_RANGE


def test_fp8_row_past_the_exchange_range_is_reported():
    h_q = 16
    k = _opposed_keys(6.0)  # 6 and -9 are E4M3 numbers
    kv8 = np.zeros((1, 64, 1, 640), dtype=np.uint8)
    kv8[0, :, 0, :512] = W._e4m3_codes(k[:, :512])
    kv8[0, :, 0, 512:] = np.ascontiguousarray(W.f32_to_bf16_bits(k[:, 512:]).astype("<u2")).view(np.uint8)
    inp = {"q": W.f32_to_bf16_bits(np.ones((1, 1, h_q, 576), dtype=np.float32)), "kv8": kv8, "kv_scale": 1.0,
           "block_table": np.zeros((1, 1), np.int32), "seqlens": np.array([64], np.int32), "scale": W.SCALE,
           "causal": False}
    _, ref_lse = oracle.decode_fp8(inp["q"], inp["kv8"], 1.0, inp["block_table"], inp["seqlens"], inp["scale"],
                                   False)
    assert np.allclose(ref_lse, np.log(62.0))
    _, _, status = _run_fp8(inp)
    assert status == MLA_ERR_RANGE


def _one_sequence(inp, i):
    """Sequence i of a batch as a batch of its own (same cache and block table row)."""
    d = dict(inp)
    d["q"] = inp["q"][i:i + 1]
    d["block_table"] = inp["block_table"][i:i + 1]
    d["seqlens"] = inp["seqlens"][i:i + 1]
    return d


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_scale_one_rows_pass_parity_or_are_reported(kv):
    """Softmax scale 1.0 on N(0,1) inputs: the partial maxima overstate the true maximum by ~34
    octaves on average, with a tail that reaches past the exchange's range. Over several draws,
    each sequence (decoded on its own, so the status is its own) either matches the oracle within
    the stated tolerances or is reported with MLA_ERR_RANGE; no other status is allowed."""
    wl = W.custom(3, 64, 1, [1000, 64, 333], scale=1.0)
    passed = reported = 0
    for seed in range(6):
        inp = (W.make_inputs if kv == "bf16" else W.make_inputs_fp8)(wl, seed=100 + seed, tail="nan")
        for i in range(wl.batch):
            one = _one_sequence(inp, i)
            out, lse, status = (_run_bf16 if kv == "bf16" else _run_fp8)(one)
            assert status in (0, MLA_ERR_RANGE), "status %d" % status
            if status == MLA_ERR_RANGE:
                reported += 1
                continue
            if kv == "bf16":
                ref_o, ref_l = oracle.decode(one["q"], one["kv"], one["block_table"], one["seqlens"], 1.0, False)
            else:
                ref_o, ref_l = oracle.decode_fp8(one["q"], one["kv8"], one["kv_scale"], one["block_table"],
                                                 one["seqlens"], 1.0, False)
            parity.compare(parity.bf16_to_f64(out), lse.cpu().numpy().astype(np.float64), ref_o, ref_l,
                           "%s scale 1.0 seed %d seq %d" % (kv, 100 + seed, i))
            passed += 1
    print("%s scale 1.0: %d sequences passed parity, %d reported" % (kv, passed, reported))
    assert passed > 0
