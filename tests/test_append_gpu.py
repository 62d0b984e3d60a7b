"""GPU parity of the cache append (bf16 and fp8) against the CPU oracle, bit for bit, and a decode
over the appended cache (needs a B200)."""
import numpy as np
import pytest
import torch

import mla_decode_attention_14_b200 as mla
import oracle
from mla_decode_attention_14_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu
N_NEW = 3


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _case(kv="bf16", kv_scale=W.F8_SCALE, seed=21):
    """Sequences whose new tokens stay in a block, cross into a new one, or start one."""
    seqlens = [5, 62, 64, 130, 0]
    wl = W.custom(len(seqlens), 16, 1, seqlens)
    gen = W.make_inputs_fp8 if kv == "fp8" else W.make_inputs
    extra = dict(kv_scale=kv_scale) if kv == "fp8" else {}
    inp = gen(wl, seed=seed, tail="normal", spare_blocks=4, **extra)
    bt = inp["block_table"]
    width = max(bt.shape[1], (max(seqlens) + N_NEW + 63) // 64)
    bt = np.concatenate([bt, np.full((bt.shape[0], width - bt.shape[1]), -1, np.int32)], axis=1)
    free = sorted(set(range(inp["num_blocks"])) - set(int(v) for v in bt[bt >= 0]))
    for b, n in enumerate(seqlens):
        for blk in range(n // 64, (n + N_NEW - 1) // 64 + 1):
            if bt[b, blk] < 0:
                bt[b, blk] = free.pop(0)
    inp["block_table"] = bt
    new = W.f32_to_bf16_bits(np.random.default_rng(seed).standard_normal((len(seqlens), N_NEW, 576), dtype=np.float32))
    return wl, inp, new


def test_bf16_append_is_bit_exact():
    wl, inp, new = _case()
    kv = torch.from_numpy(inp["kv"]).view(torch.bfloat16).cuda()
    mla.append_kv(torch.from_numpy(new).view(torch.bfloat16).cuda(), kv, torch.from_numpy(inp["block_table"]).cuda(),
                  torch.from_numpy(inp["seqlens"]).cuda())
    assert mla.check_status() == 0
    ref = oracle.append(new, inp["kv"], inp["block_table"], inp["seqlens"])
    assert np.array_equal(kv.view(torch.uint16).cpu().numpy(), ref)


@pytest.mark.parametrize("kv_scale", [W.F8_SCALE, 0.0123])
def test_fp8_append_codes_are_bit_exact(kv_scale):
    wl, inp, new = _case("fp8", kv_scale)
    kv8 = torch.from_numpy(inp["kv8"]).cuda()
    mla.append_kv_fp8(torch.from_numpy(new).view(torch.bfloat16).cuda(), kv8,
                      torch.from_numpy(inp["block_table"]).cuda(), torch.from_numpy(inp["seqlens"]).cuda(), kv_scale)
    assert mla.check_status() == 0
    inv = np.float32(1.0) / np.float32(kv_scale)  # the library's 1 / kv_scale, in fp32
    ref = oracle.append_fp8(new, inp["kv8"], inv, inp["block_table"], inp["seqlens"])
    assert np.array_equal(kv8.cpu().numpy(), ref)


def test_missing_table_entry_is_reported_and_skipped():
    wl, inp, new = _case()
    bt = inp["block_table"].copy()
    bt[1, 1] = -1  # sequence 1 (62 tokens) needs block 1 for its new tokens 2 and 3
    kv = torch.from_numpy(inp["kv"]).view(torch.bfloat16).cuda()
    mla.append_kv(torch.from_numpy(new).view(torch.bfloat16).cuda(), kv, torch.from_numpy(bt).cuda(),
                  torch.from_numpy(inp["seqlens"]).cuda())
    assert mla.check_status() == 6  # MLA_ERR_BOUNDS
    assert mla.check_status() == 0
    got = kv.view(torch.uint16).cpu().numpy().reshape(-1, 576)
    row = bt[0, 0] * 64 + 5  # sequence 0's first new token still landed
    assert np.array_equal(got[row], new[0, 0])


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_decode_after_append(kv):
    """Append N_NEW tokens, extend the lengths, decode (s_q = N_NEW, causal): parity with the oracle
    on the oracle's own appended cache."""
    wl, inp, new = _case(kv)
    bt = torch.from_numpy(inp["block_table"]).cuda()
    sl = torch.from_numpy(inp["seqlens"]).cuda()
    nk = torch.from_numpy(new).view(torch.bfloat16).cuda()
    new_len = inp["seqlens"] + N_NEW
    q = W.f32_to_bf16_bits(np.random.default_rng(5).standard_normal((len(new_len), N_NEW, 16, 576), dtype=np.float32))
    qd = torch.from_numpy(q).view(torch.bfloat16).cuda()
    sl2 = torch.from_numpy(new_len.astype(np.int32)).cuda()
    meta = mla.get_metadata(sl2, 16, N_NEW, num_parts=5)
    if kv == "bf16":
        cache = torch.from_numpy(inp["kv"]).view(torch.bfloat16).cuda()
        mla.append_kv(nk, cache, bt, sl)
        out, lse = mla.decode(qd, cache, bt, sl2, wl.scale, True, meta)
        ref_kv = oracle.append(new, inp["kv"], inp["block_table"], inp["seqlens"])
        ro, rl = oracle.decode(q, ref_kv, inp["block_table"], new_len, wl.scale, True)
    else:
        cache = torch.from_numpy(inp["kv8"]).cuda()
        mla.append_kv_fp8(nk, cache, bt, sl, inp["kv_scale"])
        out, lse = mla.decode_fp8(qd, cache, bt, sl2, wl.scale, inp["kv_scale"], True, meta)
        ref_kv = oracle.append_fp8(new, inp["kv8"], np.float32(1.0) / np.float32(inp["kv_scale"]),
                                   inp["block_table"], inp["seqlens"])
        ro, rl = oracle.decode_fp8(q, ref_kv, inp["kv_scale"], inp["block_table"], new_len, wl.scale, True)
    assert mla.check_status() == 0
    parity.compare(parity.bf16_to_f64(out), lse.cpu().numpy().astype(np.float64), ro, rl, what="decode after append")


def test_zero_new_tokens_is_a_no_op():
    wl, inp, new = _case()
    kv = torch.from_numpy(inp["kv"]).view(torch.bfloat16).cuda()
    before = kv.clone()
    mla.append_kv(torch.empty((5, 0, 576), dtype=torch.bfloat16, device="cuda"), kv,
                  torch.from_numpy(inp["block_table"]).cuda(), torch.from_numpy(inp["seqlens"]).cuda())
    assert mla.check_status() == 0
    assert torch.equal(kv, before)
