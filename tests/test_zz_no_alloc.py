"""mla_decode_noalloc: the decode entry point for callers that cannot allocate device memory.

Some callers may not call cudaMalloc at decode time (a runtime with a fixed memory pool, or
a serving path where a late allocation could fail or stall the stream). For them the library
keeps the split partials in a fixed scratch array of its own device image instead of a
caller workspace. These tests call that entry point through the C ABI and check, on two calls
in a row (the second call finds the first call's leftovers in the shared scratch), that it
matches the CPU oracle within the parity tolerances and returns what mla_decode returns on the
same inputs, with shapes whose sequences are split across parts so the scratch is really used.
"""
import ctypes

import numpy as np
import pytest
import torch

import mla_decode_attention_14_b200 as mla
import oracle
from mla_decode_attention_14_b200 import workloads as W
from tests import parity

CASES = [
    # seqlens, h_q, s_q, causal, num_parts
    ([1500, 3, 700, 1290], 64, 2, True, 11),
    ([900, 4000], 128, 1, False, 9),
    ([130, 65, 257], 16, 1, False, 7),
]


def _raw_noalloc(q, kv, bt, sl, meta, scale, causal, out, lse):
    L = mla.lib()
    b, s_q, h_q, _ = q.shape
    return L.mla_decode_noalloc(q.data_ptr(), kv.data_ptr(), kv.shape[0], bt.data_ptr(), bt.shape[1], sl.data_ptr(),
                                meta.tile_meta.data_ptr(), meta.num_splits.data_ptr(), meta.num_parts, b, s_q, h_q,
                                ctypes.c_float(scale), int(bool(causal)), out.data_ptr(), lse.data_ptr(),
                                torch.cuda.current_stream().cuda_stream)


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_noalloc_matches_oracle_and_workspace_entry_point_twice(case):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    seqlens, h_q, s_q, causal, parts = case
    wl = W.custom(len(seqlens), h_q, s_q, seqlens, causal=causal)
    inp = W.make_inputs(wl, seed=21, tail="nan", spare_blocks=3)
    q, kv, bt, sl = parity.to_device(inp)
    meta = mla.get_metadata(sl, h_q, s_q, num_parts=parts)
    assert int(np.diff(meta.num_splits.cpu().numpy()).max()) > 1, "case must split a sequence"
    assert mla.workspace_bytes(wl.batch, s_q, h_q, parts) <= mla.NOALLOC_SCRATCH_BYTES
    ref_out, ref_lse = mla.decode(q, kv, bt, sl, wl.scale, causal, meta)
    assert mla.check_status() == 0
    ref_o = parity.bf16_to_f64(ref_out)
    ref_l = ref_lse.cpu().numpy().astype(np.float64)
    orc_o, orc_l = oracle.decode(inp["q"], inp["kv"], inp["block_table"], inp["seqlens"], wl.scale, causal)
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        rc = _raw_noalloc(q, kv, bt, sl, meta, wl.scale, causal, out, lse)
        assert rc == 0, mla.lib().mla_status_string(rc)
        assert mla.check_status() == 0
        o = parity.bf16_to_f64(out)
        l = lse.cpu().numpy().astype(np.float64)
        parity.compare(o, l, orc_o, orc_l, what="noalloc call %d vs oracle" % call)
        parity.compare(o, l, ref_o, ref_l, what="noalloc call %d vs mla_decode" % call)


@pytest.mark.gpu
def test_noalloc_rejects_requests_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wl = W.custom(2, 128, 1, [100, 200])
    inp = W.make_inputs(wl, seed=1)
    q, kv, bt, sl = parity.to_device(inp)
    parts = 65535  # (batch + parts) * rows * 513 * 4 bytes is far beyond the fixed scratch
    assert mla.workspace_bytes(2, 1, 128, parts) > mla.NOALLOC_SCRATCH_BYTES
    meta = mla.get_metadata(sl, 128, 1, num_parts=parts)
    out = torch.empty((2, 1, 128, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((2, 128, 1), dtype=torch.float32, device="cuda")
    assert _raw_noalloc(q, kv, bt, sl, meta, wl.scale, False, out, lse) == 3  # MLA_ERR_WORKSPACE
