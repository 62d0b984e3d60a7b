"""Parity helpers: run the CUDA path on seeded inputs and compare with the CPU oracle.

Tolerances (stated by the library's task): max |out - ref| <= 1e-2 * max |ref|,
mean relative error sum|out - ref| / sum|ref| <= 2e-3, |lse - ref| <= 1e-3 on finite
entries, and -inf exactly where the reference is -inf. The reference is the oracle's
double result, not rounded to bf16.
"""
import numpy as np
import torch

import mla_decode_attention_14_b200 as mla
import oracle

OUT_MAX_REL = 1e-2
OUT_MEAN_REL = 2e-3
LSE_ABS = 1e-3


def to_device(inp, device="cuda"):
    q = torch.from_numpy(inp["q"]).view(torch.bfloat16).to(device)
    kv = torch.from_numpy(inp["kv"]).view(torch.bfloat16).to(device)
    bt = torch.from_numpy(inp["block_table"]).to(device)
    sl = torch.from_numpy(inp["seqlens"]).to(device)
    return q, kv, bt, sl


def run_gpu(inp, num_parts=None, fixed_cost=None):
    q, kv, bt, sl = to_device(inp)
    b, s_q, h_q, _ = q.shape
    meta = mla.get_metadata(sl, h_q, s_q, num_parts=num_parts, fixed_cost=fixed_cost)
    out, lse = mla.decode(q, kv, bt, sl, inp["scale"], inp["causal"], meta)
    status = mla.check_status()
    assert status == 0, "device error status %d" % status
    return out, lse, meta


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def compare(out, lse, ref_out, ref_lse, what=""):
    """out/lse: numpy float64 (GPU results); ref_*: oracle. Same shapes (may be row subsets)."""
    diff = np.abs(out - ref_out)
    assert np.all(np.isfinite(out)), "%s: non-finite output" % what
    mref = np.abs(ref_out).max(initial=0.0)
    sref = np.abs(ref_out).sum()
    if sref == 0.0:
        assert np.all(out == 0.0), "%s: expected all-zero output" % what
    else:
        assert diff.max() <= OUT_MAX_REL * mref, "%s: max err %g > %g" % (what, diff.max(), OUT_MAX_REL * mref)
        mre = diff.sum() / sref
        assert mre <= OUT_MEAN_REL, "%s: mean rel err %g" % (what, mre)
    ninf = np.isneginf(ref_lse)
    assert np.array_equal(np.isneginf(lse), ninf), "%s: -inf lse pattern differs" % what
    fin = ~ninf
    if fin.any():
        e = np.abs(lse[fin] - ref_lse[fin]).max()
        assert e <= LSE_ABS, "%s: lse err %g" % (what, e)


def full_parity(inp, num_parts=None, fixed_cost=None, what=""):
    out, lse, meta = run_gpu(inp, num_parts, fixed_cost)
    ref_o, ref_l = oracle.decode(inp["q"], inp["kv"], inp["block_table"], inp["seqlens"], inp["scale"],
                                 inp["causal"])
    compare(bf16_to_f64(out), lse.cpu().numpy().astype(np.float64), ref_o, ref_l, what)
    return out, lse, meta
