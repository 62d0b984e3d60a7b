"""GPU parity of the fp8 (E4M3) latent-cache decode path against the CPU oracle (needs a B200).

The oracle dequantizes every E4M3 byte exactly (kv_scale * e4m3) and computes in double; the
kernel converts the cache to fp16 exactly, rounds the latent query dims (times the scale's
mantissa) and P to fp16, and accumulates in fp32. The tolerances are the bf16 path's."""
import numpy as np
import pytest
import torch

import mla_decode_attention_14_b200 as mla
import oracle
from mla_decode_attention_14_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _to_device(inp):
    q = torch.from_numpy(inp["q"]).view(torch.bfloat16).cuda()
    kv8 = torch.from_numpy(inp["kv8"]).cuda()
    bt = torch.from_numpy(inp["block_table"]).cuda()
    sl = torch.from_numpy(inp["seqlens"]).cuda()
    return q, kv8, bt, sl


def run_fp8(inp, num_parts=None):
    q, kv8, bt, sl = _to_device(inp)
    b, s_q, h_q, _ = q.shape
    meta = mla.get_metadata(sl, h_q, s_q, num_parts=num_parts)
    out, lse = mla.decode_fp8(q, kv8, bt, sl, inp["scale"], inp["kv_scale"], inp["causal"], meta)
    st = mla.check_status()
    assert st == 0, "device error status %d" % st
    return out, lse, meta


def full_parity_fp8(inp, num_parts=None, what=""):
    out, lse, meta = run_fp8(inp, num_parts)
    ref_o, ref_l = oracle.decode_fp8(inp["q"], inp["kv8"], inp["kv_scale"], inp["block_table"], inp["seqlens"],
                                     inp["scale"], inp["causal"])
    parity.compare(parity.bf16_to_f64(out), lse.cpu().numpy().astype(np.float64), ref_o, ref_l, what)
    return out, lse, meta


def test_tiny_workload_full_parity():
    inp = W.make_inputs_fp8(W.workload("tiny"), seed=0, tail="nan")
    full_parity_fp8(inp, what="tiny fp8")


SMALL = [
    # seqlens, h_q, s_q, causal, num_parts
    ([1, 63, 64, 65, 130, 257], 16, 1, False, None),
    ([1, 63, 64, 65, 130, 257], 16, 1, False, 7),
    ([700, 5, 1290], 128, 1, False, None),
    ([700, 5, 1290], 128, 1, False, 3),
    ([129, 65, 1, 2, 200], 128, 2, True, None),
    ([129, 65, 1, 2, 200], 64, 2, True, 5),
    ([3000, 17], 64, 1, False, 20),
    ([33, 1000], 24, 3, True, 6),
    ([250, 250, 250, 250], 128, 1, False, 74),
]


@pytest.mark.parametrize("case", SMALL, ids=[str(i) for i in range(len(SMALL))])
def test_small_shapes_parity(case):
    seqlens, h_q, s_q, causal, parts = case
    wl = W.custom(len(seqlens), h_q, s_q, seqlens, causal=causal)
    inp = W.make_inputs_fp8(wl, seed=3, tail="nan", spare_blocks=2)
    full_parity_fp8(inp, num_parts=parts, what="fp8 " + str(case))


@pytest.mark.parametrize("kv_scale", [0.0123, 1.0, 3.7, 2.0 ** -20])
def test_other_latent_scales_parity(kv_scale):
    """Scales that are not powers of two (the latent query dims carry the mantissa), and extremes."""
    wl = W.custom(3, 128, 1, [500, 64, 77])
    inp = W.make_inputs_fp8(wl, seed=8, tail="nan", kv_scale=kv_scale)
    if kv_scale >= 1.0:  # latent values ~64 kv_scale N(0, 1): quieter queries keep the scores in range
        inp["q"] = W.f32_to_bf16_bits(W.bf16_bits_to_f32(inp["q"]) * np.float32(1.0 / (64 * kv_scale)))
    full_parity_fp8(inp, num_parts=4, what="kv_scale %g" % kv_scale)


@pytest.mark.parametrize("scale", [0.6, 0.3, 0.01])
def test_other_softmax_scales_parity(scale):
    """Wide score ranges: fp16 P needs the exact block max (an overstated one would push P into
    fp16's subnormal range); 0.01 makes the softmax nearly uniform."""
    wl = W.custom(3, 64, 1, [1000, 64, 333], scale=scale)
    inp = W.make_inputs_fp8(wl, seed=5, tail="nan")
    full_parity_fp8(inp, num_parts=5, what="fp8 scale %g" % scale)


def test_maximum_rows_parity():
    wl = W.custom(3, 128, 8, [300, 70, 9], causal=True)
    inp = W.make_inputs_fp8(wl, seed=11, tail="nan", spare_blocks=1)
    full_parity_fp8(inp, what="fp8 1024 rows")


def test_many_short_sequences_parity():
    rng = np.random.default_rng(17)
    seqlens = rng.integers(0, 201, size=700)
    seqlens[::97] = 0
    wl = W.custom(len(seqlens), 16, 1, seqlens)
    inp = W.make_inputs_fp8(wl, seed=6, tail="nan")
    full_parity_fp8(inp, what="fp8 700 short sequences")


@pytest.mark.parametrize("name", ["v2lite", "v3", "multitoken", "skewed"])
def test_full_size_workloads_full_parity(name):
    """Every row of every full-size workload over the fp8 cache, element by element against the
    fp8 oracle (run on all host cores)."""
    wl = W.workload(name)
    inp = W.make_inputs_fp8(wl, seed=0, tail="nan")
    out, lse, meta = run_fp8(inp)
    ref_o, ref_l = oracle.decode_fp8(inp["q"], inp["kv8"], inp["kv_scale"], inp["block_table"], inp["seqlens"],
                                     wl.scale, wl.causal)
    o = parity.bf16_to_f64(out)
    l = lse.cpu().numpy().astype(np.float64)
    parity.compare(o, l, ref_o, ref_l, what="fp8 " + name)


def test_single_token_sequences_return_dequantized_rows():
    """One key: the output is kv_scale * e4m3(latent) rounded once to bf16 (a power-of-two scale
    keeps that exact, so the comparison is bit for bit)."""
    wl = W.custom(3, 128, 1, [1, 1, 1])
    inp = W.make_inputs_fp8(wl, seed=5, kv_scale=2.0 ** -6)
    out, lse, _ = run_fp8(inp)
    for i in range(3):
        rec = inp["kv8"][inp["block_table"][i, 0], 0, 0]
        v = oracle.e4m3_decode(rec[:512]) * inp["kv_scale"]
        want = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16)
        assert torch.equal(out[i, 0].cpu(), want.expand(128, 512))


def test_subnormal_codes_are_not_flushed():
    """Every latent byte an E4M3 subnormal (exponent field 0): the kernel's fp16 form of those is
    subnormal too, and the tensor core must keep them. A latent scale of 2^6 makes the values
    ~0.1-0.9, so a flush to zero would show as a wrong output."""
    wl = W.custom(2, 64, 1, [200, 70])
    inp = W.make_inputs_fp8(wl, seed=12, tail="nan", kv_scale=2.0 ** 6)
    rng = np.random.default_rng(3)
    lat = inp["kv8"][..., :512]
    codes = rng.integers(1, 8, size=lat.shape).astype(np.uint8) | (rng.integers(0, 2, size=lat.shape).astype(np.uint8) << 7)
    nan_rows = lat == W.F8_NAN
    lat[...] = np.where(nan_rows, lat, codes)
    full_parity_fp8(inp, num_parts=3, what="subnormal codes")


def test_empty_sequences_give_zero_and_neg_inf():
    wl = W.custom(3, 16, 2, [0, 70, 1], causal=True)
    inp = W.make_inputs_fp8(wl, seed=6)
    out, lse, _ = full_parity_fp8(inp, what="fp8 empty")
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))
    assert torch.all(out[2, 0] == 0) and torch.all(torch.isneginf(lse[2, :, 0]))


def test_query_out_of_fp16_range_is_reported():
    """A latent query value that cannot be written as fp16 sets MLA_ERR_RANGE (no fault), and the
    next call runs clean."""
    wl = W.custom(2, 16, 1, [100, 5])
    inp = W.make_inputs_fp8(wl, seed=2)
    q, kv8, bt, sl = _to_device(inp)
    q[1, 0, 3, 17] = 1.0e6
    meta = mla.get_metadata(sl, 16, 1)
    mla.decode_fp8(q, kv8, bt, sl, wl.scale, inp["kv_scale"], False, meta)
    assert mla.check_status() == 7  # MLA_ERR_RANGE
    assert mla.check_status() == 0
    full_parity_fp8(inp, what="after a range error")


def test_invalid_latent_scale_rejected_on_host():
    wl = W.custom(1, 16, 1, [10])
    inp = W.make_inputs_fp8(wl, seed=2)
    q, kv8, bt, sl = _to_device(inp)
    meta = mla.get_metadata(sl, 16, 1)
    for bad in (0.0, -1.0, float("nan"), float("inf"), 2.0 ** -70):
        with pytest.raises(mla.MLAError):
            mla.decode_fp8(q, kv8, bt, sl, wl.scale, bad, False, meta)


def test_deterministic_and_graph_capturable():
    wl = W.custom(4, 128, 1, [3000, 100, 4000, 65])
    inp = W.make_inputs_fp8(wl, seed=7)
    q, kv8, bt, sl = _to_device(inp)

    def step():
        meta = mla.get_metadata(sl, 128, 1, num_parts=9)
        return mla.decode_fp8(q, kv8, bt, sl, wl.scale, inp["kv_scale"], False, meta)

    o1, l1 = step()
    o2, l2 = step()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        og, lg = step()
    graph.replay()
    torch.cuda.synchronize()
    assert mla.check_status() == 0
    assert torch.equal(og, o1) and torch.equal(lg, l1)
    del graph


def test_host_entry_point_matches_device_path():
    """mla_decode_host_fp8 (host buffers in and out) gives the device path's bits."""
    wl = W.custom(3, 64, 2, [300, 1, 129], causal=True)
    inp = W.make_inputs_fp8(wl, seed=9, kv_scale=0.0123)
    out_d, lse_d, _ = run_fp8(inp)
    dec = mla.HostDecoder(3, 2, 64, inp["kv8"].shape[0], inp["block_table"].shape[1], kv_scale=inp["kv_scale"])
    qh = torch.from_numpy(inp["q"]).view(torch.bfloat16).pin_memory()
    kvh = torch.from_numpy(inp["kv8"]).pin_memory()
    bth = torch.from_numpy(inp["block_table"]).pin_memory()
    slh = torch.from_numpy(inp["seqlens"]).pin_memory()
    oh = torch.empty((3, 2, 64, 512), dtype=torch.bfloat16).pin_memory()
    lh = torch.empty((3, 64, 2), dtype=torch.float32).pin_memory()
    dec(qh, kvh, bth, slh, inp["scale"], True, oh, lh)
    assert torch.equal(oh, out_d.cpu()) and torch.equal(lh, lse_d.cpu())
