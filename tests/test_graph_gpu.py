"""A whole decode step -- metadata, split kernel, combine kernel -- captured in one CUDA graph.

Captured on a side stream after warm-up, the step replays bit-identical to the eager calls, and
a replay after new query values are copied into the captured input tensor computes on the new
values (the graph holds pointers, not data)."""
import numpy as np
import pytest
import torch

import mla_decode_attention_14_b200 as mla
from mla_decode_attention_14_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _eager(q, kv, bt, sl, wl, parts):
    meta = mla.get_metadata(sl, wl.h_q, wl.s_q, num_parts=parts)
    return mla.decode(q, kv, bt, sl, wl.scale, wl.causal, meta)


@pytest.mark.parametrize("case", [([700, 5, 1290], 128, 1, False, 9), ([129, 65, 1, 2, 200], 64, 2, True, 5)],
                         ids=["split-128", "causal-s_q2"])
def test_decode_step_replays_from_a_cuda_graph(case):
    seqlens, h_q, s_q, causal, parts = case
    wl = W.custom(len(seqlens), h_q, s_q, seqlens, causal=causal)
    inp = W.make_inputs(wl, seed=9, tail="nan", spare_blocks=1)
    q, kv, bt, sl = parity.to_device(inp)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(2):
            _eager(q, kv, bt, sl, wl, parts)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        out_g, lse_g = _eager(q, kv, bt, sl, wl, parts)
    graph.replay()
    torch.cuda.synchronize()
    assert mla.check_status() == 0

    out_e, lse_e = _eager(q, kv, bt, sl, wl, parts)
    torch.cuda.synchronize()
    assert torch.equal(out_g, out_e)
    assert torch.equal(lse_g, lse_e)
    parity.compare(parity.bf16_to_f64(out_g), lse_g.cpu().numpy().astype(np.float64),
                   *_oracle(inp), what="graph replay")

    # new queries in the captured tensor: the replay computes on them
    inp2 = W.make_inputs(wl, seed=10, tail="nan", spare_blocks=1)
    inp2["kv"], inp2["block_table"] = inp["kv"], inp["block_table"]
    q.copy_(torch.from_numpy(inp2["q"]).view(torch.bfloat16).to(q.device))
    graph.replay()
    torch.cuda.synchronize()
    parity.compare(parity.bf16_to_f64(out_g), lse_g.cpu().numpy().astype(np.float64),
                   *_oracle(inp2), what="graph replay, new queries")
    del graph


def _oracle(inp):
    import oracle
    return oracle.decode(inp["q"], inp["kv"], inp["block_table"], inp["seqlens"], inp["scale"], inp["causal"])
