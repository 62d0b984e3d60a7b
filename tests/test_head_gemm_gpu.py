"""GPU parity of the per-head projection GEMMs (tcgen05) against the oracle (needs a B200).

Tolerance: bf16 inputs multiply exactly and accumulate in fp32 (relative error ~k 2^-24), and the
result is rounded once to bf16 (2^-9 relative): |y - ref| <= 2^-8 |ref| + 2^-12 max|ref| per
element."""
import numpy as np
import pytest
import torch

import mla_decode_attention_14_b200 as mla
import oracle
from mla_decode_attention_14_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _bf16(shape, seed, scale=1.0):
    bits = W.f32_to_bf16_bits(np.random.default_rng(seed).standard_normal(shape, dtype=np.float32) * np.float32(scale))
    return bits, W.bf16_bits_to_f32(bits).astype(np.float64)


def _close(got, ref):
    err = np.abs(got - ref)
    assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 2.0 ** -12 * np.abs(ref).max()), err.max()


@pytest.mark.parametrize("b,s_q,h", [(128, 1, 128), (100, 1, 16), (3, 2, 8)])
def test_absorb_q_writes_the_latent_query(b, s_q, h):
    k = 128
    xb, xf = _bf16((b, s_q, h, k), 1)
    wb, wf = _bf16((h, k, 512), 2, scale=k ** -0.5)
    qb, _ = _bf16((b, s_q, h, 576), 3)
    q = torch.from_numpy(qb).view(torch.bfloat16).cuda()
    mla.absorb_q(torch.from_numpy(xb).view(torch.bfloat16).cuda(), torch.from_numpy(wb).view(torch.bfloat16).cuda(), q)
    assert mla.check_status() == 0
    got = q.float().cpu().numpy().astype(np.float64)
    ref = oracle.head_gemm(xf.reshape(b * s_q, h, k), wf).reshape(b, s_q, h, 512)
    _close(got[..., :512], ref)
    assert np.array_equal(q.view(torch.uint16).cpu().numpy()[..., 512:], qb[..., 512:])  # rotary dims kept


@pytest.mark.parametrize("b,s_q,h,d", [(128, 1, 128, 128), (70, 2, 16, 64)])
def test_absorb_o_projects_the_latent_output(b, s_q, h, d):
    xb, xf = _bf16((b, s_q, h, 512), 4)
    wb, wf = _bf16((h, 512, d), 5, scale=512 ** -0.5)
    out = mla.absorb_o(torch.from_numpy(xb).view(torch.bfloat16).cuda(), torch.from_numpy(wb).view(torch.bfloat16).cuda())
    assert mla.check_status() == 0
    ref = oracle.head_gemm(xf.reshape(b * s_q, h, 512), wf).reshape(b, s_q, h, d)
    _close(out.float().cpu().numpy().astype(np.float64), ref)
