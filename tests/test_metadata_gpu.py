"""GPU split-KV metadata must equal the oracle's partition integer for integer."""
import numpy as np
import pytest
import torch

import mla_decode_attention_14_b200 as mla
import oracle
from mla_decode_attention_14_b200 import workloads as W
from tests import meta_util

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def gpu_meta(seqlens, P, C, h_q=16, s_q=1):
    sl = torch.tensor(np.asarray(seqlens, dtype=np.int32), device="cuda")
    m = mla.get_metadata(sl, h_q, s_q, num_parts=P, fixed_cost=C)
    return m.tile_meta.cpu().numpy(), m.num_splits.cpu().numpy()


def test_hand_worked_fixture_on_gpu():
    seqlens, C, cases = meta_util.load_golden()
    for P, T, meta, cum in cases:
        tm, ns = gpu_meta(seqlens, P, C)
        assert np.array_equal(tm, meta) and np.array_equal(ns, cum), P


@pytest.mark.parametrize("seed", range(20))
def test_random_bit_exact(seed):
    rng = np.random.default_rng(100 + seed)
    b = int(rng.integers(1, 3000 if seed % 4 == 0 else 300))
    sl = rng.choice([0, 1, 63, 64, 65, 100, 4096, 65536], size=b) if seed % 2 else rng.integers(0, 20000, size=b)
    sl = sl.astype(np.int32)
    P = int(rng.integers(1, 300))
    C = int(rng.integers(0, 12))
    tm, ns = gpu_meta(sl, P, C)
    otm, ons = oracle.metadata(sl, P, C)
    assert np.array_equal(tm, otm) and np.array_equal(ns, ons)
    meta_util.check_partition(sl, tm, ns, P, C)


@pytest.mark.parametrize("name", W.NAMES)
def test_workload_defaults_bit_exact(name):
    wl = W.workload(name)
    P = mla.default_num_parts(wl.h_q, wl.s_q)
    C = mla.default_fixed_cost(wl.h_q, wl.s_q)
    tm, ns = gpu_meta(wl.seqlens, P, C, wl.h_q, wl.s_q)
    otm, ons = oracle.metadata(wl.seqlens, P, C)
    assert np.array_equal(tm, otm) and np.array_equal(ns, ons)


def test_large_batch_chunked_scan():
    rng = np.random.default_rng(5)
    sl = rng.integers(0, 300, size=5000).astype(np.int32)
    tm, ns = gpu_meta(sl, 148, 3)
    otm, ons = oracle.metadata(sl, 148, 3)
    assert np.array_equal(tm, otm) and np.array_equal(ns, ons)
