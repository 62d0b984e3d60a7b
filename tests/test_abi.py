"""C-ABI checks that need no GPU: the library loads, exports every symbol include/mla.h
declares, and rejects invalid arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

import mla_decode_attention_14_b200 as mla
from mla_decode_attention_14_b200 import build as mla_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla.h")


@pytest.fixture(scope="module")
def L():
    mla_build.build()
    return mla.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(mla.EXPORTS)


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_library_links_no_cuda_driver_at_load_time():
    # the runtime is static and driver entry points are resolved lazily, so the .so
    # loads on a machine without a GPU driver
    import subprocess
    out = subprocess.run(["ldd", mla.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out


def test_status_strings(L):
    for code, name in mla.STATUS_NAMES.items():
        assert L.mla_status_string(code).decode().startswith(name)
    assert L.mla_status_string(99).decode() == "MLA: unknown status"


def test_workspace_formula(L):
    b, s_q, h_q, P = 128, 1, 128, 74
    raw = (b + P) * s_q * h_q * (512 + 3) * 4
    assert L.mla_workspace_bytes(b, s_q, h_q, P) == (raw + 255) // 256 * 256
    assert L.mla_workspace_bytes(0, 1, 1, 1) == 0
    assert L.mla_workspace_bytes(1, 1, 2000, 1) == 0   # rows above MLA_MAX_ROWS


FAKE = 1 << 20  # a 256-aligned non-null address; never dereferenced (validation fails first)


def _decode_call(L, **kw):
    a = dict(q=FAKE, kv=FAKE, nblk=10, bt=FAKE, bts=4, sl=FAKE, tm=FAKE, ns=FAKE, P=4, b=2, s_q=1,
             h_q=16, scale=0.1, causal=0, out=FAKE, lse=FAKE, ws=FAKE, wsb=1 << 30, stream=None)
    a.update(kw)
    return L.mla_decode(a["q"], a["kv"], a["nblk"], a["bt"], a["bts"], a["sl"], a["tm"], a["ns"], a["P"],
                        a["b"], a["s_q"], a["h_q"], a["scale"], a["causal"], a["out"], a["lse"], a["ws"],
                        a["wsb"], a["stream"])


@pytest.mark.parametrize("bad", [
    dict(q=None), dict(kv=None), dict(out=None), dict(ws=None), dict(q=FAKE + 8), dict(kv=FAKE + 2),
    dict(ws=FAKE + 16), dict(b=0), dict(s_q=0), dict(h_q=0), dict(h_q=1025), dict(P=0), dict(nblk=0),
    dict(bts=0), dict(scale=float("nan")), dict(scale=float("inf")), dict(scale=-0.1), dict(causal=2),
])
def test_invalid_arguments_rejected_on_host(L, bad):
    assert _decode_call(L, **bad) == 1  # MLA_ERR_INVALID_ARG


def test_small_workspace_rejected_on_host(L):
    assert _decode_call(L, wsb=1024) == 3  # MLA_ERR_WORKSPACE


def test_metadata_argument_checks(L):
    assert L.mla_get_metadata(None, 4, 16, 1, 4, 5, FAKE, FAKE, None) == 1
    assert L.mla_get_metadata(FAKE, 4, 16, 1, 0, 5, FAKE, FAKE, None) == 1
    assert L.mla_get_metadata(FAKE, 4, 16, 1, 4, -1, FAKE, FAKE, None) == 1
    assert L.mla_get_metadata(FAKE + 2, 4, 16, 1, 4, 5, FAKE, FAKE, None) == 1


def test_default_num_parts_argument_checks(L):
    n = ctypes.c_int(0)
    assert L.mla_default_num_parts(0, 0, 1, ctypes.byref(n)) == 1
    assert L.mla_default_num_parts(0, 16, 1, None) == 1


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        mla.get_metadata(torch.zeros(4, dtype=torch.int32), 16, 1, num_parts=4, fixed_cost=5)


def test_noalloc_rejects_oversized_requests_on_host(L):
    # beyond MLA_NOALLOC_SCRATCH_BYTES: rejected before any CUDA call (this host has no GPU)
    big_parts = 60000
    assert L.mla_workspace_bytes(2, 1, 128, big_parts) > mla.NOALLOC_SCRATCH_BYTES
    rc = L.mla_decode_noalloc(FAKE, FAKE, 10, FAKE, 4, FAKE, FAKE, FAKE, big_parts, 2, 1, 128, 0.1, 0,
                              FAKE, FAKE, None)
    assert rc == 3  # MLA_ERR_WORKSPACE
    assert L.mla_decode_noalloc(None, FAKE, 10, FAKE, 4, FAKE, FAKE, FAKE, 4, 2, 1, 16, 0.1, 0,
                                FAKE, FAKE, None) == 1  # MLA_ERR_INVALID_ARG


def test_noalloc_scratch_constant_matches_header():
    import re
    src = open(HEADER).read()
    m = re.search(r"#define MLA_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", src)
    assert m and int(m.group(1)) << int(m.group(2)) == mla.NOALLOC_SCRATCH_BYTES


def test_selftest_bound_is_checked_on_host(L):
    assert L.mla_selftest_wait_timeout(10, None) == 1  # MLA_ERR_INVALID_ARG: bound below 1e5 cycles
    assert L.mla_selftest_wait_timeout(5_000_000_000, None) == 1


def test_append_arguments_checked_on_host(L):
    # null pointers, batch 0, a negative token count, and (fp8) bad scales never reach a launch
    assert L.mla_append_kv(None, 1, FAKE, 10, FAKE, 4, FAKE, 2, None) == 1
    assert L.mla_append_kv(FAKE, 1, FAKE, 10, FAKE, 4, FAKE, 0, None) == 1
    assert L.mla_append_kv(FAKE, -1, FAKE, 10, FAKE, 4, FAKE, 2, None) == 1
    assert L.mla_append_kv(FAKE + 8, 1, FAKE, 10, FAKE, 4, FAKE, 2, None) == 1
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        assert L.mla_append_kv_fp8(FAKE, 1, FAKE, 10, bad, FAKE, 4, FAKE, 2, None) == 1


def test_head_gemm_arguments_checked_on_host(L):
    ok = dict(x=FAKE, ldx=2048, xh=128, w=FAKE, y=FAKE, ldy=8192, yh=512, m=4, n=512, k=128, heads=16)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return L.mla_head_gemm(a["x"], a["ldx"], a["xh"], a["w"], a["y"], a["ldy"], a["yh"], a["m"], a["n"], a["k"],
                               a["heads"], None)
    for bad in (dict(x=None), dict(w=None), dict(y=None), dict(m=0), dict(heads=0), dict(k=96), dict(n=100),
                dict(ldx=2044), dict(xh=100), dict(ldx=1024), dict(ldy=4096), dict(x=FAKE + 8)):
        assert call(**bad) == 1, bad  # MLA_ERR_INVALID_ARG


def _sparse_call(L, **kw):
    a = dict(q=FAKE, kv=FAKE, nblk=10, bt=FAKE, bts=4, sl=FAKE, ix=FAKE, topk=64, tm=FAKE, ns=FAKE, P=4, b=2,
             s_q=2, h_q=16, scale=0.1, out=FAKE, lse=FAKE, ws=FAKE, wsb=1 << 30, stream=None)
    a.update(kw)
    return L.mla_decode_sparse(a["q"], a["kv"], a["nblk"], a["bt"], a["bts"], a["sl"], a["ix"], a["topk"], a["tm"],
                               a["ns"], a["P"], a["b"], a["s_q"], a["h_q"], a["scale"], a["out"], a["lse"], a["ws"],
                               a["wsb"], a["stream"])


@pytest.mark.parametrize("bad", [
    dict(ix=None), dict(ix=FAKE + 2), dict(topk=0), dict(topk=(1 << 24) + 1), dict(q=None), dict(kv=FAKE + 2),
    dict(b=0), dict(s_q=0), dict(h_q=0), dict(h_q=1025), dict(b=1 << 20, s_q=1 << 10), dict(P=0), dict(nblk=0),
    dict(scale=float("nan")), dict(out=FAKE + 8),
])
def test_sparse_invalid_arguments_rejected_on_host(L, bad):
    assert _sparse_call(L, **bad) == 1  # MLA_ERR_INVALID_ARG


def test_sparse_workspace_is_that_of_its_work_units(L):
    # batch * s_q work units of h_q rows: the dense formula at (batch * s_q, 1, h_q)
    need = L.mla_workspace_bytes(2 * 2, 1, 16, 4)
    assert _sparse_call(L, wsb=need - 256) == 3  # MLA_ERR_WORKSPACE


def test_sparse_metadata_argument_checks(L):
    assert L.mla_get_metadata_sparse(2, 1, 16, 64, 4, 5, None, FAKE, None) == 1
    assert L.mla_get_metadata_sparse(2, 1, 16, 0, 4, 5, FAKE, FAKE, None) == 1
    assert L.mla_get_metadata_sparse(0, 1, 16, 64, 4, 5, FAKE, FAKE, None) == 1
    assert L.mla_get_metadata_sparse(2, 1, 16, 64, 0, 5, FAKE, FAKE, None) == 1
    assert L.mla_get_metadata_sparse(2, 1, 16, 64, 4, -1, FAKE, FAKE, None) == 1
