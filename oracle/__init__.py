"""CPU oracle for MLA decode attention over a paged latent KV cache.

TEST INFRASTRUCTURE ONLY. This package is loaded by the test suite, by the smoke
check in ``__graft_entry__`` and by the CPU-baseline leg of ``bench.py``; the
product (the CUDA library under ``mla_decode_attention_14_b200``) never imports it,
and the two share no code. The arithmetic lives in ``mla_oracle.c`` (plain C,
double precision, POSIX threads); this module only builds and calls it.

Sources: "Deep analysis of the DeepSeek Infra open-source releases"
(jingzhunhuoke.net/55333.html), section "DAY1 FlashMLA" (MLA glossary entry,
feature (2) 64-token KV blocks, feature (4) Gemm1/Gemm2, feature (5) variable
lengths), plus the library's task statement for the dimensions (576-d keys, first
512 dims as values), the scale, causal masking and output shapes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

D_QK = 576
D_V = 512
BLK = 64
F8_REC = 640  # fp8 cache: bytes per token


def build(force: bool = False) -> str:
    """Compile ``mla_oracle.c`` into ``liboracle.so`` next to it (gcc, -O2)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-Wall", "-Wextra",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        lib.oracle_metadata.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
        lib.oracle_metadata.restype = ctypes.c_int
        lib.oracle_decode.argtypes = [P, P, ctypes.c_int64, P, ctypes.c_int64, P,
                                      ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                      ctypes.c_int, P, P, P, ctypes.c_int64, ctypes.c_int]
        lib.oracle_decode.restype = ctypes.c_int
        lib.oracle_decode_fp8.argtypes = [P, P, ctypes.c_double, ctypes.c_int64, P, ctypes.c_int64, P,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                          ctypes.c_int, P, P, P, ctypes.c_int64, ctypes.c_int]
        lib.oracle_decode_fp8.restype = ctypes.c_int
        lib.oracle_e4m3_decode.argtypes = [P, ctypes.c_int64, P]
        lib.oracle_e4m3_decode.restype = None
        lib.oracle_decode_sparse.argtypes = [P, P, ctypes.c_int64, P, ctypes.c_int64, P, P, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, P, P,
                                             ctypes.c_int]
        lib.oracle_decode_sparse.restype = ctypes.c_int
        lib.oracle_e4m3_encode.argtypes = [P, ctypes.c_int64, P]
        lib.oracle_e4m3_encode.restype = None
        lib.oracle_append.argtypes = [P, ctypes.c_int, P, ctypes.c_int64, P, ctypes.c_int64, P, ctypes.c_int]
        lib.oracle_append.restype = ctypes.c_int
        lib.oracle_append_fp8.argtypes = [P, ctypes.c_int, P, ctypes.c_float, ctypes.c_int64, P, ctypes.c_int64, P,
                                          ctypes.c_int]
        lib.oracle_append_fp8.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def metadata(seqlens, num_parts: int, fixed_cost: int):
    """Work partition of every (sequence, 64-token block) into ``num_parts`` parts.

    Returns ``(tile_meta int32[num_parts, 8], num_splits_cum int32[batch + 1])``;
    the layout is documented in ``mla_oracle.c``.
    """
    s = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    tm = np.zeros((num_parts, 8), dtype=np.int32)
    ns = np.zeros(s.shape[0] + 1, dtype=np.int32)
    rc = _load().oracle_metadata(_ptr(s), int(s.shape[0]), int(num_parts), int(fixed_cost),
                                 _ptr(tm), _ptr(ns))
    if rc != 0:
        raise ValueError("oracle_metadata: bad arguments (rc=%d)" % rc)
    return tm, ns


def decode(q_bits, kv_bits, block_table, seqlens, scale: float, causal: bool,
           tasks=None, nthreads: int | None = None):
    """Exact (double) MLA decode attention.

    ``q_bits``: uint16 bf16 bit patterns ``[b, s_q, h_q, 576]``;
    ``kv_bits``: uint16 ``[num_blocks, 64, 1, 576]`` (or ``[num_blocks, 64, 576]``);
    ``block_table``: int32 ``[b, max_blocks]``; ``seqlens``: int32 ``[b]``.
    Returns ``(out float64[b, s_q, h_q, 512], lse float64[b, h_q, s_q])``. With
    ``tasks`` (int32 ``[k, 3]`` of (b, t, h)) only those rows are computed and the
    others are NaN.
    """
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    kv = np.ascontiguousarray(kv_bits, dtype=np.uint16)
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seqlens, dtype=np.int32)
    b, s_q, h_q, d = q.shape
    assert d == D_QK and kv.shape[-1] == D_QK and kv.shape[1] == BLK
    nblk = kv.shape[0]
    out = np.full((b, s_q, h_q, D_V), np.nan, dtype=np.float64)
    lse = np.full((b, h_q, s_q), np.nan, dtype=np.float64)
    if tasks is not None:
        tk = np.ascontiguousarray(tasks, dtype=np.int32).reshape(-1, 3)
        tptr, nt = _ptr(tk), tk.shape[0]
    else:
        tk, tptr, nt = None, None, 0
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _load().oracle_decode(_ptr(q), _ptr(kv), nblk, _ptr(bt), bt.shape[1] if bt.ndim == 2 else 0,
                               _ptr(sl), b, s_q, h_q, float(scale), int(bool(causal)),
                               _ptr(out), _ptr(lse), tptr, nt, int(nthreads))
    if rc != 0:
        raise ValueError("oracle_decode failed (rc=%d)" % rc)
    return out, lse


def decode_fp8(q_bits, kv8, kv_scale: float, block_table, seqlens, scale: float, causal: bool,
               tasks=None, nthreads: int | None = None):
    """Exact (double) MLA decode attention over the fp8 cache.

    ``kv8``: uint8 ``[num_blocks, 64, 1, 640]`` (or ``[num_blocks, 64, 640]``): per token
    512 OCP E4M3 latent bytes, each standing for ``kv_scale * e4m3(byte)``, then the 64
    rotary dims as little-endian bf16. Everything else as :func:`decode`.
    """
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    kv = np.ascontiguousarray(kv8, dtype=np.uint8)
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seqlens, dtype=np.int32)
    b, s_q, h_q, d = q.shape
    assert d == D_QK and kv.shape[-1] == F8_REC and kv.shape[1] == BLK
    out = np.full((b, s_q, h_q, D_V), np.nan, dtype=np.float64)
    lse = np.full((b, h_q, s_q), np.nan, dtype=np.float64)
    if tasks is not None:
        tk = np.ascontiguousarray(tasks, dtype=np.int32).reshape(-1, 3)
        tptr, nt = _ptr(tk), tk.shape[0]
    else:
        tk, tptr, nt = None, None, 0
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _load().oracle_decode_fp8(_ptr(q), _ptr(kv), float(kv_scale), kv.shape[0], _ptr(bt),
                                   bt.shape[1] if bt.ndim == 2 else 0, _ptr(sl), b, s_q, h_q, float(scale),
                                   int(bool(causal)), _ptr(out), _ptr(lse), tptr, nt, int(nthreads))
    if rc != 0:
        raise ValueError("oracle_decode_fp8 failed (rc=%d)" % rc)
    return out, lse


def e4m3_decode(codes) -> np.ndarray:
    """OCP E4M3 bytes -> float64, as the oracle reads the fp8 cache."""
    x = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(x.shape, dtype=np.float64)
    _load().oracle_e4m3_decode(_ptr(x), x.size, _ptr(out))
    return out


def e4m3_encode(x) -> np.ndarray:
    """float32 -> OCP E4M3 codes, round to nearest even, saturating to +-448."""
    v = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _load().oracle_e4m3_encode(_ptr(v), v.size, _ptr(out))
    return out


def append(new_kv_bits, kv_bits, block_table, seqlens):
    """Write the new tokens ``new_kv_bits`` (uint16 bf16 ``[b, n_new, 576]``) into a copy of the bf16
    cache at positions ``seqlens[b] + t``; returns the new cache."""
    nk = np.ascontiguousarray(new_kv_bits, dtype=np.uint16)
    kv = np.array(kv_bits, dtype=np.uint16, copy=True, order="C")
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seqlens, dtype=np.int32)
    rc = _load().oracle_append(_ptr(nk), nk.shape[1], _ptr(kv), kv.shape[0], _ptr(bt), bt.shape[1], _ptr(sl),
                               nk.shape[0])
    if rc != 0:
        raise ValueError("oracle_append: a row lands outside the table or the cache")
    return kv


def append_fp8(new_kv_bits, kv8, inv_scale: float, block_table, seqlens):
    """The same into a copy of the fp8 cache: latent values times ``inv_scale`` (fp32) rounded to
    E4M3, rotary dims copied; returns the new cache."""
    nk = np.ascontiguousarray(new_kv_bits, dtype=np.uint16)
    kv = np.array(kv8, dtype=np.uint8, copy=True, order="C")
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seqlens, dtype=np.int32)
    rc = _load().oracle_append_fp8(_ptr(nk), nk.shape[1], _ptr(kv), float(np.float32(inv_scale)), kv.shape[0],
                                   _ptr(bt), bt.shape[1], _ptr(sl), nk.shape[0])
    if rc != 0:
        raise ValueError("oracle_append_fp8: a row lands outside the table or the cache")
    return kv


def head_gemm(x, w):
    """Per-head products in double: ``x`` float ``[m, heads, k]``, ``w`` ``[heads, k, n]`` ->
    ``[m, heads, n]`` with ``y[r, h] = x[r, h] @ w[h]`` (numpy's matmul as the library step)."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    return np.einsum("mhk,hkn->mhn", x, w)


def decode_sparse(q_bits, kv_bits, block_table, seqlens, indices, scale: float, nthreads: int | None = None):
    """Exact (double) sparse decode: row (b, t, h) attends to the keys at positions
    ``indices[b, t, :]`` (int32 ``[b, s_q, topk]``; entries outside ``[0, seqlens[b])`` are no key).
    Returns ``(out float64[b, s_q, h_q, 512], lse float64[b, h_q, s_q])``."""
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    kv = np.ascontiguousarray(kv_bits, dtype=np.uint16)
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seqlens, dtype=np.int32)
    ix = np.ascontiguousarray(indices, dtype=np.int32)
    b, s_q, h_q, d = q.shape
    assert d == D_QK and ix.shape[:2] == (b, s_q)
    out = np.full((b, s_q, h_q, D_V), np.nan, dtype=np.float64)
    lse = np.full((b, h_q, s_q), np.nan, dtype=np.float64)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _load().oracle_decode_sparse(_ptr(q), _ptr(kv), kv.shape[0], _ptr(bt), bt.shape[1], _ptr(sl), _ptr(ix),
                                      ix.shape[2], b, s_q, h_q, float(scale), _ptr(out), _ptr(lse), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_decode_sparse failed (rc=%d)" % rc)
    return out, lse

