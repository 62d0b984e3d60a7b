"""B200-native (sm_100a) MLA decode attention over a paged latent KV cache.

Thin Python binding of the C ABI in ``include/mla.h`` (``libmla_b200.so``, built in-tree by
``python -m mla_decode_attention_14_b200.build``). It only marshals arguments: every step of
the computation runs in the library's CUDA kernels. PyTorch provides device memory and
streams. There is no CPU or framework fallback: if the library is missing or the device is
not an sm_100 GPU, the calls raise.

    meta = get_metadata(seqlens, h_q, s_q)              # split-KV schedule (device int32)
    out, lse = decode(q, kv_cache, block_table, seqlens, scale, causal, meta)

Shapes: q bf16 [b, s_q, h_q, 576]; kv_cache bf16 [num_blocks, 64, 1, 576] (64-token blocks,
"Deep analysis of the DeepSeek Infra open-source releases", DAY1 FlashMLA, feature (2));
block_table int32 [b, max_blocks]; seqlens int32 [b]; out bf16 [b, s_q, h_q, 512];
lse fp32 [b, h_q, s_q].
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

D_QK = 576
D_V = 512
BLOCK = 64
FP8_RECORD_BYTES = 640  # MLA_FP8_RECORD_BYTES in include/mla.h
META_INTS = 8

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla_b200.so")
_lib = None

MLA_OK = 0
STATUS_NAMES = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_WORKSPACE",
                4: "MLA_ERR_CUDA", 5: "MLA_ERR_TIMEOUT", 6: "MLA_ERR_BOUNDS",
                7: "MLA_ERR_RANGE"}

# exported C symbols, in the order include/mla.h declares them
EXPORTS = ("mla_status_string", "mla_default_num_parts", "mla_default_fixed_cost", "mla_workspace_bytes",
           "mla_get_metadata", "mla_decode", "mla_decode_split", "mla_decode_combine", "mla_decode_fp8",
           "mla_decode_split_fp8", "mla_get_metadata_sparse", "mla_decode_sparse", "mla_append_kv", "mla_append_kv_fp8", "mla_head_gemm",
           "mla_decode_host", "mla_decode_host_fp8",
           "mla_decode_noalloc", "mla_check_status", "mla_launch_count", "mla_last_cuda_error",
           "mla_selftest_wait_timeout")


class MLAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = lib().mla_status_string(status).decode() if _lib is not None else STATUS_NAMES.get(status, "?")
        if status == 4 and _lib is not None:  # MLA_ERR_CUDA: say which CUDA error it was
            msg += " [%s]" % lib().mla_last_cuda_error().decode()
        super().__init__("%s failed: %s (status %d)" % (fn, msg, status))


class _DeviceBuffers(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("kv_cache", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("seqlens", ctypes.c_void_p), ("tile_meta", ctypes.c_void_p), ("num_splits", ctypes.c_void_p),
                ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t), ("num_parts", ctypes.c_int), ("fixed_cost", ctypes.c_int)]


def lib():
    """Load ``libmla_b200.so`` (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libmla_b200.so not found at %s; build it with "
                               "`python -m mla_decode_attention_14_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, SZ, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
        L.mla_status_string.argtypes = [I]
        L.mla_status_string.restype = ctypes.c_char_p
        L.mla_default_num_parts.argtypes = [I, I, I, ctypes.POINTER(I)]
        L.mla_default_num_parts.restype = I
        L.mla_default_fixed_cost.argtypes = [I, I]
        L.mla_default_fixed_cost.restype = I
        L.mla_workspace_bytes.argtypes = [I, I, I, I]
        L.mla_workspace_bytes.restype = SZ
        L.mla_get_metadata.argtypes = [P, I, I, I, I, I, P, P, P]
        L.mla_get_metadata.restype = I
        dec = [P, P, I64, P, I64, P, P, P, I, I, I, I, F, I, P, P, P, SZ, P]
        for name in ("mla_decode", "mla_decode_split"):
            getattr(L, name).argtypes = dec
            getattr(L, name).restype = I
        dec8 = dec[:3] + [F] + dec[3:]  # kv_scale after num_blocks
        for name in ("mla_decode_fp8", "mla_decode_split_fp8"):
            getattr(L, name).argtypes = dec8
            getattr(L, name).restype = I
        L.mla_get_metadata_sparse.argtypes = [I, I, I, I, I, I, P, P, P]
        L.mla_get_metadata_sparse.restype = I
        L.mla_decode_sparse.argtypes = [P, P, I64, P, I64, P, P, I, P, P, I, I, I, I, F, P, P, P, SZ, P]
        L.mla_decode_sparse.restype = I
        L.mla_append_kv.argtypes = [P, I, P, I64, P, I64, P, I, P]
        L.mla_append_kv.restype = I
        L.mla_append_kv_fp8.argtypes = [P, I, P, I64, F, P, I64, P, I, P]
        L.mla_append_kv_fp8.restype = I
        L.mla_head_gemm.argtypes = [P, I64, I64, P, P, I64, I64, I, I, I, I, P]
        L.mla_head_gemm.restype = I
        L.mla_decode_noalloc.argtypes = dec[:16] + [P]
        L.mla_decode_noalloc.restype = I
        L.mla_decode_combine.argtypes = [P, I, I, I, I, P, P, P, SZ, P]
        L.mla_decode_combine.restype = I
        L.mla_decode_host.argtypes = [P, P, I64, P, I64, P, I, I, I, F, I, P, P,
                                      ctypes.POINTER(_DeviceBuffers), P]
        L.mla_decode_host.restype = I
        L.mla_decode_host_fp8.argtypes = [P, P, I64, F, P, I64, P, I, I, I, F, I, P, P,
                                          ctypes.POINTER(_DeviceBuffers), P]
        L.mla_decode_host_fp8.restype = I
        L.mla_check_status.argtypes = [P]
        L.mla_check_status.restype = I
        L.mla_launch_count.argtypes = []
        L.mla_launch_count.restype = I64
        L.mla_last_cuda_error.argtypes = []
        L.mla_last_cuda_error.restype = ctypes.c_char_p
        L.mla_selftest_wait_timeout.argtypes = [I64, P]
        L.mla_selftest_wait_timeout.restype = I
        _lib = L
    return _lib


def _check(fn: str, rc: int):
    if rc != MLA_OK:
        raise MLAError(fn, rc)


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _need(t: torch.Tensor, name: str, dtype, ndim=None, cuda=True):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if cuda and not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if ndim is not None and t.dim() != ndim:
        raise ValueError("%s must have %d dims, got shape %s" % (name, ndim, tuple(t.shape)))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


@dataclass
class Metadata:
    """Split-KV schedule produced by :func:`get_metadata` (device tensors)."""
    tile_meta: torch.Tensor   # int32 [num_parts, 8]
    num_splits: torch.Tensor  # int32 [batch + 1], cumulative piece counts
    num_parts: int
    fixed_cost: int
    h_q: int
    s_q: int
    topk: int = 0             # sparse mode (get_metadata_sparse): keys per query token; 0 = dense


def default_num_parts(h_q: int, s_q: int, device=None) -> int:
    dev = torch.cuda.current_device() if device is None else torch.device(device).index or 0
    n = ctypes.c_int(0)
    _check("mla_default_num_parts", lib().mla_default_num_parts(dev, h_q, s_q, ctypes.byref(n)))
    return n.value


def default_fixed_cost(h_q: int, s_q: int) -> int:
    return lib().mla_default_fixed_cost(h_q, s_q)


def workspace_bytes(batch: int, s_q: int, h_q: int, num_parts: int) -> int:
    return lib().mla_workspace_bytes(batch, s_q, h_q, num_parts)


def get_metadata(seqlens: torch.Tensor, h_q: int, s_q: int, num_parts: int | None = None,
                 fixed_cost: int | None = None, stream=None) -> Metadata:
    """Tile-scheduler metadata and per-sequence split counts for ``seqlens`` (int32 [b], CUDA)."""
    _need(seqlens, "seqlens", torch.int32, 1)
    b = seqlens.shape[0]
    if num_parts is None:
        num_parts = default_num_parts(h_q, s_q, seqlens.device)
    if fixed_cost is None:
        fixed_cost = default_fixed_cost(h_q, s_q)
    tm = torch.empty((num_parts, META_INTS), dtype=torch.int32, device=seqlens.device)
    ns = torch.empty((b + 1,), dtype=torch.int32, device=seqlens.device)
    with torch.cuda.device(seqlens.device):
        _check("mla_get_metadata", lib().mla_get_metadata(seqlens.data_ptr(), b, h_q, s_q, num_parts, fixed_cost,
                                                          tm.data_ptr(), ns.data_ptr(), _stream(stream)))
    return Metadata(tm, ns, num_parts, fixed_cost, h_q, s_q)


def get_metadata_sparse(batch: int, s_q: int, h_q: int, topk: int, num_parts: int | None = None,
                        fixed_cost: int | None = None, device=None, stream=None) -> Metadata:
    """Schedule for :func:`decode_sparse`: ``batch * s_q`` work units (one per query token) of
    ``topk`` keys each (``mla_get_metadata_sparse``)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if num_parts is None:
        num_parts = default_num_parts(h_q, 1, dev)
    if fixed_cost is None:
        fixed_cost = default_fixed_cost(h_q, 1)
    tm = torch.empty((num_parts, META_INTS), dtype=torch.int32, device=dev)
    ns = torch.empty((batch * s_q + 1,), dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _check("mla_get_metadata_sparse", lib().mla_get_metadata_sparse(batch, s_q, h_q, topk, num_parts, fixed_cost,
                                                                        tm.data_ptr(), ns.data_ptr(),
                                                                        _stream(stream)))
    return Metadata(tm, ns, num_parts, fixed_cost, h_q, s_q, topk)


def decode_sparse(q: torch.Tensor, kv_cache: torch.Tensor, block_table: torch.Tensor, seqlens: torch.Tensor,
                  indices: torch.Tensor, scale: float, meta: Metadata, out: torch.Tensor | None = None,
                  lse: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    """Sparse MLA decode (``mla_decode_sparse``): row (b, t, h) attends only to the cache positions
    ``indices[b, t, :]`` (int32 ``[b, s_q, topk]``; entries outside ``[0, seqlens[b])`` are no key).
    Returns ``(out bf16 [b, s_q, h_q, 512], lse fp32 [b, h_q, s_q])``."""
    _need(q, "q", torch.bfloat16, 4)
    _need(kv_cache, "kv_cache", torch.bfloat16)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seqlens, "seqlens", torch.int32, 1)
    _need(indices, "indices", torch.int32, 3)
    b, s_q, h_q, d = q.shape
    topk = indices.shape[2]
    if d != D_QK or kv_cache.shape[-1] != D_QK or kv_cache.shape[1] != BLOCK:
        raise ValueError("q must be [b, s_q, h_q, 576] and kv_cache [num_blocks, 64, 1, 576]")
    if block_table.shape[0] != b or seqlens.shape[0] != b or indices.shape[:2] != (b, s_q):
        raise ValueError("batch mismatch between q, block_table, seqlens and indices")
    if meta.topk != topk or meta.h_q != h_q or meta.s_q != s_q or meta.num_splits.shape[0] != b * s_q + 1:
        raise ValueError("metadata was computed for another shape (use get_metadata_sparse)")
    dev = q.device
    if out is None:
        out = torch.empty((b, s_q, h_q, D_V), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((b, h_q, s_q), dtype=torch.float32, device=dev)
    _need(out, "out", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    ws_bytes = workspace_bytes(b * s_q, 1, h_q, meta.num_parts)
    if workspace is None:
        workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    if workspace.numel() * workspace.element_size() < ws_bytes:
        raise ValueError("workspace too small: need %d bytes" % ws_bytes)
    with torch.cuda.device(dev):
        _check("mla_decode_sparse", lib().mla_decode_sparse(
            q.data_ptr(), kv_cache.data_ptr(), kv_cache.shape[0], block_table.data_ptr(), block_table.shape[1],
            seqlens.data_ptr(), indices.data_ptr(), topk, meta.tile_meta.data_ptr(), meta.num_splits.data_ptr(),
            meta.num_parts, b, s_q, h_q, float(scale), out.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
            ws_bytes, _stream(stream)))
    return out, lse


def _decode_args(q, kv_cache, block_table, seqlens, meta):
    _need(q, "q", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seqlens, "seqlens", torch.int32, 1)
    b, s_q, h_q, d = q.shape
    if d != D_QK:
        raise ValueError("q last dim must be %d" % D_QK)
    if kv_cache is not None:  # bf16 cache (the fp8 one is checked by decode_fp8)
        _need(kv_cache, "kv_cache", torch.bfloat16)
        if kv_cache.dim() == 4:
            if kv_cache.shape[1:] != (BLOCK, 1, D_QK):
                raise ValueError("kv_cache must be [num_blocks, 64, 1, 576], got %s" % (tuple(kv_cache.shape),))
        elif kv_cache.dim() != 3 or kv_cache.shape[1:] != (BLOCK, D_QK):
            raise ValueError("kv_cache must be [num_blocks, 64, 1, 576], got %s" % (tuple(kv_cache.shape),))
    if block_table.shape[0] != b or seqlens.shape[0] != b:
        raise ValueError("batch mismatch between q, block_table and seqlens")
    if meta.h_q != h_q or meta.s_q != s_q or meta.num_splits.shape[0] != b + 1:
        raise ValueError("metadata was computed for another shape")
    return b, s_q, h_q


def _outputs(b, s_q, h_q, meta, dev, out, lse, workspace):
    if out is None:
        out = torch.empty((b, s_q, h_q, D_V), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((b, h_q, s_q), dtype=torch.float32, device=dev)
    _need(out, "out", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    ws_bytes = workspace_bytes(b, s_q, h_q, meta.num_parts)
    if workspace is None:
        workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    if workspace.numel() * workspace.element_size() < ws_bytes:
        raise ValueError("workspace too small: need %d bytes" % ws_bytes)
    return out, lse, workspace, ws_bytes


def _append_args(new_kv, block_table, seqlens):
    _need(new_kv, "new_kv", torch.bfloat16, 3)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seqlens, "seqlens", torch.int32, 1)
    b, n_new, d = new_kv.shape
    if d != D_QK:
        raise ValueError("new_kv last dim must be %d" % D_QK)
    if block_table.shape[0] != b or seqlens.shape[0] != b:
        raise ValueError("batch mismatch between new_kv, block_table and seqlens")
    return b, n_new  # n_new == 0 is a no-op (an empty tensor may have no storage to point at)


def append_kv(new_kv: torch.Tensor, kv_cache: torch.Tensor, block_table: torch.Tensor, seqlens: torch.Tensor,
              stream=None) -> None:
    """Write ``new_kv`` (bf16 ``[b, n_new, 576]``) into the bf16 cache at positions
    ``seqlens[b] + t`` (``mla_append_kv``); ``seqlens`` are the lengths before the append."""
    b, n_new = _append_args(new_kv, block_table, seqlens)
    _need(kv_cache, "kv_cache", torch.bfloat16)
    if kv_cache.shape[-1] != D_QK or kv_cache.shape[1] != BLOCK:
        raise ValueError("kv_cache must be [num_blocks, 64, 1, 576]")
    if n_new == 0:
        return
    with torch.cuda.device(new_kv.device):
        _check("mla_append_kv", lib().mla_append_kv(new_kv.data_ptr(), n_new, kv_cache.data_ptr(), kv_cache.shape[0],
                                                    block_table.data_ptr(), block_table.shape[1], seqlens.data_ptr(),
                                                    b, _stream(stream)))


def append_kv_fp8(new_kv: torch.Tensor, kv_cache_fp8: torch.Tensor, block_table: torch.Tensor,
                  seqlens: torch.Tensor, kv_scale: float, stream=None) -> None:
    """The same into the fp8 cache (``mla_append_kv_fp8``): latent values stored as E4M3 codes of
    ``x * (1 / kv_scale)``, rotary dims as bf16."""
    b, n_new = _append_args(new_kv, block_table, seqlens)
    _need(kv_cache_fp8, "kv_cache_fp8", torch.uint8)
    if kv_cache_fp8.shape[-1] != FP8_RECORD_BYTES or kv_cache_fp8.shape[1] != BLOCK:
        raise ValueError("kv_cache_fp8 must be uint8 [num_blocks, 64, 1, %d]" % FP8_RECORD_BYTES)
    if n_new == 0:
        return
    with torch.cuda.device(new_kv.device):
        _check("mla_append_kv_fp8", lib().mla_append_kv_fp8(new_kv.data_ptr(), n_new, kv_cache_fp8.data_ptr(),
                                                            kv_cache_fp8.shape[0], float(kv_scale),
                                                            block_table.data_ptr(), block_table.shape[1],
                                                            seqlens.data_ptr(), b, _stream(stream)))


def head_gemm(x: torch.Tensor, ldx: int, x_head_stride: int, w: torch.Tensor, y: torch.Tensor, ldy: int,
              y_head_stride: int, m: int, n: int, k: int, heads: int, stream=None) -> torch.Tensor:
    """Per-head GEMM ``Y_h = X_h W_h`` (``mla_head_gemm``); strides in elements, see include/mla.h."""
    _need(x, "x", torch.bfloat16)
    _need(w, "w", torch.bfloat16)
    _need(y, "y", torch.bfloat16)
    if w.numel() != heads * k * n:
        raise ValueError("w must hold heads x k x n values")
    with torch.cuda.device(x.device):
        _check("mla_head_gemm", lib().mla_head_gemm(x.data_ptr(), ldx, x_head_stride, w.data_ptr(), y.data_ptr(), ldy,
                                                    y_head_stride, m, n, k, heads, _stream(stream)))
    return y


def absorb_q(q_nope: torch.Tensor, w_uk: torch.Tensor, q: torch.Tensor, stream=None) -> torch.Tensor:
    """Latent queries ``q[..., :512] = q_nope W_UK`` per head: ``q_nope`` bf16 ``[b, s_q, h, k]``,
    ``w_uk`` bf16 ``[h, k, 512]``, ``q`` the decode's bf16 ``[b, s_q, h, 576]`` (its rotary dims are
    left as they are)."""
    _need(q_nope, "q_nope", torch.bfloat16, 4)
    _need(q, "q", torch.bfloat16, 4)
    b, s_q, h, k = q_nope.shape
    if tuple(q.shape) != (b, s_q, h, D_QK) or tuple(w_uk.shape) != (h, k, D_V):
        raise ValueError("shapes: q_nope [b, s_q, h, k], w_uk [h, k, 512], q [b, s_q, h, 576]")
    return head_gemm(q_nope, h * k, k, w_uk, q, h * D_QK, D_QK, b * s_q, D_V, k, h, stream)


def absorb_o(o_latent: torch.Tensor, w_uv: torch.Tensor, out: torch.Tensor | None = None, stream=None):
    """Per-head output projection ``o = o_latent W_UV``: ``o_latent`` bf16 ``[b, s_q, h, 512]`` (the
    decode's output), ``w_uv`` bf16 ``[h, 512, d]``; returns bf16 ``[b, s_q, h, d]``."""
    _need(o_latent, "o_latent", torch.bfloat16, 4)
    b, s_q, h, k = o_latent.shape
    if k != D_V or w_uv.dim() != 3 or tuple(w_uv.shape[:2]) != (h, D_V):
        raise ValueError("shapes: o_latent [b, s_q, h, 512], w_uv [h, 512, d]")
    d = w_uv.shape[2]
    if out is None:
        out = torch.empty((b, s_q, h, d), dtype=torch.bfloat16, device=o_latent.device)
    return head_gemm(o_latent, h * D_V, D_V, w_uv, out, h * d, d, b * s_q, d, D_V, h, stream)


def decode_fp8(q: torch.Tensor, kv_cache_fp8: torch.Tensor, block_table: torch.Tensor, seqlens: torch.Tensor,
               scale: float, kv_scale: float, causal: bool, meta: Metadata, out: torch.Tensor | None = None,
               lse: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None,
               phase: str = "both"):
    """MLA decode attention over an fp8 cache (``mla_decode_fp8``).

    ``kv_cache_fp8``: uint8 ``[num_blocks, 64, 1, 640]`` (or ``[num_blocks, 64, 640]``), per
    token 512 E4M3 latent bytes standing for ``kv_scale * e4m3(byte)``, then 64 bf16 rotary
    dims. Returns ``(out, lse)`` as :func:`decode`; ``phase`` as there.
    """
    kv = kv_cache_fp8
    _need(kv, "kv_cache_fp8", torch.uint8)
    if not ((kv.dim() == 4 and kv.shape[1:] == (BLOCK, 1, FP8_RECORD_BYTES)) or
            (kv.dim() == 3 and kv.shape[1:] == (BLOCK, FP8_RECORD_BYTES))):
        raise ValueError("kv_cache_fp8 must be uint8 [num_blocks, 64, 1, %d], got %s"
                         % (FP8_RECORD_BYTES, tuple(kv.shape)))
    b, s_q, h_q = _decode_args(q, None, block_table, seqlens, meta)
    out, lse, workspace, ws_bytes = _outputs(b, s_q, h_q, meta, q.device, out, lse, workspace)
    st = _stream(stream)
    L = lib()
    with torch.cuda.device(q.device):
        if phase in ("both", "split"):
            fn = L.mla_decode_fp8 if phase == "both" else L.mla_decode_split_fp8
            _check("mla_decode_fp8", fn(q.data_ptr(), kv.data_ptr(), kv.shape[0], float(kv_scale),
                                        block_table.data_ptr(), block_table.shape[1], seqlens.data_ptr(),
                                        meta.tile_meta.data_ptr(), meta.num_splits.data_ptr(), meta.num_parts, b,
                                        s_q, h_q, float(scale), int(bool(causal)), out.data_ptr(), lse.data_ptr(),
                                        workspace.data_ptr(), ws_bytes, st))
        elif phase == "combine":
            _check("mla_decode_combine", L.mla_decode_combine(meta.num_splits.data_ptr(), meta.num_parts, b, s_q,
                                                              h_q, out.data_ptr(), lse.data_ptr(),
                                                              workspace.data_ptr(), ws_bytes, st))
        else:
            raise ValueError(phase)
    return out, lse


def decode(q: torch.Tensor, kv_cache: torch.Tensor, block_table: torch.Tensor, seqlens: torch.Tensor,
           scale: float, causal: bool, meta: Metadata, out: torch.Tensor | None = None,
           lse: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None,
           phase: str = "both"):
    """MLA decode attention; returns ``(out bf16 [b, s_q, h_q, 512], lse fp32 [b, h_q, s_q])``.

    ``phase`` = "split" or "combine" runs one of the two kernels only (for timing each).
    """
    b, s_q, h_q = _decode_args(q, kv_cache, block_table, seqlens, meta)
    dev = q.device
    if out is None:
        out = torch.empty((b, s_q, h_q, D_V), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((b, h_q, s_q), dtype=torch.float32, device=dev)
    _need(out, "out", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    ws_bytes = workspace_bytes(b, s_q, h_q, meta.num_parts)
    if workspace is None:
        workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    if workspace.numel() * workspace.element_size() < ws_bytes:
        raise ValueError("workspace too small: need %d bytes" % ws_bytes)
    st = _stream(stream)
    L = lib()
    with torch.cuda.device(dev):
        if phase in ("both", "split"):
            fn = L.mla_decode if phase == "both" else L.mla_decode_split
            _check("mla_decode", fn(q.data_ptr(), kv_cache.data_ptr(), kv_cache.shape[0], block_table.data_ptr(),
                                    block_table.shape[1], seqlens.data_ptr(), meta.tile_meta.data_ptr(),
                                    meta.num_splits.data_ptr(), meta.num_parts, b, s_q, h_q, float(scale),
                                    int(bool(causal)), out.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
                                    ws_bytes, st))
        elif phase == "combine":
            _check("mla_decode_combine", L.mla_decode_combine(meta.num_splits.data_ptr(), meta.num_parts, b, s_q,
                                                              h_q, out.data_ptr(), lse.data_ptr(),
                                                              workspace.data_ptr(), ws_bytes, st))
        else:
            raise ValueError(phase)
    return out, lse


NOALLOC_SCRATCH_BYTES = 16 << 20  # MLA_NOALLOC_SCRATCH_BYTES in include/mla.h


def decode_noalloc(q: torch.Tensor, kv_cache: torch.Tensor, block_table: torch.Tensor, seqlens: torch.Tensor,
                   scale: float, causal: bool, meta: Metadata, out: torch.Tensor, lse: torch.Tensor, stream=None):
    """Decode through ``mla_decode_noalloc``: no workspace, no device allocation by the library.

    For callers that cannot allocate device memory at decode time (fixed memory pools, serving
    paths where a late allocation could fail or stall): the split partials go to the library's
    fixed scratch array (``NOALLOC_SCRATCH_BYTES``), shared by every call on the device, so calls
    must not overlap on the GPU. ``out`` and ``lse`` are caller-provided.
    """
    b, s_q, h_q = _decode_args(q, kv_cache, block_table, seqlens, meta)
    _need(out, "out", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    with torch.cuda.device(q.device):
        _check("mla_decode_noalloc", lib().mla_decode_noalloc(
            q.data_ptr(), kv_cache.data_ptr(), kv_cache.shape[0], block_table.data_ptr(), block_table.shape[1],
            seqlens.data_ptr(), meta.tile_meta.data_ptr(), meta.num_splits.data_ptr(), meta.num_parts, b, s_q, h_q,
            float(scale), int(bool(causal)), out.data_ptr(), lse.data_ptr(), _stream(stream)))
    return out, lse


class HostDecoder:
    """End-to-end decode on host buffers through ``mla_decode_host`` (copies in, runs, copies out).

    Device buffers are allocated once (by torch) for the largest shapes given.
    """

    def __init__(self, batch, s_q, h_q, num_blocks, bt_stride, device="cuda", num_parts=None, fixed_cost=None,
                 kv_scale=None):
        dev = torch.device(device)
        self.kv_scale = kv_scale  # not None: the fp8 cache (mla_decode_host_fp8)
        self.device = dev
        self.num_parts = num_parts or default_num_parts(h_q, s_q, dev)
        self.fixed_cost = default_fixed_cost(h_q, s_q) if fixed_cost is None else fixed_cost
        e = lambda shape, dt: torch.empty(shape, dtype=dt, device=dev)  # noqa: E731
        self.q = e((batch, s_q, h_q, D_QK), torch.bfloat16)
        self.kv = (e((num_blocks, BLOCK, 1, FP8_RECORD_BYTES), torch.uint8) if kv_scale is not None
                   else e((num_blocks, BLOCK, 1, D_QK), torch.bfloat16))
        self.bt = e((batch, bt_stride), torch.int32)
        self.sl = e((batch,), torch.int32)
        self.tm = e((self.num_parts, META_INTS), torch.int32)
        self.ns = e((batch + 1,), torch.int32)
        self.out = e((batch, s_q, h_q, D_V), torch.bfloat16)
        self.lse = e((batch, h_q, s_q), torch.float32)
        self.ws_bytes = workspace_bytes(batch, s_q, h_q, self.num_parts)
        self.ws = e((self.ws_bytes,), torch.uint8)
        self.buf = _DeviceBuffers(self.q.data_ptr(), self.kv.data_ptr(), self.bt.data_ptr(), self.sl.data_ptr(),
                                  self.tm.data_ptr(), self.ns.data_ptr(), self.out.data_ptr(), self.lse.data_ptr(),
                                  self.ws.data_ptr(), self.ws_bytes, self.num_parts, self.fixed_cost)

    def __call__(self, q, kv_cache, block_table, seqlens, scale, causal, out, lse, stream=None):
        """Host tensors in (pinned CPU torch tensors), host tensors out; synchronous."""
        for t, n in ((q, "q"), (kv_cache, "kv_cache"), (block_table, "block_table"), (seqlens, "seqlens"),
                     (out, "out"), (lse, "lse")):
            if t.is_cuda or not t.is_contiguous():
                raise ValueError("%s must be a contiguous host tensor" % n)
        b, s_q, h_q, _ = q.shape
        with torch.cuda.device(self.device):
            if self.kv_scale is not None:
                _check("mla_decode_host_fp8", lib().mla_decode_host_fp8(
                    q.data_ptr(), kv_cache.data_ptr(), kv_cache.shape[0], float(self.kv_scale), block_table.data_ptr(),
                    block_table.shape[1], seqlens.data_ptr(), b, s_q, h_q, float(scale), int(bool(causal)),
                    out.data_ptr(), lse.data_ptr(), ctypes.byref(self.buf), _stream(stream)))
            else:
                _check("mla_decode_host", lib().mla_decode_host(
                    q.data_ptr(), kv_cache.data_ptr(), kv_cache.shape[0], block_table.data_ptr(),
                    block_table.shape[1], seqlens.data_ptr(), b, s_q, h_q, float(scale), int(bool(causal)),
                    out.data_ptr(), lse.data_ptr(), ctypes.byref(self.buf), _stream(stream)))
        return out, lse


def check_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status (0 = OK)."""
    return lib().mla_check_status(_stream(stream))


def launch_count() -> int:
    """Kernels launched through the library by this process so far."""
    return int(lib().mla_launch_count())


def selftest_wait_timeout(spin_cycles: int, stream=None) -> None:
    """Run the kernels' bounded-wait primitive on an mbarrier nothing completes (see
    mla_selftest_wait_timeout): the next check_status() returns MLA_ERR_TIMEOUT."""
    _check("mla_selftest_wait_timeout", lib().mla_selftest_wait_timeout(int(spin_cycles), _stream(stream)))
