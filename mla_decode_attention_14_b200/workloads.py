"""Seeded synthetic inputs for MLA decode attention (shared by tests, bench and oracle runs).

This module holds no arithmetic of the attention method: it only draws the inputs
(queries, a paged latent KV cache, block tables and sequence lengths) with a fixed
seed, so that the CUDA path and the CPU oracle see bit-identical data.

Recipe (the same for every workload):
  * q and every cache element ~ N(0, 1) drawn as float32 by numpy's PCG64 generator,
    then rounded to bf16 (round to nearest, ties to even);
  * sequence i has w_i = ceil(n_i / 64) blocks [64-token blocks: "Deep analysis of
    the DeepSeek Infra open-source releases", DAY1 FlashMLA, feature (2)]; the
    physical blocks are a seeded random permutation of [0, sum w_i), so a sequence's
    blocks are scattered over the cache; unused block-table entries are -1;
  * cache rows past a sequence's length inside its last block ("tail") are NaN for
    parity runs (they must not influence the result) or N(0, 1) for timing runs;
  * scale = 192 ** -0.5 for every workload.

fp8 cache (``make_inputs_fp8``): the same q, block table and tails; per token a 640-byte
record of 512 latent dims as OCP E4M3 bytes -- N(0, 1) float32 times 64, clipped to +-448
and rounded to E4M3 (nearest, ties to even, by torch's float8_e4m3fn cast) -- followed by
the 64 rotary dims as bf16 N(0, 1). The cache's latent scale (default 2^-6, which makes
the latent values ~N(0, 1)) does not change the codes.

Workloads (sizes as named by the library's benchmark list):
  tiny        b=2,   h_q=16,  s_q=1, seqlens {100, 257}
  v2lite      b=64,  h_q=16,  s_q=1, every seqlen 4096      (DeepSeek-V2-Lite head count)
  v3          b=128, h_q=128, s_q=1, seqlens uniform in [1024, 8192]  (DeepSeek-V3 head count)
  multitoken  b=64,  h_q=128, s_q=2, causal, every seqlen 16384
  skewed      b=32,  h_q=64,  s_q=1, lognormal(median 2048, sigma 1.5) rounded and clipped
              to [1, 65536], sequence 0 forced to 65536
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

D_QK = 576
D_V = 512
BLK = 64
SCALE = 192.0 ** -0.5
BF16_NAN = 0x7FC0
F8_REC = 640            # fp8 cache: bytes per token (512 E4M3 latent + 64 bf16 rotary)
F8_NAN = 0x7F           # an E4M3 NaN
F8_SCALE = 2.0 ** -6    # default latent scale of the synthetic fp8 cache


@dataclass
class Workload:
    name: str
    batch: int
    h_q: int
    s_q: int
    causal: bool
    seqlens: np.ndarray           # int32 [batch]
    scale: float = SCALE
    extra: dict = field(default_factory=dict)

    @property
    def rows(self) -> int:
        return self.s_q * self.h_q


def _seqlens(name: str, rng: np.random.Generator) -> np.ndarray:
    if name == "tiny":
        return np.array([100, 257], dtype=np.int32)
    if name == "v2lite":
        return np.full(64, 4096, dtype=np.int32)
    if name == "v3":
        return rng.integers(1024, 8192, size=128, endpoint=True).astype(np.int32)
    if name == "multitoken":
        return np.full(64, 16384, dtype=np.int32)
    if name == "skewed":
        x = np.rint(rng.lognormal(mean=math.log(2048.0), sigma=1.5, size=32))
        x = np.clip(x, 1, 65536).astype(np.int32)
        x[0] = 65536
        return x
    raise KeyError(name)


_SHAPES = {
    "tiny": (2, 16, 1, False),
    "v2lite": (64, 16, 1, False),
    "v3": (128, 128, 1, False),
    "multitoken": (64, 128, 2, True),
    "skewed": (32, 64, 1, False),
}

NAMES = tuple(_SHAPES)


def workload(name: str, seed: int = 0) -> Workload:
    """Shape and sequence lengths of a named workload (no tensors drawn)."""
    b, h, s, causal = _SHAPES[name]
    rng = np.random.default_rng([seed, 1])
    return Workload(name, b, h, s, causal, _seqlens(name, rng))


def custom(batch: int, h_q: int, s_q: int, seqlens, causal: bool = False,
           scale: float = SCALE, name: str = "custom") -> Workload:
    sl = np.asarray(seqlens, dtype=np.int32).reshape(-1)
    assert sl.shape[0] == batch
    return Workload(name, batch, h_q, s_q, causal, sl, scale)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(rng: np.random.Generator, shape, chunk: int = 1 << 24) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for lo in range(0, n, chunk):
        hi = min(n, lo + chunk)
        out[lo:hi] = f32_to_bf16_bits(rng.standard_normal(hi - lo, dtype=np.float32))
    return out.reshape(shape)


def block_layout(seqlens: np.ndarray, rng: np.random.Generator, spare_blocks: int = 0):
    """Scattered block table: returns (block_table int32[b, max_w], num_blocks)."""
    n = np.maximum(seqlens.astype(np.int64), 0)
    w = (n + BLK - 1) // BLK
    total = int(w.sum())
    num_blocks = total + spare_blocks
    perm = rng.permutation(num_blocks)[:total].astype(np.int32)
    max_w = max(1, int(w.max()) if w.size else 1)
    bt = np.full((seqlens.shape[0], max_w), -1, dtype=np.int32)
    off = 0
    for i, wi in enumerate(w):
        bt[i, :wi] = perm[off:off + wi]
        off += wi
    return bt, num_blocks


def make_inputs(wl: Workload, seed: int = 0, tail: str = "nan", spare_blocks: int = 0):
    """Draw q, the paged cache and the block table for ``wl``.

    Returns a dict of numpy arrays: ``q`` uint16 [b, s_q, h_q, 576] (bf16 bits),
    ``kv`` uint16 [num_blocks, 64, 1, 576], ``block_table`` int32 [b, max_blocks],
    ``seqlens`` int32 [b], plus ``scale``, ``causal``, ``num_blocks``.
    """
    rng = np.random.default_rng([seed, 2])
    bt, nblk = block_layout(wl.seqlens, rng, spare_blocks)
    q = _normal_bf16(rng, (wl.batch, wl.s_q, wl.h_q, D_QK))
    kv = _normal_bf16(rng, (max(nblk, 1), BLK, 1, D_QK))
    if tail == "nan":
        for i, n in enumerate(wl.seqlens):
            n = int(n)
            w = (max(n, 0) + BLK - 1) // BLK
            if w > 0 and n % BLK:
                kv[bt[i, w - 1], n % BLK:, :, :] = BF16_NAN
    elif tail != "normal":
        raise ValueError(tail)
    return {"q": q, "kv": kv, "block_table": bt, "seqlens": wl.seqlens.copy(),
            "scale": wl.scale, "causal": wl.causal, "num_blocks": nblk}


def _e4m3_codes(x: np.ndarray) -> np.ndarray:
    import torch
    t = torch.from_numpy(np.clip(x, -448.0, 448.0).astype(np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def make_inputs_fp8(wl: Workload, seed: int = 0, tail: str = "nan", spare_blocks: int = 0,
                    kv_scale: float = F8_SCALE, chunk_tokens: int = 1 << 16):
    """Draw q, an fp8 paged cache and the block table for ``wl``.

    Returns a dict with ``q`` uint16 [b, s_q, h_q, 576] (bf16 bits), ``kv8`` uint8
    [num_blocks, 64, 1, 640] (per token 512 E4M3 bytes then 64 bf16 little-endian),
    ``kv_scale`` (a latent byte x stands for kv_scale * e4m3(x)), ``block_table``,
    ``seqlens``, ``scale``, ``causal``, ``num_blocks``.
    """
    rng = np.random.default_rng([seed, 3])
    bt, nblk = block_layout(wl.seqlens, rng, spare_blocks)
    q = _normal_bf16(rng, (wl.batch, wl.s_q, wl.h_q, D_QK))
    ntok = max(nblk, 1) * BLK
    kv8 = np.empty((ntok, F8_REC), dtype=np.uint8)
    for lo in range(0, ntok, chunk_tokens):
        hi = min(ntok, lo + chunk_tokens)
        lat = rng.standard_normal((hi - lo, D_V), dtype=np.float32) * np.float32(64.0)
        kv8[lo:hi, :D_V] = _e4m3_codes(lat)
        rope = f32_to_bf16_bits(rng.standard_normal((hi - lo, D_QK - D_V), dtype=np.float32))
        kv8[lo:hi, D_V:] = np.ascontiguousarray(rope.astype("<u2")).view(np.uint8).reshape(hi - lo, -1)
    kv8 = kv8.reshape(max(nblk, 1), BLK, 1, F8_REC)
    if tail == "nan":
        nan_rope = np.frombuffer(np.array([BF16_NAN], dtype="<u2").tobytes() * (D_QK - D_V), dtype=np.uint8)
        for i, n in enumerate(wl.seqlens):
            n = int(n)
            w = (max(n, 0) + BLK - 1) // BLK
            if w > 0 and n % BLK:
                blk = kv8[bt[i, w - 1], n % BLK:, 0, :]
                blk[:, :D_V] = F8_NAN
                blk[:, D_V:] = nan_rope
    elif tail != "normal":
        raise ValueError(tail)
    return {"q": q, "kv8": kv8, "kv_scale": float(kv_scale), "block_table": bt, "seqlens": wl.seqlens.copy(),
            "scale": wl.scale, "causal": wl.causal, "num_blocks": nblk}


def sparse_indices(seqlens, s_q: int, topk: int, seed: int = 0, order: str = "sorted") -> np.ndarray:
    """Index lists for sparse decode: int32 [b, s_q, topk] positions within each sequence.

    Each (sequence, query token) draws ``min(topk, n)`` distinct positions of its sequence
    uniformly; lists longer than the sequence are padded with -1 (no key). ``order``: "sorted"
    (ascending positions) or "shuffled".
    """
    sl = np.asarray(seqlens, dtype=np.int64)
    rng = np.random.default_rng([seed, 4])
    out = np.full((sl.shape[0], s_q, topk), -1, dtype=np.int32)
    for b, n in enumerate(sl):
        n = max(int(n), 0)
        k = min(topk, n)
        for t in range(s_q):
            if k == 0:
                continue
            pos = rng.choice(n, size=k, replace=False) if k < n else np.arange(n)
            if order == "sorted":
                pos = np.sort(pos)
            elif order == "shuffled":
                pos = rng.permutation(pos)
            else:
                raise ValueError(order)
            out[b, t, :k] = pos
    return out


def sparse_counts(wl: Workload, indices: np.ndarray):
    """Algorithmic bytes and flops of one sparse decode: 1152 bytes per listed key that is a key
    (a position inside its sequence) plus 1152 per query row; 2 * (576 + 512) flops per (key, row)."""
    n = np.maximum(wl.seqlens.astype(np.int64), 0)
    ix = np.asarray(indices)
    keys = int(((ix >= 0) & (ix < n[:, None, None])).sum())
    kv_bytes = keys * D_QK * 2
    q_bytes = wl.batch * wl.rows * D_QK * 2
    return {"kv_bytes": kv_bytes, "q_bytes": q_bytes, "bytes": kv_bytes + q_bytes,
            "flops": keys * wl.h_q * 2 * (D_QK + D_V)}


def algorithmic_counts(wl: Workload, kv: str = "bf16"):
    """Algorithmic bytes and flops of one decode of ``wl``.

    bytes = 1152 per KV token (576 bf16, keys and values share the vector; 640 for the
    fp8 cache) plus 1152 per query row; flops = 2 * (576 + 512) per (visible key, query row).
    """
    n = np.maximum(wl.seqlens.astype(np.int64), 0)
    kv_bytes = int(n.sum()) * (F8_REC if kv == "fp8" else D_QK * 2)
    q_bytes = wl.batch * wl.rows * D_QK * 2
    vis = 0
    for t in range(wl.s_q):
        if wl.causal:
            v = np.clip(n - wl.s_q + t + 1, 0, n)
        else:
            v = n
        vis += int(v.sum()) * wl.h_q
    flops = vis * 2 * (D_QK + D_V)
    return {"kv_bytes": kv_bytes, "q_bytes": q_bytes, "bytes": kv_bytes + q_bytes, "flops": flops}
