"""CPU checks of the fp8 path's design arithmetic (no GPU), restated from the kernel's comments:

* the E4M3 byte placed as the fp16 bit pattern s.0eeee.mmm0000000 is the fp16 number e4m3 * 2^-8,
  for every code (checked against the oracle's E4M3 decoding);
* the converter warps' lane mapping reads every 16-byte chunk of the two raw boxes once, writes
  every chunk of the four fp16 boxes once at the address the 128-byte swizzle gives the dims it
  holds, and each 8-lane group touches 8 distinct bank groups;
* the in-place expansion (raw box 0 in fp16 box 2's place, raw box 1 in box 3's, a barrier between)
  gives the direct conversion under any interleaving of the four warps' steps.
"""
import numpy as np

import oracle

BOX = 8192  # 64 rows x 128 bytes


def _expand_pair(w, sel):
    """Two E4M3 bytes of w (chosen by the byte permute `sel`) -> two fp16 bit patterns."""
    src = [(w >> (8 * i)) & 255 for i in range(4)] + [0] * 4
    t = 0
    for i in range(4):
        t |= src[(sel >> (4 * i)) & 7] << (8 * i)
    return (t & 0x80008000) | ((t & 0x7F007F00) >> 1)


def test_fp16_pattern_is_e4m3_times_2_to_minus_8():
    codes = np.arange(256, dtype=np.uint8)
    ref = oracle.e4m3_decode(codes)
    for pos, sel in ((0, 0x1404), (1, 0x1404), (2, 0x3424), (3, 0x3424)):
        for c in range(256):
            if np.isnan(ref[c]):
                continue
            r = _expand_pair(c << (8 * pos), sel)
            h = np.array([(r >> (16 * (pos & 1))) & 0xFFFF], dtype=np.uint16).view(np.float16)[0]
            assert float(h) * 256.0 == ref[c], (c, pos)


def _lane_map(it, lane):
    u, hp, pq = lane & 7, (lane >> 3) & 1, lane >> 4
    pi = 2 * it + pq
    bx, row = pi >> 5, 2 * (pi & 31) + ((u >> 2) ^ hp)
    sw, k0 = row & 7, 2 * (u & 3)
    src = (2 + bx) * BOX + row * 128 + ((u ^ sw) << 4)
    out = (2 * bx + (u >> 2)) * BOX + row * 128
    return bx, row, u, src, (out + ((k0 ^ sw) << 4), out + (((k0 + 1) ^ sw) << 4))


def test_lane_mapping_covers_every_chunk_once_without_bank_conflicts():
    seen_src, seen_dst = set(), set()
    for it in range(32):
        groups = {}
        for lane in range(32):
            bx, row, u, src, dst = _lane_map(it, lane)
            assert src not in seen_src
            seen_src.add(src)
            dim0 = 128 * bx + 16 * u  # first latent dim of the chunk (this CTA's half)
            for d, a in ((dim0, dst[0]), (dim0 + 8, dst[1])):
                expect = (d // 64) * BOX + row * 128 + ((((d % 64) // 8) ^ (row & 7)) << 4)
                assert a == expect
                assert a not in seen_dst
                seen_dst.add(a)
            groups.setdefault(lane >> 3, []).append((src, dst[0], dst[1]))
        for g in groups.values():
            for i in range(3):
                assert len({(x[i] % 128) // 16 for x in g}) == 8
    assert len(seen_src) == 2 * 64 * 8 and len(seen_dst) == 4 * 64 * 8


def test_in_place_expansion_under_random_interleavings():
    rng = np.random.default_rng(0)
    for trial in range(12):
        valid = 64 if trial % 2 == 0 else int(rng.integers(1, 64))
        raw = [rng.integers(0, 256, (64, 128)).astype(np.uint8) for _ in range(2)]
        stage = bytearray(5 * BOX)
        for bx in range(2):  # the TMA's 128-byte-swizzled placement of the raw boxes
            for row in range(64):
                for u in range(8):
                    a = (2 + bx) * BOX + row * 128 + ((u ^ (row & 7)) << 4)
                    stage[a:a + 16] = bytes(raw[bx][row, 16 * u:16 * u + 16])
        for bx in range(2):  # the barrier of the four warps separates the two boxes
            progs = {cw: list(range(16 * bx + cw, 16 * bx + 16, 4)) for cw in range(4)}
            while any(progs.values()):
                cw = int(rng.choice([c for c in range(4) if progs[c]]))
                it = progs[cw].pop(0)
                writes = []
                for lane in range(32):  # one step: every lane reads, then every lane writes
                    _, row, u, src, dst = _lane_map(it, lane)
                    if row < valid:
                        x = [int.from_bytes(stage[src + 4 * i:src + 4 * i + 4], "little") for i in range(4)]
                        lo = [_expand_pair(x[i // 2], 0x1404 if i % 2 == 0 else 0x3424) for i in range(4)]
                        hi = [_expand_pair(x[2 + i // 2], 0x1404 if i % 2 == 0 else 0x3424) for i in range(4)]
                    else:
                        lo = hi = [0, 0, 0, 0]
                    writes += [(dst[0], lo), (dst[1], hi)]
                for a, words in writes:
                    for i, wd in enumerate(words):
                        stage[a + 4 * i:a + 4 * i + 4] = int(wd).to_bytes(4, "little")
        for bx in range(2):  # compare with the direct conversion
            for row in range(64):
                for d in range(128):
                    dim = 128 * bx + d
                    a = (dim // 64) * BOX + row * 128 + ((((dim % 64) // 8) ^ (row & 7)) << 4) + 2 * (dim % 8)
                    want = _expand_pair(int(raw[bx][row, d]), 0x1404) & 0xFFFF if row < valid else 0
                    assert int.from_bytes(stage[a:a + 2], "little") == want
