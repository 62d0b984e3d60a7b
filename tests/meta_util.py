"""Helpers for checking split-KV work partitions (test-side only)."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "metadata_hand_worked.txt")


def load_golden():
    """Parse the hand-worked partition fixture -> (seqlens, C, [(P, T, meta, cum)])."""
    seqlens, C, cases = None, None, []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("seqlens"):
                seqlens = [int(x) for x in line.split()[1:]]
            elif line.startswith("fixed_cost"):
                C = int(line.split()[1])
            elif line.startswith("case"):
                head, parts, cum = line.split("|")
                _, P, T = head.split()
                rows = [[int(x) for x in r.split()] for r in parts.split(";")]
                meta = np.zeros((int(P), 8), dtype=np.int32)
                meta[:, :5] = np.array(rows, dtype=np.int32)
                cases.append((int(P), int(T), meta, np.array([int(x) for x in cum.split()], np.int32)))
    return seqlens, C, cases


def pieces(tile_meta, num_blocks):
    """Walk every part the way the decode kernel does -> list of (part, seq, lo, hi, piece_idx)."""
    out = []
    for p, m in enumerate(np.asarray(tile_meta)):
        bs, bb, es, eb, first = (int(x) for x in m[:5])
        for s in range(bs, es + 1):
            lo = bb if s == bs else 0
            hi = eb if s == es else int(num_blocks[s])
            if hi > lo:
                out.append((p, s, lo, hi, first if s == bs else 0))
    return out


def check_partition(seqlens, tile_meta, cum, num_parts, fixed_cost):
    """Structural invariants every valid partition must satisfy (raises AssertionError)."""
    n = np.maximum(np.asarray(seqlens, dtype=np.int64), 0)
    w = (n + 63) // 64
    pcs = pieces(tile_meta, w)
    cover = [np.zeros(int(x), dtype=np.int32) for x in w]
    per_seq = [[] for _ in w]
    for p, s, lo, hi, idx in pcs:
        cover[s][lo:hi] += 1
        per_seq[s].append((p, lo, hi, idx))
    for s in range(len(w)):
        assert np.all(cover[s] == 1), "sequence %d not covered exactly once" % s
        got = per_seq[s]
        assert [x[3] for x in got] == list(range(len(got))), "piece indices of seq %d" % s
        assert [x[0] for x in got] == sorted(x[0] for x in got)
    cnt = np.array([len(x) for x in per_seq], dtype=np.int64)
    assert cum[0] == 0 and np.array_equal(np.diff(cum), cnt)
    assert cum[-1] <= len(w) + num_parts - 1 or cum[-1] == 0
    U = int(((w > 0) * fixed_cost + w).sum())
    T = max(1, -(-U // num_parts))
    work = np.zeros(num_parts, dtype=np.int64)
    for p, s, lo, hi, idx in pcs:
        work[p] += (hi - lo) + fixed_cost
    assert work.max(initial=0) <= T + fixed_cost
