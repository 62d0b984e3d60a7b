// schedule.cuh -- the walk over one work part that every role of the split kernels takes.
//
// A part is a contiguous run of (sequence, 64-token block) work units cut by the length-aware
// partition ("Deep analysis of the DeepSeek Infra open-source releases", DAY1 FlashMLA,
// feature (5)): tile_meta gives its first and last sequence and block. Each role of a kernel
// walks the same list on its own, so the roles agree on every piece without talking.
#pragma once

#include "common.cuh"

namespace mla {

// One piece: the blocks [lo, hi) of sequence `seq` (n tokens) that this part computes.
// nsplit = pieces of that sequence over all parts; slot = this piece's workspace slot.
struct Piece {
    int seq, lo, hi, n, nsplit, slot;
};

// Walks the non-empty pieces of one part (all roles walk the same list independently).
// SP: sparse mode, where every work unit has topk keys (its index list).
template <bool SP = false>
struct Cursor {
    int seq, begin_seq, begin_blk, end_seq, end_blk, first_piece;
    __device__ void init(const int32_t *meta, int batch) {
        begin_seq = meta[0];
        begin_blk = meta[1];
        end_seq = meta[2];
        end_blk = meta[3];
        first_piece = meta[4];
        if (end_seq >= begin_seq && (begin_seq < 0 || end_seq >= batch)) end_seq = begin_seq - 1;  // malformed
        seq = begin_seq;
    }
    __device__ bool next(const DecodeParams &p, Piece &pc) {
        while (seq <= end_seq) {
            const int s = seq++;
            const int n = SP ? p.topk : max(p.seqlens[s], 0);
            const int w = num_blocks_of(n);
            const int lo = s == begin_seq ? max(begin_blk, 0) : 0;
            const int hi = s == end_seq ? min(end_blk, w) : w;
            if (hi <= lo) continue;
            pc.seq = s;
            pc.lo = lo;
            pc.hi = hi;
            pc.n = n;
            pc.nsplit = p.num_splits[s + 1] - p.num_splits[s];
            pc.slot = p.num_splits[s] + (s == begin_seq ? first_piece : 0);
            if (pc.nsplit > 1 && (pc.slot < 0 || pc.slot >= p.batch + p.num_parts)) continue;  // malformed
            return true;
        }
        return false;
    }
};


}  // namespace mla
