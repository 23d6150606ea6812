// Walk over the segments of one KV chunk.
//
// The plan stage lays every sequence's 64-token tiles end to end
// (tile_prefix[b] = first tile of sequence b) and cuts that line into chunks;
// chunk c holds tiles [chunk_t[c], chunk_t[c + 1]) (the plan kernel says how
// the cuts are placed).  A chunk can cover the tail of one sequence, some
// whole sequences and the head of another; each piece is a segment, and the
// pieces of a sequence are numbered in tile order.  A segment that covers a whole sequence
// writes u/lse directly; otherwise it writes a partial row that the combine
// stage merges.  Every role of every CTA walks the same segments in the same
// order.
#pragma once

namespace mla {

struct Segment {
  int b;       // sequence
  int t0, t1;  // tiles [t0, t1) of that sequence
  int whole;   // covers every tile of the sequence
  int part;    // index of this piece among the sequence's pieces
};

struct ChunkWalk {
  const int* tp;  // tile_prefix, B + 1 entries
  int B;
  int t, t_end, b;
  int part0;  // piece index of the chunk's first segment

  // chunk_t / chunk_b come from the plan stage; the reads are independent
  // (one memory round trip)
  __device__ __forceinline__ void init(const int* tile_prefix, const int* chunk_t,
                                       const int* chunk_b, const int* header, int nseq,
                                       int chunk_id) {
    (void)header;
    tp = tile_prefix;
    B = nseq;
    t = chunk_t[chunk_id];
    t_end = chunk_t[chunk_id + 1];
    b = chunk_b[2 * chunk_id];
    part0 = chunk_b[2 * chunk_id + 1];
  }

  __device__ __forceinline__ bool next(Segment& s) {
    if (t >= t_end) return false;
    while (b < B && tp[b + 1] <= t) ++b;  // skip sequences that end at or before t
    if (b >= B) return false;
    const int begin = tp[b], end = tp[b + 1];
    const int stop = min(t_end, end);
    s.b = b;
    s.t0 = t - begin;
    s.t1 = stop - begin;
    s.whole = (t == begin && stop == end) ? 1 : 0;
    // a later segment of the chunk starts its sequence: piece 0
    s.part = t == begin ? 0 : part0;
    t = stop;
    return true;
  }
};

}  // namespace mla
