// Walk over the segments of one KV chunk.
//
// The plan stage lays every sequence's 64-token tiles end to end
// (tile_prefix[b] = first tile of sequence b) and cuts that line into chunks
// of `cs` tiles.  A chunk can cover the tail of one sequence, some whole
// sequences and the head of another; each piece is a segment.  A segment
// that covers a whole sequence writes u/lse directly; otherwise it writes a
// partial row that the combine stage merges.  Every role of every CTA walks
// the same segments in the same order.
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
  int t, t_end, cs, chunk, b;

  __device__ __forceinline__ void init(const int* tile_prefix, int nseq, int chunk_id, int chunk_size) {
    tp = tile_prefix;
    B = nseq;
    cs = chunk_size;
    chunk = chunk_id;
    const int T = tp[B];
    t = min(chunk_id * cs, T);
    t_end = min(t + cs, T);
    // largest b with tp[b] <= t
    int lo = 0, hi = B;  // invariant: tp[lo] <= t
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (tp[mid] <= t) lo = mid; else hi = mid;
    }
    b = lo;
  }

  __device__ __forceinline__ bool next(Segment& s) {
    while (b < B && tp[b + 1] <= t) ++b;  // skip sequences that end at or before t
    if (t >= t_end || b >= B) return false;
    const int begin = tp[b], end = tp[b + 1];
    const int stop = min(t_end, end);
    s.b = b;
    s.t0 = t - begin;
    s.t1 = stop - begin;
    s.whole = (t == begin && stop == end) ? 1 : 0;
    s.part = chunk - begin / cs;
    t = stop;
    return true;
  }
};

}  // namespace mla
