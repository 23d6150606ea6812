// Walk over the segments of one KV chunk.
//
// The plan stage lays every sequence's 64-token tiles end to end
// (tile_prefix[b] = first tile of sequence b) and cuts that line into chunks;
// chunk c holds tiles [chunk_t[c], chunk_t[c + 1]).  The cuts are uniform on
// a line where every sequence takes K units of start-up cost before its tiles
// (units [tile_prefix[b] + K b, tile_prefix[b] + K (b + 1))), so tile t of
// sequence b sits at unit t + K (b + 1) and lies in chunk
// (t + K (b + 1)) / units_per_chunk.  A chunk
// can cover the tail of one sequence, some whole sequences and the head of
// another; each piece is a segment.  A segment that covers a whole sequence
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
  int t, t_end, chunk, b;
  int units, K;  // line units per chunk, units per sequence start

  // chunk_t / chunk_b / header come from the plan stage; the three reads are
  // independent (one memory round trip)
  __device__ __forceinline__ void init(const int* tile_prefix, const int* chunk_t,
                                       const int* chunk_b, const int* header, int nseq,
                                       int chunk_id) {
    tp = tile_prefix;
    B = nseq;
    chunk = chunk_id;
    t = chunk_t[chunk_id];
    t_end = chunk_t[chunk_id + 1];
    b = chunk_b[chunk_id];
    units = header[1];
    K = header[4];
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
    // pieces of sequence b are numbered from the chunk holding its first tile
    s.part = chunk - (int)(((long long)begin + (long long)K * (b + 1)) / units);
    t = stop;
    return true;
  }
};

}  // namespace mla
