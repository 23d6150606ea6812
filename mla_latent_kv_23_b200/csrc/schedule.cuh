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
  int part0;            // piece index of the chunk's first segment
  int b0_begin, b0_end; // tiles [b0_begin, b0_end) of the line: the first segment's sequence

  // chunk_t and the chunk's record (sequence, piece, and that sequence's
  // first and end tile on the line) come from the plan stage; the reads are
  // independent (one memory round trip), and the first segment needs no
  // read of the tile prefix
  __device__ __forceinline__ void init(const int* tile_prefix, const int* chunk_t,
                                       const int* chunk_b, const int* header, int nseq,
                                       int chunk_id) {
    (void)header;
    tp = tile_prefix;
    B = nseq;
    t = chunk_t[chunk_id];
    t_end = chunk_t[chunk_id + 1];
    const int4 r = *reinterpret_cast<const int4*>(chunk_b + 4 * chunk_id);
    b = r.x;
    part0 = r.y;
    b0_begin = r.z;
    b0_end = r.w;
  }

  __device__ __forceinline__ bool next(Segment& s) {
    if (t >= t_end) return false;
    int begin, end;
    if (b < B && t >= b0_begin && t < b0_end) {  // still inside the first segment's sequence
      begin = b0_begin;
      end = b0_end;
    } else {
      while (b < B && tp[b + 1] <= t) ++b;  // skip sequences that end at or before t
      if (b >= B) return false;
      begin = tp[b];
      end = tp[b + 1];
    }
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
