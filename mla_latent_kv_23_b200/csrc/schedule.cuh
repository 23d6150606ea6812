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

#include "internal.h"

namespace mla {

struct Segment {
  int b;       // sequence
  int t0, t1;  // tiles [t0, t1) of that sequence
  int whole;   // covers every tile of the sequence
  int part;    // index of this piece among the sequence's pieces
  int split_base;  // first partial row of the sequence (SeqWalk only)
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

// ---------------------------------------------------------------- self plan
// The same cut computed by a kernel for its own chunk from the sequence
// lengths, so that no plan stage has to run first.  tiles(b) = ceil(L_b / 64)
// for a valid length (s_q <= L_b <= max_len), else 0.
__device__ __forceinline__ int seq_tiles(const int* seqlens, int b, int s_q, int max_len) {
  const int L = seqlens[b];
  return (L < s_q || L > max_len) ? 0 : (L + kTileTokens - 1) / kTileTokens;
}

// pieces sequence b is cut into when it is split (0 when one chunk holds it)
__device__ __forceinline__ int seq_pieces(int tp_b, int tiles, int b, int K, int units) {
  if (tiles <= 0) return 0;
  const long long u0 = (long long)tp_b + (long long)K * (b + 1);
  const int n = (int)((u0 + tiles - 1) / units - u0 / units) + 1;
  return n > 1 ? n : 0;
}

// Where chunk `chunk` of `num_chunks` starts and ends on the cost line, and
// the prefix values (first tile, first partial row) of its first sequence.
struct ChunkStart {
  int t, t_end;   // tiles [t, t_end) of the batch's tile line
  int b;          // sequence of tile t
  int tp_b;       // first tile of sequence b
  int sb_b;       // first partial row of sequence b
  int units, K;
};

// One warp computes the chunk's start (every lane returns it).  With
// `out_tp` / `out_sb` non-null the warp also writes the whole tile prefix and
// split bases ([B + 1] each), as the plan stage does, for the stage that
// merges the partials; with `err` non-null it flags invalid lengths.
__device__ __forceinline__ ChunkStart plan_chunk(const int* seqlens, int B, int s_q, int max_len,
                                                 int num_chunks, int chunk, int* out_tp,
                                                 int* out_sb, int* err) {
  const int lane = threadIdx.x & 31;
  constexpr int K = kSegCostTiles;
  // total tiles
  int T = 0;
  for (int base = 0; base < B; base += 32) {
    int x = base + lane < B ? seq_tiles(seqlens, base + lane, s_q, max_len) : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    T += x;
  }
  const long long V = (long long)T + (long long)K * B;
  const int units = V > 0 ? (int)((V + num_chunks - 1) / num_chunks) : 1;
  const long long x0 = (long long)chunk * units, x1 = (long long)(chunk + 1) * units;
  // prefixes; the last sequence whose start unit tp + K b is <= x0 (x1)
  int tp_carry = 0, sb_carry = 0;
  int b0 = 0, tp0 = 0, sb0 = 0, b1 = 0, tp1 = 0;
  for (int base = 0; base < B; base += 32) {
    const int b = base + lane;
    const int tiles = b < B ? seq_tiles(seqlens, b, s_q, max_len) : 0;
    if (err != nullptr && b < B && tiles == 0) atomicOr(err, MLA_DEVFLAG_BAD_SEQLEN);
    int incl = tiles;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int tp_b = tp_carry + incl - tiles;
    const int pieces = b < B ? seq_pieces(tp_b, tiles, b, K, units) : 0;
    int pincl = pieces;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, pincl, o);
      if (lane >= o) pincl += y;
    }
    const int sb_b = sb_carry + pincl - pieces;
    if (out_tp != nullptr && b < B) {
      out_tp[b] = tp_b;
      out_sb[b] = sb_b;
    }
    const long long start = (long long)tp_b + (long long)K * b;
    const unsigned m0 = __ballot_sync(0xffffffffu, b < B && start <= x0);
    const unsigned m1 = __ballot_sync(0xffffffffu, b < B && start <= x1);
    if (m0) {
      const int src = 31 - __clz(m0);
      b0 = base + src;
      tp0 = __shfl_sync(0xffffffffu, tp_b, src);
      sb0 = __shfl_sync(0xffffffffu, sb_b, src);
    }
    if (m1) {
      const int src = 31 - __clz(m1);
      b1 = base + src;
      tp1 = __shfl_sync(0xffffffffu, tp_b, src);
    }
    tp_carry = __shfl_sync(0xffffffffu, tp_carry + incl, 31);
    sb_carry = __shfl_sync(0xffffffffu, sb_carry + pincl, 31);
  }
  if (out_tp != nullptr && lane == 0) {
    out_tp[B] = T;
    out_sb[B] = sb_carry;
  }
  ChunkStart cs;
  cs.units = units;
  cs.K = K;
  if (x0 < V) {
    const long long off = x0 - ((long long)tp0 + (long long)K * (b0 + 1));
    cs.t = tp0 + (off > 0 ? (int)off : 0);
    cs.b = b0;
    cs.tp_b = tp0;
    cs.sb_b = sb0;
  } else {
    cs.t = T;
    cs.b = B;
    cs.tp_b = T;
    cs.sb_b = sb_carry;
  }
  if (x1 < V) {
    const long long off = x1 - ((long long)tp1 + (long long)K * (b1 + 1));
    cs.t_end = tp1 + (off > 0 ? (int)off : 0);
  } else {
    cs.t_end = T;
  }
  return cs;
}

// Walk over a chunk's segments from its ChunkStart, reading the lengths of
// the sequences it reaches (the same pieces as ChunkWalk).
struct SeqWalk {
  const int* seqlens;
  int B, s_q, max_len;
  int t, t_end, b, tp_b, tp_next, sb_b, units, K, chunk;

  __device__ __forceinline__ void init(const ChunkStart& cs, const int* lens, int nseq, int sq,
                                       int maxl, int chunk_id) {
    seqlens = lens;
    B = nseq;
    s_q = sq;
    max_len = maxl;
    t = cs.t;
    t_end = cs.t_end;
    b = cs.b;
    tp_b = cs.tp_b;
    sb_b = cs.sb_b;
    units = cs.units;
    K = cs.K;
    chunk = chunk_id;
    tp_next = b < B ? tp_b + seq_tiles(seqlens, b, s_q, max_len) : tp_b;
  }

  __device__ __forceinline__ bool next(Segment& s) {
    if (t >= t_end) return false;
    while (b < B && tp_next <= t) {  // sequences that end at or before t
      sb_b += seq_pieces(tp_b, tp_next - tp_b, b, K, units);
      tp_b = tp_next;
      ++b;
      if (b < B) tp_next = tp_b + seq_tiles(seqlens, b, s_q, max_len);
    }
    if (b >= B) return false;
    const int stop = min(t_end, tp_next);
    s.b = b;
    s.t0 = t - tp_b;
    s.t1 = stop - tp_b;
    s.whole = (t == tp_b && stop == tp_next) ? 1 : 0;
    s.part = chunk - (int)(((long long)tp_b + (long long)K * (b + 1)) / units);
    s.split_base = sb_b;
    t = stop;
    return true;
  }
};

}  // namespace mla
