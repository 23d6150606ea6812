// Attend stage on the 5th-generation tensor cores (sm_100a), for n_h <= 128
// heads, latent d_c = 512, RoPE key d_R = 64, bf16.
//
// Math ("MLA deep compression", absorption section, both equations, and its
// decoupled-RoPE section): all heads of one query row share every cached row
// [c || k^R], so the heads are the M dimension of two dense contractions per
// 64-token tile,
//     S = Q . [C || K^R]^T      (K = 576)
//     O = O * alpha + P . C     (N = 512 latent)
// with an online softmax between them; u = O / l at the end.
//
// A pair of CTAs (one 2-CTA cluster) shares every tile, and all tensor-core
// work is paired (tcgen05 cta_group::2, issued by the even CTA):
//  * Loads are split by columns.  CTA r loads, for every cached row, latent
//    columns [128r, 128r + 128) and [256 + 128r, 256 + 128r + 128) plus RoPE
//    columns [32r, 32r + 32): 288 of the 576 values, so each cache byte is
//    read from HBM by exactly one SM and never re-read.
//  * Output rows are split by heads: CTA r owns heads [64r, 64r + 64) and
//    holds their O (64 heads x 512 latent, fp32) in its TMEM.
//  * P . C is one paired MMA per 16 tokens and 256 latent columns
//    (M = 128: 64 P rows from each CTA; N = 256: each CTA supplies the 128 of
//    those columns it loaded).  The pair's tensor cores move the B halves
//    between the SMs, so no latent data crosses shared memory.
//  * S needs all 576 columns of a row, but each CTA holds only half of them.
//    A paired MMA with M = 256, N = 128 computes, in CTA r, rows
//    (head h, half j) = Q[h, columns of CTA j] against B = [CTA 0's columns of
//    the 64 tokens | CTA 1's columns of the same tokens].  Row (h, j) is
//    meaningful against CTA j's half of N, so TMEM lane (h, 0) holds the
//    partial score over CTA 0's columns and lane (h, 1) the partial over
//    CTA 1's columns; the other half of each row is discarded.  Lanes are
//    ordered (32q + 16j + i) <-> head 16q + i, so the two partials of a head
//    sit 16 lanes apart in one warp and one shuffle adds them.  Half of the
//    S arithmetic is thrown away; in exchange nothing but barrier arrivals
//    passes between the CTAs.
//
// TMEM per CTA (512 columns): S 2 x 128 (double-buffered) | O 256.
// Shared memory per CTA: Q (128 rows x 288 values, the S operand A) 72 KB;
// 4 tile stages of 36 KB; P (64 heads x 64 tokens bf16) as two 32-token
// halves with 64-byte swizzle: tokens 0-31 in the tile's own RoPE block (free
// once S of the tile is done, and held until its P . C releases the stage),
// tokens 32-63 in a two-slot 4 KB ring.
// One shared-memory copy of a tile serves both contractions: a TMA load with
// 128-byte swizzle writes each 64-column block as 64 rows x 128 B, the
// K-major layout of the S operand and the MN-major layout of the P . C
// operand at the same time.
//
// Roles (384 threads): warp 0 = TMA producer for this CTA's columns (the
// whole warp prefetches block-table entries, lane 0 issues copies); warp 1 =
// S issuer (even CTA only); warp 2 = TMEM allocator, then P . C issuer
// (even CTA only); warp 3 = relay: loads the segment's query by TMA,
// zeroes cache rows past a sequence's end in this CTA's stage, and signals
// the even CTA's barriers that this CTA's operands are in place; warps 4-11
// = softmax, two groups of four: group g takes the tiles whose S lands in S
// buffer g (every other tile), and warp 4 + 4g + q of it reads TMEM lanes
// [32q, 32q + 32) of that buffer.  Each thread adds the two column-half
// partials of one head's scores and finishes 32 of them (tokens
// [16j, 16j + 16) of each 32-token half, j = lane / 16); the group shares the
// tile's row maxima through shared memory behind a 4-warp named barrier, and
// a tile's running-maximum decision waits for the previous tile's, published
// by the other group.  O rows are rescaled by the warp that can reach their
// TMEM lanes, which reads the same published maxima.
//
// Epilogue: u = O / l leaves TMEM through the query area (free once the
// segment's last S is done) by TMA stores of whole 128-byte lines; the relay
// loads the next segment's query after those stores have read it.  u is fp32
// or bf16; the partial u of a piece of a split sequence is fp16 with an fp32
// u (bf16 with a bf16 u).
//
// Work: the plan stage cuts the batch's tiles into chunks (following the
// sequences when their lengths are equal, else of equal cost on a line that
// charges every sequence start); cluster c handles chunk
// c / s_q for query row c % s_q, walking its segments in order.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "internal.h"
#include "schedule.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace {
using namespace ptx;

constexpr int kThreads = 384;
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpAlloc = 2, kWarpRelay = 3, kWarpSoftmax0 = 4;
constexpr int kStages = 4;
constexpr int kDc = 512;

constexpr uint32_t kKvBlk = 64 * 128;                    // tile: 64 rows x 64 cols, SW128
constexpr uint32_t kKvRope = 64 * 64;                    // tile: 64 rows x 32 cols, SW64
constexpr uint32_t kStageBytes = 4 * kKvBlk + kKvRope;   // 36864
constexpr uint32_t kQBlk = 128 * 128;                    // Q: 128 rows x 64 cols, SW128
constexpr uint32_t kQRope = 128 * 64;                    // Q: 128 rows x 32 cols, SW64
constexpr uint32_t kQBytes = 4 * kQBlk + kQRope;         // 73728
constexpr uint32_t kPHalf = 64 * 64;                     // 64 heads x 32 tokens bf16, SW64

constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffKv = kOffQ + kQBytes;
constexpr uint32_t kOffP = kOffKv + kStages * kStageBytes;   // [2] second halves of P
constexpr uint32_t kOffMax = kOffP + 2 * kPHalf;             // float [2 tile parity][64 heads]
constexpr uint32_t kOffSum = kOffMax + 2 * 64 * 4;           // float [2 kind][2 group][64 heads]
constexpr uint32_t kOffScratch = kOffSum + 2 * 2 * 64 * 4;    // 16 words written by the odd CTA's signals
constexpr uint32_t kOffBar = kOffScratch + 64;

// Barriers of the even CTA that the odd CTA signals ("paired" below) count
// the even CTA's own arrivals, and the odd CTA's signals as 4-byte
// transactions (st.async) that one of the even CTA's arrivals announces.
enum Bar {
  LOCAL_FULL = 0,                  // [stage] this CTA's TMA bytes of a stage (tail tiles)
  KV_FULL = LOCAL_FULL + kStages,  // [stage] even CTA: both CTAs' stage ready; full tiles count
                                   //     both CTAs' TMA bytes, tail tiles the relays' signals
  KV_EMPTY = KV_FULL + kStages,    // [stage] P . C of the stage's tile done (paired commit)
  S_FULL = KV_EMPTY + kStages,     // [2] per S buffer (paired commit)
  S_EMPTY = S_FULL + 2,            // [2] even CTA, paired: softmax warps read the S buffer
  P_FULL = S_EMPTY + 2,            // [2] even CTA, paired: softmax warps wrote P
  PV_DONE = P_FULL + 2,            // [2] (paired commit)
  Q_LOCAL = PV_DONE + 2,           // this CTA's query bytes
  Q_FULL,                          // even CTA, paired: both queries in place (relays)
  Q_EMPTY,                         // last S of a segment done (paired commit)
  DEC,                             // [2] per softmax group: its 4 warps decided a tile's maximum
  GRP = DEC + 2,                   // the 8 softmax warps of this CTA
  EPI_FREE,                        // the 8 softmax warps' output stores have read the query area
  MMA_FINAL,                       // even CTA: all S issued so far are complete
  MMA_FINAL_PV,                    // even CTA: all P . C issued so far are complete
  BAR_COUNT
};
constexpr uint32_t kOffTmemSlot = kOffBar + BAR_COUNT * 8;
constexpr uint32_t kSmemUsed = kOffTmemSlot + 16;
constexpr size_t kSmemBytes = kSmemUsed;  // the base is 1024-byte aligned (checked at entry)

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 0;     // 2 x 128 columns
constexpr uint32_t kTmemO = 256;   // 2 x 128 columns (latent blocks 0-255, 256-511)
constexpr float kRescaleThreshold = 30.0f;  // log2 units: rescale O only if the max grows by > 2^30
constexpr int kPrefetchAhead = 4;           // tiles between an L2 prefetch and the tile's TMA load
constexpr uint16_t kBothCtas = 3;

static_assert(kOffKv % 1024 == 0 && kStageBytes % 1024 == 0 && kOffP % 1024 == 0, "align");
static_assert(kSmemBytes <= 232448, "shared memory");

// First latent column of 64-column block kc (0..3) of the columns CTA `half`
// owns; the RoPE columns of that CTA start at 512 + 32 half.
__device__ __forceinline__ int lat_col(int kc, int half) {
  return (kc >> 1) * 256 + half * 128 + (kc & 1) * 64;
}

struct Params {
  Sm100Maps maps;
  const __nv_bfloat16* q;  // [B * s_q, n_h, 576], for L2 prefetch of the next segment's rows
  const __nv_bfloat16* kv; // the cache [rows, 576], for L2 prefetch of tiles ahead of their loads
  const int* block_table;
  const int* seqlens;
  const int* header;
  const int* tile_prefix;
  const int* split_base;
  const int* chunk_t;
  const int* chunk_b;
  float* part_lse;
  float* lse;
  int* err;
  int B, s_q, n_h, max_pages, page_size, num_pages;
  int out_f32;       // u is fp32, its split partials fp16 (else both bf16)
  float scale_log2;  // softmax_scale * log2(e)
};

// Lane 0 polls (a warp of spinning lanes only adds shared-memory traffic);
// the shuffle hands the outcome, and the ordering, to the rest of the warp.
template <bool kCluster = false>
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int* err) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait<kCluster>(bar, parity, err, MLA_DEVFLAG_TIMEOUT);
  return __shfl_sync(0xffffffffu, ok, 0);
}

// Both phases complete; the two tests of each poll are independent, so their
// shared-memory latencies overlap.
__device__ __forceinline__ bool warp_wait2(uint32_t bar0, uint32_t par0, uint32_t bar1,
                                           uint32_t par1, int* err) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) {
    const uint64_t t0 = cycles();
    uint32_t n = 0;
    while (!(mbar_test_nb(bar0, par0) & mbar_test_nb(bar1, par1))) {
      if ((++n & 31u) == 0 && cycles() - t0 > kWaitLimitCycles) {
        atomicOr(err, MLA_DEVFLAG_TIMEOUT);
        ok = false;
        break;
      }
    }
  }
  return __shfl_sync(0xffffffffu, ok, 0);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_sm100_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t sbase = smem_u32(smem_raw);
  uint8_t* base = smem_raw;
  if (sbase & 1023u) {  // the swizzled layouts need it; nothing has been started yet
    if (threadIdx.x == 0) atomicOr(p.err, MLA_DEVFLAG_LAYOUT);
    return;
  }
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cid = blockIdx.x >> 1;
  const int chunk = cid / p.s_q, qrow = cid % p.s_q;
  auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8u * i; };
  // Signal a paired barrier of the even CTA: from the even CTA a local
  // arrival (with `announce`, the one arrival per phase that also expects the
  // odd CTA's `odd_bytes` of signals); from the odd CTA a non-blocking 4-byte
  // st.async into scratch word `scratch_word` of the even CTA.
  auto signal_lead = [&](int i, bool announce, uint32_t odd_bytes, int scratch_word) {
    if (leader) {
      if (announce)
        mbar_arrive_expect_tx(bar(i), odd_bytes);
      else
        mbar_arrive(bar(i));
    } else {
      st_async_b32(mapa(sbase + kOffScratch + 4u * scratch_word, 0), 0u, mapa(bar(i), 0));
    }
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(LOCAL_FULL + s), 1);
      mbar_init(bar(KV_FULL + s), 1);
      mbar_init(bar(KV_EMPTY + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(S_FULL + i), 1);
      mbar_init(bar(S_EMPTY + i), 4);
      mbar_init(bar(P_FULL + i), 4);
      mbar_init(bar(DEC + i), 4);
      mbar_init(bar(PV_DONE + i), 1);
    }
    mbar_init(bar(Q_LOCAL), 1);
    mbar_init(bar(Q_FULL), 1);
    mbar_init(bar(Q_EMPTY), 1);
    mbar_init(bar(GRP), 8);
    mbar_init(bar(EPI_FREE), 8);
    mbar_init(bar(MMA_FINAL), 1);
    mbar_init(bar(MMA_FINAL_PV), 1);
    fence_mbar_init();
  }
  if (warp == kWarpAlloc) {
    tmem_alloc_pair(sbase + kOffTmemSlot, kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == kWarpTma && lane == 0) {
    prefetch_tmap(p.maps.has_kv4 ? &p.maps.kv_lat4 : &p.maps.kv_lat);
    prefetch_tmap(&p.maps.kv_rope);
  }
  if (warp == kWarpRelay && lane == 0) {
    prefetch_tmap(p.maps.has_q5 ? &p.maps.q_lat5 : &p.maps.q_lat);
    prefetch_tmap(p.maps.has_q5 ? &p.maps.q_rope5 : &p.maps.q_rope);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers and TMEM exist before either uses the other's
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(base + kOffTmemSlot);
  // everything above overlaps the plan kernel; its results are read below
  pdl_wait_previous();
  pdl_launch_dependents();

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ producer
    // with one query row every cache tile is read once, by this cluster:
    // evict it from L2 first, so the query rows and the split partials
    // stay (measured: v3 attend 40.5 -> 38.1 us).  With two query rows the
    // other row's cluster reads the same tile, from L2 if it is still there
    // (evict_first there cost the mtp attend ~10 %).
    const uint64_t pol_stream = p.s_q == 1 ? l2_policy_evict_first() : l2_policy_evict_normal();
    ChunkWalk walk;
    walk.init(p.tile_prefix, p.chunk_t, p.chunk_b, p.header, p.B, chunk);
    Segment sg;
    int g = 0;
    int last_n[kStages], tail_n[kStages];  // uses of LOCAL_FULL per stage
    for (int s = 0; s < kStages; ++s) last_n[s] = -1, tail_n[s] = 0;
    bool ok = true;
    while (ok && walk.next(sg)) {
      const int* bt = p.block_table + (size_t)sg.b * p.max_pages;
      const int L = p.seqlens[sg.b];
      for (int t0 = sg.t0; ok && t0 < sg.t1; t0 += 32) {
        // each lane fetches the page of one upcoming tile
        int my_page = 0;
        if (t0 + lane < sg.t1) {
          my_page = bt[((t0 + lane) * kTileTokens) / p.page_size];
          if (my_page < 0 || my_page >= p.num_pages) {
            atomicOr(p.err, MLA_DEVFLAG_BAD_PAGE);
            my_page = 0;
          }
        }
        const int n_here = min(32, sg.t1 - t0);
        for (int i = 0; i < n_here; ++i, ++g) {
          const int page = __shfl_sync(0xffffffffu, my_page, i);
          // The tile kPrefetchAhead tiles later goes to L2 now: its TMA load is
          // issued only when a stage frees (after this tile's P . C), and an
          // L2 hit then lands in a fraction of the HBM latency, which would
          // otherwise keep every stage busy that much longer.  A 64-token
          // tile of one page is 64 x 1152 contiguous bytes; the even CTA
          // fetches all of it.
          // At the start of a chunk every SM is already loading its query and
          // first stages; fetching more then only delays those, so the first
          // kStages tiles of the chunk prefetch nothing.
          const int page_ahead = __shfl_sync(0xffffffffu, my_page, (i + kPrefetchAhead) & 31);
          if (leader && lane == 0 && g >= kStages && i + kPrefetchAhead < n_here) {
            const int tok_a = (t0 + i + kPrefetchAhead) * kTileTokens;
            const uint8_t* src = reinterpret_cast<const uint8_t*>(
                p.kv + ((size_t)page_ahead * p.page_size + tok_a % p.page_size) * (kDc + 64));
            constexpr uint32_t kTile = kTileTokens * (kDc + 64) * 2;
            for (uint32_t off = 0; off < kTile; off += 16384)
              bulk_prefetch_l2(src + off, min(16384u, kTile - off));
          }
          if (lane == 0) {
            const int s = g % kStages, n = g / kStages;
            ok = mbar_wait(bar(KV_EMPTY + s), (n & 1) ^ 1, p.err, MLA_DEVFLAG_TIMEOUT);
            if (ok) {
              const int tok = (t0 + i) * kTileTokens;
              const int y = page * p.page_size + tok % p.page_size;
              const uint32_t st = sbase + kOffKv + s * kStageBytes;
              if (L - tok < kTileTokens) {
                // tail tile: this CTA's relay zeroes the rows past the end
                // once they land, then signals the even CTA
                mbar_arrive_expect_tx(bar(LOCAL_FULL + s), kStageBytes);
                if (p.maps.has_kv4)
                  tma_load_4d_hint(st, &p.maps.kv_lat4, bar(LOCAL_FULL + s), 128 * (int)rank, y, 0, 0,
                                   pol_stream);
                else
                  for (int kc = 0; kc < 4; ++kc)
                    tma_load_2d_hint(st + kc * kKvBlk, &p.maps.kv_lat, bar(LOCAL_FULL + s),
                                     lat_col(kc, (int)rank), y, pol_stream);
                tma_load_2d_hint(st + 4 * kKvBlk, &p.maps.kv_rope, bar(LOCAL_FULL + s),
                                 kDc + 32 * (int)rank, y, pol_stream);
                last_n[s] = tail_n[s]++;
              } else if (leader) {
                // full tile: both CTAs' bytes complete on the even CTA's barrier
                mbar_arrive_expect_tx(bar(KV_FULL + s), 2 * kStageBytes);
                if (p.maps.has_kv4)
                  tma_load_4d_hint(st, &p.maps.kv_lat4, bar(KV_FULL + s), 0, y, 0, 0, pol_stream);
                else
                  for (int kc = 0; kc < 4; ++kc)
                    tma_load_2d_hint(st + kc * kKvBlk, &p.maps.kv_lat, bar(KV_FULL + s),
                                     lat_col(kc, 0), y, pol_stream);
                tma_load_2d_hint(st + 4 * kKvBlk, &p.maps.kv_rope, bar(KV_FULL + s), kDc, y,
                                 pol_stream);
              } else {
                const uint32_t full = mapa(bar(KV_FULL + s), 0);
                if (p.maps.has_kv4)
                  tma_load_4d_to_pair_hint(st, &p.maps.kv_lat4, full, 128, y, 0, 0, pol_stream);
                else
                  for (int kc = 0; kc < 4; ++kc)
                    tma_load_2d_to_pair_hint(st + kc * kKvBlk, &p.maps.kv_lat, full, lat_col(kc, 1), y,
                                             pol_stream);
                tma_load_2d_to_pair_hint(st + 4 * kKvBlk, &p.maps.kv_rope, full, kDc + 32, y, pol_stream);
              }
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
        }
      }
    }
    // wait for this thread's tail copies in flight before the CTA may exit
    // (full tiles are consumed by the paired MMAs before the final cluster
    // barrier)
    if (lane == 0)
      for (int s = 0; s < kStages; ++s)
        if (last_n[s] >= 0) mbar_wait(bar(LOCAL_FULL + s), last_n[s] & 1, p.err, MLA_DEVFLAG_TIMEOUT);
    __syncwarp();
  } else if (warp == kWarpRelay) {
    // ------------------------------------------------------------ relay
    ChunkWalk walk;
    walk.init(p.tile_prefix, p.chunk_t, p.chunk_b, p.header, p.B, chunk);
    Segment sg;
    int g = 0, seg_i = 0;
    int tail_n[kStages];  // uses of LOCAL_FULL per stage, in tile order
    for (int s = 0; s < kStages; ++s) tail_n[s] = 0;
    bool ok = true;
    bool q_in_flight = false;
    while (ok && walk.next(sg)) {
      // this segment's query rows (h, j) = Q[64 rank + 16 qd + i, columns of
      // CTA j], stored as row 32 qd + 16 j + i; heads >= n_h read as zero
      // (the tensor map ends there)
      // the query area is free once the previous segment's last S has read
      // it and its epilogue's output stores (staged there) have left
      if (seg_i > 0 && !(ok = warp_wait(bar(Q_EMPTY), (seg_i - 1) & 1, p.err) &&
                              warp_wait(bar(EPI_FREE), (seg_i - 1) & 1, p.err)))
        break;
      if (lane == 0) {
        const int z = sg.b * p.s_q + qrow;
        mbar_arrive_expect_tx(bar(Q_LOCAL), kQBytes);
        if (p.maps.has_q5) {
          // one copy per 64-column block: rows 32 qd + 16 j + i at once
          for (int kc = 0; kc < 4; ++kc)
            tma_load_5d(sbase + kOffQ + kc * kQBlk, &p.maps.q_lat5, bar(Q_LOCAL), lat_col(kc, 0),
                        0, 0, 4 * (int)rank, z);
          tma_load_5d(sbase + kOffQ + 4 * kQBlk, &p.maps.q_rope5, bar(Q_LOCAL), kDc, 0, 0,
                      4 * (int)rank, z);
        } else {
          for (int qd = 0; qd < 4; ++qd)
            for (int j = 0; j < 2; ++j) {
              const int y = 64 * (int)rank + 16 * qd;
              const uint32_t r0 = static_cast<uint32_t>(32 * qd + 16 * j);
              for (int kc = 0; kc < 4; ++kc)
                tma_load_3d(sbase + kOffQ + kc * kQBlk + r0 * 128, &p.maps.q_lat, bar(Q_LOCAL),
                            lat_col(kc, j), y, z);
              tma_load_3d(sbase + kOffQ + 4 * kQBlk + r0 * 64, &p.maps.q_rope, bar(Q_LOCAL),
                          kDc + 32 * j, y, z);
            }
        }
      }
      q_in_flight = true;
      // the next segment's query rows go to L2 now, so that its TMA load
      // after this segment's last S is an L2 hit
      if (lane == 0) {
        ChunkWalk peek = walk;
        Segment nx;
        const int heads = min(64, p.n_h - 64 * (int)rank);
        if (heads > 0 && peek.next(nx)) {
          const __nv_bfloat16* src =
              p.q + ((size_t)(nx.b * p.s_q + qrow) * p.n_h + 64 * rank) * (kDc + 64);
          const uint32_t bytes = static_cast<uint32_t>(heads) * (kDc + 64) * 2;
          for (uint32_t off = 0; off < bytes; off += 16384)
            bulk_prefetch_l2(reinterpret_cast<const uint8_t*>(src) + off, min(16384u, bytes - off));
        }
      }
      if (!(ok = warp_wait(bar(Q_LOCAL), seg_i & 1, p.err))) break;
      q_in_flight = false;
      if (lane == 0) signal_lead(Q_FULL, true, 4u, 8);
      __syncwarp();

      const int L = p.seqlens[sg.b];
      for (int t = sg.t0; t < sg.t1; ++t, ++g) {
        const int s = g % kStages;
        const int rows_valid = L - t * kTileTokens;
        if (rows_valid >= kTileTokens) continue;  // full tile: no relay
        if (!(ok = warp_wait(bar(LOCAL_FULL + s), (tail_n[s]++) & 1, p.err))) break;
        // rows past the sequence end may hold anything; make them zero so
        // that 0-probability x garbage cannot turn into NaN in P . C
        uint8_t* tile = base + kOffKv + s * kStageBytes;
        for (int r = max(rows_valid, 0); r < kTileTokens; ++r) {
          if (lane < 8)
            for (int kb = 0; kb < 4; ++kb)
              *reinterpret_cast<uint4*>(tile + kb * kKvBlk + r * 128 + lane * 16) =
                  make_uint4(0, 0, 0, 0);
          if (lane < 4)
            *reinterpret_cast<uint4*>(tile + 4 * kKvBlk + r * 64 + lane * 16) =
                make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) signal_lead(KV_FULL + s, true, 4u, 9);
        __syncwarp();
      }
      ++seg_i;
    }
    // a query copy still in flight must land before the CTA may exit
    if (q_in_flight && lane == 0) mbar_wait(bar(Q_LOCAL), seg_i & 1, p.err, MLA_DEVFLAG_TIMEOUT);
    __syncwarp();
  } else if (warp == kWarpMma || warp == kWarpAlloc) {
    // ------------------------------------------------------------ MMA issuers
    // Warp 1 issues every S, warp 2 (done allocating) every P . C.  The two
    // streams touch disjoint TMEM and shared memory, and each commit tracks
    // only its own thread's MMAs, so a P . C whose P is ready never waits
    // behind an S being issued (issuing blocks while the tensor pipe's queue
    // is full) and vice versa.
    if (leader) {
      constexpr uint32_t kIdS = idesc_bf16(256, 128, false);
      constexpr uint32_t kIdPV = idesc_bf16(128, 256, true);
      ChunkWalk walk;
      walk.init(p.tile_prefix, p.chunk_t, p.chunk_b, p.header, p.B, chunk);
      Segment sg;
      int g0 = 0, seg_i = 0;
      bool ok = true;
      // S for global tile g: 16 steps over the latent columns, 2 over RoPE
      auto issue_s = [&](int g, bool last) {
        tc_fence_after();
        if (lane == 0) {
          const uint32_t st = sbase + kOffKv + (g % kStages) * kStageBytes;
          const uint32_t dS = tmem + kTmemS + (g & 1) * 128;
          uint32_t acc = 0;
          for (int kc = 0; kc < 4; ++kc)
            for (int ks = 0; ks < 4; ++ks) {
              const uint64_t a =
                  smem_desc(sbase + kOffQ + kc * kQBlk + ks * 32, 16, 1024, kLayoutSW128);
              const uint64_t b = smem_desc(st + kc * kKvBlk + ks * 32, 16, 1024, kLayoutSW128);
              umma_f16_ss_pair(dS, a, b, kIdS, acc);
              acc = 1;
            }
          for (int ks = 0; ks < 2; ++ks) {
            const uint64_t a = smem_desc(sbase + kOffQ + 4 * kQBlk + ks * 32, 16, 512, kLayoutSW64);
            const uint64_t b = smem_desc(st + 4 * kKvBlk + ks * 32, 16, 512, kLayoutSW64);
            umma_f16_ss_pair(dS, a, b, kIdS, 1u);
          }
          umma_commit_pair(bar(S_FULL + (g & 1)), kBothCtas);
          if (last) umma_commit_pair(bar(Q_EMPTY), kBothCtas);
        }
        __syncwarp();
      };
      // O (+)= P . C for global tile g; `first` = first tile of its segment
      auto issue_pv = [&](int g, bool first) {
        tc_fence_after();
        if (lane == 0) {
          const uint32_t st = sbase + kOffKv + (g % kStages) * kStageBytes;
          // P tokens 0-31 sit in the stage's RoPE block (S is done with it),
          // tokens 32-63 in the second-half ring
          const uint32_t pa0 = st + 4 * kKvBlk, pa1 = sbase + kOffP + (g & 1) * kPHalf;
          for (int blk = 0; blk < 2; ++blk)
            for (int kk = 0; kk < 4; ++kk) {  // 16 tokens per MMA
              const uint64_t a = smem_desc((kk < 2 ? pa0 : pa1) + (kk & 1) * 32, 16, 512, kLayoutSW64);
              const uint64_t b =
                  smem_desc(st + 2 * blk * kKvBlk + kk * 2048, kKvBlk, 1024, kLayoutSW128);
              umma_f16_ss_pair(tmem + kTmemO + blk * 128, a, b, kIdPV,
                               (first && kk == 0) ? 0u : 1u);
            }
          umma_commit_pair(bar(KV_EMPTY + g % kStages), kBothCtas);
          umma_commit_pair(bar(PV_DONE + (g & 1)), kBothCtas);
        }
        __syncwarp();
      };
      // Fixed order per segment: S0 S1 S2, then P.C(j) S(j+3) for every tile
      // j, so S runs two tiles ahead of P.C and the softmax of tile j has
      // two S groups of tensor work to hide behind.  Each step polls only the
      // barriers it needs (a barrier test costs ~150 cycles; re-testing a
      // ready barrier is not free).
      const bool s_issuer = warp == kWarpMma;
      while (ok && walk.next(sg)) {
        const int n_t = sg.t1 - sg.t0;
        if (s_issuer) {
          // S(g) once its stage is loaded and its S buffer has been read
          if (!(ok = warp_wait(bar(Q_FULL), seg_i & 1, p.err))) break;
          for (int j = 0; ok && j < n_t; ++j) {
            const int g = g0 + j;
            if (!(ok = warp_wait2(bar(KV_FULL + g % kStages), (g / kStages) & 1,
                                  bar(S_EMPTY + (g & 1)), ((g >> 1) & 1) ^ 1, p.err)))
              break;
            issue_s(g, j == n_t - 1);
          }
        } else {
          // P . C(g) once P(g) is written
          for (int j = 0; ok && j < n_t; ++j) {
            const int g = g0 + j;
            if (!(ok = warp_wait(bar(P_FULL + (g & 1)), (g >> 1) & 1, p.err))) break;
            issue_pv(g, j == 0);
          }
        }
        g0 += n_t;
        ++seg_i;
      }
      // every MMA issued by this thread has completed before TMEM is freed
      const int fin = s_issuer ? MMA_FINAL : MMA_FINAL_PV;
      if (lane == 0) {
        umma_commit_pair(bar(fin), 1);
        mbar_wait(bar(fin), 0, p.err, MLA_DEVFLAG_TIMEOUT);
      }
      __syncwarp();
    }
  } else if (warp >= kWarpSoftmax0) {
    // ------------------------------------------------------------ softmax
    // Two groups of four warps take alternate tiles (group = g & 1, which is
    // also the tile's S buffer and P ring slot); warp q of a group reads TMEM
    // lanes [32q, 32q + 32) for all 64 tokens, so a head's tile maximum needs
    // no exchange between warps.  The running maximum after tile g is
    // published per head in shared memory (slot g & 1); a group decides tile
    // g from the maximum after tile g - 1, which the other group published.
    const int sw_warp = warp - kWarpSoftmax0;       // 0..7
    const int grp = sw_warp >> 2;                   // softmax group; also the O block it drains
    const int gw = sw_warp & 3;                     // warp within the group
    const int qd = warp & 3;                        // TMEM lanes [32 qd, 32 qd + 32)
    const int jh = lane >> 4;                       // S row half: partial over CTA jh's columns
    const int hS = 16 * qd + (lane & 15);           // head (local) of this thread's S row
    const int hO = (32 * qd + lane) & 63;           // head (local) of this thread's O lane
    const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
    const uint32_t sw64 = static_cast<uint32_t>((hS >> 1) & 3);  // 64-byte swizzle of row hS
    float* mx_pub = reinterpret_cast<float*>(base + kOffMax);  // [tile parity][head]
    float* sums = reinterpret_cast<float*>(base + kOffSum);    // [kind][group][head]
    const float c_log2 = p.scale_log2;
    uint32_t grp_phase = 0;
    // A failed wait (a broken protocol) sets the device flag; the warp then
    // skips its later waits but still runs every step, so that the group's
    // named barriers and the other roles' waits stay matched and the kernel
    // ends.
    auto rendezvous = [&](bool live) -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(GRP));
      const uint32_t ph = (grp_phase++) & 1;
      return live && warp_wait(bar(GRP), ph, p.err);
    };

    ChunkWalk walk;
    walk.init(p.tile_prefix, p.chunk_t, p.chunk_b, p.header, p.B, chunk);
    Segment sg;
    int g = 0;
    bool ok = true;
    while (walk.next(sg)) {
      const int L = p.seqlens[sg.b];
      const int L_eff = L - p.s_q + 1 + qrow;  // positions this query row may see
      const int n_t = sg.t1 - sg.t0;
      const int g0 = g;
      // the segment's output row: u's row, or its partial slot (read now,
      // used by the epilogue)
      const int out_z =
          sg.whole ? sg.b * p.s_q + qrow : (p.split_base[sg.b] + sg.part) * p.s_q + qrow;
      // this group's sums over its own tiles of the segment, in the scale of
      // m_used (the maximum it last applied)
      float m_used = -INFINITY, l = 0.f, l_exact = 0.f;
      for (int jt = (grp - g0) & 1; jt < n_t; jt += 2) {
        const int gt = g0 + jt;
        const int t = sg.t0 + jt;
        // ---- partial scores of tile gt -> registers; free the S buffer
        ok = ok && warp_wait(bar(S_FULL + grp), (gt >> 1) & 1, p.err);
        tc_fence_after();
        // sc[16 c + k]: token 32 c + 16 jh + k of the tile, for head hS.
        // S = partial(CTA 0 columns) + partial(CTA 1 columns): lane jh keeps
        // tokens [16 jh, 16 jh + 16) of each 32 and hands the rest to lane ^ 16
        float sc[32];
        const uint32_t sb = tmem + lane_base + kTmemS + grp * 128;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float va[32], vb[32];
          tmem_ld32(sb + 32 * c, va);
          tmem_ld32(sb + 64 + 32 * c, vb);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float own_lo = jh ? vb[k] : va[k], own_hi = jh ? vb[16 + k] : va[16 + k];
            const float send = jh ? own_lo : own_hi;
            const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
            sc[16 * c + k] = (jh ? own_hi : own_lo) + recv;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) signal_lead(S_EMPTY + grp, gw == 0, 16u, gw);
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int nv = L_eff - (t * kTileTokens + 32 * c + 16 * jh);  // valid of these 16
          if (nv < 16) {
#pragma unroll
            for (int k = 0; k < 16; ++k)
              if (k >= nv) sc[16 * c + k] = -INFINITY;
          }
#pragma unroll
          for (int k = 0; k < 16; k += 2) {
            mx0 = fmaxf(mx0, sc[16 * c + k]);
            mx1 = fmaxf(mx1, sc[16 * c + k + 1]);
          }
        }
        float mx = fmaxf(mx0, mx1);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        // ---- the maximum after this tile.  The running maximum may go
        // stale: it moves only when a tile's maximum exceeds it by more than
        // 2^kRescaleThreshold (weights stay below that factor), which keeps O
        // rescales rare.  Raw scores: scale > 0 commutes with max.
        const float t_s = mx * c_log2;
        float m_prev = -INFINITY;
        if (jt > 0) {  // tile gt - 1 (the other group's) is in this segment
          ok = ok && warp_wait(bar(DEC + (grp ^ 1)), ((gt - 1) >> 1) & 1, p.err);
          m_prev = mx_pub[((gt - 1) & 1) * 64 + hS];
        }
        const float m_new = (m_prev == -INFINITY || t_s > m_prev + kRescaleThreshold)
                                ? fmaxf(m_prev, t_s) : m_prev;
        if (jh == 0) mx_pub[(gt & 1) * 64 + hS] = m_new;
        named_bar_sync(1 + grp, 128);
        // O lane hO: rescale if its head's maximum moved at this tile
        float alpha_o = 1.f;
        bool resc_o = false;
        if (jt > 0) {
          const float mo_prev = mx_pub[((gt - 1) & 1) * 64 + hO];
          const float mo_new = mx_pub[(gt & 1) * 64 + hO];
          if (mo_new != mo_prev) {
            alpha_o = ex2_approx(mo_prev - mo_new);  // mo_prev = -inf: O holds only zeros
            resc_o = true;
          }
        }
        // the decision of tile gt is published (and slot (gt - 1) & 1 read)
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(DEC + grp));
        // this group's sums move to the new scale
        if (m_new != m_used) {
          const float f = m_used == -INFINITY ? 0.f : ex2_approx(m_used - m_new);
          l *= f;
          l_exact *= f;
          m_used = m_new;
        }
        const float neg_m = m_new == -INFINITY ? 0.f : -m_new;
        float r0 = 0.f, r1 = 0.f, e0 = 0.f, e1 = 0.f;
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 32; k += 2) {
          const float a = ex2_approx(fmaf(sc[k], c_log2, neg_m));
          const float b = ex2_approx(fmaf(sc[k + 1], c_log2, neg_m));
          const __nv_bfloat162 pr = __floats2bfloat162_rn(a, b);
          const float2 pf = __bfloat1622float2(pr);
          if (k & 2) { r1 += pf.x + pf.y; e1 += a + b; } else { r0 += pf.x + pf.y; e0 += a + b; }
          pk[k >> 1] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        // u is normalised by the sum of the rounded weights it was built
        // from; lse uses the unrounded weights
        l += r0 + r1;
        l_exact += e0 + e1;

        // P's ring slot grp was last read by PV(gt - 2); O may be rescaled
        // only after PV(gt - 1) (tiles of an earlier segment were retired by
        // that segment's epilogue, and the first P . C of a segment
        // overwrites O)
        if (gt >= 2) ok = ok && warp_wait(bar(PV_DONE + grp), ((gt - 2) >> 1) & 1, p.err);
        if (__any_sync(0xffffffffu, resc_o)) {
          ok = ok && warp_wait(bar(PV_DONE + (grp ^ 1)), ((gt - 1) >> 1) & 1, p.err);
          tc_fence_after();
          for (int c0 = 0; c0 < 256; c0 += 32) {  // both O blocks of these lanes
            float o[32];
            tmem_ld32(tmem + lane_base + kTmemO + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha_o;
            tmem_st32(tmem + lane_base + kTmemO + c0, o);
          }
          tmem_wait_st();
        }
        // P row hS, tokens [32c + 16jh, +16): half c of the row (32 tokens =
        // 64 B, 64-byte swizzle) lives in the stage's RoPE block (c = 0) or
        // in ring slot grp (c = 1); 16-byte chunks 2jh and 2jh + 1
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint32_t prow =
              (c == 0 ? sbase + kOffKv + (gt % kStages) * kStageBytes + 4 * kKvBlk
                      : sbase + kOffP + grp * kPHalf) + hS * 64;
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const uint32_t ch = static_cast<uint32_t>(2 * jh + k);
            st_shared_v4(prow + ((ch ^ sw64) << 4), pk[8 * c + 4 * k], pk[8 * c + 4 * k + 1],
                         pk[8 * c + 4 * k + 2], pk[8 * c + 4 * k + 3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) signal_lead(P_FULL + grp, gw == 0, 16u, gw);
      }
      g = g0 + n_t;

      // ---- epilogue: u = O / l for this thread's O lane (one head, 128
      // consecutive latent columns of O block grp)
      // the maximum after the segment's last tile (decided by either group)
      if (((g - 1) & 1) != grp) ok = ok && warp_wait(bar(DEC + (grp ^ 1)), ((g - 1) >> 1) & 1, p.err);
      const float mS_fin = mx_pub[((g - 1) & 1) * 64 + hS];
      const float mO_fin = mx_pub[((g - 1) & 1) * 64 + hO];
      {
        // this group's sums in the scale of the final maximum
        const float f = m_used == mS_fin ? 1.f : m_used == -INFINITY ? 0.f : ex2_approx(m_used - mS_fin);
        const float lf = l * f, lef = l_exact * f;
        const float l2 = lf + __shfl_xor_sync(0xffffffffu, lf, 16);
        const float e2 = lef + __shfl_xor_sync(0xffffffffu, lef, 16);
        if (jh == 0) {
          sums[(0 * 2 + grp) * 64 + hS] = l2;
          sums[(1 * 2 + grp) * 64 + hS] = e2;
        }
      }
      // every warp has read the published maxima of this segment before any
      // starts the next one
      ok = rendezvous(ok);
      const float l_o = sums[(0 * 2 + 0) * 64 + hO] + sums[(0 * 2 + 1) * 64 + hO];
      const float le_o = sums[(1 * 2 + 0) * 64 + hO] + sums[(1 * 2 + 1) * 64 + hO];
      ok = ok && warp_wait(bar(PV_DONE + ((g - 1) & 1)), ((g - 1) >> 1) & 1, p.err);
      tc_fence_after();
      const float inv = l_o > 0.f ? 1.f / l_o : 0.f;
      const int c = grp;                          // O block drained by this group
      const int col0 = 256 * c + 128 * (qd >> 1);  // latent column of TMEM column kTmemO + 128c
      // The segment's last S has read Q, so the query area stages the output:
      // 8 KB per warp, its 32 heads x 128 columns as boxes of 128-byte lines
      // (64 16-bit or 32 fp32 columns) in the 128-byte-swizzled layout of the
      // output tensor map (row = head = lane, 16-byte chunk k of a row at
      // k ^ (row & 7)).  Each box leaves by one TMA store, which writes whole
      // 128-byte lines of u; the relay loads the next segment's query only
      // after the stores have read the area.
      const uint32_t stg = sbase + kOffQ + sw_warp * 8192u;
      const int y_head = 64 * (int)rank + 32 * (qd & 1);  // first head of this warp's rows
      const CUtensorMap* omap = sg.whole ? &p.maps.u_out : &p.maps.part_out;
      if (p.out_f32 && sg.whole) {
        // fp32: four boxes of 32 columns (one 128-byte line per head), two
        // at a time through the warp's 8 KB
        for (int c0 = 0; c0 < 128; c0 += 32) {
          float o[32];
          tmem_ld32(tmem + lane_base + kTmemO + c * 128 + c0, o);
          tmem_wait_ld();
          const uint32_t box = stg + static_cast<uint32_t>((c0 >> 5) & 1) * 4096u;
          if (c0 == 64) {  // the first two boxes must have left before reuse
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
          }
#pragma unroll
          for (int e = 0; e < 8; ++e)
            st_shared_v4(box + lane * 128u + ((static_cast<uint32_t>(e ^ (lane & 7))) << 4),
                         __float_as_uint(o[4 * e] * inv), __float_as_uint(o[4 * e + 1] * inv),
                         __float_as_uint(o[4 * e + 2] * inv), __float_as_uint(o[4 * e + 3] * inv));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && y_head < p.n_h) {
            tma_store_3d(omap, box, col0 + c0, y_head, out_z);
            bulk_commit();
          }
        }
      } else {
        bool f16_range_ok = true;  // fp16 partials: every value fits
        for (int c0 = 0; c0 < 128; c0 += 32) {
          float o[32];
          tmem_ld32(tmem + lane_base + kTmemO + c * 128 + c0, o);
          tmem_wait_ld();
          // 16-bit rows: with a bf16 u, u of a whole sequence or this
          // segment's partial u, both bf16; with an fp32 u, the partial u in
          // fp16 (the merge weights and sums the partials in fp32)
          const uint32_t row = stg + static_cast<uint32_t>(c0 >> 6) * 4096u + lane * 128u;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float x0 = o[8 * e + 2 * k] * inv, x1 = o[8 * e + 2 * k + 1] * inv;
              if (p.out_f32) {
                const __half2 h2 = __floats2half2_rn(x0, x1);
                w[k] = *reinterpret_cast<const uint32_t*>(&h2);
                f16_range_ok &= fabsf(x0) <= 65504.f && fabsf(x1) <= 65504.f;
              } else {
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(x0, x1);
                w[k] = *reinterpret_cast<const uint32_t*>(&h2);
              }
            }
            const uint32_t chunk16 = static_cast<uint32_t>(((c0 & 63) >> 3) + e);
            st_shared_v4(row + ((chunk16 ^ static_cast<uint32_t>(lane & 7)) << 4), w[0], w[1],
                         w[2], w[3]);
          }
          if (c0 & 32) {  // box c0 >> 6 is complete
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && y_head < p.n_h) {
              tma_store_3d(omap, stg + static_cast<uint32_t>(c0 >> 6) * 4096u, col0 + (c0 & 64),
                           y_head, out_z);
              bulk_commit();
            }
          }
        }
        if (!__all_sync(0xffffffffu, f16_range_ok) && lane == 0) atomicOr(p.err, MLA_DEVFLAG_RANGE);
      }
      const int head = 64 * (int)rank + hO;
      if (head < p.n_h && qd < 2 && c == 0) {
        const float lse = le_o > 0.f ? (mO_fin + log2f(le_o)) * 0.69314718055994531f : -INFINITY;
        if (sg.whole) {
          if (p.lse != nullptr) p.lse[(size_t)out_z * p.n_h + head] = lse;
        } else {
          p.part_lse[(size_t)out_z * p.n_h + head] = lse;
        }
      }
      // the query area may take the next segment's rows once the stores have
      // read it
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(EPI_FREE));
      tc_fence_before();
    }
    // the last stores complete before the CTA exits
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // all paired MMAs are complete and no arrival is still on its way
  if (warp == kWarpAlloc) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
  cluster_sync();
}

}  // namespace

size_t decode_sm100_smem_bytes() { return kSmemBytes; }

// Per device, once: opt in to the shared-memory size and count how many
// 2-CTA clusters of this kernel can be resident at the same time.
int decode_sm100_prepare() {
  if (cudaFuncSetAttribute(decode_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBytes) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, decode_sm100_kernel, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    n = sms / 2;
  }
  return n;
}

cudaError_t launch_decode_sm100(const DecodeArgs& a, const Sm100Maps& maps, cudaStream_t s) {
  Params p;
  p.maps = maps;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.kv = static_cast<const __nv_bfloat16*>(a.kv);
  p.block_table = a.block_table;
  p.seqlens = a.seqlens;
  p.header = a.header;
  p.tile_prefix = a.tile_prefix;
  p.split_base = a.split_base;
  p.chunk_t = a.chunk_t;
  p.chunk_b = a.chunk_b;
  p.part_lse = a.part_lse;
  p.lse = a.lse;
  p.err = a.err;
  p.B = a.B;
  p.s_q = a.s_q;
  p.n_h = a.n_h;
  p.max_pages = a.max_pages;
  p.page_size = a.page_size;
  p.num_pages = a.num_pages;
  p.out_f32 = a.out_f32 ? 1 : 0;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * a.num_chunks * a.s_q, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, decode_sm100_kernel, p);
}

}  // namespace mla
