// Attend stage on the 5th-generation tensor cores (sm_100a), for n_h <= 128
// heads, latent d_c = 512, RoPE key d_R = 64, bf16.
//
// Math ("MLA deep compression", absorption section, both equations, and its
// decoupled-RoPE section): all heads of one query row share every cached row
// [c || k^R], so the 128 heads are the M dimension of two dense contractions
// per 64-token tile:
//     S = Q . [C || K^R]^T      (M = 128, N = 64 tokens, K = 576)
//     O = O * alpha + P . C     (M = 128, N = 512 latent, K = 64 tokens)
// with an online softmax between them; u = O / l at the end.
//
// Column split.  O for 128 heads x 512 latent in fp32 fills all 512 TMEM
// columns, which leaves no room for S.  So a cluster of two CTAs splits the
// columns: CTA r owns latent columns [256r, 256r + 256) and RoPE columns
// [32r, 32r + 32).  Each CTA loads only its own columns of every cache tile
// (each byte is read from HBM once) and computes a partial S over its 288
// columns; the partial S tiles are swapped with one 32 KB bulk copy each way
// per tile (completing on the receiver's transaction-count barrier), and both
// CTAs add own + peer.  fp32 addition commutes, so both hold the same S, make
// bit-identical softmax decisions, and each accumulates its own half of
// O = P . C (N = 256).
//
// TMEM per CTA (512 columns): O 256 | S 2 x 64 | Q latent 128 (bf16 pairs).
// Shared memory: 3 tile stages of 36 KB, the query's RoPE columns (8 KB), two
// P buffers (16 KB each), one receive and one send buffer for partial S
// (32 KB each).  One shared-memory copy of a tile serves both contractions: a
// TMA load with 128-byte swizzle writes each 64-column block as 64 rows x
// 128 B, the K-major operand layout of S = Q K^T and the MN-major operand
// layout of O = P C at the same time.
//
// Roles (384 threads): warp 0 = TMA producer (the whole warp prefetches
// block-table entries, lane 0 issues copies); warp 1 = MMA issuer, which
// issues S or P . C for whichever tile is ready (S runs up to two tiles
// ahead) and zeroes cache rows past a sequence's end; warp 2 = TMEM
// allocator; warp 3 = exchange: ships each partial S to the peer, tells the
// peer when its last shipment has been read, arms the receive barrier;
// warps 4-11 = softmax: warp 4 + 4h + q serves TMEM lanes [32q, 32q + 32)
// (head rows) and tile columns [32h, 32h + 32), so each head row has two
// threads sharing the row maximum through shared memory.  Per tile the
// softmax warps (1) add the peer's partial of tile g, (2) stage their
// partial of tile g + 1 for the exchange warp, (3) do tile g's arithmetic.
//
// Work: the plan stage cuts the batch's tiles into equal chunks; cluster c
// handles chunk c / s_q for query row c % s_q, walking its segments in order.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"
#include "schedule.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace {
using namespace ptx;

constexpr int kThreads = 384;
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpAlloc = 2, kWarpXchg = 3, kWarpSoftmax0 = 4;
constexpr int kStages = 3;
constexpr int kDc = 512, kWidth = 576;
constexpr int kLatPerCta = 256, kRopePerCta = 32;

constexpr uint32_t kKvBlk = 64 * 128;                    // tile: 64 rows x 64 cols, SW128
constexpr uint32_t kKvRope = 64 * 64;                    // tile: 64 rows x 32 cols, SW64
constexpr uint32_t kStageBytes = 4 * kKvBlk + kKvRope;   // 36864
constexpr uint32_t kQRopeBytes = 128 * 64;               // 128 rows x 32 cols bf16, SW64
constexpr uint32_t kPBytes = 128 * 128;                  // 128 rows x 64 tokens bf16, SW128
constexpr uint32_t kXBytes = 128 * 256;                  // one partial S: 128 x 64 fp32

constexpr uint32_t kOffKv = 0;
constexpr uint32_t kOffP = kOffKv + kStages * kStageBytes;    // [2]
constexpr uint32_t kOffQRope = kOffP + 2 * kPBytes;
constexpr uint32_t kOffXin = kOffQRope + kQRopeBytes;
constexpr uint32_t kOffXout = kOffXin + kXBytes;
constexpr uint32_t kOffRed = kOffXout + kXBytes;              // float [2][2][128] row maxima
constexpr uint32_t kOffSum = kOffRed + 2 * 2 * 128 * 4;       // float [2][2][128] row sums
constexpr uint32_t kOffBar = kOffSum + 2 * 2 * 128 * 4;

enum Bar {
  KV_FULL = 0,
  KV_EMPTY = KV_FULL + kStages,
  S_FULL = KV_EMPTY + kStages,   // [2] per S buffer
  S_EMPTY = S_FULL + 2,          // [2]
  P_FULL = S_EMPTY + 2,          // [2] per P buffer
  PV_DONE = P_FULL + 2,          // [2]
  X_FULL = PV_DONE + 2,          // peer's partial S landed in our receive buffer
  X_EMPTY,                       // peer has read what we sent last
  X_READ,                        // our softmax warps have read the receive buffer
  X_OUT_READY,                   // our softmax warps have staged the send buffer
  X_OUT_FREE,                    // the last send has left the send buffer
  Q_FULL,
  Q_EMPTY,
  SM_PAIR,                       // [4] the two softmax warps sharing a TMEM lane quarter
  MMA_FINAL = SM_PAIR + 4,
  BAR_COUNT
};
constexpr uint32_t kOffTmemSlot = kOffBar + BAR_COUNT * 8;
constexpr uint32_t kSmemUsed = kOffTmemSlot + 16;
constexpr size_t kSmemBytes = kSmemUsed + 1024;  // slack to align the base to 1024 B

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;     // 256 columns
constexpr uint32_t kTmemS = 256;   // 2 x 64 columns
constexpr uint32_t kTmemQ = 384;   // 128 columns: the 256 latent query values per row
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only if the max grows by > 2^8

static_assert(kStageBytes % 1024 == 0 && kOffP % 1024 == 0 && kOffQRope % 1024 == 0, "align");
static_assert(kSmemBytes <= 232448, "shared memory");

struct Params {
  Sm100Maps maps;
  const __nv_bfloat16* q;
  const int* block_table;
  const int* seqlens;
  const int* header;
  const int* tile_prefix;
  const int* split_base;
  float* part_u;
  float* part_lse;
  __nv_bfloat16* u;
  float* lse;
  int* err;
  int B, s_q, n_h, max_pages, page_size, num_pages;
  float scale_log2;  // softmax_scale * log2(e)
};

// Every lane of the warp polls; the warp agrees on the outcome.
template <bool kCluster = false>
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int* err) {
  const bool ok = mbar_wait<kCluster>(bar, parity, err, MLA_DEVFLAG_TIMEOUT);
  return __all_sync(0xffffffffu, ok);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_sm100_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (sbase - raw_addr);
  const uint32_t rank = cluster_ctarank(), peer = rank ^ 1u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cid = blockIdx.x >> 1;
  const int chunk = cid / p.s_q, qrow = cid % p.s_q;
  auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8u * i; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(KV_FULL + s), 1);
      mbar_init(bar(KV_EMPTY + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(S_FULL + i), 1);
      mbar_init(bar(S_EMPTY + i), 8);   // one arrive per softmax warp
      mbar_init(bar(P_FULL + i), 8);
      mbar_init(bar(PV_DONE + i), 1);
    }
    mbar_init(bar(X_FULL), 1);                      // armed with the 32 KB of one tile
    mbar_arrive_expect_tx(bar(X_FULL), kXBytes);    // tile 0
    mbar_init(bar(X_EMPTY), 1);
    mbar_init(bar(X_READ), 8);
    mbar_init(bar(X_OUT_READY), 8);
    mbar_init(bar(X_OUT_FREE), 1);
    mbar_init(bar(Q_FULL), 8);
    mbar_init(bar(Q_EMPTY), 1);
    for (int i = 0; i < 4; ++i) mbar_init(bar(SM_PAIR + i), 2);
    mbar_init(bar(MMA_FINAL), 1);
    fence_mbar_init();
  }
  if (warp == kWarpAlloc) {
    tmem_alloc(sbase + kOffTmemSlot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kWarpTma && lane == 0) {
    prefetch_tmap(&p.maps.kv_lat);
    prefetch_tmap(&p.maps.kv_rope);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers exist before anything is sent to them
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(base + kOffTmemSlot);
  // everything above overlaps the plan kernel; its results are read below
  pdl_wait_previous();
  pdl_launch_dependents();
  const int cs = p.header[1];

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ producer
    ChunkWalk walk;
    walk.init(p.tile_prefix, p.B, chunk, cs);
    Segment sg;
    int g = 0;
    int last_n[kStages];
    for (int s = 0; s < kStages; ++s) last_n[s] = -1;
    bool ok = true;
    while (ok && walk.next(sg)) {
      const int* bt = p.block_table + (size_t)sg.b * p.max_pages;
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
          if (lane == 0) {
            const int s = g % kStages, n = g / kStages;
            ok = mbar_wait(bar(KV_EMPTY + s), (n & 1) ^ 1, p.err, MLA_DEVFLAG_TIMEOUT);
            if (ok) {
              const int tok = (t0 + i) * kTileTokens;
              const int y = page * p.page_size + tok % p.page_size;
              const uint32_t st = sbase + kOffKv + s * kStageBytes;
              mbar_arrive_expect_tx(bar(KV_FULL + s), kStageBytes);
              for (int kb = 0; kb < 4; ++kb)
                tma_load_2d(st + kb * kKvBlk, &p.maps.kv_lat, bar(KV_FULL + s),
                            rank * kLatPerCta + kb * 64, y);
              tma_load_2d(st + 4 * kKvBlk, &p.maps.kv_rope, bar(KV_FULL + s),
                          kDc + rank * kRopePerCta, y);
              last_n[s] = n;
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
        }
      }
    }
    // wait for this thread's own copies in flight before the CTA may exit
    if (lane == 0)
      for (int s = 0; s < kStages; ++s)
        if (last_n[s] >= 0) mbar_wait(bar(KV_FULL + s), last_n[s] & 1, p.err, MLA_DEVFLAG_TIMEOUT);
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t kIdS = idesc_bf16(128, 64, false);
    constexpr uint32_t kIdPV = idesc_bf16(128, kLatPerCta, true);
    ChunkWalk walk;
    walk.init(p.tile_prefix, p.B, chunk, cs);
    Segment sg;
    int g0 = 0, seg_i = 0;
    bool ok = true;
    // S = Q . tile^T for global tile g (tile index t of the segment's sequence)
    auto issue_s = [&](int g, int t, int L, bool last) {
      const int s = g % kStages;
      const int rows_valid = L - t * kTileTokens;
      if (rows_valid < kTileTokens) {
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
      }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t st = sbase + kOffKv + s * kStageBytes;
        const uint32_t dS = tmem + kTmemS + (g & 1) * 64;
        uint32_t acc = 0;
        for (int kb = 0; kb < 4; ++kb)
          for (int ks = 0; ks < 4; ++ks) {  // 16 columns per MMA, A from TMEM
            const uint64_t b = smem_desc(st + kb * kKvBlk + ks * 32, 16, 1024, kLayoutSW128);
            umma_f16_ts(dS, tmem + kTmemQ + (kb * 4 + ks) * 8, b, kIdS, acc);
            acc = 1;
          }
        for (int ks = 0; ks < 2; ++ks) {  // RoPE columns, A from shared memory
          const uint64_t a = smem_desc(sbase + kOffQRope + ks * 32, 16, 512, kLayoutSW64);
          const uint64_t b = smem_desc(st + 4 * kKvBlk + ks * 32, 16, 512, kLayoutSW64);
          umma_f16_ss(dS, a, b, kIdS, 1u);
        }
        umma_commit(bar(S_FULL + (g & 1)));
        if (last) umma_commit(bar(Q_EMPTY));
      }
      __syncwarp();
    };
    // O (+)= P . C for global tile g; `first` = first tile of its segment
    auto issue_pv = [&](int g, bool first) {
      tc_fence_after();
      if (lane == 0) {
        const uint32_t st = sbase + kOffKv + (g % kStages) * kStageBytes;
        const uint32_t pa = sbase + kOffP + (g & 1) * kPBytes;
        for (int kk = 0; kk < 4; ++kk) {  // 16 tokens per MMA
          const uint64_t a = smem_desc(pa + kk * 32, 16, 1024, kLayoutSW128);
          const uint64_t b = smem_desc(st + kk * 2048, kKvBlk, 1024, kLayoutSW128);
          umma_f16_ss(tmem + kTmemO, a, b, kIdPV, (first && kk == 0) ? 0u : 1u);
        }
        umma_commit(bar(KV_EMPTY + g % kStages));
        umma_commit(bar(PV_DONE + (g & 1)));
      }
      __syncwarp();
    };
    while (ok && walk.next(sg)) {
      if (!(ok = warp_wait(bar(Q_FULL), seg_i & 1, p.err))) break;
      const int L = p.seqlens[sg.b];
      const int n_t = sg.t1 - sg.t0;
      int s_next = 0, pv_next = 0;
      uint64_t t_idle = 0;
      while (pv_next < n_t) {
        // P . C first when its P is ready (it frees a stage and a P buffer);
        // otherwise S for the next tile whose data and S buffer are ready
        bool did = false;
        if (pv_next < s_next) {
          const int g = g0 + pv_next;
          bool ready = false;
          if (lane == 0) ready = mbar_test_nb(bar(P_FULL + (g & 1)), (g >> 1) & 1);
          if (__shfl_sync(0xffffffffu, ready, 0)) {
            if (!(ok = warp_wait(bar(P_FULL + (g & 1)), (g >> 1) & 1, p.err))) break;
            issue_pv(g, pv_next == 0);
            ++pv_next;
            did = true;
          }
        }
        if (!did && s_next < n_t) {
          const int g = g0 + s_next;
          bool ready = false;
          if (lane == 0)
            ready = mbar_test_nb(bar(KV_FULL + g % kStages), (g / kStages) & 1) &&
                    mbar_test_nb(bar(S_EMPTY + (g & 1)), ((g >> 1) & 1) ^ 1);
          if (__shfl_sync(0xffffffffu, ready, 0)) {
            if (!(ok = warp_wait(bar(KV_FULL + g % kStages), (g / kStages) & 1, p.err) &&
                       warp_wait(bar(S_EMPTY + (g & 1)), ((g >> 1) & 1) ^ 1, p.err)))
              break;
            issue_s(g, sg.t0 + s_next, L, s_next == n_t - 1);
            ++s_next;
            did = true;
          }
        }
        if (did) {
          t_idle = 0;
        } else if (t_idle == 0) {
          t_idle = globaltimer();
        } else if (globaltimer() - t_idle > kWaitLimitNs) {
          if (lane == 0) atomicOr(p.err, MLA_DEVFLAG_TIMEOUT);
          ok = false;
          break;
        }
      }
      g0 += n_t;
      ++seg_i;
    }
    // every MMA issued by this thread has completed before TMEM is freed
    if (lane == 0) {
      umma_commit(bar(MMA_FINAL));
      mbar_wait(bar(MMA_FINAL), 0, p.err, MLA_DEVFLAG_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == kWarpXchg) {
    // ------------------------------------------------------------ exchange
    // For every tile g in order: ship our staged partial S of tile g to the
    // peer; then, once our softmax warps have read the peer's tile g, arm the
    // receive barrier for tile g + 1 and tell the peer it may send again.
    ChunkWalk walk;
    walk.init(p.tile_prefix, p.B, chunk, cs);
    Segment sg;
    int total = 0;
    while (walk.next(sg)) total += sg.t1 - sg.t0;
    const uint32_t xin_peer = mapa(sbase + kOffXin, peer);
    const uint32_t xfull_peer = mapa(bar(X_FULL), peer);
    const uint32_t xempty_peer = mapa(bar(X_EMPTY), peer);
    bool ok = true;
    for (int g = 0; ok && g < total; ++g) {
      if (!(ok = warp_wait(bar(X_OUT_READY), g & 1, p.err))) break;
      if (!(ok = warp_wait<true>(bar(X_EMPTY), (g & 1) ^ 1, p.err))) break;  // peer read g - 1
      if (lane == 0) {
        bulk_copy_to_peer(xin_peer, sbase + kOffXout, kXBytes, xfull_peer);
        bulk_commit();
        bulk_wait_read_all();
        mbar_arrive(bar(X_OUT_FREE));
      }
      if (!(ok = warp_wait(bar(X_READ), g & 1, p.err))) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(X_FULL), kXBytes);  // tile g + 1
        mbar_arrive_remote(xempty_peer);
      }
      __syncwarp();
    }
  } else if (warp >= kWarpSoftmax0) {
    // ------------------------------------------------------------ softmax
    const int sw_warp = warp - kWarpSoftmax0;       // 0..7
    const int half = sw_warp >> 2;                  // tile columns [32 half, +32)
    const int quad = warp & 3;                      // TMEM lanes [32 quad, +32)
    const int row = quad * 32 + lane;               // head
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t sw = static_cast<uint32_t>(row & 7);
    const uint32_t xout_row = sbase + kOffXout + row * 256;
    const uint32_t xin_row = sbase + kOffXin + row * 256;
    float* red = reinterpret_cast<float*>(base + kOffRed);  // [parity][half][row]
    float* sums = reinterpret_cast<float*>(base + kOffSum); // [quantity][half][row]
    const float c_log2 = p.scale_log2;
    uint32_t pair_phase = 0;
    // barrier between the two warps sharing these rows (bounded wait)
    auto sync_pair = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(SM_PAIR + quad));
      return warp_wait(bar(SM_PAIR + quad), (pair_phase++) & 1, p.err);
    };
    // S_g (this thread's 32 columns) -> registers; free the S buffer; stage
    // the row in the send buffer for the exchange warp.
    auto fetch_and_stage = [&](int g, float (&dst)[32]) -> bool {
      if (!warp_wait(bar(S_FULL + (g & 1)), (g >> 1) & 1, p.err)) return false;
      tc_fence_after();
      tmem_ld32(tmem + lane_base + kTmemS + (g & 1) * 64 + half * 32, dst);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(S_EMPTY + (g & 1)));
      if (!warp_wait(bar(X_OUT_FREE), (g & 1) ^ 1, p.err)) return false;  // send of g - 1 left
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t chunk = static_cast<uint32_t>(half * 8 + k);
        st_shared_v4(xout_row + ((chunk ^ sw) << 4), __float_as_uint(dst[4 * k]),
                     __float_as_uint(dst[4 * k + 1]), __float_as_uint(dst[4 * k + 2]),
                     __float_as_uint(dst[4 * k + 3]));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(X_OUT_READY));
      return true;
    };

    ChunkWalk walk;
    walk.init(p.tile_prefix, p.B, chunk, cs);
    Segment sg;
    int g = 0, seg_i = 0;
    bool ok = true;
    while (ok && walk.next(sg)) {
      const int L = p.seqlens[sg.b];
      const int L_eff = L - p.s_q + 1 + qrow;  // positions this query row may see
      const int n_t = sg.t1 - sg.t0;

      // ---- this segment's query: latent columns into TMEM, RoPE columns
      // into shared memory (64-byte swizzle, the S operand layout)
      if (seg_i > 0 && !(ok = warp_wait(bar(Q_EMPTY), (seg_i - 1) & 1, p.err))) break;
      {
        const __nv_bfloat16* qrow_ptr =
            row < p.n_h ? p.q + ((size_t)(sg.b * p.s_q + qrow) * p.n_h + row) * kWidth : nullptr;
        uint32_t qw[32];
        for (int part = 0; part < 2; ++part) {  // 2 x 64 latent values per thread
          const uint4* src = qrow_ptr ? reinterpret_cast<const uint4*>(
                                            qrow_ptr + rank * kLatPerCta + half * 128 + part * 64)
                                      : nullptr;
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 x = src ? src[v] : make_uint4(0, 0, 0, 0);
            qw[4 * v] = x.x;
            qw[4 * v + 1] = x.y;
            qw[4 * v + 2] = x.z;
            qw[4 * v + 3] = x.w;
          }
          tmem_st32u(tmem + lane_base + kTmemQ + half * 64 + part * 32, qw);
        }
        // RoPE: 32 values = 4 chunks of 16 B; half h writes chunks 2h, 2h + 1
        const uint4* rsrc = qrow_ptr ? reinterpret_cast<const uint4*>(
                                           qrow_ptr + kDc + rank * kRopePerCta)
                                     : nullptr;
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          const uint32_t c = static_cast<uint32_t>(half * 2 + v);
          const uint4 x = rsrc ? rsrc[c] : make_uint4(0, 0, 0, 0);
          st_shared_v4(sbase + kOffQRope + row * 64 + ((c ^ ((row >> 1) & 3)) << 4), x.x, x.y, x.z,
                       x.w);
        }
        fence_proxy_async_smem();
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(Q_FULL));
      }

      float m = -INFINITY, l = 0.f, l_exact = 0.f;
      float s[32], s_next[32];
      if (!(ok = fetch_and_stage(g, s))) break;
      for (int j = 0; j < n_t; ++j, ++g) {
        const int t = sg.t0 + j;
        // (1) the peer's partial of this tile; S = own + peer
        if (!(ok = warp_wait<true>(bar(X_FULL), g & 1, p.err))) break;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t chunk = static_cast<uint32_t>(half * 8 + k);
          const float4 v = ld_shared_v4(xin_row + ((chunk ^ sw) << 4));
          s[4 * k] += v.x;
          s[4 * k + 1] += v.y;
          s[4 * k + 2] += v.z;
          s[4 * k + 3] += v.w;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(X_READ));
        // (2) stage the next tile's partial before this tile's arithmetic
        if (j + 1 < n_t && !(ok = fetch_and_stage(g + 1, s_next))) break;

        // (3) masked online softmax in log2 units
        const int nv = L_eff - t * kTileTokens - half * 32;  // valid columns of this half
        if (nv < 32) {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c >= nv) s[c] = -INFINITY;
        }
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          mx0 = fmaxf(mx0, s[c]);
          mx1 = fmaxf(mx1, s[c + 1]);
          mx2 = fmaxf(mx2, s[c + 2]);
          mx3 = fmaxf(mx3, s[c + 3]);
        }
        float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        red[((g & 1) * 2 + half) * 128 + row] = mx;
        if (!(ok = sync_pair())) break;
        mx = fmaxf(mx, red[((g & 1) * 2 + (half ^ 1)) * 128 + row]) * c_log2;  // scale > 0
        const float m_new = fmaxf(m, mx);
        const bool resc = m_new > m + kRescaleThreshold;
        float alpha = 1.f;
        if (resc) {
          alpha = ex2_approx(m - m_new);
          m = m_new;
        }
        const float neg_m = m == -INFINITY ? 0.f : -m;
        float r0 = 0.f, r1 = 0.f, e0 = 0.f, e1 = 0.f;
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float a = ex2_approx(fmaf(s[c], c_log2, neg_m));
          const float b = ex2_approx(fmaf(s[c + 1], c_log2, neg_m));
          const __nv_bfloat162 pr = __floats2bfloat162_rn(a, b);
          const float2 pf = __bfloat1622float2(pr);
          if (c & 2) { r1 += pf.x + pf.y; e1 += a + b; } else { r0 += pf.x + pf.y; e0 += a + b; }
          pk[c >> 1] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        // u is normalised by the sum of the rounded weights it was built
        // from; lse uses the unrounded weights
        l = l * alpha + (r0 + r1);
        l_exact = l_exact * alpha + (e0 + e1);

        // P buffer g&1 was last read by PV_{g-2}; O may be rescaled only after
        // PV_{g-1} (tiles of an earlier segment were retired by that segment's
        // epilogue)
        if (j >= 2 && !(ok = warp_wait(bar(PV_DONE + (g & 1)), ((g - 2) >> 1) & 1, p.err))) break;
        if (j >= 1 && __any_sync(0xffffffffu, resc)) {
          if (!(ok = warp_wait(bar(PV_DONE + ((g - 1) & 1)), ((g - 1) >> 1) & 1, p.err))) break;
          tc_fence_after();
          for (int c0 = 0; c0 < 128; c0 += 32) {
            float o[32];
            tmem_ld32(tmem + lane_base + kTmemO + half * 128 + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tmem + lane_base + kTmemO + half * 128 + c0, o);
          }
          tmem_wait_st();
        }
        // P row (64 tokens = 128 B, 128-byte swizzle); this thread writes
        // its half: 16-byte chunks 4h .. 4h + 3
        const uint32_t prow = sbase + kOffP + (g & 1) * kPBytes + row * 128;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t c = static_cast<uint32_t>(half * 4 + k);
          st_shared_v4(prow + ((c ^ sw) << 4), pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(P_FULL + (g & 1)));
#pragma unroll
        for (int c = 0; c < 32; ++c) s[c] = s_next[c];
      }
      if (!ok) break;

      // ---- epilogue: u = O / l (this thread's 128 of the CTA's 256 columns)
      sums[(0 * 2 + half) * 128 + row] = l;
      sums[(1 * 2 + half) * 128 + row] = l_exact;
      if (!(ok = sync_pair())) break;
      l += sums[(0 * 2 + (half ^ 1)) * 128 + row];
      l_exact += sums[(1 * 2 + (half ^ 1)) * 128 + row];
      if (!(ok = warp_wait(bar(PV_DONE + ((g - 1) & 1)), ((g - 1) >> 1) & 1, p.err))) break;
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float lse = l_exact > 0.f ? (m + log2f(l_exact)) * 0.69314718055994531f : -INFINITY;
      const bool write = row < p.n_h;
      const size_t orow = (size_t)(sg.b * p.s_q + qrow) * p.n_h + row;
      const size_t slot = sg.whole ? 0 : (size_t)(p.split_base[sg.b] + sg.part) * p.s_q + qrow;
      for (int c0 = 0; c0 < 128; c0 += 32) {
        float o[32];
        tmem_ld32(tmem + lane_base + kTmemO + half * 128 + c0, o);
        tmem_wait_ld();
        if (!write) continue;
        const int col = rank * kLatPerCta + half * 128 + c0;
        if (sg.whole) {
          uint4* dst = reinterpret_cast<uint4*>(p.u + orow * kDc + col);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 h2 =
                  __floats2bfloat162_rn(o[8 * v + 2 * e] * inv, o[8 * v + 2 * e + 1] * inv);
              w[e] = *reinterpret_cast<const uint32_t*>(&h2);
            }
            dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(p.part_u + (slot * p.n_h + row) * kDc + col);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_float4(o[4 * v] * inv, o[4 * v + 1] * inv, o[4 * v + 2] * inv,
                                 o[4 * v + 3] * inv);
        }
      }
      if (write && rank == 0 && half == 0) {
        if (sg.whole) {
          if (p.lse != nullptr) p.lse[orow] = lse;
        } else {
          p.part_lse[slot * p.n_h + row] = lse;
        }
      }
      tc_fence_before();
      ++seg_i;
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpAlloc) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  cluster_sync();  // no CTA leaves while its peer may still send into its shared memory
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
  p.block_table = a.block_table;
  p.seqlens = a.seqlens;
  p.header = a.header;
  p.tile_prefix = a.tile_prefix;
  p.split_base = a.split_base;
  p.part_u = a.part_u;
  p.part_lse = a.part_lse;
  p.u = static_cast<__nv_bfloat16*>(a.u);
  p.lse = a.lse;
  p.err = a.err;
  p.B = a.B;
  p.s_q = a.s_q;
  p.n_h = a.n_h;
  p.max_pages = a.max_pages;
  p.page_size = a.page_size;
  p.num_pages = a.num_pages;
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
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_sm100_kernel, p);
}

}  // namespace mla
