// Attend stage on the 5th-generation tensor cores (sm_100a) for small latent
// widths: fp32 tensors with d_c + d_R <= 128 (kind::tf32) or bf16 tensors
// with d_c + d_R <= 256 (kind::f16), n_h <= 128.  The same math as the
// DeepSeek-V3-shape kernel ("MLA deep compression", absorption section, both
// equations; decoupled-RoPE section): per 64-token tile
//     S = Q . [C || K^R]^T      (M = 128 head rows, N = 64 tokens, K = d_c + d_R)
//     O = O * alpha + P . C     (M = 128, N = d_c, K = 64 tokens)
// with an online softmax between them; u = O / l at the end.
//
// One CTA per (KV chunk, query row).  TMEM holds S (2 buffers of 64
// columns) and O (d_c columns) for all 128 rows, so every softmax thread owns
// one head's row end to end: it reads its S row, keeps its running maximum
// and sums, rescales its own O row when the maximum grows, writes its P row
// and finally its u row.  Columns are staged in 128-byte blocks (32 fp32 or
// 64 bf16 values) with 128-byte swizzle; the last block of a row reads past
// d_c + d_R as zeros (the tensor maps end there), so Q and the cached rows
// contribute nothing beyond their width.  With bf16, one shared-memory copy of
// a tile is the K-major B operand of S and the MN-major B operand of P . C.
// An MN-major tf32 operand needs 128-byte swizzle of 32-byte atoms instead,
// so the tf32 kernel also loads the tile's latent columns a second time in
// that layout for P . C (and keeps two stages and one P slot to fit).
//
// Roles (192 threads): warp 0 = TMA producer (query per segment, cache
// tiles); warp 1 = TMEM allocator and MMA issuer (it also zeroes cache rows
// past a sequence's end in the stage before use, so that a zero weight never
// meets a non-finite value); warps 2-5 = softmax and epilogue, thread
// (warp w, lane l) owning TMEM lane / row 32 (w % 4) + l.
//
// P is rounded to the operand type before it is stored (tf32 or bf16), and
// u is normalised by the sum of the rounded weights it was built from; lse
// uses the unrounded ones.
//
// The same kernel runs the GQA path of GQLA (GQLA summary, abstract and
// method paragraphs: the same weights expose a path with a per-group expanded
// cache).  There a cached token holds, for every group g of heads, the
// expanded key K^C_g = W^UK_g c and value V_g = W^UV_g c, plus the RoPE key
// shared by all heads; one CTA takes (KV chunk, group) with every head of the
// group and every query row as the MMA rows, so a tile of the group's cache
// is read once for all s_q rows (the MTP case, s_q = 2).  S is taken over
// [K^C_g || k^R] and P . V over V_g, loaded into the stage's value region.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"
#include "schedule.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace {
using namespace ptx;

constexpr int kThreads = 192;
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpSoftmax0 = 2;
constexpr int kMaxStages = 3;
constexpr int kRows = 128;            // MMA rows: heads, padded
constexpr int kMaxBlocks = 4;         // 128-byte column blocks of a cached row
constexpr uint32_t kQBlkBytes = kRows * 128;
constexpr uint32_t kKvBlkBytes = kTileTokens * 128;

enum Bar {
  KV_FULL = 0,
  KV_EMPTY = KV_FULL + kMaxStages,
  S_FULL = KV_EMPTY + kMaxStages,  // [2]
  S_EMPTY = S_FULL + 2,         // [2] 4 softmax warps
  P_FULL = S_EMPTY + 2,         // [2] 4 softmax warps
  PV_DONE = P_FULL + 2,         // [2]
  Q_FULL = PV_DONE + 2,
  Q_EMPTY,                      // last S of a segment done
  O_FREE,                       // 4 softmax warps have read O for the epilogue
  MMA_FINAL,
  BAR_COUNT
};

struct Params {
  CUtensorMap q_map;   // q [B * s_q, n_h, W]: box (one 128-byte block) x 128 heads x 1
                       // (GQA: box (one block) x heads per group x s_q)
  CUtensorMap kv_map;  // cache [rows, W]: box (one 128-byte block) x 64 rows
                       // (GQA: the expanded cache [rows, n_g, d_h + d_v], box 64 x 1 x 64)
  CUtensorMap kv_pv_map;  // tf32: the same boxes with 32-byte-atom swizzle (P . C operand)
  CUtensorMap kr_map;  // GQA: the shared RoPE keys [rows, d_R], box 64 x 64 rows
  const int* block_table;
  const int* seqlens;
  const int* header;
  const int* tile_prefix;
  const int* split_base;
  const int* chunk_t;
  const int* chunk_b;
  void* u;
  float* lse;
  float* part_u;
  float* part_lse;
  int* err;
  int B, s_q, n_h, d_c, max_pages, page_size, num_pages;
  int blocks;          // 128-byte column blocks of the S operand
  int out_f32;         // u is fp32 (else bf16)
  float scale_log2;    // softmax_scale * log2(e)
  // GQA path: groups, heads per group, key / value / RoPE blocks
  int n_g, hpg, d_h, d_v, nbk, nbr, nbv;
};

template <bool kTf32, bool kGqa>
struct Layout {
  static constexpr int kCols = kTf32 ? 32 : 64;          // values per 128-byte block
  static constexpr int kPBlocks = kTf32 ? 2 : 1;         // P: 64 tokens per row
  static constexpr bool kValueRegion = kTf32 || kGqa;    // P . C / P . V operand apart
  static constexpr int kStages = kValueRegion ? 2 : 3;
  static constexpr int kPSlots = kTf32 ? 1 : 2;
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffKv = kOffQ + kMaxBlocks * kQBlkBytes;
  // a stage: the S operand of the tile, then (tf32, GQA) the value region:
  // the P . C copy of the latent columns, or the group's values
  static constexpr uint32_t kPvCopy = kMaxBlocks * kKvBlkBytes;
  static constexpr uint32_t kStageBytes = (kValueRegion ? 2 : 1) * kMaxBlocks * kKvBlkBytes;
  static constexpr uint32_t kOffP = kOffKv + kStages * kStageBytes;
  static constexpr uint32_t kPSlot = kPBlocks * kQBlkBytes;
  static constexpr uint32_t kOffBar = kOffP + kPSlots * kPSlot;
  static constexpr uint32_t kOffTmemSlot = kOffBar + BAR_COUNT * 8;
  static constexpr size_t kSmem = kOffTmemSlot + 16 + 1024;  // + alignment slack
};

// tf32 value of x rounded to nearest (ties away), low 13 bits zero
__device__ __forceinline__ float to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

template <bool kTf32, bool kGqa>
__global__ void __launch_bounds__(kThreads, 1) decode_small_sm100_kernel(const __grid_constant__ Params p) {
  using Lay = Layout<kTf32, kGqa>;
  constexpr int kStages = Lay::kStages;
  constexpr int kPSlots = Lay::kPSlots;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (sbase - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // MLA: (chunk, query row); GQA: (chunk, group) with every query row
  const int chunk = blockIdx.x / (kGqa ? p.n_g : p.s_q);
  const int qrow = kGqa ? 0 : blockIdx.x % p.s_q;
  const int grp = kGqa ? blockIdx.x % p.n_g : 0;
  auto bar = [&](int i) -> uint32_t { return sbase + Lay::kOffBar + 8u * i; };
  const int nb = p.blocks;
  const int d_c = kGqa ? p.d_v : p.d_c;  // width of O and of the output rows
  const int nbc = kGqa ? p.nbv : kTf32 ? d_c / Lay::kCols : 0;  // value-region blocks
  const int q_rows = kGqa ? p.hpg * p.s_q : kRows;               // query rows the TMA fills

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(KV_FULL + s), 1);
      mbar_init(bar(KV_EMPTY + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(S_FULL + i), 1);
      mbar_init(bar(S_EMPTY + i), 4);
      mbar_init(bar(P_FULL + i), 4);
      mbar_init(bar(PV_DONE + i), 1);
    }
    mbar_init(bar(Q_FULL), 1);
    mbar_init(bar(Q_EMPTY), 1);
    mbar_init(bar(O_FREE), 4);
    mbar_init(bar(MMA_FINAL), 1);
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(sbase + Lay::kOffTmemSlot, 512);
    tmem_relinquish();
  }
  if (kGqa) {
    // the query boxes fill rows [0, hpg * s_q) of each block; the rows past
    // them are zero once and stay so
    for (uint32_t off = threadIdx.x * 16; off < kMaxBlocks * kQBlkBytes; off += kThreads * 16)
      *reinterpret_cast<uint4*>(base + Lay::kOffQ + off) = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(base + Lay::kOffTmemSlot);
  constexpr uint32_t kTmemS = 0, kTmemO = 128;  // S: 2 x 64 columns; O: d_c columns
  pdl_wait_previous();
  pdl_launch_dependents();

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&p.q_map);
      prefetch_tmap(&p.kv_map);
      if (kTf32) prefetch_tmap(&p.kv_pv_map);
      if (kGqa) prefetch_tmap(&p.kr_map);
      ChunkWalk walk;
      walk.init(p.tile_prefix, p.chunk_t, p.chunk_b, p.header, p.B, chunk);
      Segment sg;
      int g = 0, seg_i = 0;
      bool ok = true;
      while (ok && walk.next(sg)) {
        // the query area is free once the previous segment's last S is done
        if (seg_i > 0 && !(ok = mbar_wait(bar(Q_EMPTY), (seg_i - 1) & 1, p.err, MLA_DEVFLAG_TIMEOUT)))
          break;
        mbar_arrive_expect_tx(bar(Q_FULL), nb * q_rows * 128);
        for (int k = 0; k < nb; ++k) {
          if (kGqa)  // rows (r, h): query row r, head h of the group
            tma_load_3d(sbase + Lay::kOffQ + k * kQBlkBytes, &p.q_map, bar(Q_FULL), k * Lay::kCols,
                        grp * p.hpg, sg.b * p.s_q);
          else
            tma_load_3d(sbase + Lay::kOffQ + k * kQBlkBytes, &p.q_map, bar(Q_FULL), k * Lay::kCols,
                        0, sg.b * p.s_q + qrow);
        }
        const int* bt = p.block_table + (size_t)sg.b * p.max_pages;
        for (int t = sg.t0; ok && t < sg.t1; ++t, ++g) {
          const int s = g % kStages, n = g / kStages;
          if (!(ok = mbar_wait(bar(KV_EMPTY + s), (n & 1) ^ 1, p.err, MLA_DEVFLAG_TIMEOUT))) break;
          const int tok = t * kTileTokens;
          int page = bt[tok / p.page_size];
          if (page < 0 || page >= p.num_pages) {
            atomicOr(p.err, MLA_DEVFLAG_BAD_PAGE);
            page = 0;
          }
          const int y = page * p.page_size + tok % p.page_size;
          const uint32_t st = sbase + Lay::kOffKv + s * Lay::kStageBytes;
          mbar_arrive_expect_tx(bar(KV_FULL + s), (nb + nbc) * kKvBlkBytes);
          if (kGqa) {
            // S operand: the group's keys, then the shared RoPE keys; the
            // value region: the group's values
            for (int k = 0; k < p.nbk; ++k)
              tma_load_3d(st + k * kKvBlkBytes, &p.kv_map, bar(KV_FULL + s), k * 64, grp, y);
            for (int k = 0; k < p.nbr; ++k)
              tma_load_2d(st + (p.nbk + k) * kKvBlkBytes, &p.kr_map, bar(KV_FULL + s), k * 64, y);
            for (int k = 0; k < nbc; ++k)
              tma_load_3d(st + Lay::kPvCopy + k * kKvBlkBytes, &p.kv_map, bar(KV_FULL + s),
                          p.d_h + k * 64, grp, y);
          } else {
            for (int k = 0; k < nb; ++k)
              tma_load_2d(st + k * kKvBlkBytes, &p.kv_map, bar(KV_FULL + s), k * Lay::kCols, y);
            for (int k = 0; k < nbc; ++k)
              tma_load_2d(st + Lay::kPvCopy + k * kKvBlkBytes, &p.kv_pv_map, bar(KV_FULL + s),
                          k * Lay::kCols, y);
          }
        }
        ++seg_i;
      }
      // copies still in flight land before the CTA may exit: the last query
      // was consumed by an S (waited for below through MMA_FINAL), and every
      // stage loaded is consumed by an MMA before the final commit
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idS = kTf32 ? idesc_tf32(kRows, kTileTokens, false)
                               : idesc_bf16(kRows, kTileTokens, false);
    const uint32_t idPV = kTf32 ? idesc_tf32(kRows, d_c, true) : idesc_bf16(kRows, d_c, true);
    ChunkWalk walk;
    walk.init(p.tile_prefix, p.chunk_t, p.chunk_b, p.header, p.B, chunk);
    Segment sg;
    int g0 = 0, seg_i = 0;
    bool ok = true;
    auto mma = [&](uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
      if (kTf32)
        umma_tf32_ss(d, a, b, id, acc);
      else
        umma_f16_ss(d, a, b, id, acc);
    };
    // S(g) may start once its stage is loaded and its S buffer was read
    auto s_ready = [&](int g) -> bool {
      const int s = g % kStages;
      return mbar_wait(bar(KV_FULL + s), (g / kStages) & 1, p.err, MLA_DEVFLAG_TIMEOUT) &&
             (g < 2 || mbar_wait(bar(S_EMPTY + (g & 1)), ((g - 2) >> 1) & 1, p.err, MLA_DEVFLAG_TIMEOUT));
    };
    while (ok && walk.next(sg)) {
      const int n_t = sg.t1 - sg.t0;
      const int L = p.seqlens[sg.b];
      bool wait_ok = true;
      if (lane == 0) wait_ok = mbar_wait(bar(Q_FULL), seg_i & 1, p.err, MLA_DEVFLAG_TIMEOUT);
      if (!(ok = __shfl_sync(0xffffffffu, wait_ok, 0))) break;
      // software pipeline: S(j + 1) is issued before P . C(j)
      for (int j = 0; ok && j <= n_t; ++j) {
        if (j < n_t) {
          const int g = g0 + j;
          const int rows_valid = L - (sg.t0 + j) * kTileTokens;
          if (lane == 0) wait_ok = s_ready(g);
          if (!(ok = __shfl_sync(0xffffffffu, wait_ok, 0))) break;
          const uint32_t st = sbase + Lay::kOffKv + (g % kStages) * Lay::kStageBytes;
          if (rows_valid < kTileTokens) {
            uint8_t* tile = base + (st - sbase);
            // (a row keeps its 128 bytes under either swizzle)
            for (int r = max(rows_valid, 0); r < kTileTokens; ++r)
              for (int k = 0; k < nb + nbc; ++k)
                if (lane < 8)
                  *reinterpret_cast<uint4*>(tile + (k < nb ? k * kKvBlkBytes
                                                           : Lay::kPvCopy + (k - nb) * kKvBlkBytes) +
                                            r * 128 + lane * 16) = make_uint4(0, 0, 0, 0);
            fence_proxy_async_smem();
            __syncwarp();
          }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t dS = tmem + kTmemS + (g & 1) * 64;
            uint32_t acc = 0;
            for (int k = 0; k < nb; ++k)
              for (int ks = 0; ks < 4; ++ks) {  // 32 bytes of K per instruction
                const uint64_t a = smem_desc(sbase + Lay::kOffQ + k * kQBlkBytes + ks * 32, 16, 1024,
                                             kLayoutSW128);
                const uint64_t b = smem_desc(st + k * kKvBlkBytes + ks * 32, 16, 1024, kLayoutSW128);
                mma(dS, a, b, idS, acc);
                acc = 1;
              }
            umma_commit(bar(S_FULL + (g & 1)));
            if (j == n_t - 1) umma_commit(bar(Q_EMPTY));
          }
          __syncwarp();
        }
        if (j >= 1) {
          // P . C(j - 1): O (+)= P [128 x 64 tokens] . C [64 tokens x d_c]
          const int g = g0 + j - 1;
          if (lane == 0) {
            wait_ok = mbar_wait(bar(P_FULL + (g & 1)), (g >> 1) & 1, p.err, MLA_DEVFLAG_TIMEOUT);
            // the first P . C of a segment overwrites O: the previous
            // segment's epilogue must have read it
            if (wait_ok && j == 1 && seg_i > 0)
              wait_ok = mbar_wait(bar(O_FREE), (seg_i - 1) & 1, p.err, MLA_DEVFLAG_TIMEOUT);
          }
          if (!(ok = __shfl_sync(0xffffffffu, wait_ok, 0))) break;
          tc_fence_after();
          if (lane == 0) {
            const uint32_t st = sbase + Lay::kOffKv + (g % kStages) * Lay::kStageBytes;
            const uint32_t pa = sbase + Lay::kOffP + (g % kPSlots) * Lay::kPSlot;
            constexpr int kStep = kTf32 ? 8 : 16;  // tokens per instruction
            for (int kk = 0; kk < kTileTokens / kStep; ++kk) {
              // A: P rows, K-major, 32 bytes per step inside its 128-byte block
              const int tok = kk * kStep;
              const uint64_t a = smem_desc(pa + (tok / Lay::kCols) * kQBlkBytes +
                                               ((tok % Lay::kCols) * (kTf32 ? 4 : 2)),
                                           16, 1024, kLayoutSW128);
              // B: the tile's latent columns, MN-major: kStep token rows
              // (128 bytes each) per step, 64-row blocks of 128-byte columns
              // kKvBlkBytes apart; K groups of 8 rows (bf16, 128-byte
              // swizzle) or 4 rows (tf32 copy, 32-byte atoms)
              const uint64_t b =
                  kTf32 ? smem_desc(st + Lay::kPvCopy + tok * 128, kKvBlkBytes, 512, kLayoutSW128Atom32)
                  : kGqa ? smem_desc(st + Lay::kPvCopy + tok * 128, kKvBlkBytes, 1024, kLayoutSW128)
                         : smem_desc(st + tok * 128, kKvBlkBytes, 1024, kLayoutSW128);
              mma(tmem + kTmemO, a, b, idPV, (j == 1 && kk == 0) ? 0u : 1u);
            }
            umma_commit(bar(KV_EMPTY + g % kStages));
            umma_commit(bar(PV_DONE + (g & 1)));
          }
          __syncwarp();
        }
      }
      g0 += n_t;
      ++seg_i;
    }
    if (lane == 0) {
      umma_commit(bar(MMA_FINAL));
      mbar_wait(bar(MMA_FINAL), 0, p.err, MLA_DEVFLAG_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int q4 = warp & 3;
    const int row = 32 * q4 + lane;  // MMA row: head (MLA) or (query row, head of the group) (GQA)
    const int r_row = kGqa ? row / p.hpg : qrow;                 // query row
    const int head = kGqa ? grp * p.hpg + row % p.hpg : row;
    const bool live = kGqa ? row < p.hpg * p.s_q : row < p.n_h;
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    const float c_log2 = p.scale_log2;
    ChunkWalk walk;
    walk.init(p.tile_prefix, p.chunk_t, p.chunk_b, p.header, p.B, chunk);
    Segment sg;
    int g = 0;
    bool ok = true;
    auto wwait = [&](uint32_t b, uint32_t par) -> bool {
      bool r = true;
      if (lane == 0) r = mbar_wait(b, par, p.err, MLA_DEVFLAG_TIMEOUT);
      return __shfl_sync(0xffffffffu, r, 0);
    };
    while (ok && walk.next(sg)) {
      const int L = p.seqlens[sg.b];
      const int L_eff = L - p.s_q + 1 + r_row;
      const int n_t = sg.t1 - sg.t0;
      float m = -INFINITY, l = 0.f, l_exact = 0.f;
      for (int j = 0; j < n_t; ++j, ++g) {
        if (!(ok = wwait(bar(S_FULL + (g & 1)), (g >> 1) & 1))) break;
        tc_fence_after();
        float s[64];
        {
          float a[32], b[32];
          tmem_ld32(tmem + lane_base + kTmemS + (g & 1) * 64, a);
          tmem_ld32(tmem + lane_base + kTmemS + (g & 1) * 64 + 32, b);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            s[k] = a[k];
            s[32 + k] = b[k];
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(S_EMPTY + (g & 1)));
        const int nv = L_eff - (sg.t0 + j) * kTileTokens;
        float tmax = -INFINITY;
#pragma unroll
        for (int k = 0; k < 64; ++k) {
          if (k >= nv) s[k] = -INFINITY;
          tmax = fmaxf(tmax, s[k]);
        }
        // exact running maximum (raw scores; scale > 0 commutes with max)
        const float mn = fmaxf(m, tmax * c_log2);
        const float alpha = (m == -INFINITY) ? 1.f : exp2f(m - mn);
        const bool resc = j > 0 && mn > m;
        m = mn;
        const float neg_m = m == -INFINITY ? 0.f : -m;
        float pr[64];
        float r_sum = 0.f, e_sum = 0.f;
#pragma unroll
        for (int k = 0; k < 64; ++k) {
          const float e = exp2f(fmaf(s[k], c_log2, neg_m));
          float v;
          if (kTf32) {
            v = to_tf32(e);
          } else {
            v = __bfloat162float(__float2bfloat16_rn(e));
          }
          pr[k] = v;
          r_sum += v;
          e_sum += e;
        }
        l = l * alpha + r_sum;
        l_exact = l_exact * alpha + e_sum;
        // the P slot g % kPSlots was last read by P . C(g - kPSlots); O may be
        // rescaled only after P . C(g - 1)
        if (g >= kPSlots &&
            !(ok = wwait(bar(PV_DONE + ((g - kPSlots) & 1)), ((g - kPSlots) >> 1) & 1)))
          break;
        if (__any_sync(0xffffffffu, resc)) {
          if (!(ok = wwait(bar(PV_DONE + ((g - 1) & 1)), ((g - 1) >> 1) & 1))) break;
          tc_fence_after();
          for (int c0 = 0; c0 < d_c; c0 += 32) {
            float o[32];
            tmem_ld32(tmem + lane_base + kTmemO + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tmem + lane_base + kTmemO + c0, o);
          }
          tmem_wait_st();
        }
        // P row: 128-byte blocks of kCols tokens, 16-byte chunk k of row r
        // at k ^ (r & 7)
        const uint32_t prow = sbase + Lay::kOffP + (g % kPSlots) * Lay::kPSlot + row * 128;
        const uint32_t sw = static_cast<uint32_t>(row & 7);
        if (kTf32) {
#pragma unroll
          for (int blk = 0; blk < 2; ++blk)
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float* v = pr + 32 * blk + 4 * k;
              st_shared_v4(prow + blk * kQBlkBytes + ((static_cast<uint32_t>(k) ^ sw) << 4),
                           __float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                           __float_as_uint(v[3]));
            }
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 h2 = __floats2bfloat162_rn(pr[8 * k + 2 * e], pr[8 * k + 2 * e + 1]);
              w[e] = *reinterpret_cast<const uint32_t*>(&h2);
            }
            st_shared_v4(prow + ((static_cast<uint32_t>(k) ^ sw) << 4), w[0], w[1], w[2], w[3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(P_FULL + (g & 1)));
      }
      if (!ok) break;
      // ---- epilogue: u = O / l for this row
      if (!(ok = wwait(bar(PV_DONE + ((g - 1) & 1)), ((g - 1) >> 1) & 1))) break;
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const size_t orow = sg.whole ? (size_t)(sg.b * p.s_q + r_row) * p.n_h + head
                                   : ((size_t)(p.split_base[sg.b] + sg.part) * p.s_q + r_row) * p.n_h + head;
      for (int c0 = 0; c0 < d_c; c0 += 32) {
        float o[32];
        tmem_ld32(tmem + lane_base + kTmemO + c0, o);
        tmem_wait_ld();
        if (!live) continue;
        if (!sg.whole || p.out_f32) {
          float* dst = (sg.whole ? static_cast<float*>(p.u) : p.part_u) + orow * d_c + c0;
#pragma unroll
          for (int k = 0; k < 32; k += 4)
            *reinterpret_cast<float4*>(dst + k) =
                make_float4(o[k] * inv, o[k + 1] * inv, o[k + 2] * inv, o[k + 3] * inv);
        } else {
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.u) + orow * d_c + c0;
#pragma unroll
          for (int k = 0; k < 32; k += 8) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 h2 = __floats2bfloat162_rn(o[k + 2 * e] * inv, o[k + 2 * e + 1] * inv);
              w[e] = *reinterpret_cast<const uint32_t*>(&h2);
            }
            *reinterpret_cast<uint4*>(dst + k) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      if (live) {
        const float lse = l_exact > 0.f ? (m + log2f(l_exact)) * 0.69314718055994531f : -INFINITY;
        if (sg.whole) {
          if (p.lse != nullptr) p.lse[orow] = lse;
        } else {
          p.part_lse[orow] = lse;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(O_FREE));
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool decode_small_sm100_supported(bool bf16, int d_c, int d_R) {
  const int W = d_c + d_R;
  if (bf16) return d_c % 64 == 0 && d_c <= 256 && W <= 256;
  return d_c % 32 == 0 && W <= 128;
}

int decode_small_sm100_prepare() {
  if (cudaFuncSetAttribute(decode_small_sm100_kernel<true, false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)Layout<true, false>::kSmem) != cudaSuccess ||
      cudaFuncSetAttribute(decode_small_sm100_kernel<false, false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)Layout<false, false>::kSmem) != cudaSuccess ||
      cudaFuncSetAttribute(decode_small_sm100_kernel<false, true>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)Layout<false, true>::kSmem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return 1;
}

cudaError_t launch_decode_small_sm100(const DecodeArgs& a, const CUtensorMap& q_map,
                                      const CUtensorMap& kv_map, const CUtensorMap& kv_pv_map,
                                      cudaStream_t s) {
  Params p;
  p.q_map = q_map;
  p.kv_map = kv_map;
  p.kv_pv_map = kv_pv_map;
  p.block_table = a.block_table;
  p.seqlens = a.seqlens;
  p.header = a.header;
  p.tile_prefix = a.tile_prefix;
  p.split_base = a.split_base;
  p.chunk_t = a.chunk_t;
  p.chunk_b = a.chunk_b;
  p.u = a.u;
  p.lse = a.lse;
  p.part_u = a.part_u;
  p.part_lse = a.part_lse;
  p.err = a.err;
  p.B = a.B;
  p.s_q = a.s_q;
  p.n_h = a.n_h;
  p.d_c = a.d_c;
  p.max_pages = a.max_pages;
  p.page_size = a.page_size;
  p.num_pages = a.num_pages;
  const int cols = a.bf16 ? 64 : 32;
  p.blocks = (a.d_c + a.d_R + cols - 1) / cols;
  p.out_f32 = a.out_f32 ? 1 : 0;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.num_chunks * a.s_q, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = a.bf16 ? Layout<false, false>::kSmem : Layout<true, false>::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 1 : 0;
  return a.bf16 ? cudaLaunchKernelEx(&cfg, decode_small_sm100_kernel<false, false>, p)
                : cudaLaunchKernelEx(&cfg, decode_small_sm100_kernel<true, false>, p);
}

cudaError_t launch_decode_gqa_sm100(const DecodeArgs& a, const GqaShape& gs, const CUtensorMap& q_map,
                                    const CUtensorMap& kv_map, const CUtensorMap& kr_map,
                                    cudaStream_t s) {
  Params p;
  memset(&p, 0, sizeof(p));
  p.q_map = q_map;
  p.kv_map = kv_map;
  p.kr_map = kr_map;
  p.block_table = a.block_table;
  p.seqlens = a.seqlens;
  p.header = a.header;
  p.tile_prefix = a.tile_prefix;
  p.split_base = a.split_base;
  p.chunk_t = a.chunk_t;
  p.chunk_b = a.chunk_b;
  p.u = a.u;
  p.lse = a.lse;
  p.part_u = a.part_u;
  p.part_lse = a.part_lse;
  p.err = a.err;
  p.B = a.B;
  p.s_q = a.s_q;
  p.n_h = a.n_h;
  p.d_c = a.d_c;  // = d_v: the output width
  p.max_pages = a.max_pages;
  p.page_size = a.page_size;
  p.num_pages = a.num_pages;
  p.n_g = gs.n_g;
  p.hpg = a.n_h / gs.n_g;
  p.d_h = gs.d_h;
  p.d_v = gs.d_v;
  p.nbk = gs.d_h / 64;
  p.nbr = (gs.d_R + 63) / 64;
  p.nbv = gs.d_v / 64;
  p.blocks = p.nbk + p.nbr;
  p.out_f32 = a.out_f32 ? 1 : 0;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.num_chunks * gs.n_g, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Layout<false, true>::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, decode_small_sm100_kernel<false, true>, p);
}

}  // namespace mla
