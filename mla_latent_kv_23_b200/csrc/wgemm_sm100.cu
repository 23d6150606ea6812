// Weight-streaming projections on the tensor cores (sm_100a):
//     Y[m, t] = sum_k W[m, k] X[t, k]
// for the token-count-wide products around the attention: the weights W
// (megabytes) are read from HBM once, the activations X (a few token rows)
// are small.  Three uses, each with its own epilogue:
//   kQuery  ("MLA deep compression", absorption section, score equation, and
//            decoupled-RoPE section): W = [W^Q ; W^QR] stacked by rows,
//            X = h.  Rows of W^Q_i give q^nope_i = W^Q_i h (128 values per
//            head); the CTA that completes head i's rows applies the second
//            product q^lat_i = W^UK_i^T q^nope_i on the tensor cores and writes
//            q[t, i, 0:d_c].  Rows of W^QR give W^QR_i h, rotated (RoPE) into
//            q[t, i, d_c:d_c + d_R].  No precomputed W^QK is read.
//   kCache  (low-rank projection section and decoupled-RoPE section):
//            W = [W^DKV ; W^KR], X = h; writes the paged cache rows
//            [c || RoPE(k^R)] of the new tokens through the block table.
//   kStore  ("Attention-head anatomy" section 5, W^UV folded into W^O):
//            Y = W X written as y[t, m]; X may hold each token twice (two
//            bf16 terms of an fp32 row), whose products are added.
//   kQueryAbsorbed (absorption section, score equation, with the offline
//            W^QK = W^UK^T W^Q): W = [W^QK ; W^QR], rows of W^QK_i give
//            q[t, i, 0:d_c] directly, rows of W^QR as in kQuery.
//
// One CTA per (128-row tile of W, slice of K): M = 128, N = token rows
// padded to 16, K streamed through a TMA pipeline of 64-column blocks with
// 128-byte swizzle.  With several K slices, every CTA adds its partial tile
// into an fp32 workspace (red.global.add) and the last one of the tile (a
// counter) runs the epilogue and returns the workspace tile and the counter
// to zero, so the workspace is zero again after every call.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {
using namespace ptx;

constexpr int kThreads = 128;
constexpr int kStages = 6;
constexpr int kMaxN = 64;                       // token rows per CTA (padded)
constexpr uint32_t kWBlk = 128 * 128;           // 128 rows x 64 bf16
constexpr uint32_t kXBlk = kMaxN * 128;         // up to 64 rows x 64 bf16
constexpr uint32_t kStageBytes = kWBlk + kXBlk;
// the query epilogue reuses the pipeline area: W^UK_i (d_h = 128 rows x
// d_c = 512 columns, 8 blocks of 16 KB) and q^nope_i as two bf16 terms
// (2 x 2 blocks of up to 64 rows x 128 bytes)
constexpr uint32_t kUkBytes = 8 * kWBlk;
constexpr uint32_t kAreaBytes =
    (kStages * kStageBytes > kUkBytes + 4 * kXBlk) ? kStages * kStageBytes : kUkBytes + 4 * kXBlk;

enum Bar { FULL = 0, EMPTY = FULL + kStages, MMA_DONE = EMPTY + kStages, UK_FULL, MMA2_DONE, BAR_COUNT };

struct Params {
  CUtensorMap w_map[2];  // the two weight tensors stacked along M: box 64 x 128 rows
  CUtensorMap x_map;     // X [N, K]: box 64 x n_pad rows
  CUtensorMap uk_map;    // kQuery: W^UK as [n_h * 128, d_c], box 64 x 128 rows
  int tiles0;            // M tiles of the first tensor; the rest come from the second
  int K, N, n_pad, ksplit;
  float* acc;            // [tiles][128][n_pad] fp32 workspace (zero on entry and exit)
  int* counters;         // [tiles]
  int* err;
  int mode;              // 0 kQuery, 1 kCache, 2 kStore, 3 kQueryAbsorbed
  // kQuery: q [N, n_h, d_c + d_R]; kCache: the cache; kStore: y [N / pair, ldo]
  __nv_bfloat16* out;
  int n_h, d_c, d_R, ldo, pair;
  const int* pos;        // kQuery, kCache: position of token t
  const int* seq;        // kCache: sequence of token t
  const int* block_table;
  int max_pages, page_size, num_pages;
  double log_base;       // ln(rope base)
};

// cos / sin of pos * base^(-2k/d) with the angle reduced in fp64 (positions
// reach 10^5 radians, where an fp32 angle is off by ~1e-2)
__device__ __forceinline__ void rope_cs(int pos, int k2, int d, double log_base, float& c, float& s) {
  const double ang = (double)pos * exp(-(double)k2 / (double)d * log_base);
  const double red = ang - 6.283185307179586 * floor(ang / 6.283185307179586);
  double sd, cd;
  sincos(red, &sd, &cd);
  c = (float)cd;
  s = (float)sd;
}

__global__ void __launch_bounds__(kThreads, 1) wgemm_sm100_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (sbase - raw);
  const uint32_t off_bar = kAreaBytes;
  auto bar = [&](int i) -> uint32_t { return sbase + off_bar + 8u * i; };
  const uint32_t tmem_slot = sbase + off_bar + BAR_COUNT * 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, slice = blockIdx.y;
  const bool second = tile >= p.tiles0;
  const int row0 = (second ? tile - p.tiles0 : tile) * 128;  // first row within its tensor
  const int kb_total = p.K / 64;
  const int kb0 = (int)((long long)kb_total * slice / p.ksplit);
  const int kb1 = (int)((long long)kb_total * (slice + 1) / p.ksplit);
  const uint32_t xblk = p.n_pad * 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(FULL + s), 1);
      mbar_init(bar(EMPTY + s), 1);
    }
    mbar_init(bar(MMA_DONE), 1);
    mbar_init(bar(UK_FULL), 1);
    mbar_init(bar(MMA2_DONE), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(base + (tmem_slot - sbase));
  // the weights never depend on the previous kernel; X may
  pdl_wait_previous();
  pdl_launch_dependents();

  bool ok = true;
  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- producer
    const CUtensorMap* wm = &p.w_map[second ? 1 : 0];
    prefetch_tmap(wm);
    prefetch_tmap(&p.x_map);
    for (int kb = kb0, i = 0; kb < kb1; ++kb, ++i) {
      const int s = i % kStages;
      if (!(ok = mbar_wait(bar(EMPTY + s), ((i / kStages) & 1) ^ 1, p.err, MLA_DEVFLAG_TIMEOUT))) break;
      const uint32_t st = sbase + s * kStageBytes;
      mbar_arrive_expect_tx(bar(FULL + s), kWBlk + xblk);
      tma_load_2d(st, wm, bar(FULL + s), kb * 64, row0);
      tma_load_2d(st + kWBlk, &p.x_map, bar(FULL + s), kb * 64, 0);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    const uint32_t idesc = idesc_bf16(128, p.n_pad, false);
    uint32_t acc = 0;
    for (int kb = kb0, i = 0; kb < kb1; ++kb, ++i) {
      const int s = i % kStages;
      if (!(ok = mbar_wait(bar(FULL + s), (i / kStages) & 1, p.err, MLA_DEVFLAG_TIMEOUT))) break;
      tc_fence_after();
      const uint32_t st = sbase + s * kStageBytes;
      for (int ks = 0; ks < 4; ++ks) {
        umma_f16_ss(tmem, smem_desc(st + ks * 32, 16, 1024, kLayoutSW128),
                    smem_desc(st + kWBlk + ks * 32, 16, 1024, kLayoutSW128), idesc, acc);
        acc = 1;
      }
      umma_commit(bar(EMPTY + s));
    }
    umma_commit(bar(MMA_DONE));
  }
  __syncwarp();
  // ------------------------------------------------------------ reduction
  bool live = true;
  if (threadIdx.x == 0) live = mbar_wait(bar(MMA_DONE), 0, p.err, MLA_DEVFLAG_TIMEOUT);
  live = __syncthreads_and(live && ok);
  tc_fence_after();
  // thread = row m of the tile; vals[t] = Y[row0 + m, t]
  const int m = threadIdx.x;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  float vals[kMaxN];
  for (int c0 = 0; c0 < p.n_pad; c0 += 32) {
    float v[32];
    tmem_ld32(tmem + lane_base + c0, v);
    tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < 32; ++k)
      if (c0 + k < kMaxN) vals[c0 + k] = v[k];
  }
  bool finisher = true;
  if (p.ksplit > 1) {
    float* at = p.acc + ((size_t)tile * 128 + m) * p.n_pad;
    for (int t = 0; t < p.n_pad; ++t)
      if (live) atomicAdd(at + t, vals[t]);
    __threadfence();
    __syncthreads();
    __shared__ int s_last;
    if (threadIdx.x == 0) s_last = atomicAdd(p.counters + tile, 1) == p.ksplit - 1;
    __syncthreads();
    finisher = s_last != 0;
    if (finisher) {
      __threadfence();
      for (int t = 0; t < p.n_pad; ++t) {
        vals[t] = __ldcg(at + t);
        at[t] = 0.f;  // the workspace is zero again for the next call
      }
      if (threadIdx.x == 0) p.counters[tile] = 0;
    }
  }

  // ------------------------------------------------------------ epilogue
  if (finisher && live) {
    if (p.mode == 2) {
      // kStore: y[t / pair, row] = sum of the pair's products
      const int row = row0 + m;
      if (row < p.ldo) {
        const int nt = p.N / p.pair;
        for (int t = 0; t < nt; ++t) {
          float v = vals[t * p.pair];
          if (p.pair == 2) v += vals[t * 2 + 1];
          p.out[(size_t)t * p.ldo + row] = __float2bfloat16_rn(v);
        }
      }
    } else if (second) {
      // RoPE rows: W^QR (two heads of d_R rows per tile when d_R = 64) or
      // W^KR; pairs (2k, 2k + 1) sit in adjacent threads
      const int r = row0 + m;           // row within the RoPE tensor
      const int head = r / p.d_R, k = r % p.d_R;
      const int k2 = k & ~1;
      const bool valid = p.mode != 1 ? head < p.n_h : r < p.d_R;
      for (int t = 0; t < p.N; ++t) {
        const float x = vals[t];
        const float y = __shfl_xor_sync(0xffffffffu, x, 1);
        if (!valid) continue;
        float c, s;
        rope_cs(p.pos[t], k2, p.d_R, p.log_base, c, s);
        // (x_even, x_odd) -> (x_even c - x_odd s, x_even s + x_odd c)
        const float out = (k & 1) ? (y * s + x * c) : (x * c - y * s);
        if (p.mode != 1) {
          p.out[((size_t)t * p.n_h + head) * (p.d_c + p.d_R) + p.d_c + k] = __float2bfloat16_rn(out);
        } else {
          const int pg_i = p.pos[t] / p.page_size;
          const int page = p.block_table[(size_t)p.seq[t] * p.max_pages + pg_i];
          if (page < 0 || page >= p.num_pages) {
            atomicOr(p.err, MLA_DEVFLAG_BAD_PAGE);
            continue;
          }
          const size_t crow = (size_t)page * p.page_size + p.pos[t] % p.page_size;
          p.out[crow * (p.d_c + p.d_R) + p.d_c + k] = __float2bfloat16_rn(out);
        }
      }
    } else if (p.mode == 3) {
      // rows (head, c) of the flattened W^QK: q[t, head, c]
      const int r = row0 + m, head = r / p.d_c, c = r % p.d_c;
      if (head < p.n_h)
        for (int t = 0; t < p.N; ++t)
          p.out[((size_t)t * p.n_h + head) * (p.d_c + p.d_R) + c] = __float2bfloat16_rn(vals[t]);
    } else if (p.mode == 1) {
      // latent rows c = row0 + m of the new tokens' cache rows
      const int c = row0 + m;
      for (int t = 0; t < p.N; ++t) {
        if (c >= p.d_c) break;
        const int page = p.block_table[(size_t)p.seq[t] * p.max_pages + p.pos[t] / p.page_size];
        if (page < 0 || page >= p.num_pages) {
          atomicOr(p.err, MLA_DEVFLAG_BAD_PAGE);
          continue;
        }
        const size_t crow = (size_t)page * p.page_size + p.pos[t] % p.page_size;
        p.out[crow * (p.d_c + p.d_R) + c] = __float2bfloat16_rn(vals[t]);
      }
    } else {
      // kQuery, head i = tile: q^nope_i [128 x N] -> q^lat_i = W^UK_i^T q^nope_i.
      // B operand: q^nope^T as [n_pad rows (t) x 128 (d)], K-major, two bf16
      // terms (hi, lo), in the swizzled layout; A: W^UK_i [128 (d) x d_c (c)]
      // as the MN-major operand (M = c).
      const int head = tile;
      const uint32_t uk = sbase;                 // 8 blocks of 128 rows (d) x 64 columns (c)
      const uint32_t bq = sbase + kUkBytes;      // [term][d block] n_pad x 128 bytes
      const int kbc = p.d_c / 64;
      if (threadIdx.x == 0) {
        prefetch_tmap(&p.uk_map);
        mbar_arrive_expect_tx(bar(UK_FULL), kbc * kWBlk);
        for (int kb = 0; kb < kbc; ++kb)
          tma_load_2d(uk + kb * kWBlk, &p.uk_map, bar(UK_FULL), kb * 64, head * 128);
      }
      // thread m = d writes element (t, d) of both terms for every t
      const int dblk = m >> 6, dcol = m & 63;
      for (int t = 0; t < p.n_pad; ++t) {
        const float v = t < p.N ? vals[t] : 0.f;
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
        const uint32_t chunk = static_cast<uint32_t>(dcol >> 3) ^ static_cast<uint32_t>(t & 7);
        const uint32_t off = dblk * xblk + t * 128 + (chunk << 4) + (dcol & 7) * 2;
        *reinterpret_cast<__nv_bfloat16*>(base + (bq - sbase) + off) = hi;
        *reinterpret_cast<__nv_bfloat16*>(base + (bq - sbase) + 2 * xblk + off) = lo;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      bool ok2 = true;
      if (threadIdx.x == 0) {
        ok2 = mbar_wait(bar(UK_FULL), 0, p.err, MLA_DEVFLAG_TIMEOUT);
        if (ok2) {
          tc_fence_after();
          // A MN-major (c contiguous): M = 128 c per instruction = two
          // 64-column blocks 16 KB apart; K = 16 rows (d) per instruction
          const uint32_t id2 = idesc_bf16(128, p.n_pad, false) | (1u << 15);
          for (int mc = 0; mc < p.d_c / 128; ++mc) {
            const uint32_t d2 = tmem + 128 + mc * kMaxN;
            uint32_t acc = 0;
            for (int term = 0; term < 2; ++term)
              for (int kk = 0; kk < 8; ++kk) {  // d = 16 kk
                const uint64_t a = smem_desc(uk + (2 * mc) * kWBlk + kk * 2048, kWBlk, 1024, kLayoutSW128);
                const uint64_t b = smem_desc(bq + term * 2 * xblk + (kk >> 2) * xblk + (kk & 3) * 32,
                                             16, 1024, kLayoutSW128);
                umma_f16_ss(d2, a, b, id2, acc);
                acc = 1;
              }
          }
        }
        umma_commit(bar(MMA2_DONE));
        if (!mbar_wait(bar(MMA2_DONE), 0, p.err, MLA_DEVFLAG_TIMEOUT)) ok2 = false;
      }
      ok2 = __syncthreads_and(ok2);
      tc_fence_after();
      if (ok2) {
        for (int mc = 0; mc < p.d_c / 128; ++mc) {
          const int c = mc * 128 + m;
          for (int c0 = 0; c0 < p.n_pad; c0 += 32) {
            float v[32];
            tmem_ld32(tmem + lane_base + 128 + mc * kMaxN + c0, v);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              const int t = c0 + k;
              if (t < p.N)
                p.out[((size_t)t * p.n_h + head) * (p.d_c + p.d_R) + c] = __float2bfloat16_rn(v[k]);
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

constexpr size_t kSmem = kAreaBytes + BAR_COUNT * 8 + 16 + 1024;

}  // namespace

int wgemm_sm100_prepare() {
  if (cudaFuncSetAttribute(wgemm_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return 1;
}

size_t wgemm_workspace_bytes(int tiles, int n_pad) {
  return ((size_t)tiles * 128 * n_pad * sizeof(float) + 255) / 256 * 256 + (size_t)tiles * sizeof(int);
}

// fp32 rows -> pairs of bf16 rows: pairs[2t] = bf16(x[t]), pairs[2t + 1] =
// bf16(x[t] - pairs[2t]); the two terms add back to x within 2^-16 of it.
__global__ void split_rows_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ pairs,
                                  int T, int K) {
  const size_t n = (size_t)T * K;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t t = i / K, k = i % K;
    const float v = x[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    pairs[(2 * t) * K + k] = hi;
    pairs[(2 * t + 1) * K + k] = __float2bfloat16_rn(v - __bfloat162float(hi));
  }
}

cudaError_t launch_split_rows(const float* x, void* pairs, int T, int K, cudaStream_t s) {
  const size_t n = (size_t)T * K;
  const int blocks = (int)std::min<size_t>((n + 255) / 256, 4096);
  split_rows_kernel<<<blocks, 256, 0, s>>>(x, static_cast<__nv_bfloat16*>(pairs), T, K);
  return cudaGetLastError();
}

cudaError_t launch_wgemm(const WgemmLaunch& L, cudaStream_t s) {
  Params p;
  memset(&p, 0, sizeof(p));
  p.w_map[0] = L.w_map[0];
  p.w_map[1] = L.w_map[1];
  p.x_map = L.x_map;
  p.uk_map = L.uk_map;
  p.tiles0 = L.tiles0;
  p.K = L.K;
  p.N = L.N;
  p.n_pad = L.n_pad;
  p.ksplit = L.ksplit;
  const size_t acc_bytes = ((size_t)L.tiles * 128 * L.n_pad * sizeof(float) + 255) / 256 * 256;
  p.acc = static_cast<float*>(L.workspace);
  p.counters = reinterpret_cast<int*>(static_cast<uint8_t*>(L.workspace) + acc_bytes);
  p.err = L.err;
  p.mode = L.mode;
  p.out = static_cast<__nv_bfloat16*>(L.out);
  p.n_h = L.n_h;
  p.d_c = L.d_c;
  p.d_R = L.d_R;
  p.ldo = L.ldo;
  p.pair = L.pair;
  p.pos = L.pos;
  p.seq = L.seq;
  p.block_table = L.block_table;
  p.max_pages = L.max_pages;
  p.page_size = L.page_size;
  p.num_pages = L.num_pages;
  p.log_base = log((double)L.rope_base);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.tiles, L.ksplit, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  return cudaLaunchKernelEx(&cfg, wgemm_sm100_kernel, p);
}

}  // namespace mla
