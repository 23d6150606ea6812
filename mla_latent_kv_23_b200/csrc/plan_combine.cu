// Plan and combine stages of mla_decode.
//
// plan:    per-sequence tile counts and their prefix sum; the cut of the tile
//          line into KV chunks; the first tile, sequence, piece index and
//          that sequence's tile range of every chunk; and the first partial row of every sequence that is
//          cut into several chunks (one block; B is small).  Two cuts:
//          * aligned: when every sequence has the same tile count t and the
//            chunks divide among the sequences (c = chunks / B pieces each),
//            sequence b takes chunks [c b, c b + c), piece k its tiles
//            [k t / c, (k + 1) t / c): no chunk holds two sequences;
//          * line: uniform on a line that charges every sequence start
//            kSegCostTiles units, so a chunk that starts new sequences takes
//            fewer tiles.
//          The aligned cut is taken when its largest chunk is no bigger than
//          the line's units per chunk plus one start charge (a chunk that
//          holds two sequences pays a second query load and epilogue, which
//          the charge only estimates).
// combine: for every row cut into pieces, merge the partial results by their
//          log-sum-exp: lse = log sum_s exp(lse_s), u = sum_s exp(lse_s - lse) u_s
//          (the split-KV merge of softmax attention; exact up to rounding).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <limits.h>
#include <math.h>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

constexpr int kPlanThreads = 256;
constexpr int kPlanSmemSeqs = 4096;  // batches up to this size keep the tile prefix on chip

// Inclusive scan of one int per thread across the block; returns the
// thread's inclusive value and writes the block total to *total.
__device__ int block_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int s = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < nw) warp_sums[lane] = s;
  }
  __syncthreads();
  const int res = x + (warp > 0 ? warp_sums[warp - 1] : 0);
  *total = warp_sums[(blockDim.x >> 5) - 1];
  __syncthreads();
  return res;
}

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int* __restrict__ seqlens, int B,
                                                            int s_q, int max_len, int num_chunks,
                                                            int* header, int* tile_prefix,
                                                            int* split_base, int* chunk_t,
                                                            int* chunk_b, int* err) {
  // let the attend kernel start its prologue while this one runs
  ptx::pdl_launch_dependents();
  __shared__ int warp_sums[32];
  __shared__ int tp_s[kPlanSmemSeqs + 1];
  __shared__ int tiles_min, tiles_max;
  const bool on_chip = B <= kPlanSmemSeqs;
  constexpr int K = kSegCostTiles;
  if (threadIdx.x == 0) {
    tiles_min = INT_MAX;
    tiles_max = 0;
  }
  __syncthreads();
  int carry = 0, total = 0;
  for (int base = 0; base < B; base += blockDim.x) {
    const int i = base + threadIdx.x;
    int tiles = 0;
    if (i < B) {
      const int L = seqlens[i];
      if (L < s_q || L > max_len) atomicOr(err, MLA_DEVFLAG_BAD_SEQLEN);
      else tiles = (L + kTileTokens - 1) / kTileTokens;
      atomicMin(&tiles_min, tiles);
      atomicMax(&tiles_max, tiles);
    }
    const int incl = block_scan(tiles, warp_sums, &total);
    if (i < B) {
      tile_prefix[i] = carry + incl - tiles;
      if (on_chip) tp_s[i] = carry + incl - tiles;
    }
    carry += total;
  }
  const int T = carry;
  // the line: sequence b takes units [tp[b] + K b, tp[b + 1] + K (b + 1)),
  // the first K of them for its start-up; tile t of sequence b is unit
  // t + K (b + 1)
  const long long V = (long long)T + (long long)K * B;
  const int units = V > 0 ? (int)((V + num_chunks - 1) / num_chunks) : 1;
  // the aligned cut: c pieces per sequence of t_seq tiles
  const int t_seq = tiles_max;
  const int cps = B > 0 ? min(num_chunks / B, t_seq) : 0;
  const bool aligned = B > 0 && tiles_min == tiles_max && t_seq > 0 && cps >= 1 &&
                       (t_seq + cps - 1) / cps <= units + K;
  if (threadIdx.x == 0) {
    tile_prefix[B] = T;
    if (on_chip) tp_s[B] = T;
  }
  __syncthreads();
  // the searches below read the prefix from shared memory when it fits
  const int* tp = on_chip ? tp_s : tile_prefix;
  for (int c = threadIdx.x; c <= num_chunks; c += blockDim.x) {
    int t = T, sb = B, part = 0;
    if (aligned) {
      if (c < B * cps) {
        sb = c / cps;
        part = c % cps;
        t = tp[sb] + (int)((long long)part * t_seq / cps);
      }
    } else {
      // chunk c starts at unit c * units: at the first tile at or after it
      const long long x = (long long)c * units;
      if (x < V) {
        int lo = 0, hi = B;  // largest b with tp[b] + K b <= x
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if ((long long)tp[mid] + (long long)K * mid <= x) lo = mid; else hi = mid;
        }
        const long long off = x - ((long long)tp[lo] + (long long)K * (lo + 1));
        t = tp[lo] + (off > 0 ? (int)off : 0);
        sb = lo;
        // pieces of sequence lo are numbered from the chunk of its first tile
        if (t > tp[lo]) part = c - (int)(((long long)tp[lo] + (long long)K * (lo + 1)) / units);
      }
    }
    chunk_t[c] = t;
    if (c < num_chunks)  // the record: sequence, piece, and the sequence's tiles on the line
      *reinterpret_cast<int4*>(chunk_b + 4 * c) =
          make_int4(sb, part, sb < B ? tp[sb] : T, sb < B ? tp[sb + 1] : T);
  }
  carry = 0;
  for (int base = 0; base < B; base += blockDim.x) {
    const int i = base + threadIdx.x;
    int pieces = 0;
    if (i < B) {
      const int t0 = tp[i], t1 = tp[i + 1];
      if (aligned) {
        pieces = cps > 1 ? cps : 0;
      } else if (t1 > t0) {
        const long long u0 = (long long)t0 + (long long)K * (i + 1);
        const int n = (int)((u0 + (t1 - t0) - 1) / units - u0 / units) + 1;
        pieces = n > 1 ? n : 0;
      }
    }
    const int incl = block_scan(pieces, warp_sums, &total);
    if (i < B) split_base[i] = carry + incl - pieces;
    carry += total;
  }
  if (threadIdx.x == 0) {
    split_base[B] = carry;
    header[0] = T;
    header[1] = units;
    header[2] = num_chunks;
    header[3] = carry * s_q;
    header[4] = K;
    header[5] = aligned ? 1 : 0;
    header[6] = aligned ? B * cps : num_chunks;  // chunks that hold tiles (at most)
  }
}

constexpr int kCombineWarps = 8;
constexpr int kCombineThreads = 32 * kCombineWarps;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Four consecutive partial values as floats (partials are fp32, or bf16 when
// the attend stage stored them so).
template <bool kPartBf16>
__device__ __forceinline__ float4 load4(const void* base, size_t idx) {
  if (kPartBf16) {
    const uint2 r = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(base) + idx);
    const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
    const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
  }
  return *reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
}

// One warp per output row (b, r, head).  Lane s holds the weight of split s
// (32 at a time); the column loop broadcasts it with a shuffle, so every
// split costs one exp per row and one 4-value load per lane per 128 columns.
template <bool kBf16, bool kPartBf16>
__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const int* __restrict__ tile_prefix, const int* __restrict__ split_base,
                   const void* __restrict__ part_u, const float* __restrict__ part_lse,
                   void* __restrict__ u_out, float* __restrict__ lse_out, int s_q, int n_h,
                   int d_c, int rows) {
  ptx::pdl_wait_previous();
  ptx::pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int h = row % n_h, br = row / n_h;
  const int b = br / s_q, r = br % s_q;
  const int nsplit = split_base[b + 1] - split_base[b];
  const bool empty = tile_prefix[b + 1] == tile_prefix[b];
  if (nsplit == 0 && !empty) return;  // written directly by the attend stage
  const size_t slot0 = static_cast<size_t>(split_base[b]) * s_q + r;  // slot of split s: slot0 + s*s_q
  float m = -INFINITY;
  for (int s = lane; s < nsplit; s += 32) m = fmaxf(m, part_lse[(slot0 + (size_t)s * s_q) * n_h + h]);
  m = warp_max(m);
  float z = 0.f;
  if (m != -INFINITY)
    for (int s = lane; s < nsplit; s += 32) z += expf(part_lse[(slot0 + (size_t)s * s_q) * n_h + h] - m);
  z = warp_sum(z);
  const float lse_all = (m == -INFINITY) ? -INFINITY : m + logf(z);
  for (int c = lane * 4; c < d_c; c += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (m != -INFINITY) {
      for (int s0 = 0; s0 < nsplit; s0 += 32) {
        const int s_me = s0 + lane;
        const float w_me = s_me < nsplit
            ? expf(part_lse[(slot0 + (size_t)s_me * s_q) * n_h + h] - lse_all) : 0.f;
        const int n_here = min(32, nsplit - s0);
#pragma unroll 4
        for (int k = 0; k < n_here; ++k) {
          const float w = __shfl_sync(0xffffffffu, w_me, k);
          const size_t slot = slot0 + (size_t)(s0 + k) * s_q;
          const float4 v = load4<kPartBf16>(part_u, (slot * n_h + h) * d_c + c);
          acc.x += w * v.x;
          acc.y += w * v.y;
          acc.z += w * v.z;
          acc.w += w * v.w;
        }
      }
    }
    const size_t orow = static_cast<size_t>(br) * n_h + h;
    if (kBf16) {
      __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
      __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&lo);
      pk.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(u_out) + orow * d_c + c) = pk;
    } else {
      *reinterpret_cast<float4*>(static_cast<float*>(u_out) + orow * d_c + c) = acc;
    }
  }
  if (lse_out != nullptr && lane == 0) lse_out[static_cast<size_t>(br) * n_h + h] = lse_all;
}

// Merge of the partials with d_c = 512 (the tensor-core path): bf16, fp16 or
// fp32 partials (kPart 1, 2, 0), bf16 or fp32 u.  One warp per output row;
// lane l owns columns [16 l, 16 l + 16).  The partials of up to kGroup splits
// (8 16-bit or 4 fp32 rows: 32 or 64 bytes per lane each) are loaded before
// any is used, so a row waits for memory about once per group instead of
// once per split.
template <bool kOutBf16, int kPart>
__global__ void __launch_bounds__(kCombineThreads)
    combine512_kernel(const int* __restrict__ tile_prefix, const int* __restrict__ split_base,
                      const void* __restrict__ part_u, const float* __restrict__ part_lse,
                      void* __restrict__ u_out, float* __restrict__ lse_out, int s_q, int n_h,
                      int rows) {
  constexpr int kDc = 512;
  constexpr bool k16 = kPart != 0;
  constexpr int kGroup = k16 ? 8 : 4;
  constexpr int kVecs = k16 ? 2 : 4;  // 16-byte loads per lane per partial row
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
  // The tile prefix and split bases come from the plan stage or from the
  // attend stage itself: read them after the wait.
  ptx::pdl_wait_previous();
  ptx::pdl_launch_dependents();
  int sb0 = 0, sb1 = 0, tp0 = 0, tp1 = 0;
  int h = 0, br = 0, r = 0;
  if (row < rows) {
    h = row % n_h;
    br = row / n_h;
    const int b = br / s_q;
    r = br % s_q;
    sb0 = split_base[b];
    sb1 = split_base[b + 1];
    tp0 = tile_prefix[b];
    tp1 = tile_prefix[b + 1];
  }
  if (row >= rows) return;
  const int nsplit = sb1 - sb0;
  if (nsplit == 0 && tp1 != tp0) return;  // written directly by the attend stage
  const size_t slot0 = static_cast<size_t>(sb0) * s_q + r;  // slot of split s: slot0 + s*s_q
  auto lse_of = [&](int s) { return part_lse[(slot0 + (size_t)s * s_q) * n_h + h]; };
  auto load_group = [&](int s0, uint4 (&v)[kGroup][kVecs]) {
#pragma unroll
    for (int k = 0; k < kGroup; ++k) {
      if (s0 + k < nsplit) {
        const size_t e0 = ((slot0 + (size_t)(s0 + k) * s_q) * n_h + h) * kDc + 16 * lane;
        const uint4* src = k16
            ? reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(part_u) + e0)
            : reinterpret_cast<const uint4*>(static_cast<const float*>(part_u) + e0);
#pragma unroll
        for (int i = 0; i < kVecs; ++i) v[k][i] = src[i];
      }
    }
  };
  // the first group of partial rows is requested together with the
  // statistics, so one memory round trip covers rows with few pieces
  uint4 v[kGroup][kVecs];
  load_group(0, v);
  // one pass: per-lane running (max, sum of exp), then the warp's
  float m = -INFINITY, z = 0.f;
  for (int s = lane; s < nsplit; s += 32) {
    const float x = lse_of(s);
    if (x > m) {
      z = z * expf(m - x) + 1.f;
      m = x;
    } else if (x != -INFINITY) {
      z += expf(x - m);
    }
  }
  const float m_all = warp_max(m);
  z = warp_sum(m == -INFINITY ? 0.f : z * expf(m - m_all));
  const float lse_all = (m_all == -INFINITY) ? -INFINITY : m_all + logf(z);
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  if (m_all != -INFINITY) {
    for (int s0 = 0; s0 < nsplit; s0 += kGroup) {
      if (s0 > 0) load_group(s0, v);
      const int n_here = min(kGroup, nsplit - s0);
      const float w_me = lane < n_here ? expf(lse_of(s0 + lane) - lse_all) : 0.f;
#pragma unroll
      for (int k = 0; k < kGroup; ++k) {
        const float w = __shfl_sync(0xffffffffu, w_me, k);
        if (k < n_here) {
          if (kPart == 1) {
            const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(v[k]);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float2 f = __bfloat1622float2(x[e]);
              acc[2 * e] += w * f.x;
              acc[2 * e + 1] += w * f.y;
            }
          } else if (kPart == 2) {
            const __half2* x = reinterpret_cast<const __half2*>(v[k]);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float2 f = __half22float2(x[e]);
              acc[2 * e] += w * f.x;
              acc[2 * e + 1] += w * f.y;
            }
          } else {
            const float* x = reinterpret_cast<const float*>(v[k]);
#pragma unroll
            for (int e = 0; e < 16; ++e) acc[e] += w * x[e];
          }
        }
      }
    }
  }
  const size_t orow = static_cast<size_t>(br) * n_h + h;
  if (kOutBf16) {
    uint32_t pk[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const __nv_bfloat162 t = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
      pk[e] = *reinterpret_cast<const uint32_t*>(&t);
    }
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(u_out) + orow * kDc + 16 * lane);
    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  } else {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(u_out) + orow * kDc + 16 * lane);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      dst[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
  }
  if (lse_out != nullptr && lane == 0) lse_out[orow] = lse_all;
}

}  // namespace

cudaError_t launch_plan(const DecodeArgs& a, cudaStream_t s) {
  plan_kernel<<<1, kPlanThreads, 0, s>>>(a.seqlens, a.B, a.s_q, a.max_pages * a.page_size,
                                         a.num_chunks, a.header, a.tile_prefix, a.split_base,
                                         a.chunk_t, a.chunk_b, a.err);
  return cudaGetLastError();
}

cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t s) {
  const int rows = a.B * a.s_q * a.n_h;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((rows + kCombineWarps - 1) / kCombineWarps, 1, 1);
  cfg.blockDim = dim3(kCombineThreads, 1, 1);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 1 : 0;
  const int* tp = a.tile_prefix;
  const int* sb = a.split_base;
  const void* pu = a.part_u;
  const float* pl = a.part_lse;
  const bool out_bf16 = !a.out_f32;
  if (a.d_c == 512) {
    if (a.part_bf16)
      return out_bf16 ? cudaLaunchKernelEx(&cfg, combine512_kernel<true, 1>, tp, sb, pu, pl, a.u,
                                           a.lse, a.s_q, a.n_h, rows)
                      : cudaLaunchKernelEx(&cfg, combine512_kernel<false, 1>, tp, sb, pu, pl,
                                           a.u, a.lse, a.s_q, a.n_h, rows);
    if (a.part_f16)
      return out_bf16 ? cudaLaunchKernelEx(&cfg, combine512_kernel<true, 2>, tp, sb, pu, pl, a.u,
                                           a.lse, a.s_q, a.n_h, rows)
                      : cudaLaunchKernelEx(&cfg, combine512_kernel<false, 2>, tp, sb, pu, pl,
                                           a.u, a.lse, a.s_q, a.n_h, rows);
    return out_bf16 ? cudaLaunchKernelEx(&cfg, combine512_kernel<true, 0>, tp, sb, pu, pl, a.u,
                                         a.lse, a.s_q, a.n_h, rows)
                    : cudaLaunchKernelEx(&cfg, combine512_kernel<false, 0>, tp, sb, pu, pl, a.u,
                                         a.lse, a.s_q, a.n_h, rows);
  }
  if (out_bf16 && a.part_bf16)
    return cudaLaunchKernelEx(&cfg, combine_kernel<true, true>, tp, sb, pu, pl, a.u, a.lse, a.s_q,
                              a.n_h, a.d_c, rows);
  if (out_bf16)
    return cudaLaunchKernelEx(&cfg, combine_kernel<true, false>, tp, sb, pu, pl, a.u, a.lse, a.s_q,
                              a.n_h, a.d_c, rows);
  return cudaLaunchKernelEx(&cfg, combine_kernel<false, false>, tp, sb, pu, pl, a.u, a.lse, a.s_q,
                            a.n_h, a.d_c, rows);
}

}  // namespace mla
