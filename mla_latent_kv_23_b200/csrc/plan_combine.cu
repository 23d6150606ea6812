// Plan and combine stages of mla_decode.
//
// plan:    per-sequence tile counts, their prefix sum, the chunk size, and the
//          first partial row of every sequence that is cut into several
//          chunks (one block; B is small).
// combine: for every row cut into pieces, merge the partial results by their
//          log-sum-exp: lse = log sum_s exp(lse_s), u = sum_s exp(lse_s - lse) u_s
//          (the split-KV merge of softmax attention; exact up to rounding).
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"

namespace mla {
namespace {

constexpr int kPlanThreads = 1024;

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
                                                            int* split_base, int* err) {
  __shared__ int warp_sums[32];
  int carry = 0, total = 0;
  for (int base = 0; base < B; base += blockDim.x) {
    const int i = base + threadIdx.x;
    int tiles = 0;
    if (i < B) {
      const int L = seqlens[i];
      if (L < s_q || L > max_len) atomicOr(err, MLA_DEVFLAG_BAD_SEQLEN);
      else tiles = (L + kTileTokens - 1) / kTileTokens;
    }
    const int incl = block_scan(tiles, warp_sums, &total);
    if (i < B) tile_prefix[i] = carry + incl - tiles;
    carry += total;
  }
  const int T = carry;
  const int cs = T > 0 ? (T + num_chunks - 1) / num_chunks : 1;
  if (threadIdx.x == 0) tile_prefix[B] = T;
  __syncthreads();
  carry = 0;
  for (int base = 0; base < B; base += blockDim.x) {
    const int i = base + threadIdx.x;
    int pieces = 0;
    if (i < B) {
      const int t0 = tile_prefix[i], t1 = tile_prefix[i + 1];
      if (t1 > t0) {
        const int n = (t1 - 1) / cs - t0 / cs + 1;
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
    header[1] = cs;
    header[2] = num_chunks;
    header[3] = carry * s_q;
  }
}

constexpr int kCombineThreads = 128;
constexpr int kCombineHeads = 4;  // heads per block

template <bool kBf16>
__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const int* __restrict__ tile_prefix, const int* __restrict__ split_base,
                   const float* __restrict__ part_u, const float* __restrict__ part_lse,
                   void* __restrict__ u_out, float* __restrict__ lse_out, int s_q, int n_h,
                   int d_c) {
  const int b = blockIdx.x / s_q, r = blockIdx.x % s_q;
  const int nsplit = split_base[b + 1] - split_base[b];
  const bool empty = tile_prefix[b + 1] == tile_prefix[b];
  if (nsplit == 0 && !empty) return;  // written directly by the attend stage
  const int h0 = blockIdx.y * kCombineHeads;
  for (int h = h0; h < min(h0 + kCombineHeads, n_h); ++h) {
    const size_t orow = (static_cast<size_t>(b) * s_q + r) * n_h + h;
    float m = -INFINITY;
    for (int s = 0; s < nsplit; ++s) {
      const size_t slot = static_cast<size_t>(split_base[b] + s) * s_q + r;
      m = fmaxf(m, part_lse[slot * n_h + h]);
    }
    float z = 0.f;
    if (m != -INFINITY)
      for (int s = 0; s < nsplit; ++s) {
        const size_t slot = static_cast<size_t>(split_base[b] + s) * s_q + r;
        z += expf(part_lse[slot * n_h + h] - m);
      }
    const float lse_all = (m == -INFINITY) ? -INFINITY : m + logf(z);
    for (int c = threadIdx.x * 4; c < d_c; c += kCombineThreads * 4) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      if (m != -INFINITY)
        for (int s = 0; s < nsplit; ++s) {
          const size_t slot = static_cast<size_t>(split_base[b] + s) * s_q + r;
          const float w = expf(part_lse[slot * n_h + h] - lse_all);
          const float4 v = *reinterpret_cast<const float4*>(part_u + (slot * n_h + h) * d_c + c);
          acc.x += w * v.x;
          acc.y += w * v.y;
          acc.z += w * v.z;
          acc.w += w * v.w;
        }
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
    if (lse_out != nullptr && threadIdx.x == 0) lse_out[orow] = lse_all;
  }
}

}  // namespace

cudaError_t launch_plan(const DecodeArgs& a, cudaStream_t s) {
  plan_kernel<<<1, kPlanThreads, 0, s>>>(a.seqlens, a.B, a.s_q, a.max_pages * a.page_size,
                                         a.num_chunks, a.header, a.tile_prefix, a.split_base,
                                         a.err);
  return cudaGetLastError();
}

cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t s) {
  dim3 grid(a.B * a.s_q, (a.n_h + kCombineHeads - 1) / kCombineHeads);
  if (a.bf16)
    combine_kernel<true><<<grid, kCombineThreads, 0, s>>>(a.tile_prefix, a.split_base, a.part_u,
                                                          a.part_lse, a.u, a.lse, a.s_q, a.n_h,
                                                          a.d_c);
  else
    combine_kernel<false><<<grid, kCombineThreads, 0, s>>>(a.tile_prefix, a.split_base, a.part_u,
                                                           a.part_lse, a.u, a.lse, a.s_q, a.n_h,
                                                           a.d_c);
  return cudaGetLastError();
}

}  // namespace mla
