// Merge of partial decode results over disjoint parts of the same query
// rows' context (context parallelism: each GPU decodes a page range of every
// sequence).  For each row,
//     lse = log sum_r exp(lse_r),    u = sum_r exp(lse_r - lse) u_r
// which is softmax attention over the union of the parts ("MLA deep
// compression", absorption section: u_i = sum_j a_ij c_j with a the softmax
// over all cached positions; exact up to rounding).
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"

namespace mla {
namespace {

constexpr int kMergeWarps = 8;
constexpr int kMergeThreads = 32 * kMergeWarps;

__device__ __forceinline__ float merge_warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float merge_warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Eight consecutive values of a part as floats.
template <bool kBf16>
__device__ __forceinline__ void load8(const void* base, size_t idx, float (&v)[8]) {
  if (kBf16) {
    const uint4 r = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + idx);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h[e]);
      v[2 * e] = f.x;
      v[2 * e + 1] = f.y;
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
    const float4 a = p[0], b = p[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

// One warp per row; lane l holds columns [8l + 256k, 8l + 256k + 8).
template <bool kBf16>
__global__ void __launch_bounds__(kMergeThreads)
    merge_kernel(const void* __restrict__ u_parts, const float* __restrict__ lse_parts,
                 void* __restrict__ u, float* __restrict__ lse, int R, int rows, int d_c) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  // log-sum-exp of the parts: per-lane running (max, sum of exp), then the warp's
  float m = -INFINITY, z = 0.f;
  for (int r = lane; r < R; r += 32) {
    const float x = lse_parts[(size_t)r * rows + row];
    if (x > m) {
      z = z * expf(m - x) + 1.f;
      m = x;
    } else if (x != -INFINITY) {
      z += expf(x - m);
    }
  }
  const float m_all = merge_warp_max(m);
  z = merge_warp_sum(m == -INFINITY ? 0.f : z * expf(m - m_all));
  const float lse_all = (m_all == -INFINITY) ? -INFINITY : m_all + logf(z);
  for (int c0 = 8 * lane; c0 < d_c; c0 += 256) {
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    if (m_all != -INFINITY) {
      for (int r = 0; r < R; ++r) {
        const float x = lse_parts[(size_t)r * rows + row];
        if (x == -INFINITY) continue;  // a part with no tokens
        const float w = expf(x - lse_all);
        float v[8];
        load8<kBf16>(u_parts, ((size_t)r * rows + row) * d_c + c0, v);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += w * v[e];
      }
    }
    const size_t o = (size_t)row * d_c + c0;
    if (kBf16) {
      uint32_t pk[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 t = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
        pk[e] = *reinterpret_cast<const uint32_t*>(&t);
      }
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(u) + o) =
          make_uint4(pk[0], pk[1], pk[2], pk[3]);
    } else {
      float4* p = reinterpret_cast<float4*>(static_cast<float*>(u) + o);
      p[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      p[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
  }
  if (lse != nullptr && lane == 0) lse[row] = lse_all;
}

}  // namespace

cudaError_t launch_merge(const void* u_parts, const float* lse_parts, void* u, float* lse, int R,
                         int rows, int d_c, bool bf16, cudaStream_t s) {
  const dim3 grid((rows + kMergeWarps - 1) / kMergeWarps);
  if (bf16)
    merge_kernel<true><<<grid, kMergeThreads, 0, s>>>(u_parts, lse_parts, u, lse, R, rows, d_c);
  else
    merge_kernel<false><<<grid, kMergeThreads, 0, s>>>(u_parts, lse_parts, u, lse, R, rows, d_c);
  return cudaGetLastError();
}

}  // namespace mla
