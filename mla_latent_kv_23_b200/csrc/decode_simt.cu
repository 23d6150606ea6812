// Attend stage on CUDA cores, for the shapes the tensor-core kernel does not
// take (fp32 tensors, latent widths other than 512, RoPE widths other than
// 64).  One block per (KV chunk, query row, head); per 64-token tile a warp
// per token computes the absorbed score q^lat.c + q^R.k^R with a warp-shuffle
// reduction, then the block updates the running max / sum and the
// softmax-weighted latent sum u ("MLA deep compression", absorption section).
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"
#include "schedule.cuh"

namespace mla {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kColsPerThread = 4;  // d_c <= 512

__device__ __forceinline__ float ld(const float* p) { return *p; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st(float* p, float v) { *p = v; }
__device__ __forceinline__ void st(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

template <typename T, typename U>
__global__ void __launch_bounds__(kThreads) decode_simt_kernel(const DecodeArgs a) {
  extern __shared__ float sm[];
  const int W = a.d_c + a.d_R;
  float* qs = sm;       // [W]
  float* ps = sm + W;   // [64] scores, then probabilities
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunk = blockIdx.x / a.s_q, r = blockIdx.x % a.s_q, h = blockIdx.y;
  const T* kv = static_cast<const T*>(a.kv);

  ChunkWalk walk;
  walk.init(a.tile_prefix, a.chunk_t, a.chunk_b, a.header, a.B, chunk);
  Segment sg;
  while (walk.next(sg)) {
    const int b = sg.b;
    const int L = a.seqlens[b];
    const int L_eff = L - a.s_q + 1 + r;  // row r sees positions < L_eff
    const T* qrow = static_cast<const T*>(a.q) + ((size_t)(b * a.s_q + r) * a.n_h + h) * W;
    for (int c = tid; c < W; c += kThreads) qs[c] = ld(qrow + c);
    __syncthreads();

    float m = -INFINITY, l = 0.f;
    float acc[kColsPerThread];
#pragma unroll
    for (int k = 0; k < kColsPerThread; ++k) acc[k] = 0.f;

    for (int t = sg.t0; t < sg.t1; ++t) {
      const int tok0 = t * kTileTokens;
      int page = a.block_table[(size_t)b * a.max_pages + tok0 / a.page_size];
      const bool bad = page < 0 || page >= a.num_pages;
      if (bad && tid == 0) atomicOr(a.err, MLA_DEVFLAG_BAD_PAGE);
      const size_t row0 = (size_t)(bad ? 0 : page) * a.page_size + tok0 % a.page_size;
      const int nv = bad ? 0 : max(0, min(kTileTokens, L_eff - tok0));
      // scores, one warp per token
      for (int j = warp; j < kTileTokens; j += kWarps) {
        float s = -INFINITY;
        if (j < nv) {
          const T* krow = kv + (row0 + j) * W;
          float d = 0.f;
          for (int c = lane; c < W; c += 32) d += qs[c] * ld(krow + c);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
          s = d * a.scale;
        }
        if (lane == 0) ps[j] = s;
      }
      __syncthreads();
      float mx = -INFINITY;
      for (int j = 0; j < nv; ++j) mx = fmaxf(mx, ps[j]);
      const float m_new = fmaxf(m, mx);
      const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      __syncthreads();
      if (tid < kTileTokens) ps[tid] = tid < nv ? expf(ps[tid] - m_use) : 0.f;
      __syncthreads();
      float psum = 0.f;
#pragma unroll
      for (int k = 0; k < kColsPerThread; ++k) acc[k] *= alpha;
      for (int j = 0; j < nv; ++j) {
        const float pj = ps[j];
        psum += pj;
        const T* crow = kv + (row0 + j) * W;
#pragma unroll
        for (int k = 0; k < kColsPerThread; ++k) {
          const int c = tid + k * kThreads;
          if (c < a.d_c) acc[k] += pj * ld(crow + c);
        }
      }
      l = l * alpha + psum;
      m = m_new;
      __syncthreads();
    }

    const float inv = l > 0.f ? 1.f / l : 0.f;
    const float lse = l > 0.f ? m + logf(l) : -INFINITY;
    const size_t orow = (size_t)(b * a.s_q + r) * a.n_h + h;
    if (sg.whole) {
      U* u = static_cast<U*>(a.u) + orow * a.d_c;
#pragma unroll
      for (int k = 0; k < kColsPerThread; ++k) {
        const int c = tid + k * kThreads;
        if (c < a.d_c) st(u + c, acc[k] * inv);
      }
      if (a.lse != nullptr && tid == 0) a.lse[orow] = lse;
    } else {
      const size_t slot = (size_t)(a.split_base[b] + sg.part) * a.s_q + r;
      float* pu = a.part_u + (slot * a.n_h + h) * a.d_c;
#pragma unroll
      for (int k = 0; k < kColsPerThread; ++k) {
        const int c = tid + k * kThreads;
        if (c < a.d_c) pu[c] = acc[k] * inv;
      }
      if (tid == 0) a.part_lse[slot * a.n_h + h] = lse;
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t s) {
  dim3 grid(a.num_chunks * a.s_q, a.n_h);
  const size_t smem = (size_t)(a.d_c + a.d_R + kTileTokens) * sizeof(float);
  if (a.bf16 && !a.out_f32)
    decode_simt_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, kThreads, smem, s>>>(a);
  else if (a.bf16)
    decode_simt_kernel<__nv_bfloat16, float><<<grid, kThreads, smem, s>>>(a);
  else
    decode_simt_kernel<float, float><<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace mla
