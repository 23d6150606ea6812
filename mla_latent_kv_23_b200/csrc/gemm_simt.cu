// Tiled CUDA-core GEMM with the store epilogues of the setup calls:
//   mla_absorb_weights   W_QK[i] = W_UK[i]^T W_Q[i]           (batched over heads)
//   mla_form_query       q = [W_QK h || RoPE(W_QR h, pos)]      (segmented columns)
//   mla_append_latent    cache row = [W_DKV h || RoPE(W_KR h, pos)] (paged rows)
//   mla_up_proj          o[t, i] = W_UV[i] u[t, i]              (fp32 / non-tensor-core shapes)
// ("MLA deep compression": low-rank projection, absorption and decoupled-RoPE
// sections).  None of these is on the per-token attention path except the
// up-projection, which has a tensor-core kernel of its own for bf16.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"

namespace mla {
namespace {

constexpr int BM = 64, BN = 64, BK = 16, TM = 4, TN = 4;
constexpr int kThreads = (BM / TM) * (BN / TN);  // 256

__device__ __forceinline__ float ld(const float* p) { return *p; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st(float* p, float v) { *p = v; }
__device__ __forceinline__ void st(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

template <typename T>
__global__ void __launch_bounds__(kThreads) gemm_kernel(const GemmArgs g) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tid = threadIdx.x;
  const int tx = tid % (BN / TN), ty = tid / (BN / TN);
  const int z = blockIdx.z;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const T* A = static_cast<const T*>(g.A) + (size_t)z * g.sAz;
  const T* B = static_cast<const T*>(g.Bm) + (size_t)z * g.sBz;
  const bool a_kfast = g.sAk == 1, b_kfast = g.sBk == 1;

  float acc[TM][TN];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < g.K; k0 += BK) {
#pragma unroll
    for (int e = 0; e < (BM * BK) / kThreads; ++e) {
      const int idx = tid + e * kThreads;
      const int mi = a_kfast ? idx / BK : idx % BM;
      const int ki = a_kfast ? idx % BK : idx / BM;
      const int m = m0 + mi, k = k0 + ki;
      As[ki][mi] = (m < g.M && k < g.K) ? ld(A + (size_t)m * g.sAm + (size_t)k * g.sAk) : 0.f;
    }
#pragma unroll
    for (int e = 0; e < (BN * BK) / kThreads; ++e) {
      const int idx = tid + e * kThreads;
      const int ni = b_kfast ? idx / BK : idx % BN;
      const int ki = b_kfast ? idx % BK : idx / BN;
      const int n = n0 + ni, k = k0 + ki;
      Bs[ki][ni] = (n < g.N && k < g.K) ? ld(B + (size_t)n * g.sBn + (size_t)k * g.sBk) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float av[TM], bv[TN];
#pragma unroll
      for (int i = 0; i < TM; ++i) av[i] = As[kk][ty * TM + i];
#pragma unroll
      for (int j = 0; j < TN; ++j) bv[j] = Bs[kk][tx * TN + j];
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }

  T* C = static_cast<T*>(g.C);
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int m = m0 + ty * TM + i;
    if (m >= g.M) continue;
    long long row_base;
    if (g.block_table != nullptr) {
      const int p = g.pos[m];
      const int page = g.block_table[(size_t)g.seq[m] * g.max_pages + p / g.page_size];
      if (page < 0 || page >= g.num_pages) {
        if (tx == 0) atomicOr(g.err, MLA_DEVFLAG_BAD_PAGE);
        continue;
      }
      row_base = ((long long)page * g.page_size + p % g.page_size) * g.sCm;
    } else {
      row_base = (long long)z * g.sCz + (long long)m * g.sCm;
    }
#pragma unroll
    for (int j = 0; j < TN; j += 2) {
      const int n = n0 + tx * TN + j;  // even; n and n + 1 share a segment
      if (n >= g.N) continue;
      float v0 = acc[i][j], v1 = acc[i][j + 1];
      const int within = n % g.seg;
      if (g.rope) {
        // pair (within, within + 1) rotates by pos * base^(-within / seg)
        const double theta = pow(g.rope_base, -(double)within / (double)g.seg);
        double sn, cs;
        sincos((double)g.pos[m] * theta, &sn, &cs);
        const float c = (float)cs, s = (float)sn;
        const float r0 = v0 * c - v1 * s, r1 = v0 * s + v1 * c;
        v0 = r0;
        v1 = r1;
      }
      const long long col = (long long)(n / g.seg) * g.seg_stride + g.col_off + within;
      st(C + row_base + col, v0);
      if (n + 1 < g.N) st(C + row_base + col + 1, v1);
    }
  }
}

}  // namespace

cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t s) {
  dim3 grid((g.N + BN - 1) / BN, (g.M + BM - 1) / BM, g.Z);
  if (g.bf16)
    gemm_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(g);
  else
    gemm_kernel<float><<<grid, kThreads, 0, s>>>(g);
  return cudaGetLastError();
}

}  // namespace mla
