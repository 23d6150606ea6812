// Per-head up-projection on the tensor cores (sm_100a), bf16:
//     o[t, i, :] = W^UV_i . u[t, i, :]
// ("MLA deep compression", absorption section, output equation).
//
// One CTA per (head i, block of up to 64 query rows t) computes
// D[v, t] = sum_c W^UV_i[v, c] u[t, i, c] as one tcgen05 MMA chain with
// M = d_v = 128, N = rows (padded to 16), K = d_c: W^UV_i (128 KB at
// d_c = 512) is the K-major A operand and the rows of u are the K-major B
// operand, both staged by TMA with 128-byte swizzle.  The weight read
// (16.8 MB over all heads, the whole cost of this step) is issued before the
// kernel waits for the decode that produces u, so with programmatic
// dependent launch it overlaps the end of the decode.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {
using namespace ptx;

constexpr int kThreads = 128;
constexpr int kDv = 128;         // M
constexpr int kMaxN = 64;        // query rows per CTA
constexpr int kMaxKb = 8;        // d_c / 64 <= 8
constexpr uint32_t kWBlk = 128 * 128;     // 128 rows x 64 cols bf16
constexpr uint32_t kUBlk = kMaxN * 128;   // up to 64 rows x 64 cols bf16

struct Params {
  CUtensorMap w_map;   // W_UV as [n_h * d_v rows, d_c cols], box 64 x 128
  CUtensorMap u_map;   // u as [T, n_h, d_c], box 64 x 1 x n_pad
  __nv_bfloat16* o;
  int* err;
  int T, n_h, d_c, n_pad;
};

__global__ void __launch_bounds__(kThreads, 1) up_proj_sm100_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (sbase - raw_addr);
  const int kb_n = p.d_c / 64;
  const uint32_t off_u = kMaxKb * kWBlk;
  const uint32_t off_bar = off_u + kMaxKb * kUBlk;
  const uint32_t bar_w = sbase + off_bar, bar_u = bar_w + 8, bar_mma = bar_w + 16;
  const uint32_t tmem_slot = bar_w + 24;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.x, t0 = blockIdx.y * kMaxN;

  if (threadIdx.x == 0) {
    mbar_init(bar_w, 1);
    mbar_init(bar_u, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(base + (tmem_slot - sbase));

  if (threadIdx.x == 0) {
    prefetch_tmap(&p.w_map);
    prefetch_tmap(&p.u_map);
    // the weights do not depend on the previous kernel: fetch them first
    mbar_arrive_expect_tx(bar_w, kb_n * kWBlk);
    for (int kb = 0; kb < kb_n; ++kb)
      tma_load_2d(sbase + kb * kWBlk, &p.w_map, bar_w, kb * 64, head * kDv);
  }
  pdl_wait_previous();
  pdl_launch_dependents();
  bool ok = true;
  if (threadIdx.x == 0) {
    const uint32_t ublk = p.n_pad * 128;
    mbar_arrive_expect_tx(bar_u, kb_n * ublk);
    for (int kb = 0; kb < kb_n; ++kb)
      tma_load_3d(sbase + off_u + kb * ublk, &p.u_map, bar_u, kb * 64, head, t0);
    ok = mbar_wait(bar_w, 0, p.err, MLA_DEVFLAG_TIMEOUT) &&
         mbar_wait(bar_u, 0, p.err, MLA_DEVFLAG_TIMEOUT);
    if (ok) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16(kDv, p.n_pad, false);
      uint32_t acc = 0;
      for (int kb = 0; kb < kb_n; ++kb)
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t a = smem_desc(sbase + kb * kWBlk + ks * 32, 16, 1024, kLayoutSW128);
          const uint64_t b = smem_desc(sbase + off_u + kb * ublk + ks * 32, 16, 1024, kLayoutSW128);
          umma_f16_ss(tmem, a, b, idesc, acc);
          acc = 1;
        }
    }
    umma_commit(bar_mma);
    if (!mbar_wait(bar_mma, 0, p.err, MLA_DEVFLAG_TIMEOUT)) ok = false;
  }
  ok = __syncthreads_and(ok);
  tc_fence_after();
  if (ok) {
    // thread (warp w, lane l) owns output row v = 32 w + l; columns are rows t
    const int v = warp * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    for (int c0 = 0; c0 < p.n_pad; c0 += 32) {
      float d[32];
      tmem_ld32(tmem + lane_base + c0, d);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const int t = t0 + c0 + k;
        if (c0 + k < p.n_pad && t < p.T)
          p.o[((size_t)t * p.n_h + head) * kDv + v] = __float2bfloat16_rn(d[k]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

constexpr size_t kSmemBytes = kMaxKb * kWBlk + kMaxKb * kUBlk + 64 + 1024;

}  // namespace

int up_proj_sm100_prepare() {
  if (cudaFuncSetAttribute(up_proj_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBytes) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return 1;
}

cudaError_t launch_up_proj_sm100(const CUtensorMap& w_map, const CUtensorMap& u_map, void* o,
                                 int* err, int T, int n_h, int d_c, cudaStream_t s) {
  Params p;
  p.w_map = w_map;
  p.u_map = u_map;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.err = err;
  p.T = T;
  p.n_h = n_h;
  p.d_c = d_c;
  const int rows = T < kMaxN ? T : kMaxN;
  p.n_pad = (rows + 15) / 16 * 16;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_h, (T + kMaxN - 1) / kMaxN, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, up_proj_sm100_kernel, p);
}

int up_proj_sm100_box_rows(int T) {
  const int rows = T < kMaxN ? T : kMaxN;
  return (rows + 15) / 16 * 16;
}

}  // namespace mla
