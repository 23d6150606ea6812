// Per-head up-projection on the tensor cores (sm_100a):
//     o[t, i, :] = W^UV_i . u[t, i, :]
// ("MLA deep compression", absorption section, output equation).
//
// One CTA per (head i, block of query rows t) computes
// D[v, t] = sum_c W^UV_i[v, c] u[t, i, c] as one tcgen05 MMA chain with
// M = 128 (rows v of W^UV_i; rows past d_v belong to the next head or lie
// past the tensor and are never stored), N = rows (padded to 16), K = d_c.
// W^UV_i is the K-major A operand and the rows of u the K-major B operand,
// both in 128-byte-swizzled shared memory.  Three input modes:
//   kBf16:   bf16 W and u, both staged by TMA (kind::f16);
//   kSplitU: bf16 W and an fp32 u, read with plain loads and split into two
//            bf16 terms hi = bf16(u), lo = bf16(u - hi) written in the
//            swizzled layout; D = W hi + W lo in one accumulator, so u is
//            used to within 2^-16 of itself (kind::f16);
//   kTf32:   fp32 W and u staged by TMA, read as tf32 (kind::tf32).
// The weight read (16.8 MB over all heads at the DeepSeek-V3 shape, the
// whole cost of this step) is issued before the kernel waits for the
// previous kernel, so under programmatic dependent launch it overlaps the
// end of the decode that produces u.
//
// kSplitU can also merge the split-KV partial results itself (the combine
// of mla_decode, fused in): a row whose sequence was cut into pieces gets
// lse = log sum_s exp(lse_s) and u = sum_s exp(lse_s - lse) u_s from the fp16
// partials (written to u and lse as well), a whole row is read as the attend
// stage wrote it; either way the fp32 row then enters the MMA as hi + lo.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {
using namespace ptx;

enum class UpMode { kBf16, kSplitU, kTf32 };

// 16 warps: the row loads and the partial merge are latency-bound (a few
// dependent memory round trips per row), so each warp takes one row of a
// 16-row block at a time; warps 0-3 drain the accumulator.
constexpr int kThreads = 512;
constexpr int kM = 128;              // MMA rows: d_v <= 128
constexpr int kMaxKb = 8;            // 128-byte column blocks of d_c
constexpr int kMaxRows = 64;         // query rows per CTA (kBf16, kTf32)
constexpr int kMaxRowsSplit = 32;    // query rows per CTA (kSplitU: hi and lo)
constexpr uint32_t kWBlk = kM * 128; // 128 rows x 128 bytes

template <UpMode kMode>
constexpr int max_rows() { return kMode == UpMode::kSplitU ? kMaxRowsSplit : kMaxRows; }
template <UpMode kMode>
constexpr uint32_t u_bytes() {  // B operand area (hi and lo for kSplitU)
  return (kMode == UpMode::kSplitU ? 2u : 1u) * kMaxKb * max_rows<kMode>() * 128u;
}
template <UpMode kMode>
constexpr size_t smem_bytes() { return kMaxKb * kWBlk + u_bytes<kMode>() + 64 + 1024; }

struct Params {
  CUtensorMap w_map;   // W_UV as [n_h * d_v rows, d_c cols], box (128 bytes) x 128 rows
  CUtensorMap u_map;   // u as [T, n_h, d_c], box (128 bytes) x 1 x n_pad (kBf16, kTf32)
  const float* u_f32;  // u (kSplitU)
  // kSplitU with merge: the decode workspace's plan and partials (d_c = 512)
  int merge, s_q;
  const int* tile_prefix;
  const int* split_base;
  const __half* part_u;  // fp16 partial u of split rows
  const float* part_lse;
  float* u_out;        // = u_f32: merged rows are written back
  float* lse_out;      // may be null
  void* o;             // [T, n_h, d_v]: bf16 (kBf16, kSplitU) or fp32 (kTf32)
  int* err;
  int T, n_h, d_c, d_v, n_pad;
};

template <UpMode kMode>
__global__ void __launch_bounds__(kThreads, 1) up_proj_sm100_kernel(const __grid_constant__ Params p) {
  constexpr bool kF32 = kMode == UpMode::kTf32;
  constexpr int kColsPerBlk = kF32 ? 32 : 64;  // elements in one 128-byte row
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (sbase - raw_addr);
  const int kb_n = p.d_c / kColsPerBlk;
  const uint32_t off_u = kMaxKb * kWBlk;
  const uint32_t off_bar = off_u + u_bytes<kMode>();
  const uint32_t bar_w = sbase + off_bar, bar_u = bar_w + 8, bar_mma = bar_w + 16;
  const uint32_t tmem_slot = bar_w + 24;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.x, t0 = blockIdx.y * max_rows<kMode>();
  const uint32_t ublk = p.n_pad * 128;  // one 128-byte column block of the B operand

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
    if (kMode != UpMode::kSplitU) prefetch_tmap(&p.u_map);
    // the weights do not depend on the previous kernel: fetch them first
    mbar_arrive_expect_tx(bar_w, kb_n * kWBlk);
    for (int kb = 0; kb < kb_n; ++kb)
      tma_load_2d(sbase + kb * kWBlk, &p.w_map, bar_w, kb * kColsPerBlk, head * p.d_v);
  }
  // kSplitU: the B operand holds 2 n_pad rows per 128-byte column block,
  // row tt = bf16(u_t) (hi) and row n_pad + tt = bf16(u_t - hi) (lo), so
  // one MMA chain over W gives W hi and W lo side by side (N = 2 n_pad)
  const uint32_t ublk2 = 2 * ublk;
  auto store_hilo = [&](int tt, int c8, const float (&v)[8]) {
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
      const float2 hf = __bfloat1622float2(h2);
      const __nv_bfloat162 l2 = __floats2bfloat162_rn(v[2 * k] - hf.x, v[2 * k + 1] - hf.y);
      hi[k] = *reinterpret_cast<const uint32_t*>(&h2);
      lo[k] = *reinterpret_cast<const uint32_t*>(&l2);
    }
    // chunk k16 of row r at byte r * 128 + ((k16 ^ (r & 7)) << 4) of its
    // block; n_pad is a multiple of 16, so rows tt and n_pad + tt share it
    const int kb = c8 >> 3, k16 = c8 & 7;
    const uint32_t sw = static_cast<uint32_t>(k16 ^ (tt & 7)) << 4;
    const uint32_t blk = sbase + off_u + kb * ublk2;
    st_shared_v4(blk + tt * 128 + sw, hi[0], hi[1], hi[2], hi[3]);
    st_shared_v4(blk + (p.n_pad + tt) * 128 + sw, lo[0], lo[1], lo[2], lo[3]);
  };
  // merged rows of split sequences, kept in registers until the product has
  // been issued: it reads only their bf16 terms in shared memory
  constexpr int kKeep = kMode == UpMode::kSplitU ? kMaxRowsSplit / (kThreads / 32) : 1;
  float keep_u[kKeep][16], keep_lse[kKeep];
  bool keep[kKeep];
#pragma unroll
  for (int j = 0; j < kKeep; ++j) keep[j] = false;
  if constexpr (kMode == UpMode::kSplitU) {
   if (p.merge) {
    // One warp per row t (rows warp and warp + 16 of the block); lane l
    // owns columns [8 l, 8 l + 8) and [256 + 8 l, 256 + 8 l + 8) of
    // d_c = 512, so each 16-byte access of the warp covers 512 contiguous
    // bytes of a row (one fp16 partial row or half an fp32 row).  The plan stage's
    // outputs are read before the wait: the plan kernel completed before
    // the attend kernel passed its own wait, and this kernel was launched
    // only after every attend CTA had passed it.
    constexpr int kRowsPerWarp = kMaxRowsSplit / (kThreads / 32);
    int kind[kRowsPerWarp], sb0[kRowsPerWarp], nsp[kRowsPerWarp];  // kind: 0 none, 1 whole, 2 empty, 3 split
#pragma unroll
    for (int j = 0; j < kRowsPerWarp; ++j) {
      const int tt = warp + j * (kThreads / 32), t = t0 + tt;
      kind[j] = 0;
      sb0[j] = 0;
      nsp[j] = 0;
      if (tt < p.n_pad && t < p.T) {
        const int b = t / p.s_q;
        const int s0 = p.split_base[b], s1 = p.split_base[b + 1];
        const bool has_tokens = p.tile_prefix[b + 1] != p.tile_prefix[b];
        sb0[j] = s0;
        nsp[j] = s1 - s0;
        kind[j] = s1 > s0 ? 3 : (has_tokens ? 1 : 2);
      }
    }
    pdl_wait_previous();
    pdl_launch_dependents();
#pragma unroll
    for (int j = 0; j < kRowsPerWarp; ++j) {
      const int tt = warp + j * (kThreads / 32), t = t0 + tt;
      if (tt >= p.n_pad) continue;
      float acc[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = 0.f;
      const size_t urow = (size_t)t * p.n_h + head;
      float* up = p.u_out + urow * 512 + 8 * lane;  // float4 i of the lane: up + 256 (i >> 1) + 4 (i & 1)
      if (kind[j] == 1) {  // written whole by the attend stage
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 v = reinterpret_cast<const float4*>(up + (i >> 1) * 256)[i & 1];
          acc[4 * i] = v.x; acc[4 * i + 1] = v.y; acc[4 * i + 2] = v.z; acc[4 * i + 3] = v.w;
        }
      } else if (kind[j] == 2) {  // no tokens (a rejected length): u = 0, lse = -inf
#pragma unroll
        for (int i = 0; i < 4; ++i)
          reinterpret_cast<float4*>(up + (i >> 1) * 256)[i & 1] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (lane == 0 && p.lse_out) p.lse_out[urow] = -INFINITY;
      } else if (kind[j] == 3) {
        const int nsplit = nsp[j];
        const size_t slot0 = (size_t)sb0[j] * p.s_q + t % p.s_q;  // slot of split s: slot0 + s s_q
        auto lse_of = [&](int sp) { return p.part_lse[(slot0 + (size_t)sp * p.s_q) * p.n_h + head]; };
        auto part_of = [&](int sp) {  // lane's 16 fp16 values: 16-byte elements 0 and 32
          return reinterpret_cast<const uint4*>(
              p.part_u + ((slot0 + (size_t)sp * p.s_q) * p.n_h + head) * 512 + 8 * lane);
        };
        // the first four partial rows are requested together with the
        // statistics: one memory round trip for rows of up to four pieces
        uint4 v[4][2];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (k < nsplit) {
#pragma unroll
            for (int i = 0; i < 2; ++i) v[k][i] = part_of(k)[32 * i];
          }
        const float x_lane = lane < nsplit ? lse_of(lane) : -INFINITY;
        float m = x_lane, z = x_lane == -INFINITY ? 0.f : 1.f;
        for (int sp = lane + 32; sp < nsplit; sp += 32) {
          const float x = lse_of(sp);
          if (x > m) {
            z = z * expf(m - x) + 1.f;
            m = x;
          } else if (x != -INFINITY) {
            z += expf(x - m);
          }
        }
        float m_all = m;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m_all = fmaxf(m_all, __shfl_xor_sync(0xffffffffu, m_all, o));
        z = m == -INFINITY ? 0.f : z * expf(m - m_all);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        const float lse = m_all == -INFINITY ? -INFINITY : m_all + logf(z);
        if (m_all != -INFINITY) {
          const float w_lane = x_lane == -INFINITY ? 0.f : expf(x_lane - lse);
          for (int s0 = 0; s0 < nsplit; s0 += 4) {
            const int n_here = min(4, nsplit - s0);
            if (s0 > 0) {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                if (k < n_here) {
#pragma unroll
                  for (int i = 0; i < 2; ++i) v[k][i] = part_of(s0 + k)[32 * i];
                }
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              // split s0 + k's weight: held by lane s0 + k for the first 32
              const float wk = s0 + k < 32 ? __shfl_sync(0xffffffffu, w_lane, (s0 + k) & 31) : 0.f;
              const float w = s0 + k < 32 ? wk : (k < n_here ? expf(lse_of(s0 + k) - lse) : 0.f);
              if (k < n_here) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  const float2 f = __half22float2(reinterpret_cast<const __half2*>(v[k])[e]);
                  acc[2 * e] += w * f.x;
                  acc[2 * e + 1] += w * f.y;
                }
              }
            }
          }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) keep_u[j][i] = acc[i];
        keep_lse[j] = lse;
        keep[j] = true;
      }
      // the row's two bf16 terms: lane l's 16 columns are chunks l, 32 + l
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float v8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) v8[k] = acc[8 * c + k];
        store_hilo(tt, lane + 32 * c, v8);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
   } else {
    pdl_wait_previous();
    pdl_launch_dependents();
    // u rows -> hi and lo bf16 terms, 8 columns (one 16-byte chunk of each
    // term) per unit; each thread requests up to four units' rows before
    // using any; rows past T are zero
    const int chunks = p.d_c / 8, units = p.n_pad * chunks;
    for (int base_u = 0; base_u < units; base_u += 4 * kThreads) {
      float v[4][8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int unit = base_u + k * kThreads + threadIdx.x;
        const int t = unit / chunks, c8 = unit % chunks;
        if (unit < units && t0 + t < p.T) {
          const float4* src = reinterpret_cast<const float4*>(
              p.u_f32 + ((size_t)(t0 + t) * p.n_h + head) * p.d_c + 8 * c8);
          const float4 a = src[0], b = src[1];
          v[k][0] = a.x; v[k][1] = a.y; v[k][2] = a.z; v[k][3] = a.w;
          v[k][4] = b.x; v[k][5] = b.y; v[k][6] = b.z; v[k][7] = b.w;
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) v[k][i] = 0.f;
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int unit = base_u + k * kThreads + threadIdx.x;
        if (unit < units) store_hilo(unit / chunks, unit % chunks, v[k]);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
   }
  } else {
    pdl_wait_previous();
    pdl_launch_dependents();
  }
  bool ok = true;
  if (threadIdx.x == 0) {
    if constexpr (kMode != UpMode::kSplitU) {
      mbar_arrive_expect_tx(bar_u, kb_n * ublk);
      for (int kb = 0; kb < kb_n; ++kb)
        tma_load_3d(sbase + off_u + kb * ublk, &p.u_map, bar_u, kb * kColsPerBlk, head, t0);
      ok = mbar_wait(bar_u, 0, p.err, MLA_DEVFLAG_TIMEOUT);
    }
    ok = ok && mbar_wait(bar_w, 0, p.err, MLA_DEVFLAG_TIMEOUT);
    if (ok) {
      tc_fence_after();
      constexpr bool kTwo = kMode == UpMode::kSplitU;  // hi and lo side by side in N
      const int n_mma = kTwo ? 2 * p.n_pad : p.n_pad;
      const uint32_t bblk = kTwo ? ublk2 : ublk;
      const uint32_t idesc = kF32 ? idesc_tf32(kM, n_mma, false) : idesc_bf16(kM, n_mma, false);
      uint32_t acc = 0;
        for (int kb = 0; kb < kb_n; ++kb)
          for (int ks = 0; ks < 4; ++ks) {  // 32 bytes of K per instruction
            const uint64_t a = smem_desc(sbase + kb * kWBlk + ks * 32, 16, 1024, kLayoutSW128);
            const uint64_t b = smem_desc(sbase + off_u + kb * bblk + ks * 32, 16, 1024, kLayoutSW128);
            if (kF32)
              umma_tf32_ss(tmem, a, b, idesc, acc);
            else
              umma_f16_ss(tmem, a, b, idesc, acc);
            acc = 1;
          }
    }
    umma_commit(bar_mma);
  }
  if constexpr (kMode == UpMode::kSplitU) {  // the merged rows leave while the product runs
#pragma unroll
    for (int j = 0; j < kKeep; ++j)
      if (keep[j]) {
        const size_t urow = (size_t)(t0 + warp + j * (kThreads / 32)) * p.n_h + head;
        float* up = p.u_out + urow * 512 + 8 * lane;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          reinterpret_cast<float4*>(up + (i >> 1) * 256)[i & 1] =
              make_float4(keep_u[j][4 * i], keep_u[j][4 * i + 1], keep_u[j][4 * i + 2], keep_u[j][4 * i + 3]);
        if (lane == 0 && p.lse_out) p.lse_out[urow] = keep_lse[j];
      }
  }
  if (threadIdx.x == 0 && !mbar_wait(bar_mma, 0, p.err, MLA_DEVFLAG_TIMEOUT)) ok = false;
  ok = __syncthreads_and(ok);
  tc_fence_after();
  if (ok && warp < 4) {
    // thread (warp w, lane l) owns output row v = 32 w + l; columns are rows t
    const int v = warp * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    for (int c0 = 0; c0 < p.n_pad; c0 += 32) {
      float d[32];
      tmem_ld32(tmem + lane_base + c0, d);
      if constexpr (kMode == UpMode::kSplitU) {  // W hi + W lo
        float e[32];
        tmem_ld32(tmem + lane_base + p.n_pad + c0, e);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) d[k] += e[k];
      }
      tmem_wait_ld();
      if (kMode == UpMode::kSplitU && p.d_v % 8 == 0) {
        // rows [c0, c0 + 32) go through the B-operand area (free once the
        // product is complete) as [t][v] bf16, then leave as 16-byte
        // stores of 8 consecutive v: one 2-byte store per value backs up
        // behind the merge's stores of u
        __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(base + off_u);
        if (v < p.d_v) {
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (c0 + k < p.n_pad) stg[k * kM + v] = __float2bfloat16_rn(d[k]);
        }
        named_bar_sync(1, 4 * 32);
        const int rows = min(32, p.n_pad - c0), per_row = p.d_v / 8;
        for (int i = threadIdx.x; i < rows * per_row; i += 4 * 32) {
          const int k = i / per_row, v8 = 8 * (i % per_row), t = t0 + c0 + k;
          if (t < p.T)
            *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + ((size_t)t * p.n_h + head) * p.d_v + v8) =
                *reinterpret_cast<const uint4*>(stg + k * kM + v8);
        }
        named_bar_sync(1, 4 * 32);  // the area is read before the next rows land in it
      } else if (v < p.d_v) {
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const int t = t0 + c0 + k;
          if (c0 + k < p.n_pad && t < p.T) {
            const size_t idx = ((size_t)t * p.n_h + head) * p.d_v + v;
            if (kF32)
              static_cast<float*>(p.o)[idx] = d[k];
            else
              static_cast<__nv_bfloat16*>(p.o)[idx] = __float2bfloat16_rn(d[k]);
          }
        }
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

template <UpMode kMode>
cudaError_t launch(const Params& p, int n_h, int T, bool pdl, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_h, (T + max_rows<kMode>() - 1) / max_rows<kMode>(), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes<kMode>();
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, up_proj_sm100_kernel<kMode>, p);
}

int pad_rows(int T, int cap) {
  const int rows = T < cap ? T : cap;
  return (rows + 15) / 16 * 16;
}

}  // namespace

int up_proj_sm100_prepare() {
  if (cudaFuncSetAttribute(up_proj_sm100_kernel<UpMode::kBf16>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem_bytes<UpMode::kBf16>()) != cudaSuccess ||
      cudaFuncSetAttribute(up_proj_sm100_kernel<UpMode::kSplitU>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem_bytes<UpMode::kSplitU>()) != cudaSuccess ||
      cudaFuncSetAttribute(up_proj_sm100_kernel<UpMode::kTf32>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem_bytes<UpMode::kTf32>()) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return 1;
}

int up_proj_sm100_box_rows(int T) { return pad_rows(T, kMaxRows); }

cudaError_t launch_up_proj_sm100(const CUtensorMap& w_map, const CUtensorMap& u_map, void* o,
                                 int* err, int T, int n_h, int d_c, int d_v, bool f32, bool pdl,
                                 cudaStream_t s) {
  Params p;
  p.w_map = w_map;
  p.u_map = u_map;
  p.u_f32 = nullptr;
  p.o = o;
  p.err = err;
  p.T = T;
  p.n_h = n_h;
  p.d_c = d_c;
  p.d_v = d_v;
  p.n_pad = pad_rows(T, kMaxRows);
  return f32 ? launch<UpMode::kTf32>(p, n_h, T, pdl, s) : launch<UpMode::kBf16>(p, n_h, T, pdl, s);
}

cudaError_t launch_up_proj_sm100_f32u(const CUtensorMap& w_map, const float* u, void* o, int* err,
                                      int T, int n_h, int d_c, int d_v, bool pdl, cudaStream_t s,
                                      const DecodeArgs* merge) {
  Params p;
  memset(&p, 0, sizeof(p));
  p.w_map = w_map;
  if (merge != nullptr) {
    p.merge = 1;
    p.s_q = merge->s_q;
    p.tile_prefix = merge->tile_prefix;
    p.split_base = merge->split_base;
    p.part_u = reinterpret_cast<const __half*>(merge->part_u);
    p.part_lse = merge->part_lse;
    p.u_out = const_cast<float*>(u);
    p.lse_out = merge->lse;
  }
  memset(&p.u_map, 0, sizeof(p.u_map));
  p.u_f32 = u;
  p.o = o;
  p.err = err;
  p.T = T;
  p.n_h = n_h;
  p.d_c = d_c;
  p.d_v = d_v;
  p.n_pad = pad_rows(T, kMaxRowsSplit);
  return launch<UpMode::kSplitU>(p, n_h, T, pdl, s);
}

}  // namespace mla
