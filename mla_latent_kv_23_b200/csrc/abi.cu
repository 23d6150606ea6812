// C ABI of libmla: argument validation, workspace sizing, TMA descriptor
// encoding and kernel selection.  No allocation happens here: every device
// buffer, the workspace included, belongs to the caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstring>
#include <functional>
#include <mutex>

#include "internal.h"
#include "mla.h"

namespace mla {

// Sticky device-side flags (MLA_DEVFLAG_*), one word per device.
__device__ int g_device_flags;

int decode_sm100_prepare();

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int sm_count = 0;
  int cc_major = 0, cc_minor = 0;
  int max_clusters = 0;  // co-resident 2-CTA clusters of the DeepSeek-V3-shape kernel
  bool small_tc = false;  // the small-latent tensor-core kernel is usable
  bool up_proj_tc = false;
  bool wgemm_tc = false;  // the weight-streaming projection kernel is usable
  int* flags = nullptr;  // device address of g_device_flags
};

DeviceInfo g_devices[kMaxDevices];
std::mutex g_mutex;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

mla_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MLA_OK;
  cudaGetLastError();
  return MLA_ERR_CUDA;
}

mla_status device_info(const DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_status(cudaErrorInvalidDevice);
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_devices[dev];
  if (!d.ready) {
    cudaError_t e;
    if ((e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_status(e);
    if ((e = cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
      return cuda_status(e);
    if ((e = cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return cuda_status(e);
    if ((e = cudaGetSymbolAddress(reinterpret_cast<void**>(&d.flags), g_device_flags)) != cudaSuccess)
      return cuda_status(e);
    d.max_clusters = (d.cc_major == 10) ? decode_sm100_prepare() : 0;
    d.small_tc = (d.cc_major == 10) && decode_small_sm100_prepare() != 0;
    d.up_proj_tc = (d.cc_major == 10) && up_proj_sm100_prepare() != 0;
    d.wgemm_tc = (d.cc_major == 10) && wgemm_sm100_prepare() != 0;
    if (g_encode == nullptr) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
              cudaSuccess &&
          q == cudaDriverEntryPointSuccess)
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
      cudaGetLastError();
    }
    d.ready = true;
  }
  *out = &d;
  return MLA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_dtype(mla_dtype d) { return d == MLA_DTYPE_BF16 || d == MLA_DTYPE_FP32; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

mla_status validate_decode(const mla_decode_params* p) {
  if (p == nullptr) return MLA_ERR_INVALID_ARG;
  if (p->B < 0) return MLA_ERR_INVALID_ARG;
  if (p->s_q < 1) return MLA_ERR_INVALID_ARG;
  if (p->s_q > 2) return MLA_ERR_UNSUPPORTED;
  if (p->n_h < 1) return MLA_ERR_INVALID_ARG;
  if (p->n_h > kMaxHeads) return MLA_ERR_UNSUPPORTED;
  if (p->d_c < 8 || p->d_c % 8 != 0) return MLA_ERR_INVALID_ARG;
  if (p->d_c > 512) return MLA_ERR_UNSUPPORTED;
  if (p->d_R < 0 || p->d_R % 8 != 0) return MLA_ERR_INVALID_ARG;
  if (p->d_R > 64) return MLA_ERR_UNSUPPORTED;
  if (p->page_size <= 0 || p->page_size % kTileTokens != 0) return MLA_ERR_INVALID_ARG;
  if (p->max_pages_per_seq < 1 || p->num_pages < 1) return MLA_ERR_INVALID_ARG;
  if ((long long)p->num_pages * p->page_size > INT_MAX) return MLA_ERR_UNSUPPORTED;
  if ((long long)p->max_pages_per_seq * p->page_size > INT_MAX) return MLA_ERR_UNSUPPORTED;
  if (!std::isfinite(p->softmax_scale) || !(p->softmax_scale > 0.f)) return MLA_ERR_INVALID_ARG;
  if (!valid_dtype(p->dtype)) return MLA_ERR_INVALID_ARG;
  if (p->num_splits < 0) return MLA_ERR_INVALID_ARG;
  if (p->B == 0) return MLA_OK;
  if ((long long)p->B * p->s_q * p->n_h > INT_MAX / 2) return MLA_ERR_UNSUPPORTED;
  if (!p->q || !p->kv_cache || !p->block_table || !p->seqlens || !p->u) return MLA_ERR_INVALID_ARG;
  if (!aligned16(p->q) || !aligned16(p->kv_cache) || !aligned16(p->u) ||
      !aligned16(p->block_table) || !aligned16(p->seqlens) || (p->lse && !aligned16(p->lse)))
    return MLA_ERR_INVALID_ARG;
  return MLA_OK;
}

// The attend kernels, each a tensor-core (tcgen05) kernel for its shapes:
// the paired-CTA kernel for the DeepSeek-V3 shape (bf16, d_c = 512,
// d_R = 64) and the one-CTA kernel for small latent widths.
enum class Kernel { kNone, kV3, kSmall };

Kernel select_kernel(const mla_decode_params* p, const DeviceInfo* d) {
  if (d->cc_major != 10 || g_encode == nullptr) return Kernel::kNone;
  const bool bf16 = p->dtype == MLA_DTYPE_BF16;
  if (bf16 && p->d_c == 512 && p->d_R == 64 && d->max_clusters > 0) return Kernel::kV3;
  if (d->small_tc && decode_small_sm100_supported(bf16, p->d_c, p->d_R)) return Kernel::kSmall;
  return Kernel::kNone;
}

int choose_chunks(const mla_decode_params* p, const DeviceInfo* d) {
  if (p->num_splits > 0) return p->num_splits;
  if (select_kernel(p, d) == Kernel::kV3) return std::max(1, d->max_clusters / p->s_q);
  return std::max(1, d->sm_count / p->s_q);  // one CTA per SM
}

struct Resolved {
  DecodeArgs a;
  long long slots = 0;  // partial rows per head the workspace holds
  Kernel kernel = Kernel::kNone;
  const DeviceInfo* dev = nullptr;
};

mla_status resolve(const mla_decode_params* p, void* ws, size_t ws_bytes, Resolved* r) {
  mla_status st = validate_decode(p);
  if (st != MLA_OK) return st;
  if ((st = device_info(&r->dev)) != MLA_OK) return st;
  r->kernel = select_kernel(p, r->dev);
  if (r->kernel == Kernel::kNone) return MLA_ERR_UNSUPPORTED;
  const int G = choose_chunks(p, r->dev);
  if ((long long)G * p->s_q * 2 > INT_MAX / 2) return MLA_ERR_UNSUPPORTED;
  const WsLayout L = ws_layout(p->B, p->s_q, p->n_h, p->d_c, G);
  if (ws_bytes < L.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MLA_ERR_INVALID_ARG;
  uint8_t* w = static_cast<uint8_t*>(ws);
  r->slots = L.slots;
  DecodeArgs& a = r->a;
  a.q = p->q;
  a.kv = p->kv_cache;
  a.block_table = p->block_table;
  a.seqlens = p->seqlens;
  a.u = p->u;
  a.lse = p->lse;
  a.header = reinterpret_cast<int*>(w + L.header);
  a.tile_prefix = reinterpret_cast<int*>(w + L.tile_prefix);
  a.split_base = reinterpret_cast<int*>(w + L.split_base);
  a.chunk_t = reinterpret_cast<int*>(w + L.chunk_t);
  a.chunk_b = reinterpret_cast<int*>(w + L.chunk_b);
  a.part_lse = reinterpret_cast<float*>(w + L.part_lse);
  a.part_u = reinterpret_cast<float*>(w + L.part_u);
  a.err = r->dev->flags;
  a.B = p->B;
  a.s_q = p->s_q;
  a.n_h = p->n_h;
  a.d_c = p->d_c;
  a.d_R = p->d_R;
  a.page_size = p->page_size;
  a.max_pages = p->max_pages_per_seq;
  a.num_pages = p->num_pages;
  a.num_chunks = G;
  a.scale = p->softmax_scale;
  a.bf16 = p->dtype == MLA_DTYPE_BF16;
  a.out_f32 = p->u_fp32 != 0 || p->dtype == MLA_DTYPE_FP32;
  a.part_bf16 = r->kernel == Kernel::kV3 && !a.out_f32;
  a.part_f16 = r->kernel == Kernel::kV3 && a.out_f32;
  a.pdl = false;
  return MLA_OK;
}

mla_status encode_2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows, uint32_t box_x,
                     uint32_t box_y, CUtensorMapSwizzle sw) {
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {box_x, box_y};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// ---------------------------------------------------------------- projections
// Token rows per projection launch (the kernel's N), and the padded N.
constexpr int kProjMaxRows = 64;
int proj_pad(int T) { return (std::min(T, kProjMaxRows) + 15) / 16 * 16; }
int tiles_of(int rows) { return (rows + 127) / 128; }

// Split of K over CTAs so that about four waves of CTAs stream the weights
// (each CTA keeps at least 4 blocks of 64 columns).
int proj_ksplit(int tiles, int K, int sm_count) {
  const int kb = K / 64;
  const int want = std::max(1, (4 * sm_count + tiles - 1) / tiles);
  return std::max(1, std::min({want, kb / 4 > 0 ? kb / 4 : 1, 64}));
}

size_t proj_acc_bytes(int tiles) { return wgemm_workspace_bytes(tiles, kProjMaxRows); }

mla_status encode_rows(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  return encode_2d(m, ptr, inner, rows, 64, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

// One projection over token rows [t0, t0 + n) of a call; the weight maps
// and the epilogue arguments are filled in by the caller.
mla_status run_projection(WgemmLaunch L, const void* X, int K, int T, int ldx_rows_per_token,
                          const DeviceInfo* d, cudaStream_t s,
                          const std::function<void(WgemmLaunch&, int t0)>& per_chunk) {
  const int chunk = kProjMaxRows / ldx_rows_per_token;
  for (int t0 = 0; t0 < T; t0 += chunk) {
    const int n = std::min(chunk, T - t0) * ldx_rows_per_token;
    WgemmLaunch C = L;
    C.N = n;
    C.n_pad = (n + 15) / 16 * 16;
    const void* xp = static_cast<const uint8_t*>(X) + (size_t)t0 * ldx_rows_per_token * K * 2;
    mla_status st = encode_2d(&C.x_map, xp, K, (uint64_t)n, 64, C.n_pad, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != MLA_OK) return st;
    C.ksplit = proj_ksplit(C.tiles, K, d->sm_count);
    per_chunk(C, t0);
    if ((st = cuda_status(launch_wgemm(C, s))) != MLA_OK) return st;
  }
  return MLA_OK;
}

// 4D map over the cache [rows, 576] (bf16) that gathers one CTA's latent
// half of 64 rows in one copy: dimensions (column, row, block & 1,
// block >> 1) with byte strides (1152, 128, 512) and box 64 x 64 x 2 x 2, so
// that the copy at column 128 r holds the blocks starting at columns
// 128 r + {0, 64, 256, 320}, block k at k x 8 KB (rows of 128 bytes, 128-byte
// swizzle).  Every address stays inside the row (column <= 511).
bool encode_kv_lat4(CUtensorMap* m, const void* ptr, uint64_t rows) {
  const cuuint64_t dims[4] = {192, rows, 2, 2};
  const cuuint64_t strides[3] = {576 * 2, 128, 512};
  const cuuint32_t box[4] = {64, 64, 2, 2};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 5D map over the queries [B * s_q, n_h, 576] (bf16, n_h % 16 == 0) that
// fills one CTA's query area in one copy per 64-column block: dimensions
// (column, head within 16, column half, group of 16 heads, query row), the
// column half's stride 128 columns (latent) or 32 (RoPE), box box_x x 16 x 2
// x 4 x 1, so that shared row 32 g + 16 j + i holds head 16 g + i at the
// columns of half j.  Latent copies start at columns {0, 64, 256, 320} and
// the RoPE copy at 512: every address stays inside the head's row.
bool encode_q5(CUtensorMap* m, const void* ptr, uint64_t n_h, uint64_t qrows, bool rope) {
  const cuuint64_t dims[5] = {rope ? 544u : 384u, 16, 2, n_h / 16, qrows};
  const cuuint64_t strides[4] = {576 * 2, rope ? 64u : 256u, 16 * 576 * 2, n_h * 576 * 2};
  const cuuint32_t box[5] = {rope ? 32u : 64u, 16, 2, 4, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  rope ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D map over the queries [B * s_q, n_h, 576] (bf16), box box_x x 16 heads x 1.
mla_status encode_q(CUtensorMap* m, const void* ptr, uint64_t n_h, uint64_t qrows, uint32_t box_x,
                    CUtensorMapSwizzle sw) {
  const cuuint64_t dims[3] = {576, n_h, qrows};
  const cuuint64_t strides[2] = {576 * 2, n_h * 576 * 2};
  const cuuint32_t box[3] = {box_x, 16, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// 3D map over an output [rows, n_h, 512] for TMA stores, 128-byte swizzle:
// 16-bit (bf16 or fp16) with boxes of 64 columns x 32 heads x 1, or fp32 with
// boxes of 32 columns x 32 heads x 1 (one 128-byte line per head either way).
enum class OutType { kBf16, kF16, kF32 };
mla_status encode_out(CUtensorMap* m, void* ptr, uint64_t n_h, uint64_t rows, OutType t) {
  const bool f32 = t == OutType::kF32;
  const uint64_t es = f32 ? 4 : 2;
  const cuuint64_t dims[3] = {512, n_h, rows};
  const cuuint64_t strides[2] = {512 * es, n_h * 512 * es};
  const cuuint32_t box[3] = {f32 ? 32u : 64u, 32, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType dt = f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                     : (t == OutType::kF16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                           : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
  CUresult r = g_encode(m, dt, 3, ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// Called on its own (pdl = false) a stage is a plain stream-ordered launch;
// inside mla_decode the attend and combine stages may start their prologues
// while the previous stage finishes.
mla_status attend(Resolved r, const mla_decode_params* p, cudaStream_t s, bool pdl) {
  r.a.pdl = pdl;
  if (r.kernel == Kernel::kSmall) {
    const bool f32 = !r.a.bf16;
    const uint64_t es = f32 ? 4 : 2, W = (uint64_t)p->d_c + p->d_R;
    const CUtensorMapDataType tdt = f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const cuuint32_t cols = static_cast<cuuint32_t>(128 / es);
    CUtensorMap q_map, kv_map, kv_pv_map;
    memset(&kv_pv_map, 0, sizeof(kv_pv_map));
    {
      const cuuint64_t dims[3] = {W, (cuuint64_t)p->n_h, (cuuint64_t)p->B * p->s_q};
      const cuuint64_t strides[2] = {W * es, (cuuint64_t)p->n_h * W * es};
      const cuuint32_t box[3] = {cols, 128, 1};
      const cuuint32_t estr[3] = {1, 1, 1};
      if (g_encode(&q_map, tdt, 3, const_cast<void*>(p->q), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return MLA_ERR_CUDA;
    }
    {
      const cuuint64_t dims[2] = {W, (cuuint64_t)p->num_pages * p->page_size};
      const cuuint64_t strides[1] = {W * es};
      const cuuint32_t box[2] = {cols, (cuuint32_t)kTileTokens};
      const cuuint32_t estr[2] = {1, 1};
      if (g_encode(&kv_map, tdt, 2, const_cast<void*>(p->kv_cache), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return MLA_ERR_CUDA;
      // an MN-major tf32 operand: 128-byte swizzle of 32-byte atoms
      if (f32 && g_encode(&kv_pv_map, tdt, 2, const_cast<void*>(p->kv_cache), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return MLA_ERR_CUDA;
    }
    return cuda_status(launch_decode_small_sm100(r.a, q_map, kv_map, kv_pv_map, s));
  }
  Sm100Maps maps;
  const uint64_t kvrows = (uint64_t)p->num_pages * p->page_size;
  mla_status st;
  if ((st = encode_2d(&maps.kv_lat, p->kv_cache, 576, kvrows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK ||
      (st = encode_2d(&maps.kv_rope, p->kv_cache, 576, kvrows, 32, 64, CU_TENSOR_MAP_SWIZZLE_64B)) != MLA_OK)
    return st;
  const uint64_t qrows = (uint64_t)p->B * p->s_q;
  if ((st = encode_q(&maps.q_lat, p->q, p->n_h, qrows, 64, CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK ||
      (st = encode_q(&maps.q_rope, p->q, p->n_h, qrows, 32, CU_TENSOR_MAP_SWIZZLE_64B)) != MLA_OK)
    return st;
  maps.has_kv4 = encode_kv_lat4(&maps.kv_lat4, p->kv_cache, kvrows) ? 1 : 0;
  maps.has_q5 = p->n_h % 16 == 0 && encode_q5(&maps.q_lat5, p->q, p->n_h, qrows, false) &&
                encode_q5(&maps.q_rope5, p->q, p->n_h, qrows, true);
  if ((st = encode_out(&maps.u_out, p->u, p->n_h, qrows,
                       r.a.out_f32 ? OutType::kF32 : OutType::kBf16)) != MLA_OK ||
      (st = encode_out(&maps.part_out, r.a.part_u, p->n_h, (uint64_t)r.slots,
                       r.a.part_f16 ? OutType::kF16 : OutType::kBf16)) !=
          MLA_OK)
    return st;
  return cuda_status(launch_decode_sm100(r.a, maps, s));
}

}  // namespace

// csrc/merge.cu: the merge of partial results over pieces of the context
cudaError_t launch_merge(const void* u_parts, const float* lse_parts, void* u, float* lse, int R,
                         int rows, int d_c, bool bf16, cudaStream_t s);

WsLayout ws_layout(int B, int s_q, int n_h, int d_c, int num_chunks) {
  WsLayout L;
  L.slots = (long long)(B + num_chunks) * s_q;
  size_t off = 0;
  L.header = off;
  off += 256;
  L.tile_prefix = off;
  off = align_up(off + sizeof(int) * (B + 1), 256);
  L.split_base = off;
  off = align_up(off + sizeof(int) * (B + 1), 256);
  L.chunk_t = off;
  off = align_up(off + sizeof(int) * (num_chunks + 1), 256);
  L.chunk_b = off;
  off = align_up(off + sizeof(int) * 4 * (size_t)num_chunks, 256);
  L.part_lse = off;
  off = align_up(off + sizeof(float) * (size_t)L.slots * n_h, 256);
  L.part_u = off;
  off = align_up(off + sizeof(float) * (size_t)L.slots * n_h * d_c, 256);
  L.total = off;
  return L;
}

}  // namespace mla

using namespace mla;

extern "C" {

const char* mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARG: return "invalid argument";
    case MLA_ERR_UNSUPPORTED: return "unsupported configuration";
    case MLA_ERR_CUDA: return "CUDA error";
    case MLA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MLA_ERR_DEVICE_CHECK: return "device-side check failed";
  }
  return "unknown status";
}

mla_status mla_decode_workspace_size(const mla_decode_params* p, size_t* bytes) {
  if (bytes == nullptr) return MLA_ERR_INVALID_ARG;
  mla_status st = validate_decode(p);
  if (st != MLA_OK) return st;
  const DeviceInfo* d = nullptr;
  if ((st = device_info(&d)) != MLA_OK) return st;
  *bytes = ws_layout(p->B, p->s_q, p->n_h, p->d_c, choose_chunks(p, d)).total;
  return MLA_OK;
}

mla_status mla_decode_kernel_info(const mla_decode_params* p, int* uses_tensor_cores,
                                  int* num_chunks) {
  mla_status st = validate_decode(p);
  if (st != MLA_OK) return st;
  const DeviceInfo* d = nullptr;
  if ((st = device_info(&d)) != MLA_OK) return st;
  if (uses_tensor_cores) *uses_tensor_cores = select_kernel(p, d) != Kernel::kNone ? 1 : 0;
  if (num_chunks) *num_chunks = choose_chunks(p, d);
  return MLA_OK;
}

mla_status mla_decode_plan(const mla_decode_params* p, void* ws, size_t ws_bytes, void* stream) {
  if (p != nullptr && p->B == 0) return validate_decode(p);
  Resolved r;
  mla_status st = resolve(p, ws, ws_bytes, &r);
  if (st != MLA_OK) return st;
  return cuda_status(launch_plan(r.a, static_cast<cudaStream_t>(stream)));
}

mla_status mla_decode_attend(const mla_decode_params* p, void* ws, size_t ws_bytes, void* stream) {
  if (p != nullptr && p->B == 0) return validate_decode(p);
  Resolved r;
  mla_status st = resolve(p, ws, ws_bytes, &r);
  if (st != MLA_OK) return st;
  return attend(r, p, static_cast<cudaStream_t>(stream), false);
}

mla_status mla_decode_combine(const mla_decode_params* p, void* ws, size_t ws_bytes, void* stream) {
  if (p != nullptr && p->B == 0) return validate_decode(p);
  Resolved r;
  mla_status st = resolve(p, ws, ws_bytes, &r);
  if (st != MLA_OK) return st;
  return cuda_status(launch_combine(r.a, static_cast<cudaStream_t>(stream)));
}

mla_status mla_decode(const mla_decode_params* p, void* ws, size_t ws_bytes, void* stream) {
  if (p != nullptr && p->B == 0) return validate_decode(p);
  Resolved r;
  mla_status st = resolve(p, ws, ws_bytes, &r);
  if (st != MLA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = cuda_status(launch_plan(r.a, s))) != MLA_OK) return st;
  if ((st = attend(r, p, s, true)) != MLA_OK) return st;
  r.a.pdl = true;
  return cuda_status(launch_combine(r.a, s));
}

mla_status mla_decode_step(const mla_decode_params* p, const void* W_UV, void* o, int d_v,
                           void* ws, size_t ws_bytes, void* stream) {
  if (p != nullptr && p->B == 0) return validate_decode(p);
  if (W_UV == nullptr || o == nullptr || d_v < 1) return MLA_ERR_INVALID_ARG;
  if (!aligned16(W_UV) || !aligned16(o)) return MLA_ERR_INVALID_ARG;
  Resolved r;
  mla_status st = resolve(p, ws, ws_bytes, &r);
  if (st != MLA_OK) return st;
  if (r.kernel != Kernel::kV3 || !r.a.out_f32 || d_v > 128 || !r.dev->up_proj_tc)
    return MLA_ERR_UNSUPPORTED;
  if ((long long)p->n_h * d_v > INT_MAX) return MLA_ERR_UNSUPPORTED;
  CUtensorMap w_map;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)p->d_c, (cuuint64_t)p->n_h * d_v};
    const cuuint64_t strides[1] = {(cuuint64_t)p->d_c * 2};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t estr[2] = {1, 1};
    if (g_encode(&w_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(W_UV), dims, strides,
                 box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = cuda_status(launch_plan(r.a, s))) != MLA_OK) return st;
  if ((st = attend(r, p, s, true)) != MLA_OK) return st;
  const int T = p->B * p->s_q;
  return cuda_status(launch_up_proj_sm100_f32u(w_map, static_cast<const float*>(p->u), o, r.dev->flags, T,
                                               p->n_h, p->d_c, d_v, true, s, &r.a));
}

mla_status mla_absorb_weights(const void* W_UK, const void* W_Q, void* W_QK, int n_h, int d_h,
                              int d_c, int d_model, mla_dtype dtype, void* stream) {
  if (!W_UK || !W_Q || !W_QK || !valid_dtype(dtype)) return MLA_ERR_INVALID_ARG;
  if (n_h < 1 || d_h < 1 || d_c < 1 || d_model < 1) return MLA_ERR_INVALID_ARG;
  if (n_h > 65535) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(W_UK) || !aligned16(W_Q) || !aligned16(W_QK)) return MLA_ERR_INVALID_ARG;
  const DeviceInfo* d = nullptr;
  mla_status st = device_info(&d);
  if (st != MLA_OK) return st;
  GemmArgs g = {};
  g.A = W_UK;  // A(z, m = c, k) = W_UK[z][k][c]
  g.Bm = W_Q;  // B(z, n = d, k) = W_Q[z][k][d]
  g.C = W_QK;
  g.M = d_c;
  g.N = d_model;
  g.K = d_h;
  g.Z = n_h;
  g.sAz = (long long)d_h * d_c;
  g.sAm = 1;
  g.sAk = d_c;
  g.sBz = (long long)d_h * d_model;
  g.sBn = 1;
  g.sBk = d_model;
  g.sCz = (long long)d_c * d_model;
  g.sCm = d_model;
  g.seg = INT_MAX;
  g.err = d->flags;
  g.bf16 = dtype == MLA_DTYPE_BF16;
  return cuda_status(launch_gemm(g, static_cast<cudaStream_t>(stream)));
}

mla_status mla_form_query(const void* h, const void* W_QK, const void* W_QR, const int* pos,
                          void* q, int T, int n_h, int d_model, int d_c, int d_R, float rope_base,
                          mla_dtype dtype, void* workspace, size_t workspace_bytes, void* stream) {
  if (!valid_dtype(dtype) || T < 0 || n_h < 1 || d_model < 1 || d_c < 1 || d_R < 0 || d_R % 2)
    return MLA_ERR_INVALID_ARG;
  if (!(rope_base > 0.f) || !std::isfinite(rope_base)) return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (!h || !W_QK || !q || (d_R > 0 && (!W_QR || !pos))) return MLA_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(W_QK) || !aligned16(q) || (W_QR && !aligned16(W_QR)))
    return MLA_ERR_INVALID_ARG;
  if (T > 65535 * 64) return MLA_ERR_UNSUPPORTED;
  const DeviceInfo* d = nullptr;
  mla_status st = device_info(&d);
  if (st != MLA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int W = d_c + d_R;
  if (dtype == MLA_DTYPE_BF16) {
    // tensor cores: W = [W^QK (n_h * d_c rows) ; W^QR (n_h * d_R rows)]
    if (!d->wgemm_tc || g_encode == nullptr) return MLA_ERR_UNSUPPORTED;
    if (d_model % 64 != 0 || d_R % 2 != 0 || (d_R > 0 && 128 % d_R != 0)) return MLA_ERR_UNSUPPORTED;
    const int rows0 = n_h * d_c, rows1 = n_h * d_R;
    WgemmLaunch L = {};
    L.tiles0 = tiles_of(rows0);
    L.tiles = L.tiles0 + tiles_of(rows1);
    if (workspace_bytes < proj_acc_bytes(L.tiles) || workspace == nullptr ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      return workspace_bytes < proj_acc_bytes(L.tiles) ? MLA_ERR_WORKSPACE_TOO_SMALL : MLA_ERR_INVALID_ARG;
    if ((st = encode_rows(&L.w_map[0], W_QK, d_model, rows0, 128)) != MLA_OK) return st;
    L.w_map[1] = L.w_map[0];
    if (rows1 > 0 && (st = encode_rows(&L.w_map[1], W_QR, d_model, rows1, 128)) != MLA_OK) return st;
    L.K = d_model;
    L.workspace = workspace;
    L.err = d->flags;
    L.mode = 3;
    L.n_h = n_h;
    L.d_c = d_c;
    L.d_R = d_R;
    L.rope_base = rope_base;
    return run_projection(L, h, d_model, T, 1, d, s, [&](WgemmLaunch& C, int t0) {
      C.out = static_cast<__nv_bfloat16*>(q) + (size_t)t0 * n_h * W;
      C.pos = pos + t0;
    });
  }
  // fp32 tensors: the tiled CUDA-core GEMM
  GemmArgs g = {};
  g.A = h;
  g.M = T;
  g.K = d_model;
  g.Z = 1;
  g.sAm = d_model;
  g.sAk = 1;
  g.sBk = 1;
  g.sBn = d_model;
  g.sCm = (long long)n_h * W;
  g.err = d->flags;
  g.bf16 = dtype == MLA_DTYPE_BF16;
  // latent part: n = i * d_c + c
  g.Bm = W_QK;
  g.C = q;
  g.N = n_h * d_c;
  g.seg = d_c;
  g.seg_stride = W;
  g.col_off = 0;
  if ((st = cuda_status(launch_gemm(g, s))) != MLA_OK) return st;
  if (d_R == 0) return MLA_OK;
  // RoPE part: n = i * d_R + k, rotated by the query position
  g.Bm = W_QR;
  g.N = n_h * d_R;
  g.seg = d_R;
  g.seg_stride = W;
  g.col_off = d_c;
  g.pos = pos;
  g.rope = 1;
  g.rope_base = rope_base;
  return cuda_status(launch_gemm(g, s));
}

mla_status mla_append_latent(const void* h, const void* W_DKV, const void* W_KR,
                             const int* seq_ids, const int* pos, const int* block_table,
                             int max_pages_per_seq, int page_size, int num_pages, void* kv_cache,
                             int T, int d_model, int d_c, int d_R, float rope_base,
                             mla_dtype dtype, void* workspace, size_t workspace_bytes,
                             void* stream) {
  if (!valid_dtype(dtype) || T < 0 || d_model < 1 || d_c < 1 || d_R < 0 || d_R % 2 ||
      page_size < 1 || max_pages_per_seq < 1 || num_pages < 1)
    return MLA_ERR_INVALID_ARG;
  if (!(rope_base > 0.f) || !std::isfinite(rope_base)) return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (!h || !W_DKV || !seq_ids || !pos || !block_table || !kv_cache || (d_R > 0 && !W_KR))
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(W_DKV) || !aligned16(kv_cache) || (W_KR && !aligned16(W_KR)))
    return MLA_ERR_INVALID_ARG;
  if (T > 65535 * 64) return MLA_ERR_UNSUPPORTED;
  const DeviceInfo* d = nullptr;
  mla_status st = device_info(&d);
  if (st != MLA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == MLA_DTYPE_BF16) {
    // tensor cores: W = [W^DKV (d_c rows) ; W^KR (d_R rows)]
    if (!d->wgemm_tc || g_encode == nullptr) return MLA_ERR_UNSUPPORTED;
    if (d_model % 64 != 0 || d_R % 2 != 0 || d_R > 128) return MLA_ERR_UNSUPPORTED;
    WgemmLaunch L = {};
    L.tiles0 = tiles_of(d_c);
    L.tiles = L.tiles0 + tiles_of(d_R);
    if (workspace_bytes < proj_acc_bytes(L.tiles) || workspace == nullptr ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      return workspace_bytes < proj_acc_bytes(L.tiles) ? MLA_ERR_WORKSPACE_TOO_SMALL : MLA_ERR_INVALID_ARG;
    if ((st = encode_rows(&L.w_map[0], W_DKV, d_model, d_c, 128)) != MLA_OK) return st;
    L.w_map[1] = L.w_map[0];
    if (d_R > 0 && (st = encode_rows(&L.w_map[1], W_KR, d_model, d_R, 128)) != MLA_OK) return st;
    L.K = d_model;
    L.workspace = workspace;
    L.err = d->flags;
    L.mode = 1;
    L.out = kv_cache;
    L.d_c = d_c;
    L.d_R = d_R;
    L.block_table = block_table;
    L.max_pages = max_pages_per_seq;
    L.page_size = page_size;
    L.num_pages = num_pages;
    L.rope_base = rope_base;
    return run_projection(L, h, d_model, T, 1, d, s, [&](WgemmLaunch& C, int t0) {
      C.pos = pos + t0;
      C.seq = seq_ids + t0;
    });
  }
  // fp32 tensors: the tiled CUDA-core GEMM
  GemmArgs g = {};
  g.A = h;
  g.C = kv_cache;
  g.M = T;
  g.K = d_model;
  g.Z = 1;
  g.sAm = d_model;
  g.sAk = 1;
  g.sBn = d_model;
  g.sBk = 1;
  g.sCm = d_c + d_R;
  g.seg = INT_MAX;
  g.pos = pos;
  g.seq = seq_ids;
  g.block_table = block_table;
  g.max_pages = max_pages_per_seq;
  g.page_size = page_size;
  g.num_pages = num_pages;
  g.err = d->flags;
  g.bf16 = dtype == MLA_DTYPE_BF16;
  g.Bm = W_DKV;
  g.N = d_c;
  g.col_off = 0;
  if ((st = cuda_status(launch_gemm(g, s))) != MLA_OK) return st;
  if (d_R == 0) return MLA_OK;
  g.Bm = W_KR;
  g.N = d_R;
  g.col_off = d_c;
  g.seg = d_R;
  g.seg_stride = 0;
  g.rope = 1;
  g.rope_base = rope_base;
  return cuda_status(launch_gemm(g, s));
}

mla_status mla_up_proj(const void* u, const void* W_UV, void* o, int T, int n_h, int d_c, int d_v,
                       mla_dtype u_dtype, mla_dtype dtype, void* stream) {
  if (!valid_dtype(dtype) || !valid_dtype(u_dtype) || T < 0 || n_h < 1 || d_c < 1 || d_v < 1)
    return MLA_ERR_INVALID_ARG;
  if (u_dtype != dtype && u_dtype != MLA_DTYPE_FP32) return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (!u || !W_UV || !o) return MLA_ERR_INVALID_ARG;
  if (!aligned16(u) || !aligned16(W_UV) || !aligned16(o)) return MLA_ERR_INVALID_ARG;
  if (n_h > 65535 || T > 65535 * 32 || d_v > 128) return MLA_ERR_UNSUPPORTED;
  const bool f32 = dtype == MLA_DTYPE_FP32;
  if (f32 ? (d_c % 32 != 0 || d_c > 256) : (d_c % 64 != 0 || d_c > 512))
    return MLA_ERR_UNSUPPORTED;
  if ((long long)n_h * d_v > INT_MAX) return MLA_ERR_UNSUPPORTED;
  const DeviceInfo* d = nullptr;
  mla_status st = device_info(&d);
  if (st != MLA_OK) return st;
  if (!d->up_proj_tc || g_encode == nullptr) return MLA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint64_t es = f32 ? 4 : 2;
  const CUtensorMapDataType tdt = f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const cuuint32_t cols = static_cast<cuuint32_t>(128 / es);  // one 128-byte row per box row
  CUtensorMap w_map, u_map;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)d_c, (cuuint64_t)n_h * d_v};
    const cuuint64_t strides[1] = {(cuuint64_t)d_c * es};
    const cuuint32_t box[2] = {cols, 128};
    const cuuint32_t estr[2] = {1, 1};
    if (g_encode(&w_map, tdt, 2, const_cast<void*>(W_UV), dims, strides, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  }
  if (!f32 && u_dtype == MLA_DTYPE_FP32)
    return cuda_status(launch_up_proj_sm100_f32u(w_map, static_cast<const float*>(u), o, d->flags,
                                                 T, n_h, d_c, d_v, false, s));
  {
    const cuuint64_t dims[3] = {(cuuint64_t)d_c, (cuuint64_t)n_h, (cuuint64_t)T};
    const cuuint64_t strides[2] = {(cuuint64_t)d_c * es, (cuuint64_t)n_h * d_c * es};
    const cuuint32_t box[3] = {cols, 1, (cuuint32_t)up_proj_sm100_box_rows(T)};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (g_encode(&u_map, tdt, 3, const_cast<void*>(u), dims, strides, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  }
  return cuda_status(launch_up_proj_sm100(w_map, u_map, o, d->flags, T, n_h, d_c, d_v, f32, false, s));
}

namespace {

mla_status validate_gqa(const mla_gqa_params* p) {
  if (p == nullptr) return MLA_ERR_INVALID_ARG;
  if (p->B < 0 || p->s_q < 1 || p->n_h < 1 || p->n_g < 1 || p->d_h < 1 || p->d_v < 1 || p->d_R < 0)
    return MLA_ERR_INVALID_ARG;
  if (p->s_q > 2 || p->n_h % p->n_g != 0) return p->s_q > 2 ? MLA_ERR_UNSUPPORTED : MLA_ERR_INVALID_ARG;
  if (p->page_size <= 0 || p->page_size % kTileTokens != 0) return MLA_ERR_INVALID_ARG;
  if (p->max_pages_per_seq < 1 || p->num_pages < 1) return MLA_ERR_INVALID_ARG;
  if (!std::isfinite(p->softmax_scale) || !(p->softmax_scale > 0.f)) return MLA_ERR_INVALID_ARG;
  if (p->d_R % 8 != 0 || p->num_splits < 0) return MLA_ERR_INVALID_ARG;
  if (p->dtype != MLA_DTYPE_BF16) return valid_dtype(p->dtype) ? MLA_ERR_UNSUPPORTED : MLA_ERR_INVALID_ARG;
  if (p->d_h % 64 != 0 || p->d_v % 64 != 0 || p->d_h + p->d_R > 256 || p->d_v > 256 ||
      (p->n_h / p->n_g) * p->s_q > 128)
    return MLA_ERR_UNSUPPORTED;
  if ((long long)p->num_pages * p->page_size > INT_MAX ||
      (long long)p->max_pages_per_seq * p->page_size > INT_MAX)
    return MLA_ERR_UNSUPPORTED;
  if (p->B == 0) return MLA_OK;
  if (!p->q || !p->kv || (p->d_R > 0 && !p->k_rope) || !p->block_table || !p->seqlens || !p->o)
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(p->q) || !aligned16(p->kv) || (p->k_rope && !aligned16(p->k_rope)) ||
      !aligned16(p->o) || !aligned16(p->block_table) || !aligned16(p->seqlens) ||
      (p->lse && !aligned16(p->lse)))
    return MLA_ERR_INVALID_ARG;
  return MLA_OK;
}

int gqa_chunks(const mla_gqa_params* p, const DeviceInfo* d) {
  if (p->num_splits > 0) return p->num_splits;
  return std::max(1, d->sm_count / p->n_g);  // one CTA per SM
}

}  // namespace

mla_status mla_decode_gqa_workspace_size(const mla_gqa_params* p, size_t* bytes) {
  if (bytes == nullptr) return MLA_ERR_INVALID_ARG;
  mla_status st = validate_gqa(p);
  if (st != MLA_OK) return st;
  const DeviceInfo* d = nullptr;
  if ((st = device_info(&d)) != MLA_OK) return st;
  *bytes = ws_layout(p->B, p->s_q, p->n_h, p->d_v, gqa_chunks(p, d)).total;
  return MLA_OK;
}

mla_status mla_decode_gqa(const mla_gqa_params* p, void* ws, size_t ws_bytes, void* stream) {
  mla_status st = validate_gqa(p);
  if (st != MLA_OK || p->B == 0) return st;
  const DeviceInfo* d = nullptr;
  if ((st = device_info(&d)) != MLA_OK) return st;
  if (d->cc_major != 10 || !d->small_tc || g_encode == nullptr) return MLA_ERR_UNSUPPORTED;
  const int G = gqa_chunks(p, d);
  const WsLayout L = ws_layout(p->B, p->s_q, p->n_h, p->d_v, G);
  if (ws_bytes < L.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MLA_ERR_INVALID_ARG;
  uint8_t* w = static_cast<uint8_t*>(ws);
  DecodeArgs a = {};
  a.q = p->q;
  a.kv = p->kv;
  a.block_table = p->block_table;
  a.seqlens = p->seqlens;
  a.u = p->o;
  a.lse = p->lse;
  a.header = reinterpret_cast<int*>(w + L.header);
  a.tile_prefix = reinterpret_cast<int*>(w + L.tile_prefix);
  a.split_base = reinterpret_cast<int*>(w + L.split_base);
  a.chunk_t = reinterpret_cast<int*>(w + L.chunk_t);
  a.chunk_b = reinterpret_cast<int*>(w + L.chunk_b);
  a.part_lse = reinterpret_cast<float*>(w + L.part_lse);
  a.part_u = reinterpret_cast<float*>(w + L.part_u);
  a.err = d->flags;
  a.B = p->B;
  a.s_q = p->s_q;
  a.n_h = p->n_h;
  a.d_c = p->d_v;  // output width for the attend epilogue and the combine
  a.d_R = p->d_R;
  a.page_size = p->page_size;
  a.max_pages = p->max_pages_per_seq;
  a.num_pages = p->num_pages;
  a.num_chunks = G;
  a.scale = p->softmax_scale;
  a.bf16 = true;
  a.out_f32 = p->o_fp32 != 0;
  a.part_bf16 = false;
  a.part_f16 = false;
  a.pdl = false;
  const int hpg = p->n_h / p->n_g;
  const uint64_t wq = (uint64_t)p->d_h + p->d_R, wkv = (uint64_t)p->d_h + p->d_v;
  const uint64_t rows = (uint64_t)p->num_pages * p->page_size;
  CUtensorMap q_map, kv_map, kr_map;
  memset(&kr_map, 0, sizeof(kr_map));
  {
    const cuuint64_t dims[3] = {wq, (cuuint64_t)p->n_h, (cuuint64_t)p->B * p->s_q};
    const cuuint64_t strides[2] = {wq * 2, (cuuint64_t)p->n_h * wq * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)hpg, (cuuint32_t)p->s_q};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (g_encode(&q_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(p->q), dims, strides,
                 box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  }
  {
    const cuuint64_t dims[3] = {wkv, (cuuint64_t)p->n_g, rows};
    const cuuint64_t strides[2] = {wkv * 2, (cuuint64_t)p->n_g * wkv * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)kTileTokens};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (g_encode(&kv_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(p->kv), dims,
                 strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  }
  if (p->d_R > 0 && (st = encode_2d(&kr_map, p->k_rope, p->d_R, rows, 64, kTileTokens,
                                    CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK)
    return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = cuda_status(launch_plan(a, s))) != MLA_OK) return st;
  const GqaShape gs{p->n_g, p->d_h, p->d_v, p->d_R};
  if ((st = cuda_status(launch_decode_gqa_sm100(a, gs, q_map, kv_map, kr_map, s))) != MLA_OK) return st;
  return cuda_status(launch_combine(a, s));
}

mla_status mla_projection_workspace_size(int rows0, int rows1, int T, int x_fp32_K,
                                         size_t* bytes) {
  if (bytes == nullptr || rows0 < 0 || rows1 < 0 || T < 0 || x_fp32_K < 0) return MLA_ERR_INVALID_ARG;
  size_t b = proj_acc_bytes(tiles_of(rows0) + tiles_of(rows1));
  if (x_fp32_K > 0) b += align_up((size_t)2 * T * x_fp32_K * 2, 256);
  *bytes = b;
  return MLA_OK;
}

mla_status mla_form_query_fused(const void* h, const void* W_Q, const void* W_UK,
                                const void* W_QR, const int* pos, void* q, int T, int n_h,
                                int d_h, int d_model, int d_c, int d_R, float rope_base,
                                void* workspace, size_t workspace_bytes, void* stream) {
  if (T < 0 || n_h < 1 || d_h < 1 || d_model < 1 || d_c < 1 || d_R < 0 || d_R % 2)
    return MLA_ERR_INVALID_ARG;
  if (!(rope_base > 0.f) || !std::isfinite(rope_base)) return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (!h || !W_Q || !W_UK || !q || (d_R > 0 && (!W_QR || !pos))) return MLA_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(W_Q) || !aligned16(W_UK) || !aligned16(q) ||
      (W_QR && !aligned16(W_QR)))
    return MLA_ERR_INVALID_ARG;
  // one 128-row tile per head of W^Q, whole heads of W^QR per tile, d_c in
  // 128-row steps of the second product
  if (d_h != 128 || d_c % 128 != 0 || d_c > 512 || d_model % 64 != 0 ||
      (d_R > 0 && 128 % d_R != 0))
    return MLA_ERR_UNSUPPORTED;
  const DeviceInfo* d = nullptr;
  mla_status st = device_info(&d);
  if (st != MLA_OK) return st;
  if (!d->wgemm_tc || g_encode == nullptr) return MLA_ERR_UNSUPPORTED;
  const int rows0 = n_h * d_h, rows1 = n_h * d_R;
  WgemmLaunch L = {};
  L.tiles0 = tiles_of(rows0);
  L.tiles = L.tiles0 + tiles_of(rows1);
  if (workspace_bytes < proj_acc_bytes(L.tiles)) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return MLA_ERR_INVALID_ARG;
  if ((st = encode_rows(&L.w_map[0], W_Q, d_model, rows0, 128)) != MLA_OK) return st;
  L.w_map[1] = L.w_map[0];
  if (rows1 > 0 && (st = encode_rows(&L.w_map[1], W_QR, d_model, rows1, 128)) != MLA_OK) return st;
  if ((st = encode_rows(&L.uk_map, W_UK, d_c, (uint64_t)n_h * d_h, 128)) != MLA_OK) return st;
  L.K = d_model;
  L.workspace = workspace;
  L.err = d->flags;
  L.mode = 0;
  L.n_h = n_h;
  L.d_c = d_c;
  L.d_R = d_R;
  L.rope_base = rope_base;
  const int W = d_c + d_R;
  return run_projection(L, h, d_model, T, 1, d, static_cast<cudaStream_t>(stream),
                        [&](WgemmLaunch& C, int t0) {
                          C.out = static_cast<__nv_bfloat16*>(q) + (size_t)t0 * n_h * W;
                          C.pos = pos + t0;
                        });
}

mla_status mla_fold_output_weights(const void* W_O, const void* W_UV, void* W_OUV, int n_h, int d_v,
                                   int d_c, int d_model, mla_dtype dtype, void* stream) {
  if (!W_O || !W_UV || !W_OUV || !valid_dtype(dtype)) return MLA_ERR_INVALID_ARG;
  if (n_h < 1 || d_v < 1 || d_c < 1 || d_model < 1) return MLA_ERR_INVALID_ARG;
  if (n_h > 65535) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(W_O) || !aligned16(W_UV) || !aligned16(W_OUV)) return MLA_ERR_INVALID_ARG;
  const DeviceInfo* d = nullptr;
  mla_status st = device_info(&d);
  if (st != MLA_OK) return st;
  // W_OUV[m][i * d_c + c] = sum_v W_O[m][i * d_v + v] W_UV[i][v][c]
  GemmArgs g = {};
  g.A = W_O;    // A(z = i, m, k = v) = W_O[m][i * d_v + v]
  g.Bm = W_UV;  // B(z, n = c, k = v) = W_UV[i][v][c]
  g.C = W_OUV;  // C(z, m, n) = W_OUV[m][i * d_c + n]
  g.M = d_model;
  g.N = d_c;
  g.K = d_v;
  g.Z = n_h;
  g.sAz = d_v;
  g.sAm = (long long)n_h * d_v;
  g.sAk = 1;
  g.sBz = (long long)d_v * d_c;
  g.sBn = 1;
  g.sBk = d_c;
  g.sCz = d_c;
  g.sCm = (long long)n_h * d_c;
  g.seg = INT_MAX;
  g.err = d->flags;
  g.bf16 = dtype == MLA_DTYPE_BF16;
  return cuda_status(launch_gemm(g, static_cast<cudaStream_t>(stream)));
}

mla_status mla_output_projection(const void* x, mla_dtype x_dtype, const void* W, void* y, int T,
                                 int K, int M, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  if (!valid_dtype(x_dtype) || T < 0 || K < 1 || M < 1) return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (!x || !W || !y) return MLA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(W) || !aligned16(y)) return MLA_ERR_INVALID_ARG;
  if (K % 64 != 0 || M % 8 != 0) return MLA_ERR_UNSUPPORTED;
  const DeviceInfo* d = nullptr;
  mla_status st = device_info(&d);
  if (st != MLA_OK) return st;
  if (!d->wgemm_tc || g_encode == nullptr) return MLA_ERR_UNSUPPORTED;
  const bool f32 = x_dtype == MLA_DTYPE_FP32;
  WgemmLaunch L = {};
  L.tiles0 = L.tiles = tiles_of(M);
  const size_t acc = proj_acc_bytes(L.tiles);
  const size_t need = acc + (f32 ? align_up((size_t)2 * T * K * 2, 256) : 0);
  if (workspace_bytes < need) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return MLA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const void* X = x;
  if (f32) {
    // an fp32 x enters as two bf16 rows per token whose products are added
    void* pairs = static_cast<uint8_t*>(workspace) + acc;
    if ((st = cuda_status(launch_split_rows(static_cast<const float*>(x), pairs, T, K, s))) != MLA_OK)
      return st;
    X = pairs;
  }
  if ((st = encode_rows(&L.w_map[0], W, K, M, 128)) != MLA_OK) return st;
  L.w_map[1] = L.w_map[0];
  L.K = K;
  L.workspace = workspace;
  L.err = d->flags;
  L.mode = 2;
  L.ldo = M;
  L.pair = f32 ? 2 : 1;
  return run_projection(L, X, K, T, L.pair, d, s, [&](WgemmLaunch& C, int t0) {
    C.out = static_cast<__nv_bfloat16*>(y) + (size_t)t0 * M;
  });
}

mla_status mla_merge_partials(const void* u_parts, const float* lse_parts, void* u, float* lse,
                              int R, int rows, int d_c, mla_dtype dtype, void* stream) {
  if (!valid_dtype(dtype) || R < 1 || rows < 0 || d_c < 8 || d_c % 8 != 0)
    return MLA_ERR_INVALID_ARG;
  if (rows == 0) return MLA_OK;
  if (!u_parts || !lse_parts || !u) return MLA_ERR_INVALID_ARG;
  if (!aligned16(u_parts) || !aligned16(u) || (lse && !aligned16(lse)) ||
      (reinterpret_cast<uintptr_t>(lse_parts) & 3u) != 0)
    return MLA_ERR_INVALID_ARG;
  if ((long long)R * rows * d_c > (1LL << 40)) return MLA_ERR_UNSUPPORTED;
  const DeviceInfo* d = nullptr;
  mla_status st = device_info(&d);
  if (st != MLA_OK) return st;
  return cuda_status(launch_merge(u_parts, lse_parts, u, lse, R, rows, d_c,
                                  dtype == MLA_DTYPE_BF16, static_cast<cudaStream_t>(stream)));
}

mla_status mla_selftest_wait(int arrive, void* stream) {
  const DeviceInfo* d = nullptr;
  mla_status st = device_info(&d);
  if (st != MLA_OK) return st;
  return cuda_status(launch_wait_selftest(d->flags, arrive != 0, static_cast<cudaStream_t>(stream)));
}

mla_status mla_check_device_errors(void* stream, int* flags) {
  const DeviceInfo* d = nullptr;
  mla_status st = device_info(&d);
  if (st != MLA_OK) return st;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_status(e);
  int v = 0;
  if ((e = cudaMemcpy(&v, d->flags, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_status(e);
  if (v != 0) {
    const int zero = 0;
    if ((e = cudaMemcpy(d->flags, &zero, sizeof(int), cudaMemcpyHostToDevice)) != cudaSuccess)
      return cuda_status(e);
  }
  if (flags) *flags = v;
  return v == 0 ? MLA_OK : MLA_ERR_DEVICE_CHECK;
}

}  // extern "C"
