// Declarations shared by the translation units of libmla (not part of the ABI).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "mla.h"

namespace mla {

constexpr int kTileTokens = 64;   // cache rows per attention tile
constexpr int kMaxHeads = 128;    // query heads packed as the MMA M dimension

// Cost of starting one more sequence inside a KV chunk (loading its queries,
// writing its output), in units of one 64-token tile.  The plan cuts chunks on
// a line where every sequence start takes this many units on top of its tiles,
// so chunks that hold several sequences get fewer tiles.  A second segment in
// a chunk costs the attend kernel about 6-8 us (epilogue, query load,
// pipeline refill), 5-6 tiles at 1.3-1.4 us each.
constexpr int kSegCostTiles = 6;

// Workspace of mla_decode.  Header ints: [0] total tiles, [1] line units per
// chunk, [2] number of chunks, [3] split rows in use, [4] units per sequence
// start, [5] 1 when the chunks follow the sequences (see the plan kernel),
// [6] the chunks in use (the others are empty).
// chunk_t[c] is the first tile of chunk c (chunk_t[chunks] = total tiles);
// chunk_b[4 c .. 4 c + 3] is chunk c's record: the sequence that tile belongs
// to, the index of that piece among its sequence's pieces (0 when the chunk
// starts at the sequence's first tile), and that sequence's first and end
// tile on the line (16-byte aligned, one load).
struct WsLayout {
  size_t header = 0, tile_prefix = 0, split_base = 0, chunk_t = 0, chunk_b = 0, part_lse = 0,
         part_u = 0, total = 0;
  long long slots = 0;  // partial (u, lse) rows per head: (B + chunks) * s_q
};
WsLayout ws_layout(int B, int s_q, int n_h, int d_c, int num_chunks);

// Everything a decode stage needs, resolved from mla_decode_params + workspace.
struct DecodeArgs {
  const void* q;
  const void* kv;
  const int* block_table;
  const int* seqlens;
  void* u;
  float* lse;
  int* header;
  int* tile_prefix;
  int* split_base;
  int* chunk_t;
  int* chunk_b;
  float* part_u;
  float* part_lse;
  int* err;
  int B, s_q, n_h, d_c, d_R, page_size, max_pages, num_pages, num_chunks;
  float scale;
  bool bf16;       // q and the cache are bf16 (else fp32)
  bool out_f32;    // u is fp32 (else bf16)
  bool part_bf16;  // split partials of u are bf16 (the DeepSeek-V3-shape kernel with a bf16 u)
  bool part_f16;   // split partials of u are fp16 (that kernel with an fp32 u); else fp32
  bool pdl;        // launch as a programmatic dependent of the previous kernel
};

cudaError_t launch_plan(const DecodeArgs& a, cudaStream_t s);
// one bounded mbarrier wait, on a phase that completes (arrive) or never does
cudaError_t launch_wait_selftest(int* err, bool arrive, cudaStream_t s);
cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t s);

// Tensor-core decode for small latent widths (one CTA per KV chunk and query
// row): fp32 with d_c a multiple of 32, d_c + d_R <= 128 (tf32), or bf16 with
// d_c a multiple of 64, d_c + d_R <= 256.  q_map: q [B * s_q, n_h, d_c + d_R]
// with boxes of 128 bytes x 128 heads x 1; kv_map: the cache [rows, d_c + d_R]
// with boxes of 128 bytes x 64 rows; both 128-byte swizzle.  kv_pv_map (fp32
// only): the cache again with 128-byte swizzle of 32-byte atoms.  Split
// partials are fp32.
bool decode_small_sm100_supported(bool bf16, int d_c, int d_R);
// GQA path of GQLA on the same kernel (bf16): one CTA per (KV chunk, group),
// every head of the group and every query row as MMA rows.  q_map: q
// [B * s_q, n_h, d_h + d_R], box 64 x heads-per-group x s_q; kv_map: the
// expanded cache [rows, n_g, d_h + d_v], box 64 x 1 x 64; kr_map: the RoPE
// keys [rows, d_R], box 64 x 64; 128-byte swizzle.  a.d_c carries d_v.
struct GqaShape {
  int n_g, d_h, d_v, d_R;
};
cudaError_t launch_decode_gqa_sm100(const DecodeArgs& a, const GqaShape& gs, const CUtensorMap& q_map,
                                    const CUtensorMap& kv_map, const CUtensorMap& kr_map,
                                    cudaStream_t s);
int decode_small_sm100_prepare();
cudaError_t launch_decode_small_sm100(const DecodeArgs& a, const CUtensorMap& q_map,
                                      const CUtensorMap& kv_map, const CUtensorMap& kv_pv_map,
                                      cudaStream_t s);

// Tensor-core decode for n_h <= 128, d_c = 512, d_R = 64, bf16.
// kv maps over the cache [rows, 576]: latent boxes 64 x 64 rows (128-byte
// swizzle), RoPE boxes 32 x 64 rows (64-byte swizzle).  q maps over the
// queries [B * s_q, n_h, 576]: latent boxes 64 x 16 heads x 1 (128-byte
// swizzle), RoPE boxes 32 x 16 heads x 1 (64-byte swizzle); heads past n_h
// read as zero.
// out maps over u [B * s_q, n_h, 512] and over the split partials
// [slots, n_h, 512], both bf16 (boxes 64 x 32 heads x 1) or both fp32
// (boxes 32 x 32 heads x 1), 128-byte swizzle, for the TMA stores of the
// epilogue; heads past n_h are not written.
//
// kv_lat4 covers one CTA's four 64-column latent blocks of 64 rows in one
// copy: dimensions (column, row, block & 1, block >> 1) with byte strides
// (1152, 128, 512); q_lat5 / q_rope5 cover a CTA's whole query area in one
// copy each: (column, head within 16, column half, group of 16 heads, query
// row) with the column half's stride 256 / 64 bytes.  has_kv4 / has_q5 say
// whether they were encoded (has_q5 needs n_h % 16 == 0); otherwise the
// kernel issues the per-block copies.
struct Sm100Maps {
  CUtensorMap kv_lat, kv_rope, q_lat, q_rope, u_out, part_out;
  CUtensorMap kv_lat4, q_lat5, q_rope5;
  int has_kv4, has_q5;
};
cudaError_t launch_decode_sm100(const DecodeArgs& a, const Sm100Maps& maps, cudaStream_t s);
size_t decode_sm100_smem_bytes();

// C[z][m][n] = sum_k A(z,m,k) * B(z,n,k), fp32 accumulation, generic strides
// (element units), with a store epilogue that can
//  - map the row through a paged block table (cache append),
//  - split columns into segments of `seg` written `seg_stride` apart plus
//    `col_off` (packed query / cache rows),
//  - rotate consecutive column pairs by pos[m] * base^(-2k/seg) (RoPE).
struct GemmArgs {
  const void* A;
  const void* Bm;
  void* C;
  int M, N, K, Z;
  long long sAz, sAm, sAk;
  long long sBz, sBn, sBk;
  long long sCz, sCm;
  int seg;               // column segment length (>= N means one segment)
  long long seg_stride;  // distance between segments in C
  long long col_off;     // added to every column
  const int* pos;        // per-row position (RoPE and paged rows)
  int rope;              // apply rotary pairs within each segment
  double rope_base;
  // paged rows: row of m = block_table[seq[m]*max_pages + pos[m]/page]*page + pos[m]%page
  const int* seq;
  const int* block_table;
  int max_pages, page_size, num_pages;
  int* err;
  bool bf16;
};
cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t s);

// Per-head up-projection on the tensor cores, d_v <= 128.  w_map: W_UV as
// [n_h * d_v, d_c] with 128-byte boxes x 128 rows, 128-byte swizzle (bf16:
// 64 columns; fp32: 32 columns).  u_map: u as [T, n_h, d_c], 128-byte boxes
// x 1 x up_proj_sm100_box_rows(T), 128-byte swizzle.  f32: W, u and o are
// fp32 (tf32 MMAs, d_c a multiple of 32 up to 256); else bf16 (d_c a
// multiple of 64 up to 512).
int up_proj_sm100_prepare();
int up_proj_sm100_box_rows(int T);
cudaError_t launch_up_proj_sm100(const CUtensorMap& w_map, const CUtensorMap& u_map, void* o,
                                 int* err, int T, int n_h, int d_c, int d_v, bool f32, bool pdl,
                                 cudaStream_t s);
// bf16 W and o with an fp32 u, read with plain loads and split into two bf16
// terms, u = hi + lo, in shared memory: o = W^UV hi + W^UV lo.  With
// `merge` (d_c = 512), the rows of split sequences are first merged from the
// decode workspace's fp16 partials (and written to u and lse): the combine
// stage fused into the up-projection.
cudaError_t launch_up_proj_sm100_f32u(const CUtensorMap& w_map, const float* u, void* o, int* err,
                                      int T, int n_h, int d_c, int d_v, bool pdl, cudaStream_t s,
                                      const DecodeArgs* merge = nullptr);

// Weight-streaming projection Y[m, t] = sum_k W[m, k] X[t, k] on the tensor
// cores (bf16): one CTA per (128-row tile, K slice), fp32 split-K
// reduction in a workspace that is zero on entry and left zero.  w_map[0]
// covers tiles [0, tiles0), w_map[1] the rest (boxes 64 x 128 rows); x_map:
// X [N, K], box 64 x n_pad rows; all 128-byte swizzle, K a multiple of 64.
// mode 0: query (W^Q rows -> q^nope -> W^UK^T on the tensor cores into
// q[t, i, 0:d_c]; W^QR rows -> RoPE into q[t, i, d_c:]); mode 1: cache rows
// [W^DKV h || RoPE(W^KR h)] through the block table; mode 2: y[t, m]
// (pair = 2: X rows 2t, 2t + 1 are two terms of token t and are added).
struct WgemmLaunch {
  CUtensorMap w_map[2];
  CUtensorMap x_map;
  CUtensorMap uk_map;  // mode 0: W^UK as [n_h * 128, d_c], box 64 x 128 rows
  int tiles, tiles0;
  int K, N, n_pad, ksplit;
  void* workspace;
  int* err;
  int mode;
  void* out;
  int n_h, d_c, d_R, ldo, pair;
  const int* pos;
  const int* seq;
  const int* block_table;
  int max_pages, page_size, num_pages;
  float rope_base;
};
int wgemm_sm100_prepare();
size_t wgemm_workspace_bytes(int tiles, int n_pad);
cudaError_t launch_wgemm(const WgemmLaunch& L, cudaStream_t s);
// x [T, K] fp32 -> pairs [2T, K] bf16 (hi, lo of every row)
cudaError_t launch_split_rows(const float* x, void* pairs, int T, int K, cudaStream_t s);

}  // namespace mla
