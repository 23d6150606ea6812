/*
 * libmla -- absorbed Multi-head Latent Attention (MLA) decode for B200 (sm_100a).
 *
 * The math (sources named by page title and section):
 *   - "MLA deep compression" (operatorworld.com), absorption section, score
 *     equation: head i scores the cached latent c directly with the absorbed
 *     query q^lat_i = W^QK_i h, where W^QK_i = (W^UK_i)^T W^Q_i is formed
 *     offline once per model.
 *   - same page, absorption section, output equation: o_i = W^UV_i u_i with
 *     u_i = sum_j a_ij c_j, the softmax-weighted sum of cached latents.
 *   - same page, decoupled-RoPE section: each cached row also holds a 64-wide
 *     RoPE key k^R shared by all heads; the score adds q^R_i . k^R_j to the
 *     latent dot product, so a cached row is [c (d_c) || k^R (d_R)], 576
 *     values at the DeepSeek-V3 shape.
 *   - "Attention-head anatomy" (romaanj.github.io) section 5: the same fold
 *     of W^UK into the query path and the sum of the two dot products.
 *
 * Conventions for every call:
 *   - Pointers named as device buffers are device pointers the caller owns;
 *     the library allocates nothing and frees nothing.  Scratch space for
 *     mla_decode is passed in as `workspace`.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call is asynchronous on that stream; arguments are
 *     validated on the host first and a non-OK status means nothing was
 *     enqueued.  A launch failure reported by the CUDA runtime returns
 *     MLA_ERR_CUDA.
 *   - Element type is chosen by `dtype`: MLA_DTYPE_BF16 tensors hold bf16,
 *     MLA_DTYPE_FP32 tensors hold fp32.  Index tensors are int32.  Softmax
 *     statistics (lse) are always fp32.  Accumulation is always fp32.
 *   - All tensors are dense row-major with the shapes given; every device
 *     pointer must be 16-byte aligned.
 *   - Problems the host cannot see (a sequence length or page id out of
 *     range in device memory, a device-side wait that ran out of time) set a
 *     sticky device flag instead of faulting; mla_check_device_errors reads
 *     and clears it.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,          /* null/unaligned pointer, bad size, bad dtype */
  MLA_ERR_UNSUPPORTED = 2,          /* valid but not implemented (e.g. n_h > 128) */
  MLA_ERR_CUDA = 3,                 /* CUDA runtime/driver error */
  MLA_ERR_WORKSPACE_TOO_SMALL = 4,  /* workspace_bytes < mla_decode_workspace_size */
  MLA_ERR_DEVICE_CHECK = 5          /* device flag raised (see mla_check_device_errors) */
} mla_status;

typedef enum { MLA_DTYPE_BF16 = 0, MLA_DTYPE_FP32 = 1 } mla_dtype;

/* Device flag bits reported by mla_check_device_errors (OR-ed together). */
#define MLA_DEVFLAG_BAD_SEQLEN 0x1  /* seqlens[b] < s_q or > max_pages_per_seq*page_size */
#define MLA_DEVFLAG_BAD_PAGE 0x2    /* block_table entry outside [0, num_pages) */
#define MLA_DEVFLAG_TIMEOUT 0x4     /* a device-side wait gave up (kernel returned early) */
#define MLA_DEVFLAG_LAYOUT 0x8      /* a kernel's shared memory was not 1024-byte aligned (it returned at once) */
#define MLA_DEVFLAG_RANGE 0x10      /* a split row's partial u did not fit fp16 (|value| > 65504): u of that row is wrong */

const char* mla_status_string(mla_status s);

/*
 * Offline weight absorption, score side ("MLA deep compression", absorption
 * section, score equation):  W_QK[i] = W_UK[i]^T . W_Q[i]  for every head i.
 *   W_UK  [n_h, d_h, d_c]      device, read
 *   W_Q   [n_h, d_h, d_model]  device, read
 *   W_QK  [n_h, d_c, d_model]  device, written
 * Run once per model; not on the per-token path.
 */
mla_status mla_absorb_weights(const void* W_UK, const void* W_Q, void* W_QK, int n_h, int d_h,
                              int d_c, int d_model, mla_dtype dtype, void* stream);

/*
 * Projections around the attention (query formation, latent append, output
 * projection) stream their weights once through the tensor cores; their K
 * dimension is split over CTAs whose partial sums meet in an fp32 scratch
 * area.  `workspace` (bf16 calls) is caller-owned device memory of at least
 * mla_projection_workspace_size bytes, 256-byte aligned, that must be ZERO
 * before its first use; every call leaves it zero again, so one zeroed
 * workspace serves any number of calls ordered on one stream.  rows0 and
 * rows1 are the row counts of the call's first and second weight tensor
 * (n_h * d_c and n_h * d_R for mla_form_query, n_h * d_h and n_h * d_R for
 * mla_form_query_fused, d_c and d_R for mla_append_latent, M and 0 for
 * mla_output_projection); x_fp32_K is K for mla_output_projection with an
 * fp32 x, else 0.
 */
mla_status mla_projection_workspace_size(int rows0, int rows1, int T, int x_fp32_K,
                                         size_t* bytes);

/*
 * Absorbed query formation ("MLA deep compression", absorption section score
 * equation and decoupled-RoPE section):
 *   q[t, i, 0:d_c]       = W_QK[i] . h[t]
 *   q[t, i, d_c:d_c+d_R] = RoPE(W_QR[i] . h[t], pos[t])
 * RoPE rotates consecutive pairs (2k, 2k+1) by angle pos * rope_base^(-2k/d_R)
 * (the pages give no convention; this is the plain rotary one).
 *   h     [T, d_model]             device, read
 *   W_QK  [n_h, d_c, d_model]      device, read (from mla_absorb_weights)
 *   W_QR  [n_h, d_R, d_model]      device, read
 *   pos   [T] int32                device, read (query positions)
 *   q     [T, n_h, d_c + d_R]      device, written (T = B * s_q rows)
 * bf16: tensor cores (d_model a multiple of 64, d_R dividing 128), with a
 * projection workspace; fp32: a tiled CUDA-core GEMM (workspace unused).
 */
mla_status mla_form_query(const void* h, const void* W_QK, const void* W_QR, const int* pos,
                          void* q, int T, int n_h, int d_model, int d_c, int d_R, float rope_base,
                          mla_dtype dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Query formation with the absorption done on the fly ("MLA deep
 * compression", absorption section, score equation read right to left, and
 * decoupled-RoPE section): no precomputed W_QK is read.
 *   q[t, i, 0:d_c]       = W_UK[i]^T . (W_Q[i] . h[t])
 *   q[t, i, d_c:d_c+d_R] = RoPE(W_QR[i] . h[t], pos[t])
 * bf16, one kernel: the products with W_Q and W_QR stream those weights once
 * through the tensor cores; the CTA that completes head i's W_Q . h applies
 * W_UK[i]^T on the tensor cores (W_Q . h split into two bf16 terms, so it
 * enters unrounded).  Reads 2 * n_h * (d_h + d_R) * d_model + 2 * n_h * d_h
 * * d_c bytes of weights (369 MB at the DeepSeek-V3 shape) instead of the
 * absorbed path's 2 * n_h * (d_c + d_R) * d_model (1057 MB).
 *   h     [T, d_model]        device, read (bf16)
 *   W_Q   [n_h, d_h, d_model] device, read
 *   W_UK  [n_h, d_h, d_c]     device, read
 *   W_QR  [n_h, d_R, d_model] device, read
 *   pos   [T] int32           device, read
 *   q     [T, n_h, d_c + d_R] device, written
 * Supported: d_h = 128, d_c a multiple of 128 up to 512, d_model a multiple
 * of 64, d_R even and dividing 128.  Needs a projection workspace.
 */
mla_status mla_form_query_fused(const void* h, const void* W_Q, const void* W_UK,
                                const void* W_QR, const int* pos, void* q, int T, int n_h,
                                int d_h, int d_model, int d_c, int d_R, float rope_base,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * Latent append ("MLA deep compression", low-rank projection section and
 * decoupled-RoPE section): for each new token t of sequence seq_ids[t] at
 * position pos[t], writes the cache row
 *   kv_cache[row] = [ W_DKV . h[t]  ||  RoPE(W_KR . h[t], pos[t]) ]
 * where row = block_table[seq_ids[t]][pos[t] / page_size] * page_size + pos[t] % page_size.
 *   h           [T, d_model]                      device, read
 *   W_DKV       [d_c, d_model]                    device, read
 *   W_KR        [d_R, d_model]                    device, read
 *   seq_ids,pos [T] int32                         device, read
 *   block_table [*, max_pages_per_seq] int32      device, read
 *   kv_cache    [num_pages*page_size, d_c + d_R]  device, written (only the T rows)
 * Out-of-range page ids raise MLA_DEVFLAG_BAD_PAGE and the row is skipped.
 * bf16: tensor cores (d_model a multiple of 64, d_R <= 128), with a
 * projection workspace; fp32: a tiled CUDA-core GEMM (workspace unused).
 */
mla_status mla_append_latent(const void* h, const void* W_DKV, const void* W_KR,
                             const int* seq_ids, const int* pos, const int* block_table,
                             int max_pages_per_seq, int page_size, int num_pages, void* kv_cache,
                             int T, int d_model, int d_c, int d_R, float rope_base,
                             mla_dtype dtype, void* workspace, size_t workspace_bytes,
                             void* stream);

/*
 * Absorbed decode over a paged latent cache ("MLA deep compression",
 * absorption section, both equations; decoupled-RoPE section):
 *   for every sequence b, query row r < s_q, head i:
 *     s_j  = q[b,r,i,:d_c] . c_j + q[b,r,i,d_c:] . kR_j     for j <= seqlens[b] - s_q + r
 *     a    = softmax(softmax_scale * s)
 *     u[b,r,i,:]  = sum_j a_j c_j
 *     lse[b,r,i]  = log(sum_j exp(softmax_scale * s_j))      (natural log)
 * The s_q query rows are the last s_q positions of the sequence (already in
 * the cache); row r sees every cached position up to and including its own.
 * Long or ragged contexts are cut into KV chunks that run in parallel and are
 * merged by a combine step (log-sum-exp weighting).
 */
typedef struct {
  const void* q;            /* [B, s_q, n_h, d_c + d_R] device; latent part first, then RoPE   */
  const void* kv_cache;     /* [num_pages * page_size, d_c + d_R] device; row = c || k^R        */
  const int* block_table;   /* [B, max_pages_per_seq] int32 device; physical page ids          */
  const int* seqlens;       /* [B] int32 device; cached tokens incl. the s_q query tokens        */
  void* u;                  /* [B, s_q, n_h, d_c] device, written; bf16 or fp32 (see u_fp32)     */
  float* lse;               /* [B, s_q, n_h] fp32 device, written; may be NULL                   */
  int B;                    /* sequences; 0 is a no-op                                           */
  int s_q;                  /* query rows per sequence: 1 or 2                                   */
  int n_h;                  /* heads, 1..128                                                     */
  int d_c;                  /* latent width (512 at the DeepSeek-V3 shape), multiple of 8, <=512 */
  int d_R;                  /* RoPE key width (64), even, multiple of 8 with d_c, <= 64          */
  int page_size;            /* tokens per page, a positive multiple of 64                         */
  int max_pages_per_seq;    /* columns of block_table                                            */
  int num_pages;            /* pages in kv_cache                                                 */
  float softmax_scale;      /* multiplies the scores before softmax, finite and > 0               */
  mla_dtype dtype;          /* of q, kv_cache and u                                              */
  int num_splits;           /* KV chunks the whole batch is cut into; 0 = one per SM pair        */
  int u_fp32;               /* nonzero: u is fp32 (the partial u of pieces of split rows fp16 on the
                               DeepSeek-V3-shape kernel, which flags MLA_DEVFLAG_RANGE if a value
                               exceeds 65504; fp32 on the small-latent kernel);
                               0: u has type `dtype`.  With bf16 inputs an fp32 u carries the
                               softmax-weighted latent sum to the up-projection unrounded: a
                               bf16 u moves o = W_UV u by up to 2^-8 |u| per element, which for
                               contexts dominated by a few large latents (|u| ~ 25) exceeds an
                               elementwise 2e-2 (1 + |o|) budget where o is near zero.  fp32
                               inputs always give an fp32 u.                                    */
} mla_decode_params;

/* Bytes of device scratch mla_decode needs for these parameters (depends on
 * B, s_q, n_h, d_c, num_splits and the current device's SM count). */
mla_status mla_decode_workspace_size(const mla_decode_params* p, size_t* bytes);

/* Runs plan + attend + combine.  `workspace` must be 256-byte aligned device
 * memory of at least mla_decode_workspace_size bytes; it is scratch (no
 * state is kept between calls).  Rows of a page past seqlens[b] may hold
 * any bit pattern (they are never used).  Calls that share a workspace must
 * be ordered on the GPU. */
mla_status mla_decode(const mla_decode_params* p, void* workspace, size_t workspace_bytes,
                      void* stream);

/* The three stages of mla_decode, for callers that time or schedule them
 * separately; calling them in this order is exactly mla_decode.
 *   plan:    per-sequence tile counts and KV-chunk boundaries into the workspace
 *   attend:  the chunked attention (writes u/lse directly for unsplit rows,
 *            partials into the workspace otherwise: see u_fp32 for their type)
 *   combine: merges the partials of split rows into u/lse
 * Called on their own, the stages launch as plain stream-ordered kernels;
 * inside mla_decode each stage may start its prologue while the previous
 * one finishes (programmatic dependent launch). */
mla_status mla_decode_plan(const mla_decode_params* p, void* workspace, size_t workspace_bytes,
                           void* stream);
mla_status mla_decode_attend(const mla_decode_params* p, void* workspace, size_t workspace_bytes,
                             void* stream);
mla_status mla_decode_combine(const mla_decode_params* p, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * One decode step of the attention output: mla_decode, then o = W_UV u
 * (as mla_up_proj), with the combine of split rows done inside the
 * up-projection: each up-projection CTA merges the fp16 partials of its
 * head's rows from the workspace (also writing u and lse), splits the fp32
 * rows into two bf16 terms and runs the tensor-core product.  The three
 * kernels (plan, attend, merge + up-projection) are chained by programmatic
 * dependent launch, so the weight read starts while the attend kernel ends.
 * Requires the DeepSeek-V3 shape kernel (bf16, d_c = 512, d_R = 64), an fp32
 * u (p->u_fp32 = 1) and d_v <= 128.  Results equal mla_decode followed by
 * mla_up_proj.  The workspace is mla_decode's.
 *   W_UV  [n_h, d_v, d_c] bf16 device, read
 *   o     [B * s_q, n_h, d_v] bf16 device, written
 */
mla_status mla_decode_step(const mla_decode_params* p, const void* W_UV, void* o, int d_v,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * mla_decode without a caller-provided workspace.  The pages have no
 * counterpart to this call; it exists for callers that cannot allocate
 * device memory, such as a host framework that owns all device memory and
 * hands a kernel library only inputs and outputs (a fixed serving pool, a
 * plugin interface without a workspace argument).
 *
 * Same parameters, results and errors as mla_decode.  The scratch space is
 * a 32 MiB array inside the library (a file-scope __device__ variable): every
 * GPU that loads the library holds it until the process exits, and this call
 * allocates nothing.  Parameters whose mla_decode_workspace_size exceeds
 * 32 MiB are rejected with MLA_ERR_WORKSPACE_TOO_SMALL before anything is
 * enqueued.  The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  All calls on a device share the array and
 * leave their data in it; nothing in it needs to start at zero, but calls
 * whose work overlaps on the GPU race on it, so order them on one stream or
 * with events.
 */
mla_status mla_decode_noalloc(const mla_decode_params* p, void* stream);

/* Which attend kernel these parameters select: 1 = tensor-core (tcgen05)
 * kernel, 0 = CUDA-core kernel; and the number of KV chunks it will use. */
mla_status mla_decode_kernel_info(const mla_decode_params* p, int* uses_tensor_cores,
                                  int* num_chunks);

/*
 * GQLA's GQA path (GQLA summary, abstract and method paragraphs: the same
 * trained weights expose, besides the MQA-absorb path above, a GQA path with
 * a per-group expanded cache; heads of a group share W^UK_g and W^UV_g).  A
 * cached token holds, for each group g, K^C_g = W^UK_g c and V_g = W^UV_g c,
 * and once the RoPE key k^R shared by all heads.  For head i of group
 * g = i / (n_h / n_g), query row r < s_q of sequence b:
 *   s_j = q[b,r,i,:d_h] . K^C_g[j] + q[b,r,i,d_h:] . k^R[j]   for j <= seqlens[b] - s_q + r
 *   o[b,r,i,:] = sum_j softmax(softmax_scale * s)_j V_g[j];  lse as in mla_decode
 * One CTA takes a KV chunk of one group with all its heads and all s_q query
 * rows as the MMA rows, so the group's cache is read once for both rows of
 * multi-token prediction (s_q = 2).  bf16 on the tensor cores; chunks and
 * their merge as in mla_decode (fp32 partials).
 */
typedef struct {
  const void* q;            /* [B, s_q, n_h, d_h + d_R] device: q^nope then q^R            */
  const void* kv;           /* [num_pages * page_size, n_g, d_h + d_v] device: K^C_g then V_g */
  const void* k_rope;       /* [num_pages * page_size, d_R] device                         */
  const int* block_table;   /* [B, max_pages_per_seq] int32 device                         */
  const int* seqlens;       /* [B] int32 device                                            */
  void* o;                  /* [B, s_q, n_h, d_v] device, written (bf16, or fp32 if o_fp32) */
  float* lse;               /* [B, s_q, n_h] fp32 device, written; may be NULL             */
  int B, s_q, n_h, n_g;     /* s_q in {1, 2}; n_h a multiple of n_g; (n_h / n_g) s_q <= 128 */
  int d_h, d_v, d_R;        /* d_h, d_v multiples of 64; d_h + d_R <= 256; d_v <= 256      */
  int page_size, max_pages_per_seq, num_pages;
  float softmax_scale;
  mla_dtype dtype;          /* MLA_DTYPE_BF16                                              */
  int num_splits;           /* KV chunks; 0 = automatic                                    */
  int o_fp32;
} mla_gqa_params;

mla_status mla_decode_gqa_workspace_size(const mla_gqa_params* p, size_t* bytes);
mla_status mla_decode_gqa(const mla_gqa_params* p, void* workspace, size_t workspace_bytes,
                          void* stream);

/*
 * Per-head up-projection ("MLA deep compression", absorption section, output
 * equation):  o[t, i, :] = W_UV[i] . u[t, i, :]
 *   u     [T, n_h, d_c]   device, read   (T = B * s_q), type u_dtype
 *   W_UV  [n_h, d_v, d_c] device, read,    type dtype
 *   o     [T, n_h, d_v]   device, written, type dtype
 * Runs on the tensor cores: bf16 weights with a bf16 u, or with an fp32 u
 * split into two bf16 terms (u = hi + lo, |u - hi - lo| <= 2^-16 |u|) whose
 * products are accumulated together, so an fp32 u is used to well below
 * bf16 rounding; fp32 weights (and then an fp32 u) run as tf32.  Supported:
 * d_v <= 128, d_c a multiple of 64 (bf16) or 32 (fp32) up to 512.
 * u_dtype must be dtype or MLA_DTYPE_FP32.
 */
mla_status mla_up_proj(const void* u, const void* W_UV, void* o, int T, int n_h, int d_c,
                       int d_v, mla_dtype u_dtype, mla_dtype dtype, void* stream);

/*
 * Output side folded offline ("Attention-head anatomy" section 5: W^UV folds
 * into W^O; "MLA deep compression", absorption section, output equation):
 *   W_OUV[m, i * d_c + c] = sum_v W_O[m, i * d_v + v] W_UV[i, v, c]
 * so that y = W_O . concat_i(W_UV[i] u_i) = W_OUV . concat_i(u_i).
 *   W_O    [d_model, n_h * d_v]   device, read
 *   W_UV   [n_h, d_v, d_c]        device, read
 *   W_OUV  [d_model, n_h * d_c]   device, written
 * Run once per model (tiled CUDA-core GEMM, fp32 accumulation).
 */
mla_status mla_fold_output_weights(const void* W_O, const void* W_UV, void* W_OUV, int n_h, int d_v,
                                   int d_c, int d_model, mla_dtype dtype, void* stream);

/*
 * Output projection y[t, m] = sum_k W[m, k] x[t, k] on the tensor cores,
 * streaming W once: with W = W_OUV and x = u flattened [T, n_h * d_c] it
 * projects the decode's u straight to the hidden size; with W = W_O and
 * x = o flattened [T, n_h * d_v] it is the unfolded output projection.
 *   x  [T, K]  device, read; bf16, or fp32 (split into two bf16 terms whose
 *              products are added, so x enters to within 2^-16 of itself)
 *   W  [M, K]  device, read, bf16
 *   y  [T, M]  device, written, bf16
 * K a multiple of 64, M a multiple of 8.  Needs a projection workspace
 * (rows0 = M, rows1 = 0, x_fp32_K = K for an fp32 x).
 */
mla_status mla_output_projection(const void* x, mla_dtype x_dtype, const void* W, void* y, int T,
                                 int K, int M, void* workspace, size_t workspace_bytes,
                                 void* stream);

/*
 * Merge of partial decode results over disjoint parts of the same query
 * rows' context ("MLA deep compression", absorption section: u is the
 * softmax-weighted sum over every cached position, so results over pieces of
 * the context combine by their log-sum-exp):
 *   lse[row]    = log sum_r exp(lse_parts[r, row])
 *   u[row, :]   = sum_r exp(lse_parts[r, row] - lse[row]) u_parts[r, row, :]
 * For context parallelism across GPUs: each GPU decodes a page range of every
 * sequence with mla_decode (s_q = 1), the (u, lse) of all GPUs are gathered,
 * and this call merges them on each GPU.
 *   u_parts    [R, rows, d_c]  device, read  (dtype)
 *   lse_parts  [R, rows] fp32  device, read; -inf marks a part without tokens
 *   u          [rows, d_c]     device, written (dtype)
 *   lse        [rows] fp32     device, written; may be NULL
 * rows = B * s_q * n_h (the flattened rows of mla_decode's u); R >= 1; d_c a
 * positive multiple of 8; u_parts, u and lse 16-byte aligned.  A row whose
 * parts are all -inf gets u = 0 and lse = -inf.  rows = 0 is a no-op.
 */
mla_status mla_merge_partials(const void* u_parts, const float* lse_parts, void* u, float* lse,
                              int R, int rows, int d_c, mla_dtype dtype, void* stream);

/*
 * Self-test of the bounded device-side wait.  Launches one kernel that
 * waits on an mbarrier phase with a limit of about 2e6 cycles (~1 ms):
 * with arrive != 0 the kernel first completes that phase and the wait
 * returns at once; with arrive == 0 nothing completes it, the wait gives up,
 * MLA_DEVFLAG_TIMEOUT is set in the device flags and the kernel returns.
 * Every kernel of the library waits this way (with a limit of 2e9 cycles),
 * so a broken hand-off ends as a flag, never as a hang.  Read the flags with
 * mla_check_device_errors.  No arithmetic of the method is involved.
 */
mla_status mla_selftest_wait(int arrive, void* stream);

/* Synchronizes `stream`, then reads and clears the device flag of the
 * current device.  Returns MLA_OK if no flag was raised, otherwise
 * MLA_ERR_DEVICE_CHECK and the MLA_DEVFLAG_* bits in *flags (may be NULL). */
mla_status mla_check_device_errors(void* stream, int* flags);

#ifdef __cplusplus
}
#endif
#endif /* MLA_H_ */
