/*
 * libattn -- fused attention forward with an online softmax, for NVIDIA B200
 * (sm_100a).
 *
 * What every entry point computes, per query row i of sequence b and query
 * head h (the pages' statement of the problem):
 *
 *   S_j   = scale * <q_i, k_j>                   CANN "flash_attn", 计算公式
 *   m     = max(sink_h, max_j S_j)               same page, the sink variant
 *   O_i   = sum_j e^{S_j - m} v_j / (sum_j e^{S_j - m} + e^{sink_h - m})
 *   LSE_i = max_j S_j + ln sum_j e^{S_j - max_j S_j}    (keys only; the
 *           softmax_lse formula of the same page is written over S alone)
 *
 * with j over the keys visible to row i:
 *   delta = L_k - L_q (the last query row sees the last key: bottom-right
 *   alignment, MindSpore "sparse_flash_attention", sparse_mode=3
 *   "rightDownCausal");
 *   causal:        j <= i + delta;
 *   window_left:   j >= i + delta - window_left   (-1 = unbounded);
 *   window_right:  j <= i + delta + window_right  (-1 = unbounded)
 *   (MindSpore Lite "flash_attention", window_size=(-1, -1); inclusive).
 * A row that sees no key gets O = 0 and LSE = -inf. GQA/MQA: query head h
 * reads KV head h / (H_q / H_kv).
 *
 * Conventions for all entry points:
 *  - Every tensor pointer is a DEVICE pointer, owned by the caller, and must
 *    stay valid until the work queued on `stream` has finished. The library
 *    allocates no device memory; workspaces come from the *_size queries.
 *  - Launches are asynchronous on `stream` (a cudaStream_t; 0 = legacy
 *    default stream). No call synchronises the host.
 *  - The innermost dimension of every tensor is contiguous; other strides are
 *    given in ELEMENTS and must make every row start 16-byte aligned.
 *  - Host-visible facts are validated (null pointers, zero-size axes, head
 *    counts, dims, dtypes, alignment, workspace size) and reported through
 *    the return code; nothing is launched on error. Any zero-size axis is an
 *    error (CANN "flash_attn", empty-tensor rule: every empty-tensor case is
 *    rejected).
 *  - Tensor VALUES (cu_seqlens, block_table, cache_seqlens, sparse indices)
 *    are not validated on the host (CANN "flash_attn", 声明: values of tensor
 *    arguments are not checked and bad values are undefined behaviour). The
 *    kernels clamp nothing; keep them in range. Sparse indices outside
 *    [0, cache_seqlens[b]) are skipped by design.
 *  - Scheduler metadata must come from attn_sched_metadata called with the
 *    same arguments as the main call (CANN "flash_attn", 声明). The kernels
 *    compare the metadata header with their own arguments and, on mismatch,
 *    write nothing and raise ATTN_DEVERR_META_MISMATCH in the device error
 *    word (see attn_get_device_error).
 */
#ifndef LIBATTN_H_
#define LIBATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,          /* a host-visible argument is wrong          */
  ATTN_ERR_UNSUPPORTED = 2,          /* valid, but not a shape/dtype we build      */
  ATTN_ERR_WORKSPACE_TOO_SMALL = 3,  /* workspace_bytes below the *_size result    */
  ATTN_ERR_CUDA = 4,                 /* a CUDA runtime/driver call failed          */
  ATTN_ERR_DEVICE = 5                /* attn_get_device_error found a device error */
} attn_status_t;

/* Device error word codes (attn_get_device_error). */
enum {
  ATTN_DEVERR_NONE = 0,
  ATTN_DEVERR_TIMEOUT = 1,        /* a bounded pipeline wait gave up            */
  ATTN_DEVERR_META_MISMATCH = 2,  /* scheduler metadata built for other args    */
  ATTN_DEVERR_SMEM_ALIGN = 3,     /* dynamic shared memory not 1024-byte aligned */
  ATTN_DEVERR_UNITS_OVERFLOW = 4  /* attn_sched_metadata: total work units of the
                                     problem above 2^31 - 1 (the metadata is left
                                     invalid, so the main call raises
                                     ATTN_DEVERR_META_MISMATCH if this word is clear) */
};

typedef enum {
  ATTN_DTYPE_BF16 = 0,
  ATTN_DTYPE_FP16 = 1,
  ATTN_DTYPE_E4M3 = 2,   /* OCP FP8 E4M3 ("e4m3fn")                           */
  ATTN_DTYPE_E5M2 = 3,   /* OCP FP8 E5M2                                      */
  ATTN_DTYPE_FP32 = 4    /* only for fp32 partial outputs of attn_combine     */
} attn_dtype_t;

/* ------------------------------------------------------------------------ */
/* attn_fwd_varlen: prefill / full-sequence attention.                      */
/*                                                                          */
/* MATE "Attention", FMHA (flash_attn_varlen_func) and its dtype notes;      */
/* MindSpore Lite "flash_attention" (padded BSND, softmax_scale, causal,     */
/* window_size); CANN "flash_attn" (cu_seqlens, sink, softmax_lse).          */
/*                                                                          */
/* Layouts (strides in elements, innermost dim contiguous):                  */
/*   varlen (cu_seqlens_q != NULL): q (total_q, H_q, D_qk) packed, k and v   */
/*     (total_k, H_kv, D), out (total_q, H_q, D_v); cu_seqlens_q/k int32     */
/*     (batch+1) prefix sums; lse (H_q, total_q) -- pass lse_stride_b = 0,   */
/*     lse_stride_h = total_q; the row index is the packed row.              */
/*   padded (cu_seqlens_q == NULL, cu_seqlens_k == NULL): q (B, S_q, H_q, D),*/
/*     k/v (B, S_k, H_kv, D), out (B, S_q, H_q, D_v), lse (B, H_q, S_q) with */
/*     S_q = max_seqlen_q, S_k = max_seqlen_k.                               */
/* Types: q/k/v one of bf16, fp16, e4m3, e5m2 (all the same); out is bf16    */
/*   for bf16/FP8 inputs and fp16 for fp16 inputs (FP8 in -> bf16 out, MATE  */
/*   FMHA dtype notes). lse fp32, nullable (CANN return_softmax_lse=False).  */
/* FP8: q/k/v_descale fp32 (batch, H_kv), contiguous, required for FP8 and   */
/*   ignored otherwise; S uses q*q_descale and k*k_descale, O uses           */
/*   v*v_descale (MATE FMHA dtype notes).                                    */
/* sink: fp32 (H_q,) per-head logit, nullable.                               */
/* seqused_q / seqused_k (CANN "flash_attn": seqused_q, seqused_kv): padded  */
/*   layout only, nullable, device int32 (batch): the rows of q and the keys */
/*   of k/v in use per sequence (<= max_seqlen_q / max_seqlen_k; values are  */
/*   not checked). Sequence b is its first seqused_q[b] rows against its     */
/*   first seqused_k[b] keys (bottom-right causal alignment on those); rows  */
/*   past seqused_q[b] are not written.                                      */
/* mask (Mojo "flash_attention_split_kv": input_mask_fn, additive mask       */
/*   values): nullable device fp32, added to scale * q.k before the softmax; */
/*   element (b, h, i, j) for sequence b, query head h, row i and key j of   */
/*   the sequence at b*mask_stride_b + h*mask_stride_h + i*mask_stride_s + j */
/*   (strides in elements, >= 0, 0 broadcasts; rows 16-byte aligned: base    */
/*   and mask_stride_s multiples of 4 elements). -inf leaves a key out. The  */
/*   causal/window masks still apply. Each row reads its mask row once per   */
/*   key tile, so the mask adds S_q x S_k x 4 bytes per (sequence, head).    */
/* Supported now: D_qk = D_v in {64, 128}; FP8 (e4m3, e5m2) with D = 128.   */
/* ------------------------------------------------------------------------ */
typedef struct {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* lse;
  const int32_t* cu_seqlens_q;
  const int32_t* cu_seqlens_k;
  int32_t batch;
  int32_t max_seqlen_q;   /* padded: S_q; varlen: an upper bound of any L_q   */
  int32_t max_seqlen_k;   /* padded: S_k; varlen: an upper bound of any L_k   */
  int32_t total_q;        /* varlen: rows of q/out; padded: ignored           */
  int32_t total_k;        /* varlen: rows of k/v;   padded: ignored           */
  int32_t num_heads_q;
  int32_t num_heads_kv;
  int32_t head_dim_qk;
  int32_t head_dim_v;
  int64_t q_stride_b, q_stride_s, q_stride_h;   /* batch stride unused if varlen */
  int64_t k_stride_b, k_stride_s, k_stride_h;
  int64_t v_stride_b, v_stride_s, v_stride_h;
  int64_t o_stride_b, o_stride_s, o_stride_h;
  int64_t lse_stride_b, lse_stride_h;
  int32_t dtype;          /* attn_dtype_t of q/k/v                            */
  float scale;            /* > 0; the pages' default is 1/sqrt(D_qk)          */
  int32_t causal;
  int32_t window_left;    /* -1 = unbounded                                   */
  int32_t window_right;   /* -1 = unbounded                                   */
  const float* sink;
  const float* q_descale;
  const float* k_descale;
  const float* v_descale;
  const int32_t* seqused_q;  /* padded layout only; nullable                  */
  const int32_t* seqused_k;  /* padded layout only; nullable                  */
  const float* mask;         /* additive score mask; nullable                 */
  int64_t mask_stride_b, mask_stride_h, mask_stride_s;
  int32_t* work_counter;     /* 4 bytes of device memory, or NULL. Given, the  */
                             /* persistent CTAs take work units (256 query     */
                             /* rows of one sequence and head, longest-running */
                             /* first) from this counter as they finish the    */
                             /* last; NULL: each CTA takes every gridDim-th    */
                             /* unit. The call zeroes it on `stream` before    */
                             /* the launch; calls in flight at the same time   */
                             /* must not share one counter.                    */
} attn_varlen_args;

attn_status_t attn_fwd_varlen(const attn_varlen_args* args, void* stream);

/* ------------------------------------------------------------------------ */
/* attn_sched_metadata: work split for the paged decode entry points.        */
/*                                                                          */
/* MATE "Attention" (get_scheduler_metadata, get_mla_metadata: precompute    */
/* the scheduler input of the main call); CANN "flash_attn" (the metadata    */
/* interface is called first and its result passed to the main operator).   */
/*                                                                          */
/* Reads cache_seqlens (device int32, batch) and writes `meta` (device       */
/* int32 buffer of attn_sched_metadata_size() bytes): a header echoing the   */
/* arguments, then a balanced split of all (sequence, KV-unit) work over     */
/* `num_ctas` persistent CTAs and the per-segment split counts the combine   */
/* step uses. One small kernel on `stream`.                                  */
/* mode: ATTN_SCHED_MHA (attn_fwd_paged_kvcache), ATTN_SCHED_MLA             */
/* (mla_fwd_paged), ATTN_SCHED_MLA_SPARSE (mla_sparse_fwd; uses topk).       */
/* num_ctas = 0 picks the device's SM count. The MLA modes schedule over     */
/* clusters of two CTAs: their slots number max(1, num_ctas / 2), and the    */
/* MLA kernels launch two CTAs per slot.                                     */
/* Limits: batch x segments per sequence at most 2^24 (ATTN_ERR_UNSUPPORTED  */
/* on the host); the problem's total units (keys in tiles of 64 for GQA,     */
/* 32 for MLA, per segment) at most 2^31 - 1, checked on the device:         */
/* above it the header is left invalid and ATTN_DEVERR_UNITS_OVERFLOW is     */
/* raised.                                                                   */
/* ------------------------------------------------------------------------ */
enum { ATTN_SCHED_MHA = 0, ATTN_SCHED_MLA = 1, ATTN_SCHED_MLA_SPARSE = 2 };

typedef struct {
  const int32_t* cache_seqlens;
  int32_t batch;
  int32_t seqlen_q;
  int32_t num_heads_q;
  int32_t num_heads_kv;
  int32_t head_dim_qk;
  int32_t head_dim_v;
  int32_t page_size;
  int32_t mode;
  int32_t topk;
  int32_t num_ctas;
  int32_t* meta;
  size_t meta_bytes;
  int32_t sparse_block_size;  /* ATTN_SCHED_MLA_SPARSE: as in mla_args          */
  int32_t seqlen_new;  /* ATTN_SCHED_MHA: the seqlen_new of the paged call (0) */
} attn_sched_args;

/* Bytes of `meta` needed for these arguments (host only, no device access). */
size_t attn_sched_metadata_size(const attn_sched_args* args);
attn_status_t attn_sched_metadata(const attn_sched_args* args, void* stream);

/* ------------------------------------------------------------------------ */
/* attn_fwd_paged_kvcache: decode against a paged KV cache, split-KV and     */
/* combined.                                                                 */
/*                                                                          */
/* MATE "Attention", FMHA (flash_attn_with_kvcache, scheduler_metadata,      */
/* flash_attn_combine) and the MLA example's paged layout; MindSpore         */
/* "sparse_flash_attention" (PA_BSND: (block_num, block_size, N, D));        */
/* CANN "flash_attn" (a non-empty block_table turns on paged attention).     */
/*                                                                          */
/* q (B, s_q, H_q, D); k_cache, v_cache (num_blocks, page_size, H_kv, D);    */
/* block_table int32 (B, max_pages_per_seq) with row stride in elements:     */
/* logical token t of sequence b is row t % page_size of physical page       */
/* block_table[b][t / page_size]; entries may repeat. cache_seqlens int32    */
/* (B,) = L_b; the s_q query rows are the last s_q positions (delta =        */
/* L_b - s_q). out (B, s_q, H_q, D) bf16 (fp16 for fp16 input); lse (B, H_q, */
/* s_q) fp32, nullable.                                                     */
/* FP8 (dtype e4m3 or e5m2; q and both caches in that format, D = 128):     */
/*   q_descale, k_descale, v_descale fp32 (B, H_kv), all required: the      */
/*   values of sequence b and KV head g are the stored codes times their     */
/*   descale [b][g] (MATE "Attention", FMHA FP8 paragraph). out is bf16.     */
/*   The descales are ignored for bf16 and fp16 input.                      */
/* Appended keys (Mojo "flash_attention_split_kv": the previous keys come    */
/*   from the cache and the current ones from separate k and v tensors, in  */
/*   one concatenated sequence): k_new, v_new (B, seqlen_new, H_kv, D) of    */
/*   the cache's dtype, with strides in elements, or both NULL. Sequence b   */
/*   then has L_b + seqlen_new keys, the new ones after its cached L_b, and  */
/*   the query rows are its last s_q positions. The cache is not written.    */
/*   The metadata must come from attn_sched_metadata with the same          */
/*   seqlen_new (checked on the device: ATTN_DEVERR_META_MISMATCH).         */
/* meta: from attn_sched_metadata(mode=ATTN_SCHED_MHA, same args), or NULL   */
/*   for one CTA per (sequence, KV head) and no splitting.                   */
/* workspace: device buffer of attn_paged_workspace_size() bytes (partial   */
/*   O and LSE of the splits); may be NULL when meta is NULL. The combine    */
/*   step runs inside this call.                                             */
/* Supported now: bf16 and fp16 with D in {64, 128}; e4m3 and e5m2 with     */
/*   D = 128; page_size in {16, 32, 64, 128, 256}; s_q * H_q / H_kv <= 16.  */
/* Errors: INVALID_ARG for NULL required pointers (the descales included    */
/*   for FP8), only one of k_new / v_new, seqlen_new < 1 with them, bad      */
/*   sizes or misaligned strides; UNSUPPORTED outside the supported shapes   */
/*   above.                                                                  */
/* ------------------------------------------------------------------------ */
typedef struct {
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_table;
  const int32_t* cache_seqlens;
  void* out;
  float* lse;
  int32_t batch;
  int32_t seqlen_q;
  int32_t num_heads_q;
  int32_t num_heads_kv;
  int32_t head_dim;
  int32_t page_size;
  int32_t num_blocks;
  int32_t max_pages_per_seq;
  int64_t block_table_stride;
  int64_t q_stride_b, q_stride_s, q_stride_h;
  int64_t kc_stride_blk, kc_stride_tok, kc_stride_h;
  int64_t vc_stride_blk, vc_stride_tok, vc_stride_h;
  int64_t o_stride_b, o_stride_s, o_stride_h;
  int32_t dtype;
  float scale;
  int32_t causal;
  int32_t window_left;
  int32_t window_right;
  const float* sink;
  const int32_t* meta;
  size_t meta_bytes;
  int32_t num_ctas;       /* the num_ctas given to attn_sched_metadata (0 = SMs) */
  void* workspace;
  size_t workspace_bytes;
  const float* q_descale; /* FP8 only: (B, H_kv) fp32 */
  const float* k_descale;
  const float* v_descale;
  const void* k_new;      /* appended keys (B, seqlen_new, H_kv, D), or NULL */
  const void* v_new;
  int32_t seqlen_new;
  int64_t kn_stride_b, kn_stride_s, kn_stride_h;
  int64_t vn_stride_b, vn_stride_s, vn_stride_h;
} attn_paged_args;

/* Bytes of workspace for these arguments (host only; 0 when meta is NULL).  */
size_t attn_paged_workspace_size(const attn_paged_args* args);
attn_status_t attn_fwd_paged_kvcache(const attn_paged_args* args, void* stream);

/* ------------------------------------------------------------------------ */
/* attn_fwd_paged_kvcache_static: the same paged split-KV decode, with no    */
/* caller-provided scratch. The pages have no counterpart of this entry      */
/* point; it exists for callers that cannot allocate device memory when      */
/* they run the decode -- for example code that runs inside a host callback  */
/* or a plugin interface that hands it only its inputs and outputs, or a     */
/* runtime whose device memory is fully reserved up front -- so they cannot  */
/* provide the metadata and workspace buffers attn_fwd_paged_kvcache needs.  */
/*                                                                          */
/* Arguments as attn_fwd_paged_kvcache, except that meta and workspace must  */
/* be NULL (ATTN_ERR_INVALID_ARG otherwise): the scheduler metadata and the  */
/* split partials live in one 16 MiB array inside the library image, which   */
/* every GPU that uses the library holds until the process exits. The call   */
/* computes the metadata itself (num_ctas as given, 0 = SM count), then runs */
/* the decode and the combine. Problems whose metadata plus partials exceed  */
/* 16 MiB (about S + G slots of 16 x D x 4 bytes, S = batch x H_kv x         */
/* ceil(s_q x H_q / H_kv / 16), G = num_ctas) return                         */
/* ATTN_ERR_WORKSPACE_TOO_SMALL and launch nothing. No device memory is     */
/* allocated or freed.                                                       */
/*                                                                          */
/* The first call on a device looks up the array's device address (a        */
/* runtime call); make that first call before any stream capture. A device   */
/* reset moves the array; the first call after it looks the address up      */
/* again, so make that call before any capture as well. All calls           */
/* share the one array and it keeps the last call's contents: calls that may */
/* overlap on the GPU (other streams, other host threads) race on it and     */
/* must be serialised by the caller. Nothing in the array needs to start at */
/* zero.                                                                     */
/* ------------------------------------------------------------------------ */
attn_status_t attn_fwd_paged_kvcache_static(const attn_paged_args* args, void* stream);

/* ------------------------------------------------------------------------ */
/* attn_combine: merge split partial results.                                */
/*                                                                          */
/* MATE "Attention", FMHA notes (flash_attn_combine merges partial outputs   */
/* and log-sum-exp buffers of a split computation). The pages print no       */
/* formula; with sink-free partials (O_s, LSE_s) over disjoint key sets:     */
/*   LSE = ln sum_s e^{LSE_s},  O = sum_s e^{LSE_s - LSE} O_s,               */
/* then, with a sink, O <- O / (1 + e^{sink_h - LSE}) (CANN "flash_attn",    */
/* 计算公式, with the keys-only LSE). Splits with LSE_s = -inf weigh 0; all  */
/* -inf gives O = 0, LSE = -inf.                                             */
/*                                                                          */
/* out_partial fp32 (num_splits, B, S, H, D_v) contiguous; lse_partial fp32  */
/* (num_splits, B, H, S) contiguous; out (B, S, H, D_v) bf16/fp16 with       */
/* strides; lse (B, H, S) fp32 contiguous, nullable. num_splits_per_seq int32*/
/* (B,), nullable: sequence b uses only its first num_splits_per_seq[b]      */
/* splits. sink fp32 (H,), nullable. D_v a multiple of 8, <= 1024.           */
/* ------------------------------------------------------------------------ */
typedef struct {
  const float* out_partial;
  const float* lse_partial;
  void* out;
  float* lse;
  const int32_t* num_splits_per_seq;
  const float* sink;
  int32_t num_splits;
  int32_t batch;
  int32_t seqlen_q;
  int32_t num_heads;
  int32_t head_dim_v;
  int64_t o_stride_b, o_stride_s, o_stride_h;
  int32_t out_dtype;      /* ATTN_DTYPE_BF16 or ATTN_DTYPE_FP16 */
} attn_combine_args;

attn_status_t attn_combine(const attn_combine_args* args, void* stream);

/* ------------------------------------------------------------------------ */
/* mla_fwd_paged: MLA-absorbed decode against a paged latent cache.          */
/*                                                                          */
/* MATE "Attention", MLA (get_mla_metadata, flash_mla_with_kvcache; example  */
/* with 576-wide rows and head_dim_v=512); MindSpore "sparse_flash_attention"*/
/* (attention_mode=2: nope (512) and rope (64) parts concatenated along D).  */
/*                                                                          */
/* q (B, s_q, H_q, 576) bf16; kv_cache (num_blocks, page_size, H_kv, 576)   */
/* bf16, each row [512 latent | 64 rope]; K is the whole row, V its first    */
/* head_dim_v (= 512) entries. Query head h reads KV head h / (H_q / H_kv)  */
/* (the MATE example's cache has 2 KV heads). block_table, cache_seqlens as  */
/* in attn_fwd_paged_kvcache. out (B, s_q, H_q, 512) bf16; lse (B, H_q, s_q) */
/* fp32 nullable. meta from attn_sched_metadata(mode=ATTN_SCHED_MLA, same    */
/* H_q and H_kv) or NULL; workspace from mla_workspace_size().               */
/* Supported now: H_q / H_kv a power of two up to 128 or a multiple of 128;  */
/*   page_size a power of two in [16, 256].                                  */
/* FP8 (MATE "Attention", FMHA dtype notes and FP8 paragraph, applied to the */
/*   latent cache): dtype = ATTN_DTYPE_E4M3 makes q and kv_cache e4m3 codes  */
/*   (strides still in elements, i.e. bytes); q_descale, k_descale and       */
/*   v_descale fp32 (B, H_kv) are all given (K = row * k_descale,            */
/*   V = row[:512] * v_descale, q * q_descale) or all NULL (= 1). The output */
/*   stays bf16. dtype = ATTN_DTYPE_BF16 (0) takes no descales.              */
/* ------------------------------------------------------------------------ */
typedef struct {
  const void* q;
  const void* kv_cache;
  const int32_t* block_table;
  const int32_t* cache_seqlens;
  const int32_t* indices;     /* mla_sparse_fwd only: (B, s_q, H_kv, topk)  */
  void* out;
  float* lse;
  int32_t batch;
  int32_t seqlen_q;
  int32_t num_heads_q;
  int32_t num_heads_kv;
  int32_t head_dim_qk;        /* 576 */
  int32_t head_dim_v;         /* 512 */
  int32_t page_size;
  int32_t num_blocks;
  int32_t max_pages_per_seq;
  int32_t topk;               /* mla_sparse_fwd only                          */
  int64_t block_table_stride;
  int64_t q_stride_b, q_stride_s, q_stride_h;
  int64_t kv_stride_blk, kv_stride_tok;
  int64_t o_stride_b, o_stride_s, o_stride_h;
  int64_t idx_stride_b, idx_stride_s;
  float scale;
  int32_t causal;
  const int32_t* meta;
  size_t meta_bytes;
  int32_t num_ctas;           /* the num_ctas given to attn_sched_metadata    */
  void* workspace;
  size_t workspace_bytes;
  int32_t sparse_block_size;  /* mla_sparse_fwd: 0 or 1 = each index is one     */
                              /* position; a power of two up to 128 = each     */
                              /* index k >= 0 lists positions k*bs .. k*bs+bs-1 */
                              /* (MindSpore sparse_flash_attention             */
                              /* sparse_block_size); dense: must be 0 or 1     */
  int64_t kv_stride_h;        /* H_kv > 1: KV-head stride of kv_cache          */
  int64_t idx_stride_h;       /* H_kv > 1, sparse: KV-head stride of indices   */
  const int32_t* cu_seqlens_q; /* mla_sparse_fwd with packed (TND) queries, or  */
                              /* NULL; see mla_sparse_fwd                       */
  int32_t dtype;              /* ATTN_DTYPE_BF16 or ATTN_DTYPE_E4M3 (q and cache) */
  const float* q_descale;     /* e4m3: (B, H_kv) each, all given or all NULL   */
  const float* k_descale;     /*   (TND: B is the number of sequences)         */
  const float* v_descale;
} mla_args;

/* Bytes of workspace for these arguments (host only; 0 when meta is NULL).  */
size_t mla_workspace_size(const mla_args* args);
attn_status_t mla_fwd_paged(const mla_args* args, void* stream);

/* ------------------------------------------------------------------------ */
/* mla_sparse_fwd: MLA decode over a top-k index set.                        */
/*                                                                          */
/* MATE "Attention", MLA (flash_mla_sparse_fwd); MindSpore                   */
/* "sparse_flash_attention" (sparse_indices int32 (B, Q_S, N2, sparse_size), */
/* sparse_size 2048, N2 = 1, PA_BSND cache with block_table).                */
/*                                                                          */
/* As mla_fwd_paged, plus indices int32 (B, s_q, 1, topk): query token       */
/* (b, i) attends to the listed logical positions p with                     */
/* 0 <= p < cache_seqlens[b]; other entries (e.g. -1 padding) are skipped.   */
/* causal = 0: no mask beyond the index set (sparse_mode=0); causal = 1:    */
/* also p <= i + cache_seqlens[b] - s_q (sparse_mode=3, "rightDownCausal").   */
/* meta from attn_sched_metadata(mode=ATTN_SCHED_MLA_SPARSE) or NULL.        */
/* Packed queries (MindSpore "sparse_flash_attention", layout_query="TND"   */
/*   with a PA_BSND cache): cu_seqlens_q int32 (B+1) prefix sums, the        */
/*   prefix-sum form of actual_seq_lengths_query. q (T, H_q, 576) with       */
/*   seqlen_q = T (q/o/idx batch strides unused), indices (T, H_kv, topk),   */
/*   out (T, H_q, 512), lse (H_q, T). Token t of sequence b (cu[b] <= t <   */
/*   cu[b+1]) reads sequence b's cache; with causal, its row i = t - cu[b]   */
/*   sees p <= i + cache_seqlens[b] - (cu[b+1] - cu[b]). The metadata is     */
/*   made with batch = 1 and seqlen_q = T. Values of cu_seqlens_q are not    */
/*   validated (cu[B] must equal T).                                         */
/* ------------------------------------------------------------------------ */
attn_status_t mla_sparse_fwd(const mla_args* args, void* stream);

/* ------------------------------------------------------------------------ */
/* Diagnostics.                                                              */
/* ------------------------------------------------------------------------ */

/* Copies the device error word of the current device into *code (an         */
/* ATTN_DEVERR_* value in the low 8 bits, the reporting site above them),    */
/* clears it, and synchronises `stream`. Returns ATTN_ERR_DEVICE when the    */
/* word was non-zero, ATTN_OK otherwise.                                     */
attn_status_t attn_get_device_error(int32_t* code, void* stream);

/* Failure-detection self-test. Launches one CTA on `stream` whose thread    */
/* waits, with the same bounded wait the kernels use, on an mbarrier that     */
/* nothing arrives on. The wait gives up after its limit (2 s), raises        */
/* ATTN_DEVERR_TIMEOUT with site ATTN_SELFTEST_SITE in the device error word, */
/* and the kernel returns; the context stays usable. Read the word with       */
/* attn_get_device_error. Returns ATTN_ERR_CUDA if the launch fails.          */
enum { ATTN_SELFTEST_SITE = 200 };
attn_status_t attn_selftest_wait_timeout(void* stream);

/* A static description of a status code. */
const char* attn_status_str(int32_t status);

/* sizeof() of the argument structs, so bindings can check their mirrors:    */
/* which = 0 varlen, 1 sched, 2 paged, 3 combine, 4 mla.                     */
size_t attn_args_sizeof(int32_t which);

#ifdef __cplusplus
}
#endif

#endif  /* LIBATTN_H_ */
