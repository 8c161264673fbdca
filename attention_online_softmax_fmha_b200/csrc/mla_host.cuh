// Host side of mla_fwd_paged and mla_sparse_fwd: argument checks, the tensor
// maps and the launch of the MLA kernels and their combine step.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "host.cuh"
#include "mla_sm100.cuh"
#include "sched_host.cuh"

namespace attn {
namespace {

// ---------------------------------------------------------------------------
// MLA decode (dense and sparse)
// ---------------------------------------------------------------------------
attn_status_t check_mla(const mla_args* a, bool sparse) {
  if (!a) return ATTN_ERR_INVALID_ARG;
  if (!a->q || !a->kv_cache || !a->block_table || !a->cache_seqlens || !a->out)
    return ATTN_ERR_INVALID_ARG;
  if (sparse && (!a->indices || a->topk <= 0)) return ATTN_ERR_INVALID_ARG;
  if (a->batch <= 0 || a->seqlen_q <= 0 || a->num_heads_q <= 0 || a->num_heads_kv <= 0 ||
      a->head_dim_qk <= 0 || a->head_dim_v <= 0 || a->page_size <= 0 || a->num_blocks <= 0 ||
      a->max_pages_per_seq <= 0 || a->num_ctas < 0)
    return ATTN_ERR_INVALID_ARG;
  if (a->block_table_stride < a->max_pages_per_seq) return ATTN_ERR_INVALID_ARG;
  if (!(a->scale > 0.f) || !std::isfinite(a->scale)) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(a->q) || !aligned16(a->kv_cache) || !aligned16(a->out)) return ATTN_ERR_INVALID_ARG;
  if (a->dtype != ATTN_DTYPE_BF16 && a->dtype != ATTN_DTYPE_E4M3) return ATTN_ERR_UNSUPPORTED;
  const bool fp8 = a->dtype == ATTN_DTYPE_E4M3;
  const int ne = (a->q_descale != nullptr) + (a->k_descale != nullptr) + (a->v_descale != nullptr);
  if (ne != 0 && (ne != 3 || !fp8)) return ATTN_ERR_INVALID_ARG;
  const int es = fp8 ? 1 : 2;  // bytes per q / cache element
  // packed (TND) queries: sparse only; there is no query batch axis
  const bool tnd = a->cu_seqlens_q != nullptr;
  if (tnd && !sparse) return ATTN_ERR_UNSUPPORTED;
  if ((!tnd && (!stride_ok(a->q_stride_b, es) || !stride_ok(a->o_stride_b, 2))) ||
      !stride_ok(a->q_stride_s, es) || !stride_ok(a->q_stride_h, es) ||
      !stride_ok(a->kv_stride_blk, es) || !stride_ok(a->kv_stride_tok, es) ||
      !stride_ok(a->o_stride_s, 2) || !stride_ok(a->o_stride_h, 2))
    return ATTN_ERR_INVALID_ARG;
  if (sparse && ((!tnd && a->idx_stride_b <= 0) || a->idx_stride_s <= 0))
    return ATTN_ERR_INVALID_ARG;
  if (a->num_heads_q % a->num_heads_kv) return ATTN_ERR_INVALID_ARG;
  if (a->num_heads_kv > 1 &&
      (!stride_ok(a->kv_stride_h, es) || (sparse && a->idx_stride_h <= 0)))
    return ATTN_ERR_INVALID_ARG;
  if (a->head_dim_qk != kMlaDqk || a->head_dim_v != kMlaDv) return ATTN_ERR_UNSUPPORTED;
  if (!mla_heads_ok(a->num_heads_q / a->num_heads_kv)) return ATTN_ERR_UNSUPPORTED;
  if (!pow2_in(a->page_size, 16, 256)) return ATTN_ERR_UNSUPPORTED;
  if (!sbs_ok(a->sparse_block_size) || (!sparse && a->sparse_block_size > 1))
    return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

// Split partials: per slot, both V halves of O (fp32) and the LSE.
size_t mla_ws_bytes(const DecodeShape& ds) {
  const size_t slots = (size_t)ds.S + ds.G;
  return slots * 2 * kMlaRows * kMlaDvHalf * sizeof(float) + slots * kMlaRows * sizeof(float) +
         256;
}

template <bool kSparse, bool kFp8>
attn_status_t run_mla(const mla_args& a, const DecodeShape& ds, cudaStream_t stream) {
  using C = MlaCfg<kFp8>;
  // a TMA box column is 128 bytes: 64 bf16 or 128 e4m3 values
  const CUtensorMapDataType dt =
      kFp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int es = kFp8 ? 1 : 2;
  const uint32_t box_c = kFp8 ? 128 : 64;
  // Q boxes: the query heads of one KV head (128 at most) x the tile's tokens
  const int box_h = ds.group >= kMlaRows ? kMlaRows : ds.group;
  const int box_t = ds.group >= kMlaRows ? 1 : ds.tokens_per_tile;
  // TND: the query side is one batch of seqlen_q = T packed tokens
  const bool tnd = a.cu_seqlens_q != nullptr;
  const int batch_q = tnd ? 1 : a.batch;
  const uint64_t q_sb = tnd ? (uint64_t)a.q_stride_s * a.seqlen_q : (uint64_t)a.q_stride_b;
  // The cache as (576, page row, block, KV head); with one KV head the last
  // stride only has to be valid.
  const uint64_t kv_sh = a.num_heads_kv > 1 ? (uint64_t)a.kv_stride_h
                                             : a.kv_stride_blk * (uint64_t)a.num_blocks;
  CUtensorMap mq, mkv;
  if (!encode_4d(&mq, a.q, dt, es, kMlaDqk, a.num_heads_q, a.seqlen_q, batch_q, a.q_stride_h,
                 a.q_stride_s, q_sb, box_c, box_h, box_t, 1) ||
      !encode_4d(&mkv, a.kv_cache, dt, es, kMlaDqk, a.page_size, a.num_blocks, a.num_heads_kv,
                 a.kv_stride_tok, a.kv_stride_blk, kv_sh, box_c,
                 a.page_size >= kMlaBN ? kMlaBN : a.page_size, 1, 1))
    return ATTN_ERR_INVALID_ARG;
  MlaParams p;
  memset(&p, 0, sizeof(p));
  p.q = a.q;
  p.out = a.out;
  p.lse = a.lse;
  p.block_table = a.block_table;
  p.cache_seqlens = a.cache_seqlens;
  p.indices = a.indices;
  p.meta = a.meta;
  p.kv = a.kv_cache;
  p.q_descale = a.q_descale;
  p.k_descale = a.k_descale;
  p.v_descale = a.v_descale;
  p.bt_stride = a.block_table_stride;
  p.q_sb = tnd ? 0 : a.q_stride_b;
  p.q_ss = a.q_stride_s;
  p.q_sh = a.q_stride_h;
  p.o_sb = tnd ? 0 : a.o_stride_b;
  p.o_ss = a.o_stride_s;
  p.o_sh = a.o_stride_h;
  p.kv_sblk = a.kv_stride_blk;
  p.kv_stok = a.kv_stride_tok;
  p.kv_sh = a.num_heads_kv > 1 ? a.kv_stride_h : 0;
  p.idx_sb = tnd ? 0 : a.idx_stride_b;
  p.idx_ss = a.idx_stride_s;
  p.idx_sh = a.num_heads_kv > 1 ? a.idx_stride_h : 0;
  p.batch = batch_q;
  p.batch_kv = a.batch;
  p.cu_q = a.cu_seqlens_q;
  p.seqlen_q = a.seqlen_q;
  p.heads_q = a.num_heads_q;
  p.heads_kv = a.num_heads_kv;
  p.group = ds.group;
  p.page_size = a.page_size;
  p.topk = a.topk;
  p.sbs = a.sparse_block_size > 1 ? a.sparse_block_size : 1;
  p.sbs_log2 = 0;
  while ((1 << p.sbs_log2) < p.sbs) ++p.sbs_log2;
  p.tiles_per_token = ds.tiles_per_token;
  p.tokens_per_tile = ds.tokens_per_tile;
  p.row_tiles = ds.row_tiles;
  p.segs_per_seq = ds.sh.segs_per_seq;
  p.num_segs = ds.S;
  p.num_ctas = ds.G;
  p.scale_log2 = a.scale * kLog2e;
  p.causal = a.causal;
  if (a.meta) {
    const size_t slots = (size_t)ds.S + ds.G;
    p.ws_o = reinterpret_cast<float*>(a.workspace);
    p.ws_lse = p.ws_o + slots * 2 * kMlaRows * kMlaDvHalf;
  }
  auto kernel = mla_kernel<kSparse, kFp8>;
  static std::atomic<uint64_t> configured{0};
  const attn_status_t cst = configure_per_device(configured, [&] {
    return launch_status(set_smem(kernel, C::kSmemBytes));
  });
  if (cst != ATTN_OK) return cst;
  // Clusters of two CTAs (the kernel's __cluster_dims__): one per segment, or
  // one per metadata slot.
  kernel<<<2 * (a.meta ? ds.G : ds.S), C::kThreads, C::kSmemBytes, stream>>>(mq, mkv, p);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  if (a.meta) {
    const int64_t warps = (int64_t)ds.S * 2 * kMlaRows;
    mla_combine_kernel<kSparse><<<(int)((warps + 7) / 8), 256, 0, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

attn_status_t mla_entry(const mla_args* a, void* stream, bool sparse) {
  attn_status_t st = check_mla(a, sparse);
  if (st != ATTN_OK) return st;
  DecodeShape ds;
  const int mode = sparse ? ATTN_SCHED_MLA_SPARSE : ATTN_SCHED_MLA;
  // TND: the work is that of one batch of seqlen_q = T tokens
  const int batch_q = a->cu_seqlens_q ? 1 : a->batch;
  st = decode_shape(mode, batch_q, a->seqlen_q, a->num_heads_q, a->num_heads_kv,
                    sparse_positions(mode, a->topk, a->sparse_block_size), a->num_ctas, ds);
  if (st != ATTN_OK) return st;
  if (a->meta) {
    if (a->meta_bytes < meta_bytes_for(ds)) return ATTN_ERR_INVALID_ARG;
    if (!a->workspace || a->workspace_bytes < mla_ws_bytes(ds))
      return ATTN_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(a->workspace)) return ATTN_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (a->dtype == ATTN_DTYPE_E4M3)
    return sparse ? run_mla<true, true>(*a, ds, s) : run_mla<false, true>(*a, ds, s);
  return sparse ? run_mla<true, false>(*a, ds, s) : run_mla<false, false>(*a, ds, s);
}

}  // namespace
}  // namespace attn
