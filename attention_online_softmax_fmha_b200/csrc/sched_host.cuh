// Host side of the scheduler metadata: the segments and units of a decode or
// MLA problem, shared by the paged decode and the MLA launch code.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "host.cuh"
#include "sched.cuh"
#include "decode_paged.cuh"
#include "mla_sm100.cuh"

namespace attn {
namespace {

// Segments and units of a decode problem (see sched.cuh).
struct DecodeShape {
  SchedShape sh;
  int group = 0, rows = 0, n_rsub = 0, S = 0, G = 0;
  int tiles_per_token = 1, tokens_per_tile = 1, row_tiles = 0;  // MLA
};

// MLA row tiles of 128 (token, head) rows: heads_q a power of two up to 128
// (tiles hold 128 / heads_q tokens) or a multiple of 128.
bool mla_heads_ok(int heads_q) {
  return heads_q > 0 && ((heads_q <= kMlaRows && (heads_q & (heads_q - 1)) == 0) ||
                         heads_q % kMlaRows == 0);
}

// sparse_block_size: 0 or 1 (one position per index) or a power of two up to
// 128 (MindSpore sparse_flash_attention range).
bool sbs_ok(int bs) { return bs == 0 || pow2_in(bs, 1, 128); }
// Key positions per token of a sparse MLA problem (topk indices of bs keys).
int sparse_positions(int mode, int topk, int bs) {
  return mode == ATTN_SCHED_MLA_SPARSE ? topk * (bs > 1 ? bs : 1) : topk;
}

attn_status_t decode_shape(int mode, int batch, int seqlen_q, int heads_q, int heads_kv,
                           int topk, int num_ctas, DecodeShape& ds) {
  if (batch <= 0 || seqlen_q <= 0 || heads_q <= 0 || heads_kv <= 0 || heads_q % heads_kv)
    return ATTN_ERR_INVALID_ARG;
  ds.sh.mode = mode;
  ds.sh.topk = topk;
  ds.sh.new_keys = 0;
  if (mode == ATTN_SCHED_MHA) {
    ds.group = heads_q / heads_kv;
    ds.rows = seqlen_q * ds.group;
    ds.n_rsub = (ds.rows + kDecRows - 1) / kDecRows;
    ds.sh.segs_per_seq = heads_kv * ds.n_rsub;
    ds.sh.unit_keys = kDecTileKeys;
  } else {
    // row tiles of each KV head's group of query heads
    ds.group = heads_q / heads_kv;
    if (!mla_heads_ok(ds.group)) return ATTN_ERR_UNSUPPORTED;
    if (mode == ATTN_SCHED_MLA_SPARSE && topk <= 0) return ATTN_ERR_INVALID_ARG;
    if (ds.group >= kMlaRows) {
      ds.tiles_per_token = ds.group / kMlaRows;
      ds.row_tiles = seqlen_q * ds.tiles_per_token;
    } else {
      ds.tokens_per_tile = mode == ATTN_SCHED_MLA_SPARSE ? 1 : kMlaRows / ds.group;
      ds.row_tiles = (seqlen_q + ds.tokens_per_tile - 1) / ds.tokens_per_tile;
    }
    // both V halves of a row tile: one cluster of two CTAs
    ds.sh.segs_per_seq = heads_kv * ds.row_tiles;
    ds.sh.unit_keys = kMlaBN;
  }
  const int64_t S = (int64_t)batch * ds.sh.segs_per_seq;
  if (S > (1 << 24)) return ATTN_ERR_UNSUPPORTED;
  ds.S = (int)S;
  ds.G = num_ctas > 0 ? num_ctas : device_sm_count();
  if (ds.G <= 0 || ds.G > 65536) return num_ctas < 0 ? ATTN_ERR_INVALID_ARG : ATTN_ERR_CUDA;
  // MLA work goes to clusters of two CTAs: the scheduler's slots are clusters.
  if (mode != ATTN_SCHED_MHA) ds.G = std::max(1, ds.G / 2);
  return ATTN_OK;
}

size_t meta_bytes_for(const DecodeShape& ds) {
  return (size_t)MetaLayout(ds.G, ds.S).words * sizeof(int32_t);
}

}  // namespace
}  // namespace attn
