// MLA-absorbed decode on sm_100a, dense (paged) and top-k sparse.
//
// MATE "Attention", MLA (flash_mla_with_kvcache: 576-wide rows, head_dim_v =
// 512; flash_mla_sparse_fwd); MindSpore "sparse_flash_attention"
// (attention_mode=2: the 512 latent ("nope") and 64 rope parts concatenated
// along D; sparse_indices of logical positions; PA_BSND cache + block table).
// Every query row (token i, head h) scores against the whole 576-wide cached
// row of its KV head g = h / (H_q / H_kv); V is the row's first 512 entries.
// With H_kv > 1 (the MATE MLA example's cache of 2 KV heads) the row tiles of
// each KV head are separate segments; a segment reads only its KV head's
// rows (and, sparse, its KV head's index list).
//
// Work decomposition. A cluster of two CTAs owns 128 query rows ("row tile")
// and streams the keys once for both V halves: CTA rank r holds the score
// dimensions of its V half (rank r: nope 256r .. 256r + 255) and a share of
// the 64 rope dimensions (dense: 32 each; sparse: all on rank 0) of Q and of
// every key, computes the partial scores
// S_r = Q_r K_r^T on its tensor core, and the two halves swap partials through
// distributed shared memory (one bulk copy per warp into the other CTA,
// completing on its barrier), so both see S = S_0 + S_1 (the same sum in the
// same order: identical P). Each CTA then accumulates O for its 256 V columns
// (its first four 64-column chunks). Q sits in TMEM (the S MMAs read A from
// there), which leaves shared memory for a deep key ring, and the cache is
// read once per row tile instead of once per V half.
//   dense : segment = (sequence, KV head, row tile), keys 0 .. L-1 in tiles of 32
//           (causal: key j visible to token i iff j <= i + L - s_q).
//   sparse: segment = (sequence, KV head, token, head tile), keys = that token's
//           listed positions in tiles of 32 entries; entries outside [0, L)
//           are skipped, and with causal (sparse_mode=3) those past
//           i + L - s_q too.
// Segments are split over persistent clusters by the scheduler metadata (a
// metadata "CTA" is a cluster); split segments go through the combine kernel.
//
// Roles (320 threads per CTA; e4m3 rows 384):
//   warps 0-3  softmax: thread r owns query row r (= TMEM lane r). Adds the
//              other CTA's partial scores to its own, writes P over S.
//   warp 4     producer: Q chunks (TMA) through two staging buffers, key
//              tiles of 32 keys into a 6-stage (e4m3: 8-stage) ring: dense by
//              TMA boxes through the block table; sparse by per-lane 16-byte
//              async copies of the gathered rows (each lane one key, zeros for
//              skipped keys), completed and fenced before the stage is handed
//              over.
//   warp 5     TMEM owner and MMA issuer (whole warp, one elected lane): Q
//              chunks into TMEM (tcgen05.cp); S_j = Q K_j^T (M=128, N=32, A
//              from TMEM) into one of three TMEM S buffers (issued three tiles
//              ahead); O += P_j V_j (M=128, N=256, K=32) with P from TMEM.
//   warps 6-7  e4m3 rows only: the fp16 copy of each tile's V half.
//   last 4     sender: loads each S tile and sends it to the other CTA, so
//              the softmax never waits on the exchange's copy.
#pragma once

#include "combine.cuh"
#include "common.cuh"
#include "sched.cuh"

namespace attn {

constexpr int kMlaDqk = 576;
constexpr int kMlaDv = 512;
constexpr int kMlaDvHalf = 256;
constexpr int kMlaBN = 32;         // keys per tile
constexpr int kMlaRows = 128;      // query rows per row tile
constexpr int kMlaMaxStages = 8;  // key stages of the deepest ring (MlaCfg::kStages)
constexpr int kMlaSBufs = 3;       // S buffers in TMEM
// S of tile g + kMlaSAhead is issued after P V of tile g. The sender needs S
// ahead of the softmax (the other CTA waits for its partials), so at least
// 2; each tile further ahead keeps one more key stage busy and leaves one
// tile less of slack for the loads.
constexpr int kMlaSAhead = 3;
static_assert(kMlaSAhead >= 2 && kMlaSAhead <= kMlaSBufs, "S lookahead");
// The O barriers (one per S buffer) rely on S of tile g being issued after P V
// of tile g - kMlaSBufs.
static_assert(kMlaSAhead == kMlaSBufs, "O barrier phases");
constexpr int kMlaXsBufs = 2;      // partial-S exchange buffers in shared memory
constexpr int kGatherLag = 1;      // sparse: tiles of gathers in flight before a stage is signalled
constexpr int kMlaQChunkBytes = kMlaRows * 128;                // 16 KB
constexpr int kMlaKVChunkBytes = kMlaBN * 128;                 // 4 KB
constexpr int kMlaXsBytes = kMlaRows * kMlaBN * 4;             // one partial S tile, 16 KB
constexpr uint32_t kMlaTmemCols = 512;
constexpr uint32_t kMlaTmemS = 0;      // three S buffers of 32 columns
constexpr uint32_t kMlaTmemQ = 96;     // Q: 32 columns per 128-byte chunk, 5 chunks at most
constexpr uint32_t kMlaTmemO = 256;    // 256 columns of O
constexpr int kMlaQStages = 2;         // Q staging buffers of one chunk (128 rows x 128 bytes)

// Shared-memory layout of the bf16 (kFp8 = false) and the e4m3 kernel. A
// chunk is one 128-byte column of a TMA box: 64 bf16 or 128 e4m3 values.
// e4m3 rows also need an fp16 copy of the tile's V half for P V (FP8 has no
// fp16 partner type in one MMA, and P stays fp16), made by two extra warps.
template <bool kFp8>
struct MlaCfg {
  static constexpr int kMaxChunks = kFp8 ? 3 : 5;          // chunks per CTA (at most)
  static constexpr int kKVBytes = kMaxChunks * kMlaKVChunkBytes;
  // Q passes through two one-chunk staging buffers into TMEM, where the S
  // MMAs read it; the shared memory this frees holds more key stages.
  static constexpr int kQSOff = 0;
  static constexpr int kXsOff = kQSOff + kMlaQStages * kMlaQChunkBytes;  // partial S received here
  static constexpr int kXoOff = kXsOff + kMlaXsBufs * kMlaXsBytes;       // and staged here to send
  static constexpr int kKVOff = kXoOff + kMlaXsBufs * kMlaXsBytes;
  static constexpr int kStages = kFp8 ? 8 : 6;
  static constexpr int kVHStages = kFp8 ? 2 : 0;
  static constexpr int kVHBytes = 4 * kMlaKVChunkBytes;  // fp16 V half: 4 chunks of 64 columns
  static constexpr int kVHOff = kKVOff + kStages * kKVBytes;
  static constexpr int kBarOff = kVHOff + kVHStages * kVHBytes;
  static constexpr int kSmemBytes = kBarOff + 512;
  // softmax 0-3, producer 4, MMA 5, (e4m3: conversion 6-7), sender warpgroup
  static constexpr int kSendWarp0 = kFp8 ? 8 : 6;
  static constexpr int kThreads = (kSendWarp0 + 4) * 32;
  static_assert(kStages <= kMlaMaxStages && kGatherLag < kStages, "key ring");
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  static_assert(kMlaTmemQ + 32 * kMaxChunks <= kMlaTmemO, "TMEM columns");
};

// Columns held by each CTA. A CTA's first 256 columns are its V half: rank r
// holds the nope (latent) columns 256r .. 256r + 255. The 64 rope columns
// (512..575) sit in one more box: bf16 chunk 4 (64 columns at 512); e4m3
// chunk 2 (the box at 448, whose second half is the rope). Dense kernels
// split the rope, 32 columns to each CTA (both load its box), so the two
// CTAs' S MMAs take 18 (e4m3: 9) K steps each; sparse kernels, bound by the
// gathered bytes rather than the MMAs, leave it all to rank 0 (20 and 16
// steps; e4m3 10 and 8) and rank 1 loads no rope box.
template <bool kFp8, bool kSplitRope>
DEVI int mla_nchunks(int rank) {
  return (kSplitRope || rank == 0) ? (kFp8 ? 3 : 5) : (kFp8 ? 2 : 4);
}
// First element column of local chunk c of rank r.
template <bool kFp8>
DEVI int mla_col(int rank, int c) {
  if constexpr (kFp8) return c < 2 ? 256 * rank + 128 * c : 448;
  return c < 4 ? 64 * (4 * rank + c) : 512;
}
// 32-byte K steps of this CTA's partial score, and the (chunk, step within
// the chunk) of step k. The rope steps start at step 2 of the e4m3 box (its
// first half is latent columns 448..511, counted by rank 1) and, with a split
// rope, rank 1 takes the second half of the rope.
template <bool kFp8, bool kSplitRope>
DEVI int mla_ksteps(int rank) {
  return kSplitRope ? (kFp8 ? 9 : 18) : (kFp8 ? (rank == 0 ? 10 : 8) : (rank == 0 ? 20 : 16));
}
template <bool kFp8>
DEVI void mla_kstep(int k, int rope_off, int& chunk, int& sub) {
  chunk = k >> 2;
  sub = k & 3;
  if (kFp8 && k >= 8) {
    chunk = 2;
    sub = 2 + (k - 8) + rope_off;
  } else if (!kFp8 && k >= 16) {
    chunk = 4;
    sub = (k - 16) + rope_off;
  }
}

struct MlaParams {
  const void* q;
  void* out;
  float* lse;
  const int32_t* block_table;
  const int32_t* cache_seqlens;
  const int32_t* indices;
  const int32_t* meta;
  float* ws_o;    // [slot][V half][128][256]
  float* ws_lse;  // [slot][128]
  const void* kv;
  const float* q_descale;  // FP8: (B, H_kv) each, or nullptr (all 1)
  const float* k_descale;
  const float* v_descale;
  int64_t bt_stride;
  int64_t q_sb, q_ss, q_sh;
  int64_t o_sb, o_ss, o_sh;
  int64_t kv_sblk, kv_stok, kv_sh;
  int64_t idx_sb, idx_ss, idx_sh;
  int32_t batch, seqlen_q, heads_q, page_size, topk;
  int32_t heads_kv, group;  // latent KV heads; query heads per KV head (H_q / H_kv)
  // Packed (TND) sparse queries: the query side is one sequence of seqlen_q = T
  // tokens (batch = 1); token t belongs to KV sequence b with
  // cu_q[b] <= t < cu_q[b + 1] (batch_kv sequences). nullptr: BSND.
  const int32_t* cu_q;
  int32_t batch_kv;
  int32_t sbs;              // sparse: positions per index (sparse_block_size, >= 1)
  int32_t sbs_log2;         // log2(sbs) (sbs is a power of two)
  int32_t tiles_per_token;  // group >= 128: group / 128 (else 1)
  int32_t tokens_per_tile;  // group < 128: 128 / group (else 1)
  int32_t row_tiles;        // row tiles per (sequence, KV head)
  int32_t segs_per_seq, num_segs, num_ctas;  // num_ctas: clusters (metadata slots)
  float scale_log2;
  int32_t causal;
};

struct MlaBarriers {
  uint64_t qs_full[kMlaQStages], qs_empty[kMlaQStages];  // Q chunk staging buffers
  uint64_t q_done;  // the segment's last S has completed: TMEM Q may be replaced
  uint64_t kv_full[kMlaMaxStages], kv_empty[kMlaMaxStages];
  uint64_t vh_full[2], vh_empty[2];  // FP8: the fp16 copies of V
  uint64_t s_full[kMlaSBufs], p_full[2];
  uint64_t xs_full[kMlaXsBufs];   // the other CTA's partial S tile has landed here
  uint64_t xs_empty[kMlaXsBufs];  // the other CTA has read the tile this CTA sent it
  uint64_t s_read[kMlaSBufs];     // the sender has loaded S buffer k: P may overwrite it
  // o_full[k]: P V of every tile g with g % 3 == k has completed. One barrier
  // per S buffer: S of tile g is issued after P V of tile g - 3, so a waiter
  // for P V of tile x knows P V of tile x - 3 (the same barrier's previous
  // phase) is done, and the barrier is never two phases past the awaited one.
  uint64_t o_full[kMlaSBufs], o_empty;
  uint64_t mma_drain;
  uint32_t tmem_base;
  int32_t abort;
};
static_assert(sizeof(MlaBarriers) <= 512, "barrier block");

// A segment and its rows.
struct MlaSeg {
  int b, len;        // query-side batch index; cached keys of the KV sequence
  int bk;            // KV-side sequence (block table, cache length): b, or TND's
  int q0, sq;        // first token and token count of the query rows of sequence bk
  int kvg;           // KV head; its query heads are kvg * group .. + group - 1
  int tok0, head0;   // first (token, head within the group) of the row tile
  int rows_valid;    // rows of the tile that exist (the rest are padding)
  int units;         // KV tiles of the segment
};

template <bool kSparse>
DEVI void mla_seg(const MlaParams& p, int s, MlaSeg& g) {
  g.b = s / p.segs_per_seq;
  const int rem = s - g.b * p.segs_per_seq;  // (KV head, row tile) within the sequence
  g.kvg = rem / p.row_tiles;
  const int rt = rem - g.kvg * p.row_tiles;
  if (p.group >= kMlaRows) {
    g.tok0 = rt / p.tiles_per_token;
    g.head0 = (rt % p.tiles_per_token) * kMlaRows;
    g.rows_valid = kMlaRows;
  } else {
    g.tok0 = kSparse ? rt : rt * p.tokens_per_tile;
    g.head0 = 0;
    g.rows_valid = kSparse ? p.group : min(kMlaRows, (p.seqlen_q - g.tok0) * p.group);
  }
  g.bk = g.b;
  g.q0 = 0;
  g.sq = p.seqlen_q;
  if (kSparse && p.cu_q) {
    // the packed token's sequence: the last b with cu_q[b] <= tok0
    int lo = 0, hi = p.batch_kv - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.cu_q[mid] <= g.tok0) lo = mid; else hi = mid - 1;
    }
    g.bk = lo;
    g.q0 = p.cu_q[lo];
    g.sq = p.cu_q[lo + 1] - g.q0;
  }
  g.len = p.cache_seqlens[g.bk];
  if (kSparse)
    g.units = (p.topk * p.sbs + kMlaBN - 1) / kMlaBN;
  else
    g.units = g.len > 0 ? (g.len + kMlaBN - 1) / kMlaBN : 0;
}

// Key position of entry e of token tok's sparse list (-1: skipped): with
// sparse_block_size bs, index k >= 0 lists positions k*bs .. k*bs + bs - 1.
DEVI int mla_sparse_pos(const MlaParams& p, int b, int kvg, int tok, int e) {
  if (e >= (p.topk << p.sbs_log2)) return -1;
  const int blk = e >> p.sbs_log2;
  const int k = __ldg(p.indices + b * p.idx_sb + (int64_t)tok * p.idx_ss + kvg * p.idx_sh + blk);
  return k >= 0 ? (k << p.sbs_log2) + (e & (p.sbs - 1)) : -1;
}
// The same in two steps, so that the index load can be issued a tile early
// and stay in flight until its value is used: the raw index word of entry e
// (-1 past the list), then the position it gives.
DEVI int mla_sparse_raw(const MlaParams& p, int b, int kvg, int tok, int e) {
  if (e >= (p.topk << p.sbs_log2)) return -1;
  return __ldg(p.indices + b * p.idx_sb + (int64_t)tok * p.idx_ss + kvg * p.idx_sh +
               (e >> p.sbs_log2));
}
DEVI int mla_pos_of(const MlaParams& p, int k, int e) {
  return k >= 0 ? (k << p.sbs_log2) + (e & (p.sbs - 1)) : -1;
}

// Token and (global) query head of tile row x.
DEVI void mla_row(const MlaParams& p, const MlaSeg& g, int x, int& tok, int& head) {
  if (p.group >= kMlaRows) {
    tok = g.tok0;
    head = g.kvg * p.group + g.head0 + x;
  } else {
    tok = g.tok0 + x / p.group;
    head = g.kvg * p.group + x % p.group;
  }
}

// The cluster's unit range [ub, ue) and first segment (metadata, or one
// segment per cluster).
template <bool kSparse>
DEVI void mla_range(const MlaParams& p, int& ub, int& ue, int& s0, const int32_t*& prefix) {
  const int cl = blockIdx.x >> 1;
  if (p.meta) {
    const MetaLayout ml(p.num_ctas, p.num_segs);
    ub = p.meta[ml.cta_begin + cl];
    ue = p.meta[ml.cta_begin + cl + 1];
    s0 = p.meta[ml.cta_seg + cl];
    prefix = p.meta + ml.seg_begin;
  } else {
    MlaSeg g;
    mla_seg<kSparse>(p, cl, g);
    s0 = cl;
    ub = 0;
    ue = g.units;  // an empty sequence: the softmax warps write O = 0, LSE = -inf
    prefix = nullptr;
  }
}

// ---------------------------------------------------------------------------
// Producer warp
// ---------------------------------------------------------------------------
template <bool kSparse, bool kFp8>
DEVI void mla_producer(const MlaParams& p, const CUtensorMap* mq, const CUtensorMap* mkv,
                       uint8_t* smem, MlaBarriers* bars, int rank) {
  using C = MlaCfg<kFp8>;
  constexpr int kEsize = kFp8 ? 1 : 2;
  volatile int* abort = &bars->abort;
  const int lane = threadIdx.x & 31;
  const int nch = mla_nchunks<kFp8, !kSparse>(rank);
  if (lane == 0) {
    tma_prefetch_desc(mq);
    if (!kSparse) tma_prefetch_desc(mkv);
  }
  int ub, ue, s;
  const int32_t* prefix;
  mla_range<kSparse>(p, ub, ue, s, prefix);
  int it = 0, nqc = 0;  // key tiles and Q chunks issued
  const int P = p.page_size;
  // Sparse gathers issued and not yet signalled: tiles it - pend .. it - 1.
  int pend = 0;
  auto flush_gathers = [&]() {
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    fence_proxy_async_smem();
    for (; pend > 0; --pend) mbar_arrive(&bars->kv_full[(it - pend) % C::kStages]);
  };
  int u = ub;
  // After a failed wait the producer stops issuing and falls through to the
  // drains below, so no copy it issued lands after the CTA exits.
  bool stop = false;
  while (u < ue && !stop) {
    int sb, se;
    if (prefix) {
      sb = prefix[s];
      se = prefix[s + 1];
      if (se <= u) { ++s; continue; }
    } else {
      sb = u;
      se = ue;
    }
    MlaSeg g;
    mla_seg<kSparse>(p, s, g);
    const int a = u - sb, e = min(ue, se) - sb;
    if (e <= a) {
      u = min(ue, se);
      ++s;
      continue;
    }
    // Q tile of the segment: this CTA's chunks of the 576 columns, one at a
    // time through the staging buffers (the MMA warp copies each into TMEM).
    const int box_rows =
        p.group >= kMlaRows ? kMlaRows : p.group * (kSparse ? 1 : p.tokens_per_tile);
    for (int c = 0; c < nch && !stop; ++c) {
      const int qb = nqc % kMlaQStages;
      bool ok = true;
      if (lane == 0) {
        ok = nqc < kMlaQStages ||
             mbar_wait(&bars->qs_empty[qb], ((nqc / kMlaQStages) - 1) & 1, abort, 60);
        if (ok) {
          mbar_expect_tx(&bars->qs_full[qb], box_rows * 128);
          tma_load_4d(smem + C::kQSOff + qb * kMlaQChunkBytes, mq, &bars->qs_full[qb],
                      mla_col<kFp8>(rank, c), g.kvg * p.group + g.head0, g.tok0, g.b);
        }
      }
      if (__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) ++nqc;
      else stop = true;
    }
    if (stop) break;
    const int32_t* bt = p.block_table + (int64_t)g.bk * p.bt_stride;
    // sparse: this lane's index word is loaded two tiles ahead and its cache
    // block one tile ahead, so no dependent global load sits between a stage
    // becoming free and the gathers into it.
    int pos_c = -1, blk_c = 0, raw_n = -1;  // tile t's position and block; tile t + 1's index
    if constexpr (kSparse) {
      pos_c = mla_sparse_pos(p, g.b, g.kvg, g.tok0, a * kMlaBN + lane);
      if (pos_c >= 0 && pos_c < g.len) blk_c = __ldg(bt + pos_c / P);
      if (a + 1 < e) raw_n = mla_sparse_raw(p, g.b, g.kvg, g.tok0, (a + 1) * kMlaBN + lane);
    }
    for (int t = a; t < e; ++t, ++it) {
      const int st = it % C::kStages;
      uint8_t* dst = smem + C::kKVOff + st * C::kKVBytes;
      bool ok = true;
      if (it >= C::kStages) {
        const uint32_t parity = ((it / C::kStages) - 1) & 1;
        if constexpr (kSparse) {
          // About to block on a stage: signal every gathered tile first (the
          // MMA warp may need them to free that stage).
          const bool free_now = lane == 0 && mbar_test(smem_u32(&bars->kv_empty[st]), parity);
          if (!__shfl_sync(0xffffffffu, free_now ? 1 : 0, 0)) flush_gathers();
        }
        if (lane == 0) ok = mbar_wait(&bars->kv_empty[st], parity, abort, 61);
      }
      if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
        if constexpr (kSparse) flush_gathers();
        stop = true;
        break;
      }
      if constexpr (!kSparse) {
        // keys [32t, 32t + 32): pages of the block table, one TMA box per
        // (page, 64-column chunk)
        const int key0 = t * kMlaBN;
        const int npages = (g.len + P - 1) / P;
        const int box = P >= kMlaBN ? kMlaBN : P;
        const int nload = P >= kMlaBN ? 1 : min(kMlaBN / P, npages - key0 / P);
        int page = 0;
        if (lane < nload) page = bt[key0 / P + lane];
        if (lane == 0) {
          mbar_expect_tx(&bars->kv_full[st], nch * nload * box * 128);
        }
        for (int j = 0; j < nload; ++j) {
          const int pg = __shfl_sync(0xffffffffu, page, j);
          if (lane == 0)
            for (int c = 0; c < nch; ++c)
              tma_load_4d(dst + c * kMlaKVChunkBytes + j * box * 128, mkv, &bars->kv_full[st],
                          mla_col<kFp8>(rank, c), key0 % P, pg, g.kvg);
        }
      } else {
        // lane k gathers key t*32 + k: 8 async copies of 16 bytes per chunk
        // into the 128-byte-swizzled layout, or zeros if the entry is skipped.
        const int pos = pos_c, blk = blk_c;
        const bool valid = pos >= 0 && pos < g.len;
        // ahead: the position and block of tile t + 1, the index of tile t + 2
        pos_c = mla_pos_of(p, raw_n, (t + 1) * kMlaBN + lane);
        blk_c = (pos_c >= 0 && pos_c < g.len) ? __ldg(bt + pos_c / P) : 0;
        raw_n = t + 2 < e ? mla_sparse_raw(p, g.b, g.kvg, g.tok0, (t + 2) * kMlaBN + lane) : -1;
        const uint8_t* src = nullptr;  // the cached row, in bytes
        if (valid)
          src = static_cast<const uint8_t*>(p.kv) +
                (g.kvg * p.kv_sh + (int64_t)blk * p.kv_sblk + (int64_t)(pos % P) * p.kv_stok) *
                    kEsize;
        const uint32_t dbase = smem_u32(dst) + lane * 128;
        for (int c = 0; c < nch; ++c) {
          const int gcol = mla_col<kFp8>(rank, c) * kEsize;  // byte column of the chunk
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const uint32_t d = dbase + c * kMlaKVChunkBytes + ((x ^ (lane & 7)) << 4);
            if (valid) {
              asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d),
                           "l"(src + gcol + x * 16)
                           : "memory");
            } else {
              asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" ::"r"(d), "r"(0) : "memory");
            }
          }
        }
        // The stage is signalled kGatherLag tiles later, once this lane's
        // copies of it have landed (made visible to the tensor core, the async
        // proxy), so the gathers of several tiles are in flight at once.
        asm volatile("cp.async.commit_group;" ::: "memory");
        ++pend;
        if (pend > kGatherLag) {
          asm volatile("cp.async.wait_group %0;" ::"n"(kGatherLag) : "memory");
          fence_proxy_async_smem();
          mbar_arrive(&bars->kv_full[(it - kGatherLag) % C::kStages]);
          --pend;
        }
      }
    }
    if (stop) break;
    // The segment's last S needs its last tiles before TMEM Q may be replaced
    // (and the next segment's Q chunks wait for that).
    if constexpr (kSparse) flush_gathers();
    u = min(ue, se);
    ++s;
  }
  if constexpr (!kSparse) {
    if (lane == 0) {  // the last stages' copies must land before the CTA exits
      int zero = 0;
      for (int i = max(0, it - C::kStages); i < it; ++i)
        mbar_wait(&bars->kv_full[i % C::kStages], (i / C::kStages) & 1, &zero, 62);
    }
  }
  if (lane == 0) {  // and the last Q chunks
    int zero = 0;
    for (int i = max(0, nqc - kMlaQStages); i < nqc; ++i)
      mbar_wait(&bars->qs_full[i % kMlaQStages], (i / kMlaQStages) & 1, &zero, 63);
  }
}

// ---------------------------------------------------------------------------
// MMA warp (whole warp; one elected lane issues)
// ---------------------------------------------------------------------------
// Shared memory to TMEM: 128 rows of 32 bytes (row i to lane i, 8 columns
// from taddr's), the source given by a shared-memory matrix descriptor. Runs
// in order with the MMAs this thread issues after it; one elected lane.
DEVI void tc_cp_128x256b_w(uint32_t taddr, uint64_t sdesc) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.cp.cta_group::1.128x256b [%0], %1;\n\t}" ::"r"(taddr),
      "l"(sdesc)
      : "memory");
}

// S of the tile with global index g (this CTA's partial scores), A = Q from
// TMEM: waits for its key stage, writes S buffer g % 3; the segment's last S
// also signals q_done (TMEM Q may then be replaced).
// e4m3: S runs on the FP8 codes (kind::f8f6f4); P V reads the fp16 copy of V,
// so the stage is released here (with the conversion warps' arrivals).
template <bool kFp8>
DEVI bool mla_issue_s(MlaBarriers* bars, int g, uint64_t dkv, uint32_t tmem, int nk, int rope_off,
                      bool last) {
  // kind::f16 format 1 = bf16; kind::f8f6f4 format 0 = e4m3
  constexpr uint32_t idesc_s = make_idesc(128, kMlaBN, kFp8 ? 0 : 1, 0, 0);
  constexpr int kStages = MlaCfg<kFp8>::kStages;
  const int st = g % kStages;
  if (!warp_wait(&bars->kv_full[st], (g / kStages) & 1, &bars->abort, 71)) return false;
  tc_fence_after();
  const uint32_t sbuf = tmem + kMlaTmemS + (g % kMlaSBufs) * kMlaBN;
  const uint64_t kst = dkv + st * (MlaCfg<kFp8>::kKVBytes >> 4);
#pragma unroll 4
  for (int k = 0; k < nk; ++k) {
    int ch, sub;
    mla_kstep<kFp8>(k, rope_off, ch, sub);
    // 32 bytes of each Q row per K step: 8 TMEM columns
    const uint32_t qa = tmem + kMlaTmemQ + ch * 32 + sub * 8;
    const uint32_t ko = ch * (kMlaKVChunkBytes >> 4) + sub * 2;
    if constexpr (kFp8)
      mma_f8_ts_w(sbuf, qa, kst + ko, idesc_s, k > 0 ? 1u : 0u);
    else
      mma_f16_ts_w(sbuf, qa, kst + ko, idesc_s, k > 0 ? 1u : 0u);
  }
  tc_commit_w(&bars->s_full[g % kMlaSBufs]);
  if constexpr (kFp8) tc_commit_w(&bars->kv_empty[st]);
  if (last) tc_commit_w(&bars->q_done);
  return true;
}

template <bool kSparse, bool kFp8>
DEVI void mla_mma(const MlaParams& p, uint8_t* smem, MlaBarriers* bars, uint32_t tmem, int rank) {
  using C = MlaCfg<kFp8>;
  volatile int* abort = &bars->abort;
  const int nk = mla_ksteps<kFp8, !kSparse>(rank);  // 32-byte K steps of the partial score
  // with a split rope, rank 1 takes its second half (2 bf16 or 1 e4m3 K steps on)
  const int rope_off = (!kSparse && rank == 1) ? (kFp8 ? 1 : 2) : 0;
  // P V: bf16 P and V, or (e4m3 rows) fp16 P and the fp16 copy of V
  constexpr uint32_t idesc_pv = make_idesc(128, kMlaDvHalf, kFp8 ? 0 : 1, 0, 1);
  // Q staging buffers, 128-byte swizzled K-major: 32-byte K steps
  const uint64_t dqs = sdesc_sw128(smem_u32(smem + C::kQSOff), 16, 1024);
  const int nch = mla_nchunks<kFp8, !kSparse>(rank);
  const uint64_t dkv = sdesc_sw128(smem_u32(smem + C::kKVOff), 16, 1024);
  // This CTA's V half: local chunks 0..3 of the bf16 key tile (or of the
  // fp16 copy), MN-major (leading byte offset = chunk stride, stride byte
  // offset = 8 keys x 128 bytes).
  const uint64_t dv = sdesc_sw128(smem_u32(smem + (kFp8 ? C::kVHOff : C::kKVOff)),
                                  kMlaKVChunkBytes, 1024);
  int ub, ue, s;
  const int32_t* prefix;
  mla_range<kSparse>(p, ub, ue, s, prefix);
  int it = 0, nqc = 0, nseg = 0, pieces = 0;
  int u = ub;
  while (u < ue) {
    int sb, se;
    if (prefix) {
      sb = prefix[s];
      se = prefix[s + 1];
      if (se <= u) { ++s; continue; }
    } else {
      sb = u;
      se = ue;
    }
    MlaSeg g;
    mla_seg<kSparse>(p, s, g);
    const int a = u - sb, e = min(ue, se) - sb;
    const int n = max(0, e - a);
    if (n == 0) {  // empty sequence without metadata: the softmax writes O = 0
      u = min(ue, se);
      ++s;
      continue;
    }
    // Q into TMEM once the previous segment's S MMAs have read the old one:
    // each staged chunk as 4 copies of 128 rows x 32 bytes (lane = row, 8
    // columns each, the layout of an A operand in TMEM), then the staging
    // buffer goes back to the producer.
    if (nseg > 0 && !warp_wait(&bars->q_done, (nseg - 1) & 1, abort, 70)) goto drain;
    ++nseg;
    for (int c = 0; c < nch; ++c, ++nqc) {
      const int qb = nqc % kMlaQStages;
      if (!warp_wait(&bars->qs_full[qb], (nqc / kMlaQStages) & 1, abort, 78)) goto drain;
      tc_fence_after();
#pragma unroll
      for (int sub = 0; sub < 4; ++sub)
        tc_cp_128x256b_w(tmem + kMlaTmemQ + c * 32 + sub * 8,
                         dqs + qb * (kMlaQChunkBytes >> 4) + sub * 2);
      tc_commit_w(&bars->qs_empty[qb]);
    }
    // S of the first kMlaSAhead tiles, then per tile g: PV_g, S_{g+kMlaSAhead}
    // (into buffer (g + kMlaSAhead) % 3, whose last P the tensor core has read
    // in an earlier P V: the pipe runs in order). The softmax thus finds
    // S_{g+1} ready while it finishes tile g.
    for (int j = 0; j < kMlaSAhead && j < n; ++j)
      if (!mla_issue_s<kFp8>(bars, it + j, dkv, tmem, nk, rope_off, j == n - 1)) goto drain;
    for (int j = 0; j < n; ++j) {
      const int gi = it + j, sp = gi % C::kStages;
      if (!warp_wait(&bars->p_full[gi & 1], (gi >> 1) & 1, abort, 72)) goto drain;
      if (j == 0 && pieces > 0 && !warp_wait(&bars->o_empty, (pieces - 1) & 1, abort, 73))
        goto drain;
      uint64_t vst;
      if constexpr (kFp8) {
        if (!warp_wait(&bars->vh_full[gi & 1], (gi >> 1) & 1, abort, 75)) goto drain;
        vst = dv + (gi & 1) * (C::kVHBytes >> 4);
      } else {
        vst = dv + sp * (C::kKVBytes >> 4);
      }
      tc_fence_after();
      const uint32_t pbuf = tmem + kMlaTmemS + (gi % kMlaSBufs) * kMlaBN;
#pragma unroll
      for (int kk = 0; kk < kMlaBN / 16; ++kk)
        mma_f16_ts_w(tmem + kMlaTmemO, pbuf + kk * 8, vst + kk * (16 * 128 >> 4), idesc_pv,
                     (j > 0 || kk > 0) ? 1u : 0u);
      if constexpr (kFp8)
        tc_commit_w(&bars->vh_empty[gi & 1]);
      else
        tc_commit_w(&bars->kv_empty[sp]);
      tc_commit_w(&bars->o_full[gi % kMlaSBufs]);
      if (j + kMlaSAhead < n &&
          !mla_issue_s<kFp8>(bars, gi + kMlaSAhead, dkv, tmem, nk, rope_off,
                             j + kMlaSAhead == n - 1))
        goto drain;
    }
    it += n;
    ++pieces;
    u = min(ue, se);
    ++s;
  }
drain : {
  int zero = 0;
  tc_commit_w(&bars->mma_drain);
  warp_wait(&bars->mma_drain, 0, &zero, 74);
}
}

// ---------------------------------------------------------------------------
// e4m3 rows only: conversion warps (warps 6, 7). Each key tile's V half (the
// CTA's first two 128-column chunks of e4m3 codes) is rewritten as fp16, which
// holds every e4m3 value exactly, in the layout the P V MMA reads (four
// 64-column chunks, 128-byte swizzled); keys past the end of the cache become
// zeros so that P = 0 never meets a NaN code. The FP8 stage is then released
// (with the S MMA's commit) and the fp16 copy handed to the MMA warp.
// ---------------------------------------------------------------------------
template <bool kSparse>
DEVI void mla_convert(const MlaParams& p, uint8_t* smem, MlaBarriers* bars) {
  using C = MlaCfg<true>;
  volatile int* abort = &bars->abort;
  const int t = threadIdx.x - 192;  // 0..63
  int ub, ue, s;
  const int32_t* prefix;
  mla_range<kSparse>(p, ub, ue, s, prefix);
  int it = 0;
  int u = ub;
  while (u < ue) {
    int sb, se;
    if (prefix) {
      sb = prefix[s];
      se = prefix[s + 1];
      if (se <= u) { ++s; continue; }
    } else {
      sb = u;
      se = ue;
    }
    MlaSeg g;
    mla_seg<kSparse>(p, s, g);
    const int a = u - sb, e = min(ue, se) - sb;
    for (int j = 0; j < e - a; ++j, ++it) {
      const int st = it % C::kStages, hb = it & 1;
      if (!mbar_wait(&bars->kv_full[st], (it / C::kStages) & 1, abort, 76)) return;
      if (it >= 2 && !mbar_wait(&bars->vh_empty[hb], ((it >> 1) - 1) & 1, abort, 77)) return;
      // keys of the tile that exist (sparse: skipped entries are zeros already)
      const int nvalid = kSparse ? kMlaBN : g.len - (a + j) * kMlaBN;
      const uint8_t* src = smem + C::kKVOff + st * C::kKVBytes;
      uint8_t* dst = smem + C::kVHOff + hb * C::kVHBytes;
#pragma unroll 2
      for (int x = t; x < kMlaBN * 16; x += 64) {
        // key row, source chunk (0, 1) and its 16-byte unit: e4m3 columns
        // 128 * c + 16 * unit .. + 15
        const int row = x >> 4, c = (x >> 3) & 1, unit = x & 7;
        uint4 v = *reinterpret_cast<const uint4*>(src + c * kMlaKVChunkBytes + row * 128 +
                                                  ((unit ^ (row & 7)) << 4));
        if (row >= nvalid) v = make_uint4(0, 0, 0, 0);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t h[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          h[2 * q] = fp8x2_to_f16x2<2>((unsigned short)(w[q] & 0xffff));
          h[2 * q + 1] = fp8x2_to_f16x2<2>((unsigned short)(w[q] >> 16));
        }
        // fp16 columns 128 c + 16 unit .. + 15: chunk 2c + unit / 4, units
        // 2 (unit % 4) and + 1 of that chunk's 128-byte row
        const int dchunk = 2 * c + (unit >> 2), du = (unit & 3) * 2;
        uint8_t* drow = dst + dchunk * kMlaKVChunkBytes + row * 128;
        *reinterpret_cast<uint4*>(drow + ((du ^ (row & 7)) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(drow + (((du + 1) ^ (row & 7)) << 4)) =
            make_uint4(h[4], h[5], h[6], h[7]);
      }
      fence_proxy_async_smem();  // the fp16 tile is read by the tensor core
      mbar_arrive(&bars->vh_full[hb]);
      mbar_arrive(&bars->kv_empty[st]);
    }
    u = min(ue, se);
    ++s;
  }
}

// ---------------------------------------------------------------------------
// Softmax warpgroup
// ---------------------------------------------------------------------------
// ---------------------------------------------------------------------------
// Sender warpgroup
// ---------------------------------------------------------------------------
// Remote arrivals with relaxed semantics. A release at cluster scope here
// cost about a thousand cycles per tile on the softmax's critical path.
// expect_tx publishes nothing (the bulk copy's complete_tx carries the data);
// the release of a receive buffer follows loads whose values the thread has
// already consumed (the adds before it), and a warp issues in order, so the
// loads have returned before the arrival leaves.
DEVI void mbar_arrive_remote_relaxed(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
DEVI void mbar_expect_tx_remote_relaxed(uint32_t cluster_addr, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.relaxed.cluster.shared::cluster.b64 _, [%0], %1;" ::"r"(
                   cluster_addr),
               "r"(bytes)
               : "memory");
}

// For every tile, in the MMA warp's order: loads this CTA's partial scores
// (thread = row = TMEM lane) and tells the softmax the S buffer may take P
// (s_read), then sends the rows to the other CTA's receive buffer g % 2:
// each warp stages its 32 rows (16-byte pieces permuted by row to spread the
// banks), fences them for the async proxy and sends one 4 KB bulk copy that
// completes on that CTA's barrier. Before writing buffer b it waits until the
// other CTA's softmax has read the tile sent there before (xs_empty), and
// staging buffer b until the copy two tiles ago has read it. The softmax
// threads thus never wait on the exchange's staging, fence or copy.
template <bool kSparse, bool kFp8>
DEVI void mla_sender(const MlaParams& p, uint8_t* smem, MlaBarriers* bars, uint32_t tmem,
                     int rank, int quarter) {
  using C = MlaCfg<kFp8>;
  volatile int* abort = &bars->abort;
  const int r = quarter * 32 + (threadIdx.x & 31);  // row = TMEM lane
  const uint32_t lane = (uint32_t)(quarter * 32) << 16;
  const bool leader = (threadIdx.x & 31) == 0;
  int ub, ue, s;
  const int32_t* prefix;
  mla_range<kSparse>(p, ub, ue, s, prefix);
  int g = 0;
  int u = ub;
  while (u < ue) {
    int sb, se;
    if (prefix) {
      sb = prefix[s];
      se = prefix[s + 1];
      if (se <= u) { ++s; continue; }
    } else {
      sb = u;
      se = ue;
    }
    const int n = max(0, min(ue, se) - u);
    for (int j = 0; j < n; ++j, ++g) {
      const int sbuf = g % kMlaSBufs, b = g % kMlaXsBufs;
      uint32_t sv[kMlaBN];
      if (!warp_wait(&bars->s_full[sbuf], (g / kMlaSBufs) & 1, abort, 80)) return;
      tc_fence_after();
      tmem_load<32>(tmem + kMlaTmemS + sbuf * kMlaBN + lane, sv);
      tc_fence_before();
      __syncwarp();
      if (leader) mbar_arrive(&bars->s_read[sbuf]);
      if (g >= kMlaXsBufs &&
          !warp_wait_cluster(&bars->xs_empty[b], ((g / kMlaXsBufs) - 1) & 1, abort, 84))
        return;
      const int warp_row0 = r & ~31;
      if (leader) bulk_wait_read<1>();
      __syncwarp();
      uint8_t* stage = smem + C::kXoOff + b * kMlaXsBytes + r * 128;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        *reinterpret_cast<uint4*>(stage + ((k ^ (r & 7)) << 4)) =
            make_uint4(sv[4 * k], sv[4 * k + 1], sv[4 * k + 2], sv[4 * k + 3]);
      fence_proxy_async_smem();  // the copy reads through the async proxy
      __syncwarp();
      if (leader) {
        const uint32_t bar = mapa_shared(smem_u32(&bars->xs_full[b]), rank ^ 1);
        const uint32_t off = b * kMlaXsBytes + warp_row0 * 128;
        mbar_expect_tx_remote_relaxed(bar, 32 * 128);
        bulk_copy_to_cluster(mapa_shared(smem_u32(smem + C::kXsOff + off), rank ^ 1),
                             smem_u32(smem + C::kXoOff + off), 32 * 128, bar);
        bulk_commit();
      }
    }
    u = min(ue, se);
    ++s;
  }
}

// ---------------------------------------------------------------------------
// Softmax warpgroup
// ---------------------------------------------------------------------------
template <bool kSparse, bool kFp8>
DEVI void mla_softmax(const MlaParams& p, uint8_t* smem, MlaBarriers* bars, uint32_t tmem,
                      int rank) {
  using C = MlaCfg<kFp8>;
  volatile int* abort = &bars->abort;
  const int r = threadIdx.x;  // 0..127
  const uint32_t lane = (uint32_t)(r & ~31) << 16;
  const uint32_t o_tmem = tmem + kMlaTmemO + lane;
  const MetaLayout ml(p.num_ctas, p.num_segs);
  int ub, ue, s;
  const int32_t* prefix;
  mla_range<kSparse>(p, ub, ue, s, prefix);
  int it = 0;
  if (!p.meta && ue == 0) {
    // empty sequence without metadata: O = 0, LSE = -inf
    MlaSeg g;
    mla_seg<kSparse>(p, blockIdx.x >> 1, g);
    int tok, head;
    mla_row(p, g, r, tok, head);
    if (r < g.rows_valid && tok < p.seqlen_q) {
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) + g.b * p.o_sb +
                            (int64_t)tok * p.o_ss + (int64_t)head * p.o_sh + rank * kMlaDvHalf;
      for (int c = 0; c < kMlaDvHalf; c += 8)
        *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
      if (p.lse && rank == 0) p.lse[((int64_t)g.b * p.heads_q + head) * p.seqlen_q + tok] = -INFINITY;
    }
    return;
  }
  int u = ub;
  while (u < ue) {
    int sb, se;
    if (prefix) {
      sb = prefix[s];
      se = prefix[s + 1];
      if (se <= u) { ++s; continue; }
    } else {
      sb = u;
      se = ue;
    }
    MlaSeg g;
    mla_seg<kSparse>(p, s, g);
    const int a = u - sb, e = min(ue, se) - sb;
    const int n = max(0, e - a);
    int tok, head;
    mla_row(p, g, r, tok, head);
    const bool valid_row = r < g.rows_valid && tok < p.seqlen_q;
    // dense: visible keys [0, hi]; causal aligns the last token with the last key
    int hi = g.len - 1;
    if (p.causal) hi = min(hi, (tok - g.q0) + g.len - g.sq);
    // sparse: every row of the tile is token tok0, so key visibility is the
    // same for all rows; lane c of each warp evaluates key c of a tile and
    // the warp shares the result by ballot. The index is loaded one tile ahead.
    int hi0 = g.len - 1;
    if (kSparse && p.causal) hi0 = min(hi0, (g.tok0 - g.q0) + g.len - g.sq);
    const int lane_c = threadIdx.x & 31;
    int raw_next = -1;
    if (kSparse && n > 0) raw_next = mla_sparse_raw(p, g.b, g.kvg, g.tok0, a * kMlaBN + lane_c);
    // FP8: S and O use the dequantised rows (MATE FMHA dtype notes): the q and
    // k descales of (sequence, KV head) scale the scores, the v descale O.
    float sl2 = p.scale_log2, v_scale = 1.f;
    if (kFp8 && p.q_descale != nullptr) {
      const int di = g.bk * p.heads_kv + g.kvg;
      sl2 *= p.q_descale[di] * p.k_descale[di];
      v_scale = p.v_descale[di];
    }
    float m_run = -INFINITY, l_run = 0.f, l_rnd = 0.f;
    bool seen = false;
    uint32_t sv[kMlaBN];
    for (int j = 0; j < n; ++j) {
      const int gi = it + j;
      const int t = a + j;
      {
        // This CTA's partial scores of the tile, plus the other CTA's.
        const int b = gi % kMlaXsBufs, sbuf = gi % kMlaSBufs;
        if (!warp_wait(&bars->s_full[sbuf], (gi / kMlaSBufs) & 1, abort, 86)) return;
        tc_fence_after();
        tmem_load<32>(tmem + kMlaTmemS + sbuf * kMlaBN + lane, sv);
        if (!warp_wait_cluster(&bars->xs_full[b], (gi / kMlaXsBufs) & 1, abort, 83)) return;
        const uint8_t* src = smem + C::kXsOff + b * kMlaXsBytes + r * 128;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint4 v = *reinterpret_cast<const uint4*>(src + ((k ^ (r & 7)) << 4));
          sv[4 * k] = __float_as_uint(__uint_as_float(sv[4 * k]) + __uint_as_float(v.x));
          sv[4 * k + 1] = __float_as_uint(__uint_as_float(sv[4 * k + 1]) + __uint_as_float(v.y));
          sv[4 * k + 2] = __float_as_uint(__uint_as_float(sv[4 * k + 2]) + __uint_as_float(v.z));
          sv[4 * k + 3] = __float_as_uint(__uint_as_float(sv[4 * k + 3]) + __uint_as_float(v.w));
        }
        // This warp's rows of the buffer have been read: the other CTA may
        // send its next tile there.
        __syncwarp();
        if ((threadIdx.x & 31) == 0)
          mbar_arrive_remote_relaxed(mapa_shared(smem_u32(&bars->xs_empty[b]), rank ^ 1));
      }
      if constexpr (kSparse) {
        // Key position of entry e (see mla_sparse_pos); visible iff
        // 0 <= pos <= hi (hi = L - 1, or with sparse_mode=3, "rightDownCausal",
        // also tok + L - s_q).
        const int pos = mla_pos_of(p, raw_next, t * kMlaBN + lane_c);
        if (j + 1 < n) raw_next = mla_sparse_raw(p, g.b, g.kvg, g.tok0, (t + 1) * kMlaBN + lane_c);
        const uint32_t vis = __ballot_sync(0xffffffffu, pos >= 0 && pos <= hi0);
#pragma unroll
        for (int c = 0; c < kMlaBN; ++c)
          if (!valid_row || !((vis >> c) & 1u)) sv[c] = __float_as_uint(-INFINITY);
      } else {
        const int k0 = t * kMlaBN;
        if (k0 + kMlaBN - 1 > hi) {
#pragma unroll
          for (int c = 0; c < kMlaBN; ++c)
            if (k0 + c > hi) sv[c] = __float_as_uint(-INFINITY);
        }
        // Rows of the tile past the end of the cache hold whatever the page
        // has there: zero this V half of them so P = 0 never meets a NaN. S
        // of this tile has been computed already. (e4m3: the conversion warps
        // zero them in the fp16 copy.)
        const int nvalid = g.len - k0;
        if (!kFp8 && nvalid < kMlaBN) {
          uint8_t* kvs = smem + C::kKVOff + (gi % C::kStages) * C::kKVBytes;
          const int bad = kMlaBN - nvalid;
          for (int x = r; x < 4 * bad * 8; x += 128) {
            const int c = x / (bad * 8), rem = x % (bad * 8);
            const int row = nvalid + rem / 8, u16 = rem % 8;
            *reinterpret_cast<uint4*>(kvs + c * kMlaKVChunkBytes + row * 128 +
                                      u16 * 16) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kMlaBN; ++c) mx = fmaxf(mx, __uint_as_float(sv[c]));
      seen |= mx != -INFINITY;
      mx *= sl2;
      float alpha = 1.f;
      const bool grow = (j == 0) ? (mx > m_run) : (mx > m_run + kRescaleThreshold);
      if (grow) {
        if (j > 0 && m_run != -INFINITY) alpha = ex2(m_run - mx);
        m_run = mx;
        l_run *= alpha;
        l_rnd *= alpha;
      }
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        // O may be rescaled once P V of the previous tile (global index
        // gi - 1) has landed: phase (gi - 1) / 3 of o_full[(gi - 1) % 3]. Its
        // previous phase (P V gi - 4) is done, since S gi was issued after P V
        // gi - 3, and its next one needs P of tile gi + 2, not yet made.
        const int pv = gi - 1;
        if (!warp_wait(&bars->o_full[pv % kMlaSBufs], (pv / kMlaSBufs) & 1, abort, 81)) return;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < kMlaDvHalf; c += 32) {
          uint32_t o[32];
          tmem_load<32>(o_tmem + c, o);
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
          tmem_store<32>(o_tmem + c, o);
        }
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      uint32_t pk[kMlaBN / 2];
      float le = 0.f, lr = 0.f;
#pragma unroll
      for (int c = 0; c < kMlaBN / 2; ++c) {
        const float p0 = ex2(fmaf(__uint_as_float(sv[2 * c]), sl2, -m_use));
        const float p1 = ex2(fmaf(__uint_as_float(sv[2 * c + 1]), sl2, -m_use));
        le += p0 + p1;
        if constexpr (kFp8) {
          // fp16 P (to nearest even); O is normalised by the sum of the same
          // rounded values
          pk[c] = pack_f16x2(p0, p1);
          lr += sum2<true>(pk[c]);
        } else {
          // bf16 P rounded to nearest (ties away from zero; P >= 0); O is
          // normalised by the sum of the same rounded values
          const uint32_t r0 = __float_as_uint(p0) + 0x8000u, r1 = __float_as_uint(p1) + 0x8000u;
          pk[c] = __byte_perm(r0, r1, 0x7632);
          lr += __uint_as_float(r0 & 0xffff0000u) + __uint_as_float(r1 & 0xffff0000u);
        }
      }
      l_run += le;
      l_rnd += lr;
      // P replaces S in the buffer once the sender has loaded S from it
      if (!warp_wait(&bars->s_read[gi % kMlaSBufs], (gi / kMlaSBufs) & 1, abort, 87)) return;
      tc_fence_after();
      tmem_store<16>(tmem + kMlaTmemS + (gi % kMlaSBufs) * kMlaBN + lane, pk);
      tmem_store_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_full[gi & 1]);
    }
    it += n;

    // --- epilogue: O / l (or a sink-free partial for the combine step) -------
    int slot = -1;
    if (p.meta && n > 0) {
      const int ns = p.meta[ml.seg_nsplit + s];
      if (ns > 1) slot = p.meta[ml.seg_slot + s] + ((blockIdx.x >> 1) - p.meta[ml.seg_first + s]);
    }
    if (n > 0) {
      // the segment's last P V (global index it + n - 1; it now counts it);
      // its barrier's previous phase is done, as for the rescale
      const int pv = it - 1;
      if (!warp_wait(&bars->o_full[pv % kMlaSBufs], (pv / kMlaSBufs) & 1, abort, 82)) return;
      tc_fence_after();
    }
    if (!seen) l_run = l_rnd = 0.f;
    const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
    const float inv = (l_rnd > 0.f && seen) ? v_scale / l_rnd : 0.f;
    const float lse = (l_run > 0.f && seen) ? (m_use + log2f(l_run)) * kLn2 : -INFINITY;
    __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) + g.b * p.o_sb +
                          (int64_t)tok * p.o_ss + (int64_t)head * p.o_sh + rank * kMlaDvHalf;
    float* wrow =
        slot >= 0 ? p.ws_o + (((int64_t)slot * 2 + rank) * kMlaRows + r) * kMlaDvHalf : nullptr;
#pragma unroll 1
    for (int c = 0; c < kMlaDvHalf; c += 32) {
      uint32_t o[32];
      if (n > 0) {
        tmem_load<32>(o_tmem + c, o);
      } else {
#pragma unroll
        for (int x = 0; x < 32; ++x) o[x] = 0u;
      }
      if (valid_row) {
        if (slot < 0) {
#pragma unroll
          for (int x = 0; x < 32; x += 8) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[x + 0]) * inv, __uint_as_float(o[x + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(o[x + 2]) * inv, __uint_as_float(o[x + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(o[x + 4]) * inv, __uint_as_float(o[x + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(o[x + 6]) * inv, __uint_as_float(o[x + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + c + x) = v;
          }
        } else {
#pragma unroll
          for (int x = 0; x < 32; x += 4)
            *reinterpret_cast<float4*>(wrow + c + x) =
                make_float4(__uint_as_float(o[x]) * inv, __uint_as_float(o[x + 1]) * inv,
                            __uint_as_float(o[x + 2]) * inv, __uint_as_float(o[x + 3]) * inv);
        }
      }
    }
    if (n > 0) {
      tc_fence_before();
      mbar_arrive(&bars->o_empty);
    }
    if (valid_row) {
      if (slot >= 0) {
        if (rank == 0) p.ws_lse[(int64_t)slot * kMlaRows + r] = lse;
      } else if (p.lse && rank == 0)
        p.lse[((int64_t)g.b * p.heads_q + head) * p.seqlen_q + tok] = lse;
    }
    u = min(ue, se);
    ++s;
  }
}

template <bool kSparse, bool kFp8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(MlaCfg<kFp8>::kThreads, 1)
    mla_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_kv,
               const MlaParams p) {
  using C = MlaCfg<kFp8>;
  // 128-byte swizzled TMA tiles need 1024-byte aligned shared memory; both
  // CTAs of the cluster share the layout, so both leave here or neither.
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) raise_error(ATTN_DEVERR_SMEM_ALIGN, 2);
    return;
  }
  MlaBarriers* bars = reinterpret_cast<MlaBarriers*>(smem + C::kBarOff);
  const int warp = threadIdx.x >> 5;
  const int rank = (int)cluster_ctarank();
  if (threadIdx.x == 0) {
    for (int i = 0; i < kMlaQStages; ++i) {
      mbar_init(&bars->qs_full[i], 1);
      mbar_init(&bars->qs_empty[i], 1);
    }
    mbar_init(&bars->q_done, 1);
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&bars->kv_full[i], kSparse ? 32 : 1);
      // e4m3: released by the S MMA's commit and the 64 conversion threads
      mbar_init(&bars->kv_empty[i], kFp8 ? 1 + 64 : 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->vh_full[i], 64);
      mbar_init(&bars->vh_empty[i], 1);
    }
    for (int i = 0; i < kMlaSBufs; ++i) mbar_init(&bars->s_full[i], 1);
    for (int i = 0; i < kMlaXsBufs; ++i) {
      mbar_init(&bars->xs_full[i], 4);   // one bulk copy from each sender warp of the other CTA
      mbar_init(&bars->xs_empty[i], 4);  // each softmax warp of the other CTA has read
    }
    for (int i = 0; i < kMlaSBufs; ++i) mbar_init(&bars->s_read[i], 4);  // each sender warp
    for (int i = 0; i < 2; ++i) mbar_init(&bars->p_full[i], 128);
    for (int i = 0; i < kMlaSBufs; ++i) mbar_init(&bars->o_full[i], 1);
    mbar_init(&bars->o_empty, 128);
    mbar_init(&bars->mma_drain, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  __shared__ int s_bad;
  if (threadIdx.x == 0) {
    s_bad = 0;
    if (p.meta) {
      const int mode = kSparse ? ATTN_SCHED_MLA_SPARSE : ATTN_SCHED_MLA;
      if (!(meta_matches(p.meta, mode, p.batch, p.seqlen_q, p.heads_q, p.heads_kv, p.page_size,
                         p.num_segs, kMlaBN, kMlaDqk, kMlaDv) &&
            p.meta[kMetaNumCtas] == p.num_ctas &&
            (!kSparse || p.meta[kMetaTopk] == p.topk * p.sbs))) {
        raise_error(ATTN_DEVERR_META_MISMATCH, 90);
        s_bad = 1;
      }
    }
  }
  if (warp == 5) {
    tmem_alloc(&bars->tmem_base, kMlaTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // The other CTA's barriers are initialised before any remote arrival.
  cluster_sync();
  const uint32_t tmem = bars->tmem_base;
  if (!s_bad) {
    if (warp < 4)
      mla_softmax<kSparse, kFp8>(p, smem, bars, tmem, rank);
    else if (warp == 4)
      mla_producer<kSparse, kFp8>(p, &map_q, &map_kv, smem, bars, rank);
    else if (warp == 5)
      mla_mma<kSparse, kFp8>(p, smem, bars, tmem, rank);
    else if (warp >= C::kSendWarp0)
      mla_sender<kSparse, kFp8>(p, smem, bars, tmem, rank, warp & 3);
    else if constexpr (kFp8)
      mla_convert<kSparse>(p, smem, bars);
  }
  // The partial-score copies this CTA sent have landed in the other CTA.
  if (warp >= C::kSendWarp0 && (threadIdx.x & 31) == 0) bulk_wait_all();
  tc_fence_before();
  __syncthreads();
  // No remote arrival or store into this CTA's shared memory after this.
  cluster_sync();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kMlaTmemCols);
  }
}

// Merges split MLA segments: one warp per (segment, V half, row); each half
// covers 256 of the 512 output columns; half 0 writes the LSE.
template <bool kSparse>
__global__ void __launch_bounds__(256) mla_combine_kernel(const MlaParams p) {
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int s = gw / (2 * kMlaRows);
  const int vh = (gw / kMlaRows) & 1, r = gw % kMlaRows;
  if (s >= p.num_segs) return;
  const int mode = kSparse ? ATTN_SCHED_MLA_SPARSE : ATTN_SCHED_MLA;
  if (!(meta_matches(p.meta, mode, p.batch, p.seqlen_q, p.heads_q, p.heads_kv, p.page_size,
                     p.num_segs, kMlaBN, kMlaDqk, kMlaDv) &&
        p.meta[kMetaNumCtas] == p.num_ctas))
    return;
  const MetaLayout ml(p.num_ctas, p.num_segs);
  const int ns = p.meta[ml.seg_nsplit + s];
  if (ns == 1) return;
  MlaSeg g;
  mla_seg<kSparse>(p, s, g);
  int tok, head;
  mla_row(p, g, r, tok, head);
  if (r >= g.rows_valid || tok >= p.seqlen_q) return;
  const int slot0 = ns > 1 ? p.meta[ml.seg_slot + s] : 0;
  __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + g.b * p.o_sb +
                       (int64_t)tok * p.o_ss + (int64_t)head * p.o_sh + vh * kMlaDvHalf;
  const float lse = combine_row(
      ns, kMlaDvHalf, 0.f, false,
      [&](int k) { return p.ws_lse[(int64_t)(slot0 + k) * kMlaRows + r]; },
      [&](int k) { return p.ws_o + (((int64_t)(slot0 + k) * 2 + vh) * kMlaRows + r) * kMlaDvHalf; },
      [&](int c, float v) { store_out(dst + c, v); });
  if (p.lse && vh == 0 && (threadIdx.x & 31) == 0)
    p.lse[((int64_t)g.b * p.heads_q + head) * p.seqlen_q + tok] = lse;
}

}  // namespace attn
