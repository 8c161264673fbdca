// Scheduler metadata: a balanced split of the decode work over persistent
// CTAs (MATE "Attention": get_scheduler_metadata / get_mla_metadata precompute
// the scheduler input of the main call; CANN "flash_attn": the metadata
// interface runs first and its result is passed to the main operator).
//
// Work model: the decode problem is a list of segments (a sequence and a
// group of query rows that share one KV stream: (b, kv head, row block) for
// GQA decode, (b, row tile, V half) for MLA), each a run of `units` KV tiles.
// The units of all segments are laid end to end and cut into num_ctas equal
// ranges (fewer if there are fewer units than CTAs; the idle CTAs come last);
// CTA c processes units [cta_begin[c], cta_begin[c+1]). A segment
// touched by n >= 2 CTAs is split n ways; its partial (O, LSE) go to slots
// seg_slot[s] .. seg_slot[s] + n - 1 of the workspace and are merged by the
// combine kernel. Segments with n = 1 are written directly by their CTA.
#pragma once

#include "common.cuh"

namespace attn {

// Header of the metadata buffer (int32 words).
enum MetaHeader {
  kMetaMagic = 0,
  kMetaMode,
  kMetaBatch,
  kMetaSeqlenQ,
  kMetaHeadsQ,
  kMetaHeadsKV,
  kMetaPageSize,
  kMetaNumCtas,
  kMetaNumSegs,
  kMetaUnitKeys,
  kMetaTopk,
  kMetaDimQK,
  kMetaDimV,
  kMetaTotalSlots,  // written by the device
  kMetaSegsPerSeq,
  kMetaNewKeys,  // keys appended after each sequence's cache (GQA decode)
  kMetaHeaderWords = 16
};
constexpr int32_t kMetaMagicValue = 0x4154544d;  // "MTTA"

// Offsets (int32 words) of the tables that follow the header.
struct MetaLayout {
  int64_t cta_begin, cta_seg, seg_begin, seg_first, seg_nsplit, seg_slot, words;
  __host__ __device__ MetaLayout(int G, int S) {
    cta_begin = kMetaHeaderWords;        // G + 1 entries
    cta_seg = cta_begin + G + 1;         // G
    seg_begin = cta_seg + G;             // S + 1 (prefix sums of units)
    seg_first = seg_begin + S + 1;       // S   first CTA touching the segment
    seg_nsplit = seg_first + S;          // S   CTAs touching the segment
    seg_slot = seg_nsplit + S;           // S   first workspace slot (nsplit >= 2)
    words = seg_slot + S;
  }
};

// How a mode maps sequences to segments and KV lengths to units.
struct SchedShape {
  int32_t segs_per_seq;  // segments per sequence
  int32_t unit_keys;     // keys per unit (dense modes)
  int32_t mode;
  int32_t topk;
  int32_t new_keys;      // GQA decode: keys appended after the cache (own tiles)
};

// Units (KV tiles) of one segment of a sequence with `len` cached keys. The
// appended keys of GQA decode start a tile of their own after the cache's
// last (partial) tile.
DEVI int32_t sched_units(const SchedShape& sh, int32_t len) {
  if (sh.mode == ATTN_SCHED_MLA_SPARSE) return (sh.topk + sh.unit_keys - 1) / sh.unit_keys;
  const int32_t cached = len > 0 ? (len - 1) / sh.unit_keys + 1 : 0;  // no overflow at 2^31 - 1
  return cached + (sh.new_keys + sh.unit_keys - 1) / sh.unit_keys;
}

struct SchedParams {
  const int32_t* cache_seqlens;
  int32_t* meta;
  SchedShape sh;
  int32_t batch, seqlen_q, heads_q, heads_kv, page_size, G, S, dim_qk, dim_v;
};

// Block-wide exclusive scan of `n` values in place (one CTA, blockDim 1024).
DEVI void block_exclusive_scan(int32_t* data, int64_t n, int32_t* sh_warp, int32_t& total) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  int32_t carry = 0;
  for (int64_t base = 0; base < n; base += blockDim.x) {
    const int64_t i = base + tid;
    const int32_t v = i < n ? data[i] : 0;
    int32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) sh_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int32_t w = lane < nw ? sh_warp[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      if (lane < nw) sh_warp[lane] = w;  // inclusive warp totals
    }
    __syncthreads();
    const int32_t before = (warp > 0 ? sh_warp[warp - 1] : 0) + carry;
    if (i < n) data[i] = before + x - v;
    const int32_t chunk_total = sh_warp[nw - 1];
    __syncthreads();
    carry += chunk_total;
  }
  total = carry;
}

__global__ void __launch_bounds__(1024, 1) sched_kernel(const SchedParams p) {
  __shared__ int32_t sh_warp[32];
  const MetaLayout ml(p.G, p.S);
  int32_t* cta_begin = p.meta + ml.cta_begin;
  int32_t* cta_seg = p.meta + ml.cta_seg;
  int32_t* seg_begin = p.meta + ml.seg_begin;
  int32_t* seg_first = p.meta + ml.seg_first;
  int32_t* seg_nsplit = p.meta + ml.seg_nsplit;
  int32_t* seg_slot = p.meta + ml.seg_slot;
  const int tid = threadIdx.x;

  // 1. units per segment, then their exclusive prefix sums. The sums are
  //    int32: a problem with more units than that is refused (an invalid
  //    header, which the main kernels reject, and a device error).
  __shared__ unsigned long long sh_units;
  if (tid == 0) sh_units = 0;
  __syncthreads();
  unsigned long long mine = 0;
  for (int s = tid; s < p.S; s += blockDim.x) {
    const int b = s / p.sh.segs_per_seq;
    const int32_t n = sched_units(p.sh, p.cache_seqlens[b]);
    seg_begin[s] = n;
    mine += (unsigned long long)max(n, 0);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, o);
  if ((tid & 31) == 0) atomicAdd(&sh_units, mine);
  __syncthreads();
  if (sh_units > (unsigned long long)INT32_MAX) {
    if (tid == 0) {
      p.meta[kMetaMagic] = 0;
      raise_error(ATTN_DEVERR_UNITS_OVERFLOW, 50);
    }
    return;
  }
  int32_t total;
  block_exclusive_scan(seg_begin, p.S, sh_warp, total);
  if (tid == 0) seg_begin[p.S] = total;
  __syncthreads();

  // 2. equal unit ranges per CTA. With fewer units than CTAs only the first
  //    `total` CTAs get work, so every CTA that touches a segment is non-empty
  //    and consecutive (the split index of CTA c is c - first CTA).
  const int ge = min(p.G, total);
  for (int c = tid; c <= p.G; c += blockDim.x)
    cta_begin[c] = c >= ge ? total : (int32_t)(((int64_t)total * c) / ge);
  __syncthreads();

  // CTA whose range holds unit u (the last c with cta_begin[c] <= u).
  auto cta_of = [&](int32_t u) {
    int lo = 0, hi = p.G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (cta_begin[mid] <= u) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  // 3. per segment: the CTAs that touch it
  for (int s = tid; s < p.S; s += blockDim.x) {
    const int32_t a = seg_begin[s], e = seg_begin[s + 1];
    if (e > a) {
      const int first = cta_of(a), last = cta_of(e - 1);
      seg_first[s] = first;
      seg_nsplit[s] = last - first + 1;
      seg_slot[s] = last > first ? last - first + 1 : 0;  // scanned below
    } else {
      seg_first[s] = -1;
      seg_nsplit[s] = 0;
      seg_slot[s] = 0;
    }
  }
  __syncthreads();
  int32_t slots;
  block_exclusive_scan(seg_slot, p.S, sh_warp, slots);
  __syncthreads();
  // 4. the first segment of each CTA range (the one containing its first unit)
  for (int c = tid; c < p.G; c += blockDim.x) {
    const int32_t u = cta_begin[c];
    int lo = 0, hi = p.S - 1;  // last s with seg_begin[s] <= u
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (seg_begin[mid] <= u) lo = mid; else hi = mid - 1;
    }
    cta_seg[c] = lo;
  }
  if (tid == 0) {
    int32_t* h = p.meta;
    h[kMetaMagic] = kMetaMagicValue;
    h[kMetaMode] = p.sh.mode;
    h[kMetaBatch] = p.batch;
    h[kMetaSeqlenQ] = p.seqlen_q;
    h[kMetaHeadsQ] = p.heads_q;
    h[kMetaHeadsKV] = p.heads_kv;
    h[kMetaPageSize] = p.page_size;
    h[kMetaNumCtas] = p.G;
    h[kMetaNumSegs] = p.S;
    h[kMetaUnitKeys] = p.sh.unit_keys;
    h[kMetaTopk] = p.sh.topk;
    h[kMetaDimQK] = p.dim_qk;
    h[kMetaDimV] = p.dim_v;
    h[kMetaTotalSlots] = slots;
    h[kMetaSegsPerSeq] = p.sh.segs_per_seq;
    h[kMetaNewKeys] = p.sh.new_keys;
  }
}

// Checks a metadata header against the main call's own view of the problem.
DEVI bool meta_matches(const int32_t* meta, int32_t mode, int32_t batch, int32_t seqlen_q,
                       int32_t heads_q, int32_t heads_kv, int32_t page_size, int32_t num_segs,
                       int32_t unit_keys, int32_t dim_qk, int32_t dim_v) {
  return meta[kMetaMagic] == kMetaMagicValue && meta[kMetaMode] == mode &&
         meta[kMetaBatch] == batch && meta[kMetaSeqlenQ] == seqlen_q &&
         meta[kMetaHeadsQ] == heads_q && meta[kMetaHeadsKV] == heads_kv &&
         meta[kMetaPageSize] == page_size && meta[kMetaNumSegs] == num_segs &&
         meta[kMetaUnitKeys] == unit_keys && meta[kMetaDimQK] == dim_qk &&
         meta[kMetaDimV] == dim_v;
}

}  // namespace attn
