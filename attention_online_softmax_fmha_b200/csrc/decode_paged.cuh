// Decode against a paged KV cache, split over persistent CTAs (MATE
// "Attention", FMHA: flash_attn_with_kvcache with scheduler metadata and
// flash_attn_combine; MindSpore "sparse_flash_attention": PA_BSND cache of
// (block_num, block_size, N, D) with a block table).
//
// One segment = (sequence b, KV head g, block of <= 16 query rows that read
// g: (query token, head) pairs). Its KV stream is cut into 64-key tiles;
// logical key t lives in row t % page_size of physical page
// block_table[b][t / page_size].
//
// The work is HBM-bound (about 4 flop per KV byte at s_q = 1, H_q/H_kv = 4),
// so the design goal is a full memory pipe, not tensor throughput:
//   warp 4      producer: reads the block-table entries 32 at a time and
//               issues one TMA box per (page, 64-column chunk) for K and V,
//               128-byte swizzled, into a 6-stage ring (32 KB per stage).
//   warps 0-7   consumers, two warpgroups taking alternate tiles (warpgroup
//               it % 2 takes the CTA's it-th tile, so each stage of the even
//               ring always goes to the same warpgroup). Warp w of a
//               warpgroup owns keys [16w, 16w + 16) of its tiles and keeps its
//               own online-softmax state (running max, sums, O in registers).
//               S = Q K^T and O += P V use mma.sync m16n8k16 with fp32
//               accumulation. Two consumer warps per SM sub-partition hide
//               each other's per-tile latency chain (wait, ldmatrix, MMA,
//               shuffles, exp2). At the end of a segment piece the eight warp
//               states are merged through shared memory in a fixed order, so
//               repeated runs agree bit for bit.
// FP8 caches (e4m3 / e5m2, D = 128) arrive as 128-byte rows. S = Q K^T runs
// on the FP8 codes directly (mma.sync m16n8k32, Q kept in FP8); each warp
// rewrites its 16 V rows as fp16 (exact for both formats) in a private
// tile, and O += P V runs in fp16 from there. The q/k descales fold into the
// score scale and the v descale into the output scale.
// A piece that is the whole segment writes O (bf16) and LSE directly; a piece
// of a split segment writes a sink-free partial (O / l, LSE) to the workspace
// for the combine kernel.
// Appended keys (Mojo "flash_attention_split_kv": the current k and v are read
// in place after the cached ones, as one sequence) come from their own
// (B, s_new, H_kv, D) tensors through a second pair of tensor maps. They
// start a tile of their own after the cache's last tile, so no tile mixes the
// two sources; rows past s_new read as zeros.
#pragma once

#include "common.cuh"
#include "sched.cuh"

namespace attn {

constexpr int kDecTileKeys = 64;
constexpr int kDecRows = 16;       // query rows per segment (mma M)
constexpr int kDecConsumerWarps = 8;  // two warpgroups
constexpr int kDecConsumerThreads = 32 * kDecConsumerWarps;
constexpr int kDecThreads = kDecConsumerThreads + 32;  // + the producer warp

struct DecodeParams {
  const void* q;
  void* out;
  float* lse;
  const int32_t* block_table;
  const int32_t* cache_seqlens;
  const int32_t* meta;       // nullptr: one CTA per segment, no split
  float* ws_o;               // [slot][kDecRows][D]
  float* ws_lse;             // [slot][kDecRows]
  const float* sink;
  const float* q_descale;    // FP8: (B, H_kv) fp32, else unused
  const float* k_descale;
  const float* v_descale;
  int64_t bt_stride;
  int64_t q_sb, q_ss, q_sh;
  int64_t o_sb, o_ss, o_sh;
  int32_t batch, seqlen_q, heads_q, heads_kv, group, rows, n_rsub, segs_per_seq, num_segs;
  int32_t page_size;
  int32_t num_ctas;          // grid size with metadata
  float scale_log2;
  int32_t causal, window_left, window_right;
  int32_t seqlen_new;        // appended keys per sequence (0: none)
};

template <int D, bool kFp8>
struct DecodeCfg {
  static_assert(!kFp8 || D == 128, "FP8 caches: D = 128 (one 128-byte chunk per row)");
  static constexpr int kElt = kFp8 ? 1 : 2;                    // bytes per cached element
  static constexpr int kChunkCols = 128 / kElt;                // columns per 128-byte chunk
  static constexpr int kChunks = D / kChunkCols;
  static constexpr int kTileBytes = kDecTileKeys * D * kElt;  // K or V tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  // Stages in flight: about 190 KB of K/V per SM either way, enough bytes in
  // flight to cover the memory latency at the SM's share of HBM bandwidth.
  // Even: stage st always feeds warpgroup st % 2.
  static constexpr int kStages = kFp8 ? 10 : 6;
  static_assert(kStages % 2 == 0, "alternate tiles keep a stage with one warpgroup");
  static constexpr int kQStride = D * 2 + 16;                  // padded 16-bit Q row (bytes)
  static constexpr int kStageOff = 0;
  static constexpr int kQOff = kStages * kStageBytes;
  // FP8: each consumer warp's fp16 copy of its 16 V rows
  static constexpr int kStgWarpBytes = kFp8 ? 16 * D * 2 : 0;
  static constexpr int kStgOff = kQOff + kDecRows * kQStride;
  static constexpr int kRedOff = kStgOff + kDecConsumerWarps * kStgWarpBytes;  // merge buffers
  // two O buffers (one per warpgroup), then m, l and the rounded l per warp
  static constexpr int kRedBytes = 2 * kDecRows * D * 4 + kDecConsumerWarps * kDecRows * 4 * 3;
  static constexpr int kBarOff = kRedOff + kRedBytes;
  static constexpr int kSmemBytes = kBarOff + 2 * kStages * 8 + 64 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

struct DecodeSeg {
  int b, g, rsub;
  int len;     // cached keys
  int ltot;    // cached + appended keys
  int nct;     // tiles of the cache; appended keys start at tile nct
  int t0, t1;  // visible cache tiles [t0, t1)
  int tn0, tn1;  // visible appended tiles [tn0, tn1)
  DEVI bool visible(int t) const { return (t >= t0 && t < t1) || (t >= tn0 && t < tn1); }
  // position in the sequence of row 0 of tile t, and the end of the valid
  // positions of that tile's source
  DEVI int pos0(int t) const { return t < nct ? t * kDecTileKeys : len + (t - nct) * kDecTileKeys; }
  DEVI int pend(int t) const { return t < nct ? len : ltot; }
};

DEVI void decode_seg(const DecodeParams& p, int s, DecodeSeg& sg) {
  sg.b = s / p.segs_per_seq;
  const int rem = s - sg.b * p.segs_per_seq;
  sg.g = rem / p.n_rsub;
  sg.rsub = rem - sg.g * p.n_rsub;
  sg.len = p.cache_seqlens[sg.b];
  sg.ltot = sg.len + p.seqlen_new;
  sg.nct = sg.len > 0 ? (sg.len + kDecTileKeys - 1) / kDecTileKeys : 0;
  // union of the rows' visible ranges (row i = 0 has the smallest left edge,
  // i = s_q - 1 the largest right edge)
  const int delta = sg.ltot - p.seqlen_q;
  int lo = 0, hi = sg.ltot - 1;
  if (p.window_left >= 0) lo = max(lo, delta - p.window_left);
  if (p.causal) hi = min(hi, p.seqlen_q - 1 + delta);
  if (p.window_right >= 0) hi = min(hi, p.seqlen_q - 1 + delta + p.window_right);
  const int chi = min(hi, sg.len - 1);  // cached part
  if (chi < lo) {
    sg.t0 = sg.t1 = 0;
  } else {
    sg.t0 = lo / kDecTileKeys;
    sg.t1 = chi / kDecTileKeys + 1;
  }
  const int nlo = max(lo, sg.len);      // appended part
  if (hi < nlo) {
    sg.tn0 = sg.tn1 = 0;
  } else {
    sg.tn0 = sg.nct + (nlo - sg.len) / kDecTileKeys;
    sg.tn1 = sg.nct + (hi - sg.len) / kDecTileKeys + 1;
  }
}

// ---- mma.sync / ldmatrix helpers -------------------------------------------
DEVI void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
DEVI void ldsm_x4_t(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
template <bool kFp16>
DEVI void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  if (kFp16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}
// FP8 x FP8 -> fp32, m16n8k32 (kType 3 = e5m2, otherwise e4m3).
template <int kType>
DEVI void mma16832_fp8(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  if constexpr (kType == 3) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e5m2.e5m2.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}
DEVI void named_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Address of the 16-byte chunk holding (row, col..col+7) of a 128-byte-
// swizzled tile made of 64-column chunks of `rows` rows each.
DEVI uint32_t sw128_addr(uint32_t base, int rows, int row, int col) {
  const int chunk = col >> 6;
  const int c16 = (col & 63) >> 3;
  return base + chunk * rows * 128 + row * 128 + ((c16 ^ (row & 7)) << 4);
}

// Sixteen FP8 values (one 16-byte unit of a cached row) as fp16 into columns
// col .. col + 15 of `row` of a 128-byte-swizzled fp16 tile of 16 rows.
template <int kType>
DEVI void fp8x16_to_f16_tile(uint32_t tile, int row, int col, uint4 w) {
  const uint32_t in[4] = {w.x, w.y, w.z, w.w};
  uint32_t h[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const unsigned short lo = (unsigned short)(in[i] & 0xffffu);
    const unsigned short hi = (unsigned short)(in[i] >> 16);
    if constexpr (kType == 3) {
      asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h[2 * i]) : "h"(lo));
      asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h[2 * i + 1]) : "h"(hi));
    } else {
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h[2 * i]) : "h"(lo));
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h[2 * i + 1]) : "h"(hi));
    }
  }
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(sw128_addr(tile, 16, row, col)),
               "r"(h[0]), "r"(h[1]), "r"(h[2]), "r"(h[3]) : "memory");
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(sw128_addr(tile, 16, row, col + 8)),
               "r"(h[4]), "r"(h[5]), "r"(h[6]), "r"(h[7]) : "memory");
}

// ---------------------------------------------------------------------------
template <int D, bool kFp8>
DEVI void decode_producer(const DecodeParams& p, const CUtensorMap* mk, const CUtensorMap* mv,
                          const CUtensorMap* mkn, const CUtensorMap* mvn, uint8_t* smem,
                          uint64_t* full, uint64_t* empty, volatile int* abort,
                          int seg_begin_units, int seg_end_units, int first_seg,
                          const int32_t* seg_prefix) {
  using C = DecodeCfg<D, kFp8>;
  const int lane = threadIdx.x & 31;
  if (lane == 0) {
    tma_prefetch_desc(mk);
    tma_prefetch_desc(mv);
    if (p.seqlen_new > 0) {
      tma_prefetch_desc(mkn);
      tma_prefetch_desc(mvn);
    }
  }
  int it = 0;
  const int P = p.page_size;
  const int loads_per_tile = P >= kDecTileKeys ? 1 : kDecTileKeys / P;
  const int box_rows = P >= kDecTileKeys ? kDecTileKeys : P;
  int u = seg_begin_units, s = first_seg;
  bool stop = false;
  while (u < seg_end_units && !stop) {
    // segment s covers units [seg_prefix(s), seg_prefix(s+1)) (or all of
    // one segment without metadata)
    int sb, se;
    if (seg_prefix) {
      sb = seg_prefix[s];
      se = seg_prefix[s + 1];
      if (se <= u) { ++s; continue; }
    } else {
      sb = u;
      se = seg_end_units;
    }
    DecodeSeg sg;
    decode_seg(p, s, sg);
    const int a = u - sb, e = min(seg_end_units, se) - sb;  // tiles [a, e) of this segment
    const int32_t* bt = p.block_table + (int64_t)sg.b * p.bt_stride;
    const int npages_seq = (sg.len + P - 1) / P;
    // A window of 32 block-table entries lives in the lanes' registers
    // (lane x holds entry win0 + x) and is refilled when a tile leaves it.
    int win0 = -(1 << 30), win_val = 0;
    for (int t = a; t < e; ++t) {
      if (!sg.visible(t)) continue;  // no visible key: skipped by all roles
      const int st = it % C::kStages;
      if (it >= C::kStages) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(&empty[st], ((it / C::kStages) - 1) & 1, abort, 31);
        if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
          stop = true;  // abort: stop issuing, but still drain what is in flight
          break;
        }
      }
      if (t >= sg.nct) {
        // appended keys: one 64-row box of the new k / v per 128-byte chunk
        // (rows past s_new are outside the tensor and read as zeros)
        if (lane == 0) {
          mbar_expect_tx(&full[st], 2u * kDecTileKeys * D * C::kElt);
          uint8_t* kdst = smem + C::kStageOff + st * C::kStageBytes;
          uint8_t* vdst = kdst + C::kTileBytes;
          const int row = (t - sg.nct) * kDecTileKeys;
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c) {
            tma_load_4d(kdst + c * kDecTileKeys * 128, mkn, &full[st], c * C::kChunkCols, sg.g,
                        row, sg.b);
            tma_load_4d(vdst + c * kDecTileKeys * 128, mvn, &full[st], c * C::kChunkCols, sg.g,
                        row, sg.b);
          }
        }
        __syncwarp();
        ++it;
        continue;
      }
      const int first_page = (t * kDecTileKeys) / P;
      const int nload = min(loads_per_tile, npages_seq - first_page);
      if (first_page < win0 || first_page + nload > win0 + 32) {
        win0 = first_page;
        win_val = (win0 + lane < npages_seq) ? bt[win0 + lane] : 0;
      }
      const int row_in_page = (t * kDecTileKeys) % P;  // 0 unless P > 64
      if (lane == 0)
        mbar_expect_tx(&full[st], 2u * nload * box_rows * D * C::kElt);
      __syncwarp();
      uint8_t* kdst = smem + C::kStageOff + st * C::kStageBytes;
      uint8_t* vdst = kdst + C::kTileBytes;
      for (int j = 0; j < nload; ++j) {
        const int page = __shfl_sync(0xffffffffu, win_val, first_page + j - win0);
        if (lane == 0) {
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c) {
            tma_load_4d(kdst + c * kDecTileKeys * 128 + j * box_rows * 128, mk, &full[st],
                        c * C::kChunkCols, sg.g, row_in_page, page);
            tma_load_4d(vdst + c * kDecTileKeys * 128 + j * box_rows * 128, mv, &full[st],
                        c * C::kChunkCols, sg.g, row_in_page, page);
          }
        }
      }
      ++it;
    }
    u = min(seg_end_units, se);
    ++s;
  }
  // drain (also after an abort): the last stages' copies must land before
  // the CTA exits
  if (lane == 0) {
    int zero = 0;
    for (int i = max(0, it - C::kStages); i < it; ++i)
      mbar_wait(&full[i % C::kStages], (i / C::kStages) & 1, &zero, 32);
  }
}

// ---------------------------------------------------------------------------
// kType: 0 bf16, 1 fp16, 2 e4m3, 3 e5m2.
template <int D, int kType>
DEVI void decode_consumer(const DecodeParams& p, uint8_t* smem, uint64_t* full, uint64_t* empty,
                          volatile int* abort, int seg_begin_units, int seg_end_units,
                          int first_seg, const int32_t* seg_prefix) {
  constexpr bool kFp8 = kType >= 2;
  constexpr bool kFp16 = kType != 0;      // MMA operand type: fp16 unless bf16
  constexpr bool kOutF16 = kType == 1;    // output: fp16 for fp16 input, else bf16
  using C = DecodeCfg<D, kFp8>;
  using InT = typename std::conditional<kOutF16, __half, __nv_bfloat16>::type;
  const int tid = threadIdx.x;  // 0 .. kDecConsumerThreads - 1
  const int gw = tid >> 5, lane = tid & 31;  // consumer warp 0..7
  const int wg = gw >> 2, warp = gw & 3;     // warpgroup; key slice of its tiles
  const int qr = lane >> 2;          // fragment row (and row + 8)
  const int qc = (lane & 3) * 2;     // fragment column pair
  uint8_t* qs = smem + C::kQOff;
  float* red_o = reinterpret_cast<float*>(smem + C::kRedOff);  // [2 warpgroups][16][D]
  float* red_m = red_o + 2 * kDecRows * D;                      // [8 warps][16]
  float* red_l = red_m + kDecConsumerWarps * kDecRows;
  float* red_r = red_l + kDecConsumerWarps * kDecRows;
  // After a failed wait (timeout or abort) a warp skips the rest of its tiles
  // but still takes every named barrier, so no other consumer warp is left
  // waiting at one.
  bool dead = false;
  const int32_t* meta = p.meta;
  const MetaLayout ml(p.num_ctas, p.num_segs);
  int it = 0;
  int u = seg_begin_units, s = first_seg;
  while (u < seg_end_units) {
    int sb, se;
    if (seg_prefix) {
      sb = seg_prefix[s];
      se = seg_prefix[s + 1];
      if (se <= u) { ++s; continue; }
    } else {
      sb = u;
      se = seg_end_units;
    }
    DecodeSeg sg;
    decode_seg(p, s, sg);
    const int a = u - sb, e = min(seg_end_units, se) - sb;
    const int row0 = sg.rsub * kDecRows;
    const int nrows = min(kDecRows, p.rows - row0);

    // --- Q rows of the segment -> shared memory (16-bit, or the FP8 codes
    //     as they are; zero padded) ---
    named_barrier(1, kDecConsumerThreads);  // previous piece finished with qs / red
    constexpr int kQUnit = kFp8 ? 16 : 8;  // elements per 16-byte unit
    for (int x = tid; x < kDecRows * (D / kQUnit); x += kDecConsumerThreads) {
      const int r = x / (D / kQUnit), cu = x % (D / kQUnit);
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < nrows) {
        const int rr = row0 + r;
        const int i = rr / p.group, h = sg.g * p.group + rr % p.group;
        const int64_t off = sg.b * p.q_sb + i * p.q_ss + h * p.q_sh + cu * kQUnit;
        if constexpr (kFp8)
          v = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(p.q) + off);
        else
          v = *reinterpret_cast<const uint4*>(reinterpret_cast<const InT*>(p.q) + off);
      }
      *reinterpret_cast<uint4*>(qs + r * C::kQStride + cu * 16) = v;
    }
    named_barrier(1, kDecConsumerThreads);
    // A fragments of Q: one per 32-byte k-step (16 bf16/fp16 values, or 32
    // FP8 codes read through the same 16-bit ldmatrix view)
    constexpr int kKSteps = D * C::kElt / 32;
    uint32_t qa[kKSteps][4];
    {
      const int r = (lane & 7) + ((lane >> 3) & 1) * 8;
      const int cofs = (lane >> 4) * 8;
#pragma unroll
      for (int k = 0; k < kKSteps; ++k)
        ldsm_x4(smem_u32(qs + r * C::kQStride + (k * 16 + cofs) * 2), qa[k]);
    }
    // per-row visible key range (rows qr and qr + 8)
    int lo[2], hi[2];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int rr = row0 + qr + h2 * 8;
      const int i = min(rr, p.rows - 1) / p.group;
      const int delta = sg.ltot - p.seqlen_q;
      lo[h2] = 0;
      hi[h2] = sg.ltot - 1;
      if (p.window_left >= 0) lo[h2] = max(lo[h2], i + delta - p.window_left);
      if (p.causal) hi[h2] = min(hi[h2], i + delta);
      if (p.window_right >= 0) hi[h2] = min(hi[h2], i + delta + p.window_right);
    }
    float o[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f}, l_rnd[2] = {0.f, 0.f};
    float sl2 = p.scale_log2, vscale = 1.f;
    if constexpr (kFp8) {
      const int di = sg.b * p.heads_kv + sg.g;
      sl2 *= p.q_descale[di] * p.k_descale[di];
      vscale = p.v_descale[di];
    }
    // FP8: this warp's fp16 V tile (16 keys)
    const uint32_t vstg = smem_u32(smem + C::kStgOff + gw * C::kStgWarpBytes);

    for (int t = a; t < e; ++t) {
      if (!sg.visible(t)) continue;
      const int st = it % C::kStages;
      if ((it & 1) != wg || dead) {  // the other warpgroup's tile, or given up
        ++it;
        continue;
      }
      if (!warp_wait(&full[st], (it / C::kStages) & 1, abort, 33)) {
        dead = true;
        ++it;
        continue;
      }
      const uint32_t kbase = smem_u32(smem + C::kStageOff + st * C::kStageBytes);
      const uint32_t vbase = kbase + C::kTileBytes;
      // sequence position of this warp's first key, and the end of the valid
      // rows of the tile's source (the cache, or the appended keys)
      const int key0 = sg.pos0(t) + warp * 16;
      const int kend = sg.pend(t);
      if constexpr (kFp8) {
        // FP8 -> fp16 copy of this warp's 16 V rows; rows past the end of the
        // sequence become zeros (P = 0 must not meet a NaN there).
        __syncwarp();  // the previous tile's reads of the copy are done
        const uint8_t* vt = smem + C::kStageOff + st * C::kStageBytes + C::kTileBytes;
#pragma unroll 2
        for (int x = lane; x < 16 * (D / 16); x += 32) {
          const int kr = x / (D / 16), u = x % (D / 16);
          const int row = warp * 16 + kr;
          uint4 vw = *reinterpret_cast<const uint4*>(vt + row * 128 + ((u ^ (row & 7)) << 4));
          if (key0 + kr >= kend) vw = make_uint4(0, 0, 0, 0);
          fp8x16_to_f16_tile<kType>(vstg, kr, u * 16, vw);
        }
      } else if (key0 + 16 > kend) {
        // Keys past the end of the sequence hold whatever the page has there:
        // zero their V rows so that P = 0 never meets a NaN.
        for (int x = lane; x < 16 * (D / 8); x += 32) {
          const int kr = x / (D / 8), c8 = x % (D / 8);
          if (key0 + kr >= kend) {
            const uint32_t ad = sw128_addr(vbase, kDecTileKeys, warp * 16 + kr, c8 * 8);
            asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" ::"r"(ad), "r"(0) : "memory");
          }
        }
        __syncwarp();
      }
      // S = Q K^T for this warp's 16 keys: two n-tiles of 8 keys. K is read
      // from the stage (FP8 rows through the same 16-bit ldmatrix view).
      float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      {
        const int kr = warp * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int cofs = ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int k = 0; k < kKSteps; ++k) {
          uint32_t b[4];
          ldsm_x4(sw128_addr(kbase, kDecTileKeys, kr, k * 16 + cofs), b);
          if constexpr (kFp8) {
            mma16832_fp8<kType>(sacc[0], qa[k], b[0], b[1]);
            mma16832_fp8<kType>(sacc[1], qa[k], b[2], b[3]);
          } else {
            mma16816<kFp16>(sacc[0], qa[k], b[0], b[1]);
            mma16816<kFp16>(sacc[1], qa[k], b[2], b[3]);
          }
        }
      }
      if constexpr (kFp8) {
        // this warp no longer reads the stage (K above, V in the copy)
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
      }
      // the P V operand: the stage's V tile, or for FP8 this warp's copy
      const uint32_t vop = kFp8 ? vstg : vbase;
      constexpr int kOpRows = kFp8 ? 16 : kDecTileKeys;
      const int row0w = kFp8 ? 0 : warp * 16;
      // mask, running max (rows qr, qr+8 across the 4 lanes of a quad)
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int key = key0 + nt * 8 + qc + (x & 1);
          const int h2 = x >> 1;
          if (key >= kend || key < lo[h2] || key > hi[h2]) sacc[nt][x] = -INFINITY;
          mx[h2] = fmaxf(mx[h2], sacc[nt][x]);
        }
      float alpha[2], m_use[2];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        mx[h2] = fmaxf(mx[h2], __shfl_xor_sync(0xffffffffu, mx[h2], 1));
        mx[h2] = fmaxf(mx[h2], __shfl_xor_sync(0xffffffffu, mx[h2], 2));
        const float mn = fmaxf(m_run[h2], mx[h2] * sl2);
        alpha[h2] = (m_run[h2] == -INFINITY) ? 1.f : ex2(m_run[h2] - mn);
        m_run[h2] = mn;
        m_use[h2] = (mn == -INFINITY) ? 0.f : mn;
        l_run[h2] *= alpha[h2];
        l_rnd[h2] *= alpha[h2];
      }
      // O is rescaled only when some row of the warp raised its max (the
      // product by 1 would change nothing).
      if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
          o[n][0] *= alpha[0];
          o[n][1] *= alpha[0];
          o[n][2] *= alpha[1];
          o[n][3] *= alpha[1];
        }
      }
      // P (rounded to the input type) as the A operand of P V
      uint32_t pa[4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const float p0 = ex2(fmaf(sacc[nt][2 * h2], sl2, -m_use[h2]));
          const float p1 = ex2(fmaf(sacc[nt][2 * h2 + 1], sl2, -m_use[h2]));
          const uint32_t pk = pack2<kFp16>(p0, p1);
          pa[nt * 2 + h2] = pk;
          l_run[h2] += p0 + p1;
          l_rnd[h2] += sum2<kFp16>(pk);
        }
      // O += P V over this warp's 16 keys: 16 d-tiles of 8
      {
        const int kr = row0w + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int cofs = (lane >> 4) * 8;
#pragma unroll
        for (int n2 = 0; n2 < D / 16; ++n2) {
          uint32_t b[4];
          ldsm_x4_t(sw128_addr(vop, kOpRows, kr, n2 * 16 + cofs), b);
          mma16816<kFp16>(o[2 * n2], pa, b[0], b[1]);
          mma16816<kFp16>(o[2 * n2 + 1], pa, b[2], b[3]);
        }
      }
      if constexpr (!kFp8) {
        // this warp is done with the stage (zeroed rows included)
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
      }
      ++it;
    }

    // --- merge the eight warps' states ----------------------------------
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      l_run[h2] += __shfl_xor_sync(0xffffffffu, l_run[h2], 1);
      l_run[h2] += __shfl_xor_sync(0xffffffffu, l_run[h2], 2);
      l_rnd[h2] += __shfl_xor_sync(0xffffffffu, l_rnd[h2], 1);
      l_rnd[h2] += __shfl_xor_sync(0xffffffffu, l_rnd[h2], 2);
    }
    if ((lane & 3) == 0) {
      red_m[gw * kDecRows + qr] = m_run[0];
      red_m[gw * kDecRows + qr + 8] = m_run[1];
    }
    named_barrier(1, kDecConsumerThreads);
    float scale_w[2];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int r = qr + h2 * 8;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kDecConsumerWarps; ++w) M = fmaxf(M, red_m[w * kDecRows + r]);
      scale_w[h2] = (m_run[h2] == -INFINITY) ? 0.f : ex2(m_run[h2] - M);
      if ((lane & 3) == 0) {
        red_l[gw * kDecRows + r] = l_run[h2] * scale_w[h2];
        red_r[gw * kDecRows + r] = l_rnd[h2] * scale_w[h2];
      }
    }
    // O: the warps of each warpgroup add into that warpgroup's buffer one
    // after another in warp order, then the second buffer is added to the
    // first: a fixed order of the sums, so repeated runs agree bit for bit.
    {
      float* acc = red_o + wg * kDecRows * D;
      for (int w = 0; w < 4; ++w) {
        if (warp == w) {
#pragma unroll
          for (int n = 0; n < D / 8; ++n) {
            const int c = n * 8 + qc;
            float2* r0 = reinterpret_cast<float2*>(&acc[qr * D + c]);
            float2* r1 = reinterpret_cast<float2*>(&acc[(qr + 8) * D + c]);
            float2 v0 = make_float2(o[n][0] * scale_w[0], o[n][1] * scale_w[0]);
            float2 v1 = make_float2(o[n][2] * scale_w[1], o[n][3] * scale_w[1]);
            if (w > 0) {
              const float2 a0 = *r0, a1 = *r1;
              v0.x += a0.x; v0.y += a0.y;
              v1.x += a1.x; v1.y += a1.y;
            }
            *r0 = v0;
            *r1 = v1;
          }
        }
        named_barrier(1, kDecConsumerThreads);
      }
      for (int x = tid; x < kDecRows * D; x += kDecConsumerThreads)
        red_o[x] += red_o[kDecRows * D + x];
      named_barrier(1, kDecConsumerThreads);
    }

    // --- write: thread -> (row, 16 columns) --------------------------------
    {
      int nsplit = 1, slot = -1;
      if (meta) {
        nsplit = meta[ml.seg_nsplit + s];
        if (nsplit > 1) slot = meta[ml.seg_slot + s] + (blockIdx.x - meta[ml.seg_first + s]);
      }
      constexpr int kPer = D / 8;  // columns per thread (8 threads per row, 128 threads)
      const int r = tid >> 3, c0 = (tid & 7) * kPer;
      if (r < nrows) {  // tid < 128: r < 16 = kDecRows
        float M = -INFINITY, L = 0.f, LR = 0.f;
#pragma unroll
        for (int w = 0; w < kDecConsumerWarps; ++w) {
          M = fmaxf(M, red_m[w * kDecRows + r]);
          L += red_l[w * kDecRows + r];
          LR += red_r[w * kDecRows + r];
        }
        const float m_use = (M == -INFINITY) ? 0.f : M;
        const float lse2 = L > 0.f ? m_use + log2f(L) : -INFINITY;
        const int rr = row0 + r;
        const int i = rr / p.group, h = sg.g * p.group + rr % p.group;
        if (slot < 0) {
          float denom = LR;
          if (p.sink) denom += ex2(p.sink[h] * kLog2e - m_use);
          const float inv = denom > 0.f ? vscale / denom : 0.f;
          InT* dst = reinterpret_cast<InT*>(p.out) + sg.b * p.o_sb + i * p.o_ss + h * p.o_sh + c0;
#pragma unroll
          for (int c = 0; c < kPer; c += 8) {
            uint4 w;
            w.x = pack2<kOutF16>(red_o[r * D + c0 + c] * inv, red_o[r * D + c0 + c + 1] * inv);
            w.y = pack2<kOutF16>(red_o[r * D + c0 + c + 2] * inv, red_o[r * D + c0 + c + 3] * inv);
            w.z = pack2<kOutF16>(red_o[r * D + c0 + c + 4] * inv, red_o[r * D + c0 + c + 5] * inv);
            w.w = pack2<kOutF16>(red_o[r * D + c0 + c + 6] * inv, red_o[r * D + c0 + c + 7] * inv);
            *reinterpret_cast<uint4*>(dst + c) = w;
          }
          if (p.lse && (tid & 7) == 0)
            p.lse[((int64_t)sg.b * p.heads_q + h) * p.seqlen_q + i] = lse2 * kLn2;
        } else {
          const float inv = LR > 0.f ? vscale / LR : 0.f;
          float* dst = p.ws_o + ((int64_t)slot * kDecRows + r) * D + c0;
#pragma unroll
          for (int c = 0; c < kPer; c += 4)
            *reinterpret_cast<float4*>(dst + c) =
                make_float4(red_o[r * D + c0 + c] * inv, red_o[r * D + c0 + c + 1] * inv,
                            red_o[r * D + c0 + c + 2] * inv, red_o[r * D + c0 + c + 3] * inv);
          if ((tid & 7) == 0) p.ws_lse[(int64_t)slot * kDecRows + r] = lse2 * kLn2;
        }
      }
    }
    u = min(seg_end_units, se);
    ++s;
  }
}

template <int D, int kType>
__global__ void __launch_bounds__(kDecThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap map_k,
                  const __grid_constant__ CUtensorMap map_v,
                  const __grid_constant__ CUtensorMap map_kn,
                  const __grid_constant__ CUtensorMap map_vn, const DecodeParams p) {
  constexpr bool kFp8 = kType >= 2;
  using C = DecodeCfg<D, kFp8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* empty = full + C::kStages;
  int* abort = reinterpret_cast<int*>(empty + C::kStages);
  __shared__ int s_bad;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 4);
    }
    *abort = 0;
    s_bad = 0;
    fence_barrier_init();
  }
  __syncthreads();

  // This CTA's unit range and first segment.
  int ub, ue, s0;
  const int32_t* seg_prefix = nullptr;
  if (p.meta) {
    const MetaLayout ml(p.num_ctas, p.num_segs);
    if (threadIdx.x == 0 &&
        !(meta_matches(p.meta, ATTN_SCHED_MHA, p.batch, p.seqlen_q, p.heads_q, p.heads_kv,
                       p.page_size, p.num_segs, kDecTileKeys, D, D) &&
          p.meta[kMetaNumCtas] == p.num_ctas && p.meta[kMetaNewKeys] == p.seqlen_new)) {
      raise_error(ATTN_DEVERR_META_MISMATCH, 40);
      s_bad = 1;
    }
    __syncthreads();
    if (s_bad) return;
    ub = p.meta[ml.cta_begin + blockIdx.x];
    ue = p.meta[ml.cta_begin + blockIdx.x + 1];
    s0 = p.meta[ml.cta_seg + blockIdx.x];
    seg_prefix = p.meta + ml.seg_begin;
  } else {
    // one CTA per segment: all of its tiles
    s0 = blockIdx.x;
    const int b = s0 / p.segs_per_seq;
    const int len = p.cache_seqlens[b];
    ub = 0;
    ue = (len > 0 ? (len + kDecTileKeys - 1) / kDecTileKeys : 0) +
         (p.seqlen_new + kDecTileKeys - 1) / kDecTileKeys;
    if (ue == 0) ue = 1;  // still write O = 0, LSE = -inf for an empty sequence
  }
  if (threadIdx.x >= kDecConsumerThreads) {
    decode_producer<D, kFp8>(p, &map_k, &map_v, &map_kn, &map_vn, smem, full, empty, abort, ub,
                             ue, s0, seg_prefix);
  } else {
    decode_consumer<D, kType>(p, smem, full, empty, abort, ub, ue, s0, seg_prefix);
  }
}

}  // namespace attn
