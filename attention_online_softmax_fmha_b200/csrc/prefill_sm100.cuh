// Prefill / full-sequence attention forward on sm_100a.
//
// Computes, per query row, O = softmax(scale * q K^T + mask) V with the sink
// folded into the max and the denominator, and the keys-only LSE (CANN
// "flash_attn", 计算公式: the sink variant and the softmax_lse definition),
// for dense (BSHD) and packed varlen (THD + cu_seqlens) layouts with GQA,
// bottom-right causal and sliding-window masks (MindSpore Lite
// "flash_attention": causal, window_size; MindSpore "sparse_flash_attention":
// sparse_mode=3 "rightDownCausal").
//
// Design: one CTA per SM, persistent over work units of 256 query rows (two
// 128-row tiles Q0, Q1 of one sequence and head). Units are numbered
// heaviest first (last row block of every sequence and head first); with a
// work counter each CTA takes the next number when it starts a unit, so
// CTAs that drew short units take more of them, otherwise every
// gridDim-th number. The producer takes the numbers, decodes the units and
// hands both to the other roles through a small ring in shared memory. Both
// tiles stream the same K/V tiles of 128 keys.
//   warpgroup 0, 1   softmax of Q0 / Q1: thread r owns query row r of its
//                    tile (= TMEM lane r). Online softmax in the log2 domain;
//                    O in TMEM is rescaled only when a row's max grows by more
//                    than 2^8 (exact after the final division).
//   warp 8           TMA producer: Q0, Q1 and a ring of K/V tiles, 128-byte
//                    swizzled, one head per box.
//   warp 9           TMEM owner and MMA issuer (one thread), in the order
//                    PV0_{j-1}, S0_j, PV1_{j-1}, S1_j, ... so that the tensor
//                    core works on one tile while the other tile's softmax
//                    runs. S_w = Q_w K^T lands in TMEM; P_w (bf16) overwrites
//                    it and is the TMEM A operand of O_w += P_w V, started on
//                    the first 96 keys while the last 32 are exponentiated.
//   warps 10, 11     FP8: convert each e4m3 V tile to fp16 for P V. 16-bit
//                    inputs: warp 10 issues the output TMA stores, warp 11
//                    is idle (they complete the register warpgroup).
// Output: whole 128-row tiles go through a shared-memory staging tile and a
// TMA store, ragged tiles are stored directly by their threads.
// Registers move from warpgroup 2 to the softmax warpgroups with setmaxnreg;
// the host checks the kernel's register count before launching.
// Every mbarrier wait is bounded; a timeout raises ATTN_DEVERR_TIMEOUT and the
// roles unwind, draining in-flight copies and MMAs before TMEM is freed.
#pragma once

#include "common.cuh"

namespace attn {

struct PrefillParams {
  void* out;
  float* lse;
  const int32_t* cu_q;
  const int32_t* cu_k;
  const int32_t* seqused_q;  // padded layout: rows / keys in use per sequence
  const int32_t* seqused_k;
  const float* mask;         // additive score mask [b, h, i, j] (strides in elements)
  int64_t m_sb, m_sh, m_ss;
  const float* sink;
  const float* q_descale;
  const float* k_descale;
  const float* v_descale;
  int64_t o_sb, o_ss, o_sh;
  int64_t lse_sb, lse_sh;
  int32_t batch;
  int32_t seqlen_q;     // padded S_q (unused for varlen)
  int32_t seqlen_k;
  int32_t num_units_q;  // ceil(max_seqlen_q / 256)
  int32_t num_heads_q;
  int32_t num_heads_kv;
  int32_t group;        // H_q / H_kv
  int32_t total_units;
  float scale_log2;     // scale * log2(e)
  int32_t causal;
  int32_t window_left;
  int32_t window_right;
  int32_t* work_counter;  // next unit number (zeroed before the launch), or nullptr
};

constexpr int kPrefillBM = 128;               // query rows per tile
constexpr int kPrefillUnit = 2 * kPrefillBM;  // query rows per work unit
constexpr int kPrefillBN = 128;               // keys per tile

// Of every 16 P pairs, this many are exponentiated on the FMA pipe (a
// polynomial) and the rest on the MUFU pipe, to balance the two.
constexpr int kEmuPairs = 0;
// The softmax hands P to the MMA warp in two parts: the first kSplitKeys keys
// (p_head), then the rest (p_full), so that the P V MMA starts on the head
// while the tail is exponentiated.
constexpr int kSplitKeys = 96;
static_assert(kSplitKeys % 32 == 0 && kSplitKeys > 0 && kSplitKeys < kPrefillBN,
              "split on a 32-key chunk");
constexpr int kPrefillThreads = 384;
constexpr int kPrefillLaunchRegs = 168;       // 65536 / 384, rounded down to 8
constexpr int kPrefillSoftmaxRegs = 216;
constexpr int kPrefillOtherRegs = 72;
static_assert(2 * 128 * kPrefillSoftmaxRegs + 128 * kPrefillOtherRegs <=
                  kPrefillThreads * kPrefillLaunchRegs,
              "register split exceeds the launch allocation");

// Input types: 0 = bf16, 1 = fp16, 2 = FP8 E4M3, 3 = FP8 E5M2.
// With FP8 inputs S = Q K^T runs as an FP8 MMA; P is kept in fp16 (FP8 has
// too few mantissa bits for P: rows with few visible keys would miss the
// accuracy bound), so V is converted to fp16 in shared memory (exact: every
// e4m3 and every e5m2 value is an fp16 value) for the fp16 P V MMA.
template <int D, int kType>
struct PrefillCfg {
  static constexpr bool kFp8 = kType == 2 || kType == 3;
  static constexpr int kInBytes = kFp8 ? 1 : 2;
  static constexpr int kChunkElems = 128 / kInBytes;     // elements per 128-byte row chunk
  static constexpr int kChunks = D * kInBytes / 128;     // 128-byte column chunks
  // K and V tiles have separate rings: K is released as soon as both S MMAs
  // have read it, V after both P V MMAs (FP8: after the conversion).
  static constexpr int kKStages = kFp8 ? 4 : ((D == 64) ? 4 : 2);
  static constexpr int kVStages = (D == 64) ? 4 : 2;
  static constexpr int kVHStages = kFp8 ? 2 : 0;         // fp16 copies of V (FP8)
  static constexpr int kChunkBytes = 128 * 128;          // 128 rows x 128 bytes
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kVHBytes = (D / 64) * kChunkBytes;
  static constexpr int kQOff = 0;                        // Q0, Q1
  static constexpr int kKOff = 2 * kTileBytes;
  static constexpr int kVOff = kKOff + kKStages * kTileBytes;
  static constexpr int kVHOff = kVOff + kVStages * kTileBytes;
  // The output staging tile: 128 rows of D 16-bit values in 64-column chunks,
  // the box layout of the output tensor map (TMA store).
  static constexpr int kOutChunks = D / 64;
  static constexpr int kOStageOff = kVHOff + kVHStages * kVHBytes;
  static constexpr int kOStageBytes = kOutChunks * kChunkBytes;
  static constexpr int kBarOff = kOStageOff + kOStageBytes;
  static constexpr int kBarBytes = 1024;
  static constexpr int kSmemBytes = kBarOff + kBarBytes;
  // The dynamic shared memory base is 1024-byte aligned (the kernel checks).
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemS0 = 0, kTmemS1 = 128;
  static constexpr uint32_t kTmemO0 = 256, kTmemO1 = 256 + D;
};

// Unit numbers in flight from the producer to the other roles.
constexpr int kUnitRing = 4;

struct PrefillUnit {
  int b, h, m;
  int len_q, len_k;
  int row_q, row_k;  // first packed row of this sequence (0 for padded)
  int bcoord;        // batch coordinate of the tensor maps (0 for varlen)
  int kt0, kt1;      // key tiles [kt0, kt1)
};

struct PrefillBarriers {
  uint64_t unit_full[kUnitRing], unit_empty[kUnitRing];
  int32_t unit_idx[kUnitRing];  // a unit number, or -1 after the CTA's last unit
  // The producer's decoding of each unit in the ring, so that no other role
  // reads the sequence offsets from global memory between two units.
  PrefillUnit units[kUnitRing];
  uint64_t q_full, q_empty;
  uint64_t k_full[4], v_full[4], k_empty[4], v_empty[4];
  uint64_t vh_full[4], vh_empty[4];
  uint64_t s_full[2], p_head[2], p_full[2], o_full[2], o_empty[2];
  // The output staging tile, used by the two softmax warpgroups in turn
  // (use u = 2 * unit + warpgroup): full once all 128 rows are written,
  // free once the TMA store has read it.
  uint64_t ostage_full, ostage_free;
  // What the staged tile is: whether to store it, and its box coordinates
  // (written by the warpgroup's first thread before it arrives).
  int32_t ostage_store, ostage_c1, ostage_c2, ostage_c3;
  uint64_t mma_drain;
  uint32_t tmem_base;
  int32_t abort;
};
static_assert(sizeof(PrefillBarriers) <= 1024, "barrier block");


// Maps a linear work index to a unit; returns false for units past the end
// of their sequence. Every role calls this with the same index and gets the
// same answer, so all roles skip the same units.
DEVI bool prefill_unit(const PrefillParams& p, int t, PrefillUnit& u) {
  const int bh = p.batch * p.num_heads_q;
  const int mr = t / bh;
  const int rem = t - mr * bh;
  u.b = rem / p.num_heads_q;
  u.h = rem - u.b * p.num_heads_q;
  u.m = p.num_units_q - 1 - mr;
  if (p.cu_q != nullptr) {
    u.row_q = p.cu_q[u.b];
    u.len_q = p.cu_q[u.b + 1] - u.row_q;
    u.row_k = p.cu_k[u.b];
    u.len_k = p.cu_k[u.b + 1] - u.row_k;
    u.bcoord = 0;
  } else {
    u.row_q = u.row_k = 0;
    u.len_q = p.seqused_q ? p.seqused_q[u.b] : p.seqlen_q;
    u.len_k = p.seqused_k ? p.seqused_k[u.b] : p.seqlen_k;
    u.bcoord = u.b;
  }
  const int q0 = u.m * kPrefillUnit;
  if (q0 >= u.len_q) return false;
  const int q1 = min(q0 + kPrefillUnit, u.len_q) - 1;
  const int delta = u.len_k - u.len_q;
  int lo = 0, hi = u.len_k - 1;
  if (p.window_left >= 0) lo = max(lo, q0 + delta - p.window_left);
  if (p.causal) hi = min(hi, q1 + delta);
  if (p.window_right >= 0) hi = min(hi, q1 + delta + p.window_right);
  if (hi < lo) {
    u.kt0 = u.kt1 = 0;
  } else {
    u.kt0 = lo / kPrefillBN;
    u.kt1 = hi / kPrefillBN + 1;
  }
  return true;
}

// Takes the k-th unit number of this CTA, and its decoding, from the ring
// (warp-collective; each consuming warp releases the slot once). Returns
// false if the wait gave up.
DEVI bool take_unit(PrefillBarriers* bars, int k, int& t, PrefillUnit& u, int site) {
  const int slot = k % kUnitRing;
  if (!warp_wait(&bars->unit_full[slot], (k / kUnitRing) & 1, &bars->abort, site)) return false;
  t = *reinterpret_cast<volatile int32_t*>(&bars->unit_idx[slot]);
  if (t >= 0) {
    const volatile int* src = reinterpret_cast<const volatile int*>(&bars->units[slot]);
    int* dst = reinterpret_cast<int*>(&u);
#pragma unroll
    for (int x = 0; x < (int)(sizeof(PrefillUnit) / sizeof(int)); ++x) dst[x] = src[x];
  }
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&bars->unit_empty[slot]);
  return true;
}

// Inclusive visible key range of query row i.
DEVI void row_key_range(const PrefillParams& p, int i, int len_q, int len_k, int& lo, int& hi) {
  const int delta = len_k - len_q;
  lo = 0;
  hi = len_k - 1;
  if (p.window_left >= 0) lo = max(lo, i + delta - p.window_left);
  if (p.causal) hi = min(hi, i + delta);
  if (p.window_right >= 0) hi = min(hi, i + delta + p.window_right);
}

// bf16 inputs: a query tile with a row that sees fewer than kShortRow keys
// runs P V twice, on P rounded to bf16 and on the rounding remainder (also
// bf16), so P carries about 16 significant bits. With few keys the bf16
// rounding of P does not average out: for two keys it moves O by up to
// 2^-9 * |v_1 - v_0| / 4, which, on top of the final rounding of O to bf16,
// can exceed 1e-2. Rows with many keys need no remainder.
constexpr int kShortRow = 128;

// Whether Q tile w of unit u holds a row with fewer than kShortRow visible
// keys. The count of a row is concave in the row index (the upper bound is a
// minimum of increasing lines, the lower bound a maximum of them), so its
// minimum over the tile is at the tile's first or last row.
DEVI bool prefill_short_tile(const PrefillParams& p, const PrefillUnit& u, int w) {
  const int i0 = u.m * kPrefillUnit + w * kPrefillBM;
  if (i0 >= u.len_q) return false;
  const int i1 = min(i0 + kPrefillBM, u.len_q) - 1;
  int lo0, hi0, lo1, hi1;
  row_key_range(p, i0, u.len_q, u.len_k, lo0, hi0);
  row_key_range(p, i1, u.len_q, u.len_k, lo1, hi1);
  return min(hi0 - lo0, hi1 - lo1) + 1 < kShortRow;
}

// ---------------------------------------------------------------------------
// Producer warp (one thread)
// ---------------------------------------------------------------------------
template <int D, int kType>
DEVI void prefill_producer(const PrefillParams& p, const CUtensorMap* mq, const CUtensorMap* mk,
                           const CUtensorMap* mv, uint8_t* smem, PrefillBarriers* bars) {
  using C = PrefillCfg<D, kType>;
  volatile int* abort = &bars->abort;
  tma_prefetch_desc(mq);
  tma_prefetch_desc(mk);
  tma_prefetch_desc(mv);
  int it = 0, nq = 0, k = 0;
  for (int fetched = 0;; ++fetched) {
    // The next unit number: from the counter, or every gridDim-th. Numbers
    // past a sequence's end are passed over; the roles get the rest, then -1.
    const int t = p.work_counter ? atomicAdd(p.work_counter, 1)
                                 : blockIdx.x + fetched * (int)gridDim.x;
    const bool end = t >= p.total_units;
    PrefillUnit u;
    if (!end && !prefill_unit(p, t, u)) continue;
    {
      const int slot = k % kUnitRing;
      if (k >= kUnitRing &&
          !mbar_wait(&bars->unit_empty[slot], ((k / kUnitRing) - 1) & 1, abort, 5))
        goto drain;
      bars->unit_idx[slot] = end ? -1 : t;
      if (!end) bars->units[slot] = u;
      mbar_arrive(&bars->unit_full[slot]);  // release: the unit is visible to the waiters
      ++k;
    }
    if (end) break;
    const int n = u.kt1 - u.kt0;
    if (n <= 0) continue;
    const int hk = u.h / p.group;
    if (nq > 0 && !mbar_wait(&bars->q_empty, (nq - 1) & 1, abort, 1)) goto drain;
    mbar_expect_tx(&bars->q_full, 2 * C::kTileBytes);
#pragma unroll
    for (int w = 0; w < 2; ++w)
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_4d(smem + C::kQOff + w * C::kTileBytes + c * C::kChunkBytes, mq, &bars->q_full,
                    c * C::kChunkElems, u.h, u.row_q + u.m * kPrefillUnit + w * kPrefillBM,
                    u.bcoord);
    ++nq;
    for (int j = 0; j < n; ++j, ++it) {
      const int row = u.row_k + (u.kt0 + j) * kPrefillBN;
      const int sk = it % C::kKStages, sv = it % C::kVStages;
      if (it >= C::kKStages &&
          !mbar_wait(&bars->k_empty[sk], ((it / C::kKStages) - 1) & 1, abort, 2))
        goto drain;
      mbar_expect_tx(&bars->k_full[sk], C::kTileBytes);
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_4d(smem + C::kKOff + sk * C::kTileBytes + c * C::kChunkBytes, mk,
                    &bars->k_full[sk], c * C::kChunkElems, hk, row, u.bcoord);
      if (it >= C::kVStages &&
          !mbar_wait(&bars->v_empty[sv], ((it / C::kVStages) - 1) & 1, abort, 4))
        goto drain;
      mbar_expect_tx(&bars->v_full[sv], C::kTileBytes);
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_4d(smem + C::kVOff + sv * C::kTileBytes + c * C::kChunkBytes, mv,
                    &bars->v_full[sv], c * C::kChunkElems, hk, row, u.bcoord);
    }
  }
drain:
  // Wait (bounded, abort flag ignored) for the copies this thread may still
  // have in flight, so none lands in shared memory after the CTA exits.
  {
    int zero = 0;
    if (nq > 0) mbar_wait(&bars->q_full, (nq - 1) & 1, &zero, 3);
    for (int i = max(0, it - C::kKStages); i < it; ++i)
      mbar_wait(&bars->k_full[i % C::kKStages], (i / C::kKStages) & 1, &zero, 3);
    for (int i = max(0, it - C::kVStages); i < it; ++i)
      mbar_wait(&bars->v_full[i % C::kVStages], (i / C::kVStages) & 1, &zero, 3);
  }
}

// ---------------------------------------------------------------------------
// MMA warp (one thread issues)
// ---------------------------------------------------------------------------
// Descriptors are built once; a K step or a stage moves the start address,
// which is the low 14-bit field (in 16-byte units) of the descriptor, so an
// integer add of the offset in 16-byte units advances it (shared memory is
// below 256 KB, the field never carries).
// One MMA consumes 32 bytes of K (16 bf16/fp16 or 32 FP8 elements).
template <int D, int kType>
DEVI void prefill_issue_s(uint32_t d_tmem, uint64_t dq, uint64_t dk, uint32_t idesc) {
  using C = PrefillCfg<D, kType>;
#pragma unroll
  for (int k = 0; k < D * C::kInBytes / 32; ++k) {
    const uint32_t off16 = (k >> 2) * (C::kChunkBytes >> 4) + (k & 3) * 2;
    if constexpr (C::kFp8)
      mma_f8_ss_w(d_tmem, dq + off16, dk + off16, idesc, k > 0 ? 1u : 0u);
    else
      mma_f16_ss_w(d_tmem, dq + off16, dk + off16, idesc, k > 0 ? 1u : 0u);
  }
}
template <int kK0, int kK1>
DEVI void prefill_issue_pv(uint32_t d_tmem, uint32_t a_tmem, uint64_t dv, uint32_t idesc,
                           bool first) {
#pragma unroll
  for (int kk = kK0; kk < kK1; ++kk)
    mma_f16_ts_w(d_tmem, a_tmem + kk * 8, dv + kk * (16 * 128 >> 4), idesc,
               (!first || kk > 0) ? 1u : 0u);
}

// O_w += P_w V for the key tile with global index g: the head of P as soon as
// the softmax has released it, then the tail; with `split`, then the rounding
// remainder of P (TMEM columns 64 .. 127 of the tile's S buffer).
DEVI bool prefill_pv(PrefillBarriers* bars, int w, int g, uint32_t t_o, uint32_t t_p, uint64_t dv,
                     uint32_t idesc, bool first, bool split) {
  volatile int* abort = &bars->abort;
  constexpr int kHead = kSplitKeys / 16;
  if constexpr (kHead > 0) {
    if (!warp_wait(&bars->p_head[w], g & 1, abort, 16)) return false;
    tc_fence_after();
    prefill_issue_pv<0, kHead>(t_o, t_p, dv, idesc, first);
  }
  if (!warp_wait(&bars->p_full[w], g & 1, abort, 11)) return false;
  tc_fence_after();
  prefill_issue_pv<kHead, kPrefillBN / 16>(t_o, t_p, dv, idesc, first);
  if (split) {
    // a rolled loop: the MMA warp runs on few registers
#pragma unroll 1
    for (int kk = 0; kk < kPrefillBN / 16; ++kk)
      mma_f16_ts_w(t_o, t_p + kPrefillBN / 2 + kk * 8, dv + kk * (16 * 128 >> 4), idesc, 1u);
  }
  return true;
}

template <int D, int kType, bool kMask>
DEVI void prefill_mma(const PrefillParams& p, uint8_t* smem, PrefillBarriers* bars,
                      uint32_t tmem) {
  using C = PrefillCfg<D, kType>;
  volatile int* abort = &bars->abort;
  // Operand formats: kind::f16 0 = fp16, 1 = bf16; kind::f8f6f4 0 = e4m3,
  // 1 = e5m2. P V runs in fp16 for FP8 inputs.
  constexpr int fmt_qk = (kType == 0 || kType == 3) ? 1 : 0;
  constexpr int fmt_pv = kType == 0 ? 1 : 0;
  constexpr uint32_t idesc_qk = make_idesc(128, kPrefillBN, fmt_qk, 0, 0);
  // V is MN-major (d contiguous): one MMA covers all D columns; the 64-column
  // chunks of the tile are kChunkBytes apart (leading byte offset), groups
  // of 8 keys are 1024 bytes apart (stride byte offset).
  constexpr uint32_t idesc_pv = make_idesc(128, D, fmt_pv, 0, 1);
  constexpr int kPVStages = C::kFp8 ? C::kVHStages : C::kVStages;
  constexpr int kPVBytes = C::kFp8 ? C::kVHBytes : C::kTileBytes;
  uint64_t* pv_full = C::kFp8 ? bars->vh_full : bars->v_full;
  uint64_t* pv_empty = C::kFp8 ? bars->vh_empty : bars->v_empty;
  const uint64_t dq0 = sdesc_sw128(smem_u32(smem + C::kQOff), 16, 1024);
  const uint64_t dq1 = dq0 + (C::kTileBytes >> 4);
  const uint64_t dk_base = sdesc_sw128(smem_u32(smem + C::kKOff), 16, 1024);
  const uint64_t dv_base =
      sdesc_sw128(smem_u32(smem + (C::kFp8 ? C::kVHOff : C::kVOff)), C::kChunkBytes, 1024);
  const uint32_t tS0 = tmem + C::kTmemS0, tS1 = tmem + C::kTmemS1;
  const uint32_t tO0 = tmem + C::kTmemO0, tO1 = tmem + C::kTmemO1;
  int it = 0, nq = 0, units = 0;

  for (int k = 0;; ++k) {
    int t;
    PrefillUnit u;
    if (!take_unit(bars, k, t, u, 9)) goto drain;
    if (t < 0) break;
    const int n = u.kt1 - u.kt0;
    if (n <= 0) continue;
    if (!warp_wait(&bars->q_full, nq & 1, abort, 10)) goto drain;
    ++nq;
    const bool split0 = kType == 0 && !kMask && prefill_short_tile(p, u, 0);
    const bool split1 = kType == 0 && !kMask && prefill_short_tile(p, u, 1);
    // Order per key tile j: PV0_{j-1}, S0_j, PV1_{j-1}, S1_j. S_w needs the
    // S_w/P_w buffer that PV_w_{j-1} reads; the tensor pipe runs in order.
    for (int j = 0; j <= n; ++j) {
      const int g = it + j;
      const int s = g % C::kKStages;
      const int sp = (g - 1) % kPVStages;
      if (j < n) {
        if (!warp_wait(&bars->k_full[s], (g / C::kKStages) & 1, abort, 14)) goto drain;
      }
      if (j > 0) {
        if (!warp_wait(&pv_full[sp], ((g - 1) / kPVStages) & 1, abort, 12)) goto drain;
        if (j == 1 && units > 0 && !warp_wait(&bars->o_empty[0], (units - 1) & 1, abort, 13))
          goto drain;
        if (!prefill_pv(bars, 0, g - 1, tO0, tS0, dv_base + sp * (kPVBytes >> 4), idesc_pv,
                        j == 1, split0))
          goto drain;
        if (j == n) tc_commit_w(&bars->o_full[0]);
      } else {
        tc_fence_after();
      }
      if (j < n) {
        prefill_issue_s<D, kType>(tS0, dq0, dk_base + s * (C::kTileBytes >> 4), idesc_qk);
        tc_commit_w(&bars->s_full[0]);
      }
      if (j > 0) {
        if (j == 1 && units > 0 && !warp_wait(&bars->o_empty[1], (units - 1) & 1, abort, 13))
          goto drain;
        if (!prefill_pv(bars, 1, g - 1, tO1, tS1, dv_base + sp * (kPVBytes >> 4), idesc_pv,
                        j == 1, split1))
          goto drain;
        if (j == n) tc_commit_w(&bars->o_full[1]);
        tc_commit_w(&pv_empty[sp]);
      }
      if (j < n) {
        prefill_issue_s<D, kType>(tS1, dq1, dk_base + s * (C::kTileBytes >> 4), idesc_qk);
        tc_commit_w(&bars->s_full[1]);
        tc_commit_w(&bars->k_empty[s]);
        if (j == n - 1) tc_commit_w(&bars->q_empty);
      }
    }
    it += n;
    ++units;
  }
drain : {
  // All issued MMAs must finish before TMEM is released.
  int zero = 0;
  tc_commit_w(&bars->mma_drain);
  warp_wait(&bars->mma_drain, 0, &zero, 15);
}
}

// ---------------------------------------------------------------------------
// FP8 only: V conversion warps (warps 10, 11). Each e4m3 V tile (128-byte
// swizzled rows of 128 elements) is rewritten as an fp16 tile in the layout
// the P V MMA reads (two 64-column chunks, 128-byte swizzled); the e4m3 stage
// is then released to the producer and the fp16 stage handed to the MMA.
// ---------------------------------------------------------------------------

template <int D, int kType>
DEVI void prefill_convert(const PrefillParams& p, uint8_t* smem, PrefillBarriers* bars) {
  using C = PrefillCfg<D, kType>;
  static_assert(D == 128, "FP8 prefill is built for D = 128");
  volatile int* abort = &bars->abort;
  const int t = threadIdx.x - 320;  // 0..63
  int it = 0;
  for (int k = 0;; ++k) {
    int wu;
    PrefillUnit u;
    if (!take_unit(bars, k, wu, u, 52)) return;
    if (wu < 0) break;
    const int n = u.kt1 - u.kt0;
    for (int j = 0; j < n; ++j, ++it) {
      const int sv = it % C::kVStages, sh = it % C::kVHStages;
      if (!mbar_wait(&bars->v_full[sv], (it / C::kVStages) & 1, abort, 50)) return;
      if (it >= C::kVHStages &&
          !mbar_wait(&bars->vh_empty[sh], ((it / C::kVHStages) - 1) & 1, abort, 51))
        return;
      const uint8_t* src = smem + C::kVOff + sv * C::kTileBytes;
      uint8_t* dst = smem + C::kVHOff + sh * C::kVHBytes;
#pragma unroll 4
      for (int x = t; x < 128 * 8; x += 64) {
        const int row = x >> 3, unit = x & 7;  // 16 e4m3 values = d 16*unit .. +15
        const uint4 v = *reinterpret_cast<const uint4*>(src + row * 128 + ((unit ^ (row & 7)) << 4));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t h[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          h[2 * q] = fp8x2_to_f16x2<kType>((unsigned short)(w[q] & 0xffff));
          h[2 * q + 1] = fp8x2_to_f16x2<kType>((unsigned short)(w[q] >> 16));
        }
        const int chunk = unit >> 2, u16 = (unit & 3) * 2;
        uint8_t* drow = dst + chunk * C::kChunkBytes + row * 128;
        *reinterpret_cast<uint4*>(drow + ((u16 ^ (row & 7)) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(drow + (((u16 + 1) ^ (row & 7)) << 4)) =
            make_uint4(h[4], h[5], h[6], h[7]);
      }
      fence_proxy_async_smem();  // the fp16 tile is read by the tensor core
      mbar_arrive(&bars->vh_full[sh]);
      mbar_arrive(&bars->v_empty[sv]);
    }
  }
}

// ---------------------------------------------------------------------------
// Softmax warpgroups: warpgroup w owns tile Q_w, thread r query row r of it
// (= TMEM lane r). The two warpgroups run offset by about half a tile, so one
// exponentiates while the other waits for its next S.
// ---------------------------------------------------------------------------
// TMA store of one box from shared memory (the tensor map's swizzled layout).
DEVI void tma_store_4d(const CUtensorMap* map, const void* src, int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

struct PrefillRow {
  float m_run;  // running max (log2 domain, includes the sink)
  float l_run;  // sum of the fp32 P (for the LSE)
  float l_rnd;  // sum of the rounded P the MMA consumes (for O)
  int lo, hi;   // visible key range
  bool seen;    // some key of this row is visible
};

// P = 2^(s * scale * log2e - m) rounded to the MMA's input type (to nearest
// even), written over S 32 keys (16 packed words) at a time, the head
// released first; the row sums (kRnd: also the sum of the rounded P).
// split (bf16, kRnd instance): the rounding remainder P - bf16(P), itself
// rounded to bf16, goes to TMEM columns 64 .. 127 of the buffer; O is then
// normalised by the fp32 sum, which the two parts together match to about
// 2^-16.
template <int kType, bool kRnd, class Sig>
DEVI void prefill_exp_tile(const Sig& sig, uint32_t s_tmem, float sl2, uint32_t* s,
                           PrefillRow& row, bool split) {
  constexpr bool kSplit = kRnd && kType == 0;  // the remainder pass may run
  constexpr bool kFp16 = kType != 0;  // P in fp16 (fp16 and FP8 inputs)
  const float m_use = (row.m_run == -INFINITY) ? 0.f : row.m_run;
  const uint64_t negm = f2pack(-m_use, -m_use);
  const uint64_t sl2x2 = f2pack(sl2, sl2);
  uint64_t acc_e[4];
  float acc_r[4];
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    acc_e[x] = 0ull;
    acc_r[x] = 0.f;
  }
#pragma unroll
  for (int ch = 0; ch < kPrefillBN / 32; ++ch) {
    uint32_t pk[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int e = ch * 32 + 2 * c;
      const uint64_t arg =
          fma2(f2pack(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), sl2x2, negm);
      float a0, a1;
      f2unpack(arg, a0, a1);
      float p0, p1;
      if (c >= 16 - kEmuPairs) {
        f2unpack(exp2_poly_x2(a0, a1), p0, p1);
      } else {
        p0 = ex2(a0);
        p1 = ex2(a1);
      }
      acc_e[c & 3] = add2(acc_e[c & 3], f2pack(p0, p1));
      pk[c] = pack2<kFp16>(p0, p1);
      if constexpr (kRnd) acc_packed<kFp16>(acc_r[c & 1], acc_r[2 + (c & 1)], pk[c]);
      if constexpr (kSplit) {  // keep P itself: S of this element is no longer needed
        s[e] = __float_as_uint(p0);
        s[e + 1] = __float_as_uint(p1);
      }
    }
    tmem_store<16>(s_tmem + ch * 16, pk);
    if (kSplit && split) {
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int e = ch * 32 + 2 * c;
        // the bf16 halves of pk[c] widened exactly; P minus them is exact
        const float r0 = __uint_as_float(s[e]) - __uint_as_float(pk[c] << 16);
        const float r1 = __uint_as_float(s[e + 1]) - __uint_as_float(pk[c] & 0xffff0000u);
        pk[c] = pack_bf16x2(r0, r1);
      }
      tmem_store<16>(s_tmem + kPrefillBN / 2 + ch * 16, pk);
    }
    if (ch == kSplitKeys / 32 - 1) {
      // The head of P: the P V MMA starts on it.
      tmem_store_wait();
      tc_fence_before();
      sig.p_head();
    }
  }
  {
    const uint64_t e = add2(add2(acc_e[0], acc_e[1]), add2(acc_e[2], acc_e[3]));
    float e0, e1;
    f2unpack(e, e0, e1);
    row.l_run += e0 + e1;
    row.l_rnd += (kRnd && !(kSplit && split)) ? (acc_r[0] + acc_r[1]) + (acc_r[2] + acc_r[3])
                                              : e0 + e1;
  }
  tmem_store_wait();
  tc_fence_before();
  sig.p_full();
}

// The softmax's hand-offs with the MMA warp of the one-CTA kernel: S of tile
// w is ready (a commit on this CTA's barrier); the head / all of P is in TMEM
// (every thread arrives).
struct PrefillSig {
  PrefillBarriers* bars;
  int w;
  DEVI bool wait_s(int g) const {
    return warp_wait(&bars->s_full[w], g & 1, &bars->abort, 20 + w);
  }
  DEVI void p_head() const { mbar_arrive(&bars->p_head[w]); }
  DEVI void p_full() const { mbar_arrive(&bars->p_full[w]); }
};

// One S tile of keys [k0, k0 + 128) of this thread's row: mask, row max,
// lazy O rescale, P = 2^(s * scale * log2e - m) written over S (head first),
// row sums. Returns false if a wait gave up.
template <int D, int kType, bool kMask, class Sig>
DEVI bool prefill_softmax_tile(const Sig& sig, uint32_t s_tmem, uint32_t o_tmem, int j, int g,
                               int k0, float sl2, PrefillRow& row, const float* mrow, int len_k,
                               bool few, bool split) {
  if (!sig.wait_s(g)) return false;
  tc_fence_after();
  uint32_t s[kPrefillBN];
  tmem_load128(s_tmem, s);
  if constexpr (kMask) {
    // Additive mask: scores become log2-domain s * scale * log2e + mask *
    // log2e here (keys past the sequence end read nothing; they are masked
    // below), and the rest of the tile uses a unit scale.
#pragma unroll
    for (int c = 0; c < kPrefillBN; c += 4) {
      const int key = k0 + c;
      float4 mv = make_float4(0.f, 0.f, 0.f, 0.f);
      if (mrow != nullptr) {
        if (key + 3 < len_k) {
          mv = __ldg(reinterpret_cast<const float4*>(mrow + key));
        } else {
          if (key < len_k) mv.x = __ldg(mrow + key);
          if (key + 1 < len_k) mv.y = __ldg(mrow + key + 1);
          if (key + 2 < len_k) mv.z = __ldg(mrow + key + 2);
        }
      }
      s[c] = __float_as_uint(fmaf(__uint_as_float(s[c]), sl2, mv.x * kLog2e));
      s[c + 1] = __float_as_uint(fmaf(__uint_as_float(s[c + 1]), sl2, mv.y * kLog2e));
      s[c + 2] = __float_as_uint(fmaf(__uint_as_float(s[c + 2]), sl2, mv.z * kLog2e));
      s[c + 3] = __float_as_uint(fmaf(__uint_as_float(s[c + 3]), sl2, mv.w * kLog2e));
    }
    sl2 = 1.f;
  }
  const bool partial = !(k0 >= row.lo && k0 + kPrefillBN - 1 <= row.hi);
  if (partial) {
#pragma unroll
    for (int c = 0; c < kPrefillBN; ++c) {
      const bool vis = (k0 + c >= row.lo) && (k0 + c <= row.hi);
      s[c] = vis ? s[c] : __float_as_uint(-INFINITY);
    }
  }
  // Row max: four independent chains of three-input maxima.
  float mx4[4];
#pragma unroll
  for (int x = 0; x < 4; ++x)
    mx4[x] = fmax3(__uint_as_float(s[x]), __uint_as_float(s[4 + x]), __uint_as_float(s[8 + x]));
#pragma unroll
  for (int c = 12; c + 8 <= kPrefillBN; c += 8)
#pragma unroll
    for (int x = 0; x < 4; ++x)
      mx4[x] = fmax3(mx4[x], __uint_as_float(s[c + x]), __uint_as_float(s[c + 4 + x]));
#pragma unroll
  for (int x = 0; x < 4; ++x) mx4[x] = fmaxf(mx4[x], __uint_as_float(s[kPrefillBN - 4 + x]));
  const float tmax = fmaxf(fmax3(mx4[0], mx4[1], mx4[2]), mx4[3]);
  const float mx = tmax * sl2;
  row.seen |= tmax != -INFINITY;
  // The first tile sets the max exactly (the row's largest P is then 1
  // unless the sink is larger); later tiles raise it only when it grows by
  // more than 2^8, and then O is rescaled in TMEM. The previous P V of this
  // tile has completed: it was issued before this S. tcgen05.ld/st are
  // warp-collective, so the warp rescales together, each thread with its own
  // factor (1 if unchanged).
  float alpha = 1.f;
  const bool grow = (j == 0) ? (mx > row.m_run) : (mx > row.m_run + kRescaleThreshold);
  if (grow) {
    if (j > 0 && row.m_run != -INFINITY) alpha = ex2(row.m_run - mx);
    row.m_run = mx;
    row.l_run *= alpha;
    row.l_rnd *= alpha;
  }
  if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
    const uint64_t a2 = f2pack(alpha, alpha);
#pragma unroll
    for (int c = 0; c < D; c += 32) {
      uint32_t o[32];
      tmem_load<32>(o_tmem + c, o);
#pragma unroll
      for (int x = 0; x < 32; x += 2) {
        const uint64_t v = mul2(f2pack(__uint_as_float(o[x]), __uint_as_float(o[x + 1])), a2);
        float a, b;
        f2unpack(v, a, b);
        o[x] = __float_as_uint(a);
        o[x + 1] = __float_as_uint(b);
      }
      tmem_store<32>(o_tmem + c, o);
    }
  }
  // O is normalised by the sum of the rounded P the MMA consumes (the
  // weights then stay a convex combination and the rounding error scales
  // with the spread of V, not with |O|); the LSE uses the fp32 sum. The
  // difference matters only for rows with few visible keys (fewer than
  // kShortRow): tiles that hold such a row, first tiles and masked tiles add
  // the rounded sum; other tiles, diagonal and window-edge tiles of long rows
  // included, add their fp32 sum to both (their rounding errors average out
  // over the row's many keys).
  if (j == 0 || kMask || few)
    prefill_exp_tile<kType, true>(sig, s_tmem, sl2, s, row, split);
  else
    prefill_exp_tile<kType, false>(sig, s_tmem, sl2, s, row, false);
  return true;
}

template <int D, int kType, bool kMask>
DEVI void prefill_softmax(const PrefillParams& p, const CUtensorMap* mo, uint8_t* smem,
                          PrefillBarriers* bars, uint32_t tmem, int w) {
  using C = PrefillCfg<D, kType>;
  using OutT = typename std::conditional<kType == 1, __half, __nv_bfloat16>::type;
  volatile int* abort = &bars->abort;
  const int r = threadIdx.x & 127;
  const uint32_t lane = (uint32_t)(r & ~31) << 16;
  const uint32_t s_tmem = tmem + (w ? C::kTmemS1 : C::kTmemS0) + lane;
  const uint32_t o_tmem = tmem + (w ? C::kTmemO1 : C::kTmemO0) + lane;
  int sj = 0, units = 0;
  // The output goes out through the staging tile, one warpgroup at a time
  // (use number ouse = 2 * unit + w): a tile whose 128 rows all belong to
  // the sequence is written there and stored by TMA (one thread, in the
  // background); other rows are stored directly. Every unit takes its turn,
  // so the two warpgroups alternate.
  int ouse = w;
  auto turn_begin = [&]() -> bool {
    return ouse < 1 || warp_wait(&bars->ostage_free, (ouse - 1) & 1, abort, 26 + w);
  };
  auto turn_end = [&](bool staged, const PrefillUnit& u, int i0) -> bool {
    if (staged) fence_proxy_async_smem();  // the TMA store reads through the async proxy
    if constexpr (!C::kFp8) {
      // 16-bit inputs: the store warp issues the TMA store and passes the turn on
      if (r == 0) {
        bars->ostage_store = staged ? 1 : 0;
        bars->ostage_c1 = u.h;
        bars->ostage_c2 = u.row_q + i0;
        bars->ostage_c3 = u.bcoord;
      }
      mbar_arrive(&bars->ostage_full);
      ouse += 2;
      return true;
    }
    mbar_arrive(&bars->ostage_full);
    bool ok = true;
    if (r < 32) {  // warp 0 of the warpgroup; its lane 0 stores and passes the turn on
      if (r == 0) {
        ok = mbar_wait(&bars->ostage_full, ouse & 1, abort, 28 + w);
        if (ok && staged) {
#pragma unroll
          for (int c = 0; c < C::kOutChunks; ++c)
            tma_store_4d(mo, smem + C::kOStageOff + c * C::kChunkBytes, c * 64, u.h, u.row_q + i0,
                         u.bcoord);
          bulk_commit();
          bulk_wait_read<0>();  // the staging tile has been read
        }
        if (ok) mbar_arrive(&bars->ostage_free);
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    ouse += 2;
    return ok;
  };
  for (int k = 0;; ++k) {
    int t;
    PrefillUnit u;
    if (!take_unit(bars, k, t, u, 24 + w)) return;
    if (t < 0) break;
    const int n = u.kt1 - u.kt0;
    const int i = u.m * kPrefillUnit + w * kPrefillBM + r;
    const bool valid = i < u.len_q;
    OutT* orow = reinterpret_cast<OutT*>(p.out) + u.bcoord * p.o_sb +
                 (int64_t)(u.row_q + i) * p.o_ss + (int64_t)u.h * p.o_sh;
    float* lrow = p.lse ? p.lse + u.b * p.lse_sb + u.h * p.lse_sh + (u.row_q + i) : nullptr;
    if (n <= 0) {
      if (!turn_begin()) return;
      if (valid) {
        const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(orow)[c] = z;
        if (lrow) *lrow = -INFINITY;
      }
      if (!turn_end(false, u, 0)) return;
      continue;
    }
    float sl2 = p.scale_log2;
    float v_scale = 1.f;
    if constexpr (C::kFp8) {
      // S and O use the dequantised inputs: q * q_descale, k * k_descale,
      // v * v_descale, per (sequence, KV head) (MATE FMHA dtype notes).
      const int dk = u.b * p.num_heads_kv + u.h / p.group;
      sl2 *= p.q_descale[dk] * p.k_descale[dk];
      v_scale = p.v_descale[dk];
    }
    const bool has_sink = p.sink != nullptr;
    const float sink2 = has_sink ? p.sink[u.h] * kLog2e : -INFINITY;
    PrefillRow row;
    row_key_range(p, i, u.len_q, u.len_k, row.lo, row.hi);
    row.m_run = sink2;
    row.l_run = row.l_rnd = 0.f;
    row.seen = false;
    const float* mrow =
        (kMask && valid) ? p.mask + u.b * p.m_sb + u.h * p.m_sh + (int64_t)i * p.m_ss : nullptr;
    const bool few = !kMask && prefill_short_tile(p, u, w);
    const bool split = kType == 0 && few;
    for (int j = 0; j < n; ++j, ++sj)
      if (!prefill_softmax_tile<D, kType, kMask>(PrefillSig{bars, w}, s_tmem, o_tmem, j, sj,
                                                 (u.kt0 + j) * kPrefillBN, sl2, row, mrow,
                                                 u.len_k, few, split))
        return;
    // Epilogue: wait for the last P V, read O, release O, normalise, store.
    if (!warp_wait(&bars->o_full[w], units & 1, abort, 22 + w)) return;
    ++units;
    tc_fence_after();
    uint32_t o[D];
    if constexpr (D == 128) {
      tmem_load128(o_tmem, o);
    } else {
#pragma unroll
      for (int c = 0; c < D; c += 32) tmem_load<32>(o_tmem + c, o + c);
    }
    tc_fence_before();
    mbar_arrive(&bars->o_empty[w]);
    // A row that saw no key: O = 0, LSE = -inf (polynomial exponentials of
    // masked scores are tiny but not 0, so the sums alone cannot tell).
    if (!row.seen) row.l_run = row.l_rnd = 0.f;
    const float m_use = (row.m_run == -INFINITY) ? 0.f : row.m_run;
    const float denom = row.l_rnd + (has_sink ? ex2(sink2 - m_use) : 0.f);
    const float inv = (denom > 0.f && row.seen) ? v_scale / denom : 0.f;
    constexpr bool kOutF16 = kType == 1;
    auto word = [&](int c) {
      return pack2<kOutF16>(__uint_as_float(o[2 * c]) * inv, __uint_as_float(o[2 * c + 1]) * inv);
    };
    const int i0 = i - r;
    const bool staged = i0 + kPrefillBM <= u.len_q;
    if (!turn_begin()) return;
    if (staged) {
      // row r into the staging tile: 64-column chunks, 16-byte pieces
      // permuted by row (the 128-byte swizzle of the tensor map)
      uint8_t* srow = smem + C::kOStageOff + r * 128;
#pragma unroll
      for (int c = 0; c < C::kOutChunks; ++c)
#pragma unroll
        for (int x = 0; x < 8; ++x)
          *reinterpret_cast<uint4*>(srow + c * C::kChunkBytes + ((x ^ (r & 7)) << 4)) =
              make_uint4(word(32 * c + 4 * x), word(32 * c + 4 * x + 1),
                         word(32 * c + 4 * x + 2), word(32 * c + 4 * x + 3));
    } else if (valid) {
#pragma unroll
      for (int c = 0; c < D / 8; ++c)
        reinterpret_cast<uint4*>(orow)[c] =
            make_uint4(word(4 * c), word(4 * c + 1), word(4 * c + 2), word(4 * c + 3));
    }
    if (!turn_end(staged, u, i0)) return;
    if (valid) {
      if (lrow) *lrow = row.l_run > 0.f ? (m_use + log2f(row.l_run)) * kLn2 : -INFINITY;
    }
  }
  if (r == 0) bulk_wait_all();  // this warpgroup's output stores have completed
}

// 16-bit inputs only: the output store warp (warp 10, one thread). For every
// unit, in the softmax warpgroups' order of turns (warpgroup 0, then 1), it
// waits for the staged tile, stores it with TMA when it is a whole tile,
// waits until the stores have read the staging tile and passes the turn on.
// The softmax warps never wait on the store.
template <int D, int kType>
DEVI void prefill_store(const PrefillParams& p, const CUtensorMap* mo, uint8_t* smem,
                        PrefillBarriers* bars) {
  using C = PrefillCfg<D, kType>;
  volatile int* abort = &bars->abort;
  int ouse = 0;
  for (int k = 0;; ++k) {
    const int slot = k % kUnitRing;
    if (!mbar_wait(&bars->unit_full[slot], (k / kUnitRing) & 1, abort, 29)) break;
    const int t = *reinterpret_cast<volatile int32_t*>(&bars->unit_idx[slot]);
    mbar_arrive(&bars->unit_empty[slot]);
    if (t < 0) break;
    bool ok = true;
    for (int w = 0; w < 2 && ok; ++w, ++ouse) {
      ok = mbar_wait(&bars->ostage_full, ouse & 1, abort, 30);
      if (!ok) break;
      if (*reinterpret_cast<volatile int32_t*>(&bars->ostage_store)) {
        const int c1 = bars->ostage_c1, c2 = bars->ostage_c2, c3 = bars->ostage_c3;
#pragma unroll
        for (int c = 0; c < C::kOutChunks; ++c)
          tma_store_4d(mo, smem + C::kOStageOff + c * C::kChunkBytes, c * 64, c1, c2, c3);
        bulk_commit();
        bulk_wait_read<0>();  // the staging tile has been read
      }
      mbar_arrive(&bars->ostage_free);
    }
    if (!ok) break;
  }
  bulk_wait_all();
}

template <int D, int kType, bool kMask>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap map_q,
                   const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v,
                   const __grid_constant__ CUtensorMap map_o, const PrefillParams p) {
  using C = PrefillCfg<D, kType>;
  // 128-byte swizzled TMA tiles need 1024-byte aligned shared memory. The
  // layout leaves no slack for aligning at run time (the tiles take 224 KB),
  // so a misaligned base is reported and the CTA exits before any barrier.
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) raise_error(ATTN_DEVERR_SMEM_ALIGN, 1);
    return;
  }
  PrefillBarriers* bars = reinterpret_cast<PrefillBarriers*>(smem + C::kBarOff);
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kUnitRing; ++i) {
      mbar_init(&bars->unit_full[i], 1);
      // released by the MMA warp, the 8 softmax warps and the 2 conversion
      // warps (FP8) or the output store warp (16-bit inputs)
      mbar_init(&bars->unit_empty[i], 9 + (C::kFp8 ? 2 : 1));
    }
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], C::kFp8 ? 64 : 1);  // FP8: released by the 64 converters
    }
    for (int s = 0; s < C::kVHStages; ++s) {
      mbar_init(&bars->vh_full[s], 64);
      mbar_init(&bars->vh_empty[s], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&bars->s_full[w], 1);
      mbar_init(&bars->p_head[w], 128);
      mbar_init(&bars->p_full[w], 128);
      mbar_init(&bars->o_full[w], 1);
      mbar_init(&bars->o_empty[w], 128);
    }
    mbar_init(&bars->ostage_full, 128);
    mbar_init(&bars->ostage_free, 1);
    mbar_init(&bars->mma_drain, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&bars->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < 8) {
    regs_inc<kPrefillSoftmaxRegs>();
    prefill_softmax<D, kType, kMask>(p, &map_o, smem, bars, tmem, warp >> 2);
  } else {
    regs_dec<kPrefillOtherRegs>();
    if (warp == 8) {
      if (elect_lane0()) prefill_producer<D, kType>(p, &map_q, &map_k, &map_v, smem, bars);
    } else if (warp == 9) {
      prefill_mma<D, kType, kMask>(p, smem, bars, tmem);  // whole warp, one lane issues
    } else if constexpr (C::kFp8) {
      prefill_convert<D, kType>(p, smem, bars);
    } else if (warp == 10) {
      if (elect_lane0()) prefill_store<D, kType>(p, &map_o, smem, bars);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace attn
