// Prefill on a pair of CTAs (tcgen05 cta_group::2): bf16 inputs, D = 128,
// no additive mask. Same results as prefill_kernel (CANN "flash_attn",
// 计算公式: O with the sink in the max and denominator, keys-only LSE; causal
// and window masks of MindSpore Lite "flash_attention"); a different split of
// the work over the SMs.
//
// Why two CTAs: in the one-CTA kernel each S MMA (M=128, N=128, both operands
// in shared memory) needs the SM's whole shared-memory read bandwidth, so the
// P V operand reads and the TMA writes of the next tiles slow it down. Here a
// cluster of two CTAs on two SMs runs each MMA as one M=256 instruction:
// every CTA supplies its own 128 query rows (A) and half of B -- 64 of the
// 128 keys of a K tile for S = Q K^T, 64 of the 128 columns of a V tile for
// O += P V -- so each SM reads and loads half the K and V bytes per MMA.
//
// Work unit: 512 query rows of one (sequence, head), as two MMA tiles of 256
// rows (w = 0, 1); CTA rank r holds rows 128 r .. 128 r + 127 of each. Each
// MMA tile runs over its own key range; the K/V ring covers their union.
// Roles per CTA (384 threads):
//   warpgroups 0, 1  softmax of tile w's 128 rows of this CTA (one row per
//                    thread, TMEM lane r); as in prefill_kernel, with the
//                    P-ready and O-free signals sent to the leader CTA.
//   warp 8           TMA producer: this CTA's Q rows and halves of K and V;
//                    all copies complete on the leader's barriers. The
//                    leader's producer also takes the unit numbers and
//                    hands them to both CTAs.
//   warp 9           TMEM allocation (both CTAs); in the leader CTA also the
//                    MMA issuer, PV0_{j-1}, S0_j, PV1_{j-1}, S1_j as in
//                    prefill_kernel, each commit signalling both CTAs.
// Every wait is bounded; a timeout raises ATTN_DEVERR_TIMEOUT and both CTAs
// unwind; the leader drains its MMAs before either CTA frees TMEM.
#pragma once

#include "prefill_sm100.cuh"

namespace attn {

constexpr int kP2Unit = 4 * kPrefillBM;          // 512 query rows per unit
constexpr int kP2KStages = 4;
constexpr int kP2VStages = 4;
constexpr int kP2QTile = kPrefillBM * 128 * 2;   // 128 rows x 128 bf16: 32 KB (two 16 KB chunks)
constexpr int kP2QChunk = kPrefillBM * 128;      // 16 KB
constexpr int kP2KHalf = 64 * 128 * 2;           // 64 keys x 128 bf16: 16 KB (two 8 KB chunks)
constexpr int kP2KChunk = 64 * 128;              // 8 KB
constexpr int kP2VHalf = kPrefillBN * 64 * 2;    // 128 keys x 64 bf16: 16 KB (one chunk)
constexpr int kP2QOff = 0;
constexpr int kP2KOff = kP2QOff + 2 * kP2QTile;
constexpr int kP2VOff = kP2KOff + kP2KStages * kP2KHalf;
constexpr int kP2BarOff = kP2VOff + kP2VStages * kP2VHalf;
constexpr int kP2SmemBytes = kP2BarOff + 512;
static_assert(kP2SmemBytes <= 232448, "shared memory per CTA");

struct P2Barriers {
  uint64_t unit_full[kUnitRing], unit_empty[kUnitRing];  // unit_empty: leader only
  int32_t unit_idx[kUnitRing];
  uint64_t q_full;                        // leader: both CTAs' Q copies
  uint64_t q_empty;                       // both: the unit's last S is done
  uint64_t k_full[kP2KStages], v_full[kP2VStages];    // leader: both halves
  uint64_t k_empty[kP2KStages], v_empty[kP2VStages];  // both
  uint64_t s_full[2], o_full[2];          // both
  uint64_t p_head[2], p_full[2], o_empty[2];  // leader: 4 warps of each CTA
  uint64_t mma_drain;                     // leader
  uint32_t tmem_base;
  int32_t abort;
};
static_assert(sizeof(P2Barriers) <= 512, "barrier block");

// ---------------------------------------------------------------------------
// cta_group::2 forms (every tcgen05 instruction of the kernel uses them)
// ---------------------------------------------------------------------------
DEVI void tmem_alloc2(uint32_t* dst_smem, uint32_t ncols) {  // one warp of each CTA
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
DEVI void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
DEVI void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// M=256 across the pair: A rows 0..127 from the leader, 128..255 from the
// other CTA (each from its own shared memory or TMEM at the same address);
// B's N columns split in halves the same way; D rows land in each CTA's TMEM.
DEVI void mma2_ss_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                    uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
DEVI void mma2_ts_w(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                    uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the barrier at this offset in both CTAs when every tcgen05
// operation issued so far by this thread has completed.
DEVI void commit2_both_w(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
      "h"((unsigned short)3)
      : "memory");
}
// The same, on this CTA's barrier only.
DEVI void commit2_self_w(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}
// A tiled TMA load into this CTA's shared memory that completes on a barrier
// of either CTA of the pair (`bar_cluster`: a shared::cluster address). No
// multicast: each CTA loads its own rows.
DEVI void tma2_load_4d(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int c0, int c1,
                       int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar_cluster)
      : "memory");
}
// One thread's bounded wait with cluster-scope acquire (arrivals and
// completions come from both CTAs).
DEVI bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort, int site) {
  const uint32_t a = smem_u32(bar);
  if (mbar_test_cluster(a, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_test_cluster(a, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort) return false;
      if (globaltimer() - t0 > kWaitTimeoutNs) {
        raise_error(ATTN_DEVERR_TIMEOUT, site);
        *abort = 1;
        return false;
      }
    }
  }
}
DEVI uint32_t leader_addr(const void* p) { return mapa_shared(smem_u32(p), 0); }
DEVI void st_cluster_b32(uint32_t addr, int32_t v) {
  asm volatile("st.shared::cluster.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// ---------------------------------------------------------------------------
// Work units
// ---------------------------------------------------------------------------
struct P2Unit {
  int b, h, m;
  int len_q, len_k;
  int row_q, row_k;  // first packed row of the sequence (0 for padded)
  int bcoord;        // batch coordinate of the tensor maps (0 for varlen)
  int kt0[2], kt1[2];  // key tiles of MMA tile w (empty if kt1 <= kt0)
  int K0, K1;          // their union
};

// Unit t: rows m*512 .. m*512 + 511 of (sequence b, head h), numbered as in
// prefill_unit (last row block of every sequence and head first). False for a
// unit past its sequence's end.
template <bool kUnion>
DEVI bool p2_unit(const PrefillParams& p, int t, P2Unit& u) {
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
  if (u.m * kP2Unit >= u.len_q) return false;
  u.K0 = INT_MAX;
  u.K1 = 0;
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    u.kt0[w] = u.kt1[w] = 0;
    const int i0 = u.m * kP2Unit + w * 2 * kPrefillBM;
    if (i0 >= u.len_q) continue;
    const int i1 = min(i0 + 2 * kPrefillBM, u.len_q) - 1;
    int lo, hi, lo1, hi1;
    row_key_range(p, i0, u.len_q, u.len_k, lo, hi);
    row_key_range(p, i1, u.len_q, u.len_k, lo1, hi1);
    hi = max(hi, hi1);  // the bounds rise with the row
    if (hi < lo) continue;
    u.kt0[w] = lo / kPrefillBN;
    u.kt1[w] = hi / kPrefillBN + 1;
    u.K0 = min(u.K0, u.kt0[w]);
    u.K1 = max(u.K1, u.kt1[w]);
  }
  if (u.K1 == 0) u.K0 = 0;
  if (kUnion) {
#pragma unroll
    for (int w = 0; w < 2; ++w)
      if (u.kt1[w] > u.kt0[w]) {
        u.kt0[w] = u.K0;
        u.kt1[w] = u.K1;
      }
  }
  return true;
}

DEVI bool p2_in(const P2Unit& u, int w, int j) { return j >= u.kt0[w] && j < u.kt1[w]; }

// As prefill_short_tile, over the 256 rows of MMA tile w.
DEVI bool p2_short_tile(const PrefillParams& p, const P2Unit& u, int w) {
  const int i0 = u.m * kP2Unit + w * 2 * kPrefillBM;
  if (i0 >= u.len_q) return false;
  const int i1 = min(i0 + 2 * kPrefillBM, u.len_q) - 1;
  int lo0, hi0, lo1, hi1;
  row_key_range(p, i0, u.len_q, u.len_k, lo0, hi0);
  row_key_range(p, i1, u.len_q, u.len_k, lo1, hi1);
  return min(hi0 - lo0, hi1 - lo1) + 1 < kShortRow;
}

// Takes the k-th unit number from this CTA's ring (warp-collective) and
// releases the slot on the leader's barrier (one arrival per warp).
DEVI bool p2_take_unit(P2Barriers* bars, int k, int& t, int site) {
  const int slot = k % kUnitRing;
  if (!warp_wait_cluster(&bars->unit_full[slot], (k / kUnitRing) & 1, &bars->abort, site))
    return false;
  t = *reinterpret_cast<volatile int32_t*>(&bars->unit_idx[slot]);
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive_remote(leader_addr(&bars->unit_empty[slot]));
  return true;
}

// ---------------------------------------------------------------------------
// Producer (one thread per CTA)
// ---------------------------------------------------------------------------
template <bool kUnion>
DEVI void p2_producer(const PrefillParams& p, const CUtensorMap* mq, const CUtensorMap* mk,
                      const CUtensorMap* mv, uint8_t* smem, P2Barriers* bars, int rank) {
  volatile int* abort = &bars->abort;
  tma_prefetch_desc(mq);
  tma_prefetch_desc(mk);
  tma_prefetch_desc(mv);
  const uint32_t q_full_l = leader_addr(&bars->q_full);
  const uint32_t k_full_l = leader_addr(&bars->k_full[0]);
  const uint32_t v_full_l = leader_addr(&bars->v_full[0]);
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  int it = 0, nq = 0, k = 0;
  for (int fetched = 0;; ++fetched) {
    int t;
    P2Unit u;
    if (rank == 0) {
      // The leader takes the next number and hands it to both CTAs' roles.
      t = p.work_counter ? atomicAdd(p.work_counter, 1) : cluster + fetched * nclusters;
      if (t < p.total_units && !p2_unit<kUnion>(p, t, u)) continue;
      if (t >= p.total_units) t = -1;
      const int slot = k % kUnitRing;
      if (k >= kUnitRing &&
          !mbar_wait_cluster(&bars->unit_empty[slot], ((k / kUnitRing) - 1) & 1, abort, 5))
        goto drain;
      bars->unit_idx[slot] = t;
      mbar_arrive(&bars->unit_full[slot]);
      st_cluster_b32(mapa_shared(smem_u32(&bars->unit_idx[slot]), 1), t);
      mbar_arrive_remote(mapa_shared(smem_u32(&bars->unit_full[slot]), 1));  // after the store
    } else {
      const int slot = k % kUnitRing;
      if (!mbar_wait_cluster(&bars->unit_full[slot], (k / kUnitRing) & 1, abort, 6)) goto drain;
      t = *reinterpret_cast<volatile int32_t*>(&bars->unit_idx[slot]);
      mbar_arrive_remote(leader_addr(&bars->unit_empty[slot]));
      if (t >= 0) p2_unit<kUnion>(p, t, u);
    }
    ++k;
    if (t < 0) break;
    if (u.K1 <= u.K0) continue;
    {
      const int hk = u.h / p.group;
      if (nq > 0 && !mbar_wait_cluster(&bars->q_empty, (nq - 1) & 1, abort, 1)) goto drain;
      if (rank == 0) mbar_expect_tx(&bars->q_full, 2 * 2 * kP2QTile);  // Q0, Q1 of both CTAs
#pragma unroll
      for (int w = 0; w < 2; ++w)
#pragma unroll
        for (int c = 0; c < 2; ++c)
          tma2_load_4d(smem + kP2QOff + w * kP2QTile + c * kP2QChunk, mq, q_full_l, c * 64, u.h,
                       u.row_q + u.m * kP2Unit + w * 2 * kPrefillBM + rank * kPrefillBM,
                       u.bcoord);
      ++nq;
      for (int j = u.K0; j < u.K1; ++j, ++it) {
        const int row = u.row_k + j * kPrefillBN;
        const int sk = it % kP2KStages, sv = it % kP2VStages;
        if (it >= kP2KStages &&
            !mbar_wait_cluster(&bars->k_empty[sk], ((it / kP2KStages) - 1) & 1, abort, 2))
          goto drain;
        if (rank == 0) mbar_expect_tx(&bars->k_full[sk], 2 * kP2KHalf);
#pragma unroll
        for (int c = 0; c < 2; ++c)
          tma2_load_4d(smem + kP2KOff + sk * kP2KHalf + c * kP2KChunk, mk, k_full_l + sk * 8,
                       c * 64, hk, row + rank * 64, u.bcoord);
        if (it >= kP2VStages &&
            !mbar_wait_cluster(&bars->v_empty[sv], ((it / kP2VStages) - 1) & 1, abort, 4))
          goto drain;
        if (rank == 0) mbar_expect_tx(&bars->v_full[sv], 2 * kP2VHalf);
        tma2_load_4d(smem + kP2VOff + sv * kP2VHalf, mv, v_full_l + sv * 8, rank * 64, hk, row,
                     u.bcoord);
      }
    }
  }
drain:
  // The leader waits (bounded, abort flag ignored) for the copies of both
  // CTAs still in flight; every copy completes on its barriers.
  if (rank == 0) {
    int zero = 0;
    if (nq > 0) mbar_wait_cluster(&bars->q_full, (nq - 1) & 1, &zero, 3);
    for (int i = max(0, it - kP2KStages); i < it; ++i)
      mbar_wait_cluster(&bars->k_full[i % kP2KStages], (i / kP2KStages) & 1, &zero, 3);
    for (int i = max(0, it - kP2VStages); i < it; ++i)
      mbar_wait_cluster(&bars->v_full[i % kP2VStages], (i / kP2VStages) & 1, &zero, 3);
  }
}

// ---------------------------------------------------------------------------
// MMA warp of the leader CTA (one lane issues)
// ---------------------------------------------------------------------------
// S_w = Q_w K^T over D = 128: eight K steps of 32 bytes. Q chunks (64
// columns of 128 rows) are 16 KB apart, K chunks (64 columns of 64 keys) 8 KB.
DEVI void p2_issue_s(uint32_t d_tmem, uint64_t dq, uint64_t dk, uint32_t idesc) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t oq = (k >> 2) * (kP2QChunk >> 4) + (k & 3) * 2;
    const uint32_t ok = (k >> 2) * (kP2KChunk >> 4) + (k & 3) * 2;
    mma2_ss_w(d_tmem, dq + oq, dk + ok, idesc, k > 0 ? 1u : 0u);
  }
}

// O_w += P_w V (tile w's np-th P): the head of P once released, then the
// tail, then (split) the rounding remainder in TMEM columns 64 .. 127.
DEVI bool p2_pv(P2Barriers* bars, int w, int np, uint32_t t_o, uint32_t t_p, uint64_t dv,
                uint32_t idesc, bool first, bool split) {
  volatile int* abort = &bars->abort;
  constexpr int kHead = kSplitKeys / 16;
  if (!warp_wait_cluster(&bars->p_head[w], np & 1, abort, 16)) return false;
  tc_fence_after();
#pragma unroll
  for (int kk = 0; kk < kHead; ++kk)
    mma2_ts_w(t_o, t_p + kk * 8, dv + kk * (16 * 128 >> 4), idesc, (!first || kk > 0) ? 1u : 0u);
  if (!warp_wait_cluster(&bars->p_full[w], np & 1, abort, 11)) return false;
  tc_fence_after();
#pragma unroll
  for (int kk = kHead; kk < kPrefillBN / 16; ++kk)
    mma2_ts_w(t_o, t_p + kk * 8, dv + kk * (16 * 128 >> 4), idesc, 1u);
  if (split) {
#pragma unroll 1
    for (int kk = 0; kk < kPrefillBN / 16; ++kk)
      mma2_ts_w(t_o, t_p + kPrefillBN / 2 + kk * 8, dv + kk * (16 * 128 >> 4), idesc, 1u);
  }
  return true;
}

template <bool kUnion>
DEVI void p2_mma(const PrefillParams& p, uint8_t* smem, P2Barriers* bars, uint32_t tmem) {
  volatile int* abort = &bars->abort;
  constexpr uint32_t idesc_qk = make_idesc(256, kPrefillBN, 1, 0, 0);
  // V is MN-major; each CTA supplies one 64-column chunk (the leading byte
  // offset is unused), 8 keys x 128 bytes apart.
  constexpr uint32_t idesc_pv = make_idesc(256, 128, 1, 0, 1);
  const uint64_t dq0 = sdesc_sw128(smem_u32(smem + kP2QOff), 16, 1024);
  const uint64_t dk_base = sdesc_sw128(smem_u32(smem + kP2KOff), 16, 1024);
  const uint64_t dv_base = sdesc_sw128(smem_u32(smem + kP2VOff), kP2VHalf, 1024);
  int it = 0, nq = 0;
  int np[2] = {0, 0}, pieces[2] = {0, 0};
  for (int k = 0;; ++k) {
    int t;
    if (!p2_take_unit(bars, k, t, 9)) goto drain;
    if (t < 0) break;
    P2Unit u;
    p2_unit<kUnion>(p, t, u);
    if (u.K1 <= u.K0) continue;
    if (!warp_wait_cluster(&bars->q_full, nq & 1, abort, 10)) goto drain;
    ++nq;
    {
      const bool split[2] = {p2_short_tile(p, u, 0), p2_short_tile(p, u, 1)};
      bool started[2] = {false, false};
      for (int j = u.K0; j <= u.K1; ++j) {
        const int g = it + (j - u.K0);
        const int s = g % kP2KStages;
        const int sp = (g - 1 + kP2VStages) % kP2VStages;
        if (j < u.K1 &&
            !warp_wait_cluster(&bars->k_full[s], (g / kP2KStages) & 1, abort, 14))
          goto drain;
        if (j > u.K0 &&
            !warp_wait_cluster(&bars->v_full[sp], ((g - 1) / kP2VStages) & 1, abort, 12))
          goto drain;
        tc_fence_after();
        const uint64_t dv = dv_base + sp * (kP2VHalf >> 4);
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          // P V of tile w for key tile j - 1, then S of tile w for key tile j
          if (j > u.K0 && p2_in(u, w, j - 1)) {
            if (!started[w] && pieces[w] > 0 &&
                !warp_wait_cluster(&bars->o_empty[w], (pieces[w] - 1) & 1, abort, 13))
              goto drain;
            if (!p2_pv(bars, w, np[w], tmem + 256 + w * 128, tmem + w * 128, dv, idesc_pv,
                       !started[w], split[w]))
              goto drain;
            started[w] = true;
            ++np[w];
            if (j == u.kt1[w]) commit2_both_w(&bars->o_full[w]);
          }
          if (w == 1 && j > u.K0) commit2_both_w(&bars->v_empty[sp]);
          if (j < u.K1 && p2_in(u, w, j)) {
            p2_issue_s(tmem + w * 128, dq0 + w * (kP2QTile >> 4),
                       dk_base + s * (kP2KHalf >> 4), idesc_qk);
            commit2_both_w(&bars->s_full[w]);
          }
        }
        if (j < u.K1) {
          commit2_both_w(&bars->k_empty[s]);
          if (j == u.K1 - 1) commit2_both_w(&bars->q_empty);
        }
      }
      it += u.K1 - u.K0;
#pragma unroll
      for (int w = 0; w < 2; ++w)
        if (started[w]) ++pieces[w];
    }
  }
drain : {
  // Every MMA issued must finish before either CTA frees its TMEM.
  int zero = 0;
  commit2_self_w(&bars->mma_drain);
  warp_wait_cluster(&bars->mma_drain, 0, &zero, 15);
}
}

// ---------------------------------------------------------------------------
// Softmax warpgroups (both CTAs)
// ---------------------------------------------------------------------------
// Hand-offs with the leader's MMA warp: S of tile w is ready (a commit into
// this CTA's barrier); the head / all of P is in this CTA's TMEM (one
// arrival per warp on the leader's barrier).
struct P2Sig {
  P2Barriers* bars;
  int w;
  uint32_t head_l, full_l;
  DEVI bool wait_s(int g) const {
    return warp_wait_cluster(&bars->s_full[w], g & 1, &bars->abort, 20 + w);
  }
  DEVI void p_head() const {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive_remote(head_l);
  }
  DEVI void p_full() const {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive_remote(full_l);
  }
};

template <bool kUnion>
DEVI void p2_softmax(const PrefillParams& p, P2Barriers* bars, uint32_t tmem, int w, int rank) {
  using OutT = __nv_bfloat16;
  volatile int* abort = &bars->abort;
  const int r = threadIdx.x & 127;
  const uint32_t lane = (uint32_t)(r & ~31) << 16;
  const uint32_t s_tmem = tmem + w * 128 + lane;
  const uint32_t o_tmem = tmem + 256 + w * 128 + lane;
  const P2Sig sig{bars, w, leader_addr(&bars->p_head[w]), leader_addr(&bars->p_full[w])};
  const uint32_t o_empty_l = leader_addr(&bars->o_empty[w]);
  int sj = 0, pieces = 0;
  for (int k = 0;; ++k) {
    int t;
    if (!p2_take_unit(bars, k, t, 24 + w)) return;
    if (t < 0) break;
    P2Unit u;
    p2_unit<kUnion>(p, t, u);
    const int n = u.kt1[w] - u.kt0[w];
    const int i = u.m * kP2Unit + w * 2 * kPrefillBM + rank * kPrefillBM + r;
    const bool valid = i < u.len_q;
    OutT* orow = reinterpret_cast<OutT*>(p.out) + u.bcoord * p.o_sb +
                 (int64_t)(u.row_q + i) * p.o_ss + (int64_t)u.h * p.o_sh;
    float* lrow = p.lse ? p.lse + u.b * p.lse_sb + u.h * p.lse_sh + (u.row_q + i) : nullptr;
    if (n <= 0) {
      if (valid) {
        const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int c = 0; c < 128 / 8; ++c) reinterpret_cast<uint4*>(orow)[c] = z;
        if (lrow) *lrow = -INFINITY;
      }
      continue;
    }
    const float sl2 = p.scale_log2;
    const bool has_sink = p.sink != nullptr;
    const float sink2 = has_sink ? p.sink[u.h] * kLog2e : -INFINITY;
    PrefillRow row;
    row_key_range(p, i, u.len_q, u.len_k, row.lo, row.hi);
    row.m_run = sink2;
    row.l_run = row.l_rnd = 0.f;
    row.seen = false;
    const bool split = p2_short_tile(p, u, w);
    for (int j = 0; j < n; ++j, ++sj)
      if (!prefill_softmax_tile<128, 0, false>(sig, s_tmem, o_tmem, j, sj,
                                               (u.kt0[w] + j) * kPrefillBN, sl2, row, nullptr,
                                               u.len_k, split))
        return;
    // Epilogue: wait for the last P V, read O, release O, normalise, store.
    if (!warp_wait_cluster(&bars->o_full[w], pieces & 1, abort, 22 + w)) return;
    ++pieces;
    tc_fence_after();
    uint32_t o[128];
    tmem_load128(o_tmem, o);
    tc_fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive_remote(o_empty_l);
    if (!row.seen) row.l_run = row.l_rnd = 0.f;
    const float m_use = (row.m_run == -INFINITY) ? 0.f : row.m_run;
    const float denom = row.l_rnd + (has_sink ? ex2(sink2 - m_use) : 0.f);
    const float inv = (denom > 0.f && row.seen) ? 1.f / denom : 0.f;
    if (valid) {
#pragma unroll
      for (int c = 0; c < 128 / 8; ++c) {
        uint4 v;
        v.x = pack_bf16x2(__uint_as_float(o[8 * c + 0]) * inv, __uint_as_float(o[8 * c + 1]) * inv);
        v.y = pack_bf16x2(__uint_as_float(o[8 * c + 2]) * inv, __uint_as_float(o[8 * c + 3]) * inv);
        v.z = pack_bf16x2(__uint_as_float(o[8 * c + 4]) * inv, __uint_as_float(o[8 * c + 5]) * inv);
        v.w = pack_bf16x2(__uint_as_float(o[8 * c + 6]) * inv, __uint_as_float(o[8 * c + 7]) * inv);
        reinterpret_cast<uint4*>(orow)[c] = v;
      }
      if (lrow) *lrow = row.l_run > 0.f ? (m_use + log2f(row.l_run)) * kLn2 : -INFINITY;
    }
  }
}

template <bool kUnion>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPrefillThreads, 1)
    prefill2_kernel(const __grid_constant__ CUtensorMap map_q,
                    const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, const PrefillParams p) {
  // 128-byte swizzled TMA tiles need 1024-byte aligned shared memory; both
  // CTAs share the layout, so both leave here or neither.
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) raise_error(ATTN_DEVERR_SMEM_ALIGN, 3);
    return;
  }
  P2Barriers* bars = reinterpret_cast<P2Barriers*>(smem + kP2BarOff);
  const int warp = threadIdx.x >> 5;
  const int rank = (int)cluster_ctarank();
  if (threadIdx.x == 0) {
    for (int i = 0; i < kUnitRing; ++i) {
      mbar_init(&bars->unit_full[i], 1);
      // leader: its MMA warp and 8 softmax warps, the other CTA's producer
      // and 8 softmax warps
      mbar_init(&bars->unit_empty[i], 18);
    }
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < kP2KStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < kP2VStages; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&bars->s_full[w], 1);
      mbar_init(&bars->o_full[w], 1);
      mbar_init(&bars->p_head[w], 8);
      mbar_init(&bars->p_full[w], 8);
      mbar_init(&bars->o_empty[w], 8);
    }
    mbar_init(&bars->mma_drain, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc2(&bars->tmem_base, 512);
    tmem_relinquish2();
  }
  tc_fence_before();
  __syncthreads();
  // Both CTAs' barriers are initialised before any remote arrival or copy.
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < 8) {
    regs_inc<kPrefillSoftmaxRegs>();
    p2_softmax<kUnion>(p, bars, tmem, warp >> 2, rank);
  } else {
    regs_dec<kPrefillOtherRegs>();
    if (warp == 8) {
      if (elect_lane0()) p2_producer<kUnion>(p, &map_q, &map_k, &map_v, smem, bars, rank);
    } else if (warp == 9 && rank == 0) {
      p2_mma<kUnion>(p, smem, bars, tmem);  // whole warp, one lane issues
    }
  }

  tc_fence_before();
  __syncthreads();
  // The leader's MMAs have drained; no arrival into either CTA follows.
  cluster_sync();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc2(tmem, 512);
  }
}

}  // namespace attn
