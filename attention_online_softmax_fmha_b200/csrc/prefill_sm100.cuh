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
// Design (one CTA per SM, persistent over (q-tile, batch, head) work tiles,
// heaviest q tiles first):
//   warp 4      TMA producer: Q tile (128 rows) and a ring of K/V tiles of
//               128 keys, 128-byte swizzled, one head per box.
//   warp 5      TMEM owner and MMA issuer (one thread): S = Q K^T into one of
//               two TMEM S buffers (128 x 128 fp32), then O += P V with P read
//               from TMEM (bf16, written over its S buffer) and V from smem.
//   warps 0-3   softmax: thread r owns query row r (= TMEM lane r). Online
//               softmax in the log2 domain: running max m, running sum l;
//               O in TMEM is rescaled only when the max grows by more than
//               2^8 (exact after the final division by l).
// Every mbarrier wait is bounded; a timeout raises ATTN_DEVERR_TIMEOUT, the
// roles unwind, in-flight copies and MMAs are drained and TMEM is freed.
#pragma once

#include "common.cuh"

namespace attn {

struct PrefillParams {
  void* out;
  float* lse;
  const int32_t* cu_q;
  const int32_t* cu_k;
  const float* sink;
  const float* q_descale;
  const float* k_descale;
  const float* v_descale;
  int64_t o_sb, o_ss, o_sh;
  int64_t lse_sb, lse_sh;
  int32_t batch;
  int32_t seqlen_q;     // padded S_q (unused for varlen)
  int32_t seqlen_k;
  int32_t num_q_tiles;  // ceil(max_seqlen_q / 128)
  int32_t num_heads_q;
  int32_t num_heads_kv;
  int32_t group;        // H_q / H_kv
  int32_t total_tiles;
  float scale_log2;     // scale * log2(e)
  int32_t causal;
  int32_t window_left;
  int32_t window_right;
};

constexpr int kPrefillBM = 128;   // query rows per tile
constexpr int kPrefillBN = 128;   // keys per tile
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct PrefillCfg {
  static constexpr int kChunks = D / 64;                 // 128-byte column chunks
  static constexpr int kStages = (D == 64) ? 4 : 3;
  static constexpr int kChunkBytes = 128 * 128;          // 128 rows x 128 bytes
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kTileBytes;
  static constexpr int kVOff = kKOff + kStages * kTileBytes;
  static constexpr int kBarOff = kVOff + kStages * kTileBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;  // + barriers, + alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemS0 = 0, kTmemS1 = 128, kTmemO = 256;
};

struct PrefillBarriers {
  uint64_t q_full, q_empty;
  uint64_t k_full[4], v_full[4], kv_empty[4];
  uint64_t s_full[2], p_full[2];
  uint64_t o_full, o_empty;
  uint64_t mma_drain;
  uint32_t tmem_base;
  int32_t abort;
};

struct PrefillTile {
  int b, h, m;
  int len_q, len_k;
  int row_q, row_k;  // first packed row of this sequence (0 for padded)
  int bcoord;        // batch coordinate of the tensor maps (0 for varlen)
  int kt0, kt1;      // key tiles [kt0, kt1)
};

// Maps a linear work index to a tile; returns false for tiles past the end
// of their sequence. Every role calls this with the same t and gets the same
// answer, so all roles skip the same tiles.
DEVI bool prefill_tile(const PrefillParams& p, int t, PrefillTile& ti) {
  const int bh = p.batch * p.num_heads_q;
  const int mr = t / bh;
  const int rem = t - mr * bh;
  ti.b = rem / p.num_heads_q;
  ti.h = rem - ti.b * p.num_heads_q;
  ti.m = p.num_q_tiles - 1 - mr;
  if (p.cu_q != nullptr) {
    ti.row_q = p.cu_q[ti.b];
    ti.len_q = p.cu_q[ti.b + 1] - ti.row_q;
    ti.row_k = p.cu_k[ti.b];
    ti.len_k = p.cu_k[ti.b + 1] - ti.row_k;
    ti.bcoord = 0;
  } else {
    ti.row_q = ti.row_k = 0;
    ti.len_q = p.seqlen_q;
    ti.len_k = p.seqlen_k;
    ti.bcoord = ti.b;
  }
  const int q0 = ti.m * kPrefillBM;
  if (q0 >= ti.len_q) return false;
  const int q1 = min(q0 + kPrefillBM, ti.len_q) - 1;
  const int delta = ti.len_k - ti.len_q;
  int lo = 0, hi = ti.len_k - 1;
  if (p.window_left >= 0) lo = max(lo, q0 + delta - p.window_left);
  if (p.causal) hi = min(hi, q1 + delta);
  if (p.window_right >= 0) hi = min(hi, q1 + delta + p.window_right);
  if (hi < lo) {
    ti.kt0 = ti.kt1 = 0;
  } else {
    ti.kt0 = lo / kPrefillBN;
    ti.kt1 = hi / kPrefillBN + 1;
  }
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

// ---------------------------------------------------------------------------
// Producer warp (one thread)
// ---------------------------------------------------------------------------
template <int D>
DEVI void prefill_producer(const PrefillParams& p, const CUtensorMap* mq, const CUtensorMap* mk,
                           const CUtensorMap* mv, uint8_t* smem, PrefillBarriers* bars) {
  using C = PrefillCfg<D>;
  volatile int* abort = &bars->abort;
  tma_prefetch_desc(mq);
  tma_prefetch_desc(mk);
  tma_prefetch_desc(mv);
  int it = 0, nq = 0;
  for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x) {
    PrefillTile ti;
    if (!prefill_tile(p, t, ti)) continue;
    const int n = ti.kt1 - ti.kt0;
    if (n <= 0) continue;
    const int hk = ti.h / p.group;
    if (nq > 0 && !mbar_wait(&bars->q_empty, (nq - 1) & 1, abort, 1)) goto drain;
    mbar_expect_tx(&bars->q_full, C::kTileBytes);
#pragma unroll
    for (int c = 0; c < C::kChunks; ++c)
      tma_load_4d(smem + C::kQOff + c * C::kChunkBytes, mq, &bars->q_full, c * 64, ti.h,
                  ti.row_q + ti.m * kPrefillBM, ti.bcoord);
    ++nq;
    for (int j = 0; j < n; ++j, ++it) {
      const int s = it % C::kStages;
      if (it >= C::kStages &&
          !mbar_wait(&bars->kv_empty[s], ((it / C::kStages) - 1) & 1, abort, 2))
        goto drain;
      const int row = ti.row_k + (ti.kt0 + j) * kPrefillBN;
      mbar_expect_tx(&bars->k_full[s], C::kTileBytes);
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_4d(smem + C::kKOff + s * C::kTileBytes + c * C::kChunkBytes, mk,
                    &bars->k_full[s], c * 64, hk, row, ti.bcoord);
      mbar_expect_tx(&bars->v_full[s], C::kTileBytes);
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_4d(smem + C::kVOff + s * C::kTileBytes + c * C::kChunkBytes, mv,
                    &bars->v_full[s], c * 64, hk, row, ti.bcoord);
    }
  }
drain:
  // Wait (bounded, abort flag ignored) for the copies this thread may still
  // have in flight, so none lands in shared memory after the CTA exits.
  {
    int zero = 0;
    if (nq > 0) mbar_wait(&bars->q_full, (nq - 1) & 1, &zero, 3);
    for (int i = max(0, it - C::kStages); i < it; ++i) {
      mbar_wait(&bars->k_full[i % C::kStages], (i / C::kStages) & 1, &zero, 3);
      mbar_wait(&bars->v_full[i % C::kStages], (i / C::kStages) & 1, &zero, 3);
    }
  }
}

// ---------------------------------------------------------------------------
// MMA warp (one thread issues)
// ---------------------------------------------------------------------------
template <int D, bool kFp16>
DEVI void prefill_mma(const PrefillParams& p, uint8_t* smem, PrefillBarriers* bars,
                      uint32_t tmem) {
  using C = PrefillCfg<D>;
  volatile int* abort = &bars->abort;
  constexpr int fmt = kFp16 ? 0 : 1;
  constexpr uint32_t idesc_qk = make_idesc(128, kPrefillBN, fmt, 0, 0);
  constexpr uint32_t idesc_pv = make_idesc(128, 64, fmt, 0, 1);
  const uint32_t q_base = smem_u32(smem + C::kQOff);
  const uint32_t k_base = smem_u32(smem + C::kKOff);
  const uint32_t v_base = smem_u32(smem + C::kVOff);
  int it = 0, sj = 0, nq = 0, o_tiles = 0;

  auto issue_pv = [&](int jj, int tile_it, int tile_sj) -> bool {
    const int b = (tile_sj + jj) & 1;
    const int s = (tile_it + jj) % C::kStages;
    if (!mbar_wait(&bars->p_full[b], ((tile_sj + jj) >> 1) & 1, abort, 11)) return false;
    if (!mbar_wait(&bars->v_full[s], ((tile_it + jj) / C::kStages) & 1, abort, 12)) return false;
    if (jj == 0 && o_tiles > 0 &&
        !mbar_wait(&bars->o_empty, (o_tiles - 1) & 1, abort, 13))
      return false;
    tc_fence_after();
    const uint32_t s_tmem = tmem + (b ? C::kTmemS1 : C::kTmemS0);
    const uint32_t vs = v_base + s * C::kTileBytes;
#pragma unroll
    for (int kk = 0; kk < kPrefillBN / 16; ++kk) {
#pragma unroll
      for (int dc = 0; dc < C::kChunks; ++dc) {
        const uint64_t bdesc = sdesc_sw128(vs + dc * C::kChunkBytes + kk * 16 * 128, 1024, 1024);
        mma_f16_ts(tmem + C::kTmemO + dc * 64, s_tmem + kk * 8, bdesc, idesc_pv,
                   (jj > 0 || kk > 0) ? 1u : 0u);
      }
    }
    tc_commit(&bars->o_full);
    tc_commit(&bars->kv_empty[s]);
    return true;
  };

  for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x) {
    PrefillTile ti;
    if (!prefill_tile(p, t, ti)) continue;
    const int n = ti.kt1 - ti.kt0;
    if (n <= 0) continue;
    if (!mbar_wait(&bars->q_full, nq & 1, abort, 10)) goto drain;
    ++nq;
    for (int j = 0; j < n; ++j) {
      const int s = (it + j) % C::kStages;
      const int b = (sj + j) & 1;
      if (!mbar_wait(&bars->k_full[s], ((it + j) / C::kStages) & 1, abort, 14)) goto drain;
      tc_fence_after();
      const uint32_t s_tmem = tmem + (b ? C::kTmemS1 : C::kTmemS0);
      const uint32_t ks = k_base + s * C::kTileBytes;
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k >> 2) * C::kChunkBytes + (k & 3) * 32;
        mma_f16_ss(s_tmem, sdesc_sw128(q_base + off, 16, 1024), sdesc_sw128(ks + off, 16, 1024),
                   idesc_qk, k > 0 ? 1u : 0u);
      }
      tc_commit(&bars->s_full[b]);
      if (j == n - 1) tc_commit(&bars->q_empty);
      if (j > 0 && !issue_pv(j - 1, it, sj)) goto drain;
    }
    if (!issue_pv(n - 1, it, sj)) goto drain;
    it += n;
    sj += n;
    ++o_tiles;
  }
drain : {
  // All issued MMAs must finish before TMEM is released.
  int zero = 0;
  tc_commit(&bars->mma_drain);
  mbar_wait(&bars->mma_drain, 0, &zero, 15);
}
}

// ---------------------------------------------------------------------------
// Softmax warpgroup (warps 0-3): one query row per thread
// ---------------------------------------------------------------------------
template <int D, bool kFp16>
DEVI void prefill_softmax(const PrefillParams& p, PrefillBarriers* bars, uint32_t tmem) {
  using C = PrefillCfg<D>;
  volatile int* abort = &bars->abort;
  const int r = threadIdx.x;  // 0..127
  const uint32_t lane = (uint32_t)(r & ~31) << 16;
  int sj = 0, pv = 0;
  for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x) {
    PrefillTile ti;
    if (!prefill_tile(p, t, ti)) continue;
    const int n = ti.kt1 - ti.kt0;
    const int i = ti.m * kPrefillBM + r;
    const bool valid = i < ti.len_q;
    using OutT = typename std::conditional<kFp16, __half, __nv_bfloat16>::type;
    OutT* orow = reinterpret_cast<OutT*>(p.out) + ti.bcoord * p.o_sb +
                 (int64_t)(ti.row_q + i) * p.o_ss + (int64_t)ti.h * p.o_sh;
    float* lrow = p.lse ? p.lse + ti.b * p.lse_sb + ti.h * p.lse_sh + (ti.row_q + i) : nullptr;
    if (n <= 0) {
      if (valid) {
        uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(orow)[c] = z;
        if (lrow) *lrow = -INFINITY;
      }
      continue;
    }
    int lo_i, hi_i;
    row_key_range(p, i, ti.len_q, ti.len_k, lo_i, hi_i);
    const float sl2 = p.scale_log2;
    const bool has_sink = p.sink != nullptr;
    const float sink2 = has_sink ? p.sink[ti.h] * kLog2e : -INFINITY;
    float m_run = sink2;
    float l_run = 0.f;  // sum of the fp32 P (for the LSE)
    float l_rnd = 0.f;  // sum of the rounded P the MMA consumes (for O)

    for (int j = 0; j < n; ++j) {
      const int b = (sj + j) & 1;
      if (!warp_wait(&bars->s_full[b], ((sj + j) >> 1) & 1, abort, 20)) return;
      tc_fence_after();
      const uint32_t s_tmem = tmem + (b ? C::kTmemS1 : C::kTmemS0) + lane;
      uint32_t s[kPrefillBN];
#pragma unroll
      for (int c = 0; c < kPrefillBN; c += 32) tmem_load<32>(s_tmem + c, s + c);
      const int k0 = (ti.kt0 + j) * kPrefillBN;
      if (!(k0 >= lo_i && k0 + kPrefillBN - 1 <= hi_i)) {
#pragma unroll
        for (int c = 0; c < kPrefillBN; ++c) {
          const bool vis = (k0 + c >= lo_i) && (k0 + c <= hi_i);
          if (!vis) s[c] = __float_as_uint(-INFINITY);
        }
      }
      float tmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < kPrefillBN; ++c) tmax = fmaxf(tmax, __uint_as_float(s[c]));
      const float mx = tmax * sl2;
      if (j > 0) {
        if (!warp_wait(&bars->o_full, pv & 1, abort, 21)) return;
        ++pv;
        tc_fence_after();
      }
      // Raise the running max only when it grows by more than 2^8; O is then
      // rescaled in TMEM. tcgen05.ld/st are warp-collective, so the warp
      // rescales together, each thread with its own factor (1 if unchanged).
      // On the first tile the max is set exactly (so the row's largest P is
      // exactly 1 when it is not the sink).
      float alpha = 1.f;
      const bool grow = (j == 0) ? (mx > m_run) : (mx > m_run + kRescaleThreshold);
      if (grow) {
        if (j > 0 && m_run != -INFINITY) alpha = ex2(m_run - mx);
        m_run = mx;
        l_run *= alpha;
        l_rnd *= alpha;
      }
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          tmem_load<32>(tmem + C::kTmemO + lane + c, o);
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
          tmem_store<32>(tmem + C::kTmemO + lane + c, o);
        }
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      float lsum = 0.f, lsum_rnd = 0.f;
      uint32_t pk[kPrefillBN / 2];
#pragma unroll
      for (int c = 0; c < kPrefillBN / 2; ++c) {
        const float p0 = ex2(fmaf(__uint_as_float(s[2 * c]), sl2, -m_use));
        const float p1 = ex2(fmaf(__uint_as_float(s[2 * c + 1]), sl2, -m_use));
        pk[c] = pack2<kFp16>(p0, p1);
        // O is normalised by the sum of the rounded P that the MMA consumes:
        // the weights then stay a convex combination and the rounding error
        // scales with the spread of V, not with |O|. The LSE uses the fp32 sum.
        lsum += p0 + p1;
        lsum_rnd += sum2<kFp16>(pk[c]);
      }
      l_run += lsum;
      l_rnd += lsum_rnd;
      const uint32_t p_tmem = tmem + (b ? C::kTmemS1 : C::kTmemS0) + lane;
      tmem_store<32>(p_tmem, pk);
      tmem_store<32>(p_tmem + 32, pk + 32);
      tmem_store_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_full[b]);
    }
    sj += n;
    // Epilogue: wait for the last P V, read O, release O, normalise, store.
    if (!warp_wait(&bars->o_full, pv & 1, abort, 22)) return;
    ++pv;
    tc_fence_after();
    uint32_t o[D];
#pragma unroll
    for (int c = 0; c < D; c += 32) tmem_load<32>(tmem + C::kTmemO + lane + c, o + c);
    tc_fence_before();
    mbar_arrive(&bars->o_empty);
    const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
    const float denom = l_rnd + (has_sink ? ex2(sink2 - m_use) : 0.f);
    const float inv = denom > 0.f ? 1.f / denom : 0.f;
    if (valid) {
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        uint4 w;
        w.x = pack2<kFp16>(__uint_as_float(o[8 * c + 0]) * inv, __uint_as_float(o[8 * c + 1]) * inv);
        w.y = pack2<kFp16>(__uint_as_float(o[8 * c + 2]) * inv, __uint_as_float(o[8 * c + 3]) * inv);
        w.z = pack2<kFp16>(__uint_as_float(o[8 * c + 4]) * inv, __uint_as_float(o[8 * c + 5]) * inv);
        w.w = pack2<kFp16>(__uint_as_float(o[8 * c + 6]) * inv, __uint_as_float(o[8 * c + 7]) * inv);
        reinterpret_cast<uint4*>(orow)[c] = w;
      }
      if (lrow) *lrow = l_run > 0.f ? (m_use + log2f(l_run)) * kLn2 : -INFINITY;
    }
  }
}

template <int D, bool kFp16>
__global__ void __launch_bounds__(192, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap map_q,
                   const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const PrefillParams p) {
  using C = PrefillCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  PrefillBarriers* bars = reinterpret_cast<PrefillBarriers*>(smem + C::kBarOff);
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->p_full[b], 128);
    }
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->o_empty, 128);
    mbar_init(&bars->mma_drain, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(&bars->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < 4) {
    prefill_softmax<D, kFp16>(p, bars, tmem);
  } else if (warp == 4) {
    if (elect_lane0()) prefill_producer<D>(p, &map_q, &map_k, &map_v, smem, bars);
  } else {
    if (elect_lane0()) prefill_mma<D, kFp16>(p, smem, bars, tmem);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace attn
