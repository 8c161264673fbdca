// Split-KV combine (MATE "Attention", FMHA notes: flash_attn_combine merges
// the partial outputs and log-sum-exp buffers of a split computation).
//
// With sink-free partials (O_s, LSE_s) over disjoint key sets:
//   LSE = ln sum_s e^{LSE_s},   O = sum_s e^{LSE_s - LSE} O_s,
// and, if a sink is given, O <- O / (1 + e^{sink - LSE}) once after the merge
// (the sink formula of CANN "flash_attn", 计算公式, with the keys-only LSE).
// Splits with LSE_s = -inf weigh 0; if all are -inf, O = 0 and LSE = -inf.
// One warp per output row; lanes split the D_v columns.
#pragma once

#include "common.cuh"
#include "decode_paged.cuh"
#include "sched.cuh"

namespace attn {

constexpr int kCombineMaxSplits = 1024;

// Merges n partial rows; `lse_at(k)` and `o_at(k)` (a pointer to D_v floats)
// give split k. Writes D_v outputs through `store(col, value)`; returns LSE.
template <typename LseAt, typename OAt, typename Store>
DEVI float combine_row(int n, int dv, float sink, bool has_sink, LseAt lse_at, OAt o_at,
                       Store store) {
  const int lane = threadIdx.x & 31;
  float M = -INFINITY;
  for (int k = lane; k < n; k += 32) M = fmaxf(M, lse_at(k));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float m_use = (M == -INFINITY) ? 0.f : M;
  float tot = 0.f;
  for (int k = lane; k < n; k += 32) {
    const float l = lse_at(k);
    tot += (l == -INFINITY) ? 0.f : ex2((l - m_use) * kLog2e);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  const float lse = tot > 0.f ? m_use + logf(tot) : -INFINITY;
  float factor = tot > 0.f ? 1.f / tot : 0.f;
  if (has_sink && tot > 0.f) factor *= 1.f / (1.f + ex2((sink - lse) * kLog2e));
  for (int c0 = lane * 4; c0 < dv; c0 += 128) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k = 0; k < n; ++k) {
      const float l = lse_at(k);
      if (l == -INFINITY) continue;
      const float w = ex2((l - m_use) * kLog2e);
      const float4 v = *reinterpret_cast<const float4*>(o_at(k) + c0);
      acc[0] += w * v.x;
      acc[1] += w * v.y;
      acc[2] += w * v.z;
      acc[3] += w * v.w;
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) store(c0 + x, acc[x] * factor);
  }
  return lse;
}

// Merges the split segments of a paged decode (metadata layout).
template <int D, bool kFp16>
__global__ void __launch_bounds__(256) decode_combine_kernel(const DecodeParams p) {
  using OutT = typename std::conditional<kFp16, __half, __nv_bfloat16>::type;
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int s = gw / kDecRows, r = gw % kDecRows;
  if (s >= p.num_segs) return;
  if (!(meta_matches(p.meta, ATTN_SCHED_MHA, p.batch, p.seqlen_q, p.heads_q, p.heads_kv,
                     p.page_size, p.num_segs, kDecTileKeys, D, D) &&
        p.meta[kMetaNumCtas] == p.num_ctas && p.meta[kMetaNewKeys] == p.seqlen_new))
    return;  // the decode kernel has reported the mismatch
  const MetaLayout ml(p.num_ctas, p.num_segs);
  const int ns = p.meta[ml.seg_nsplit + s];
  if (ns == 1) return;  // written by the decode kernel
  DecodeSeg sg;
  sg.b = s / p.segs_per_seq;
  const int rem = s - sg.b * p.segs_per_seq;
  sg.g = rem / p.n_rsub;
  sg.rsub = rem - sg.g * p.n_rsub;
  const int rr = sg.rsub * kDecRows + r;
  if (rr >= p.rows) return;
  const int i = rr / p.group, h = sg.g * p.group + rr % p.group;
  const int slot0 = ns > 1 ? p.meta[ml.seg_slot + s] : 0;
  OutT* dst = reinterpret_cast<OutT*>(p.out) + sg.b * p.o_sb + i * p.o_ss + h * p.o_sh;
  const float lse = combine_row(
      ns, D, p.sink ? p.sink[h] : 0.f, p.sink != nullptr,
      [&](int k) { return p.ws_lse[(int64_t)(slot0 + k) * kDecRows + r]; },
      [&](int k) { return p.ws_o + ((int64_t)(slot0 + k) * kDecRows + r) * D; },
      [&](int c, float v) { store_out(dst + c, v); });
  if (p.lse && (threadIdx.x & 31) == 0)
    p.lse[((int64_t)sg.b * p.heads_q + h) * p.seqlen_q + i] = lse;
}

// attn_combine: dense partial layout
//   out_partial (num_splits, B, S, H, D_v), lse_partial (num_splits, B, H, S).
struct CombineParams {
  const float* o_part;
  const float* lse_part;
  void* out;
  float* lse;
  const int32_t* nsplit_per_seq;
  const float* sink;
  int32_t num_splits, batch, seqlen_q, heads, dv;
  int64_t o_sb, o_ss, o_sh;
};

template <bool kFp16>
__global__ void __launch_bounds__(256) combine_kernel(const CombineParams p) {
  using OutT = typename std::conditional<kFp16, __half, __nv_bfloat16>::type;
  const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t rows = (int64_t)p.batch * p.seqlen_q * p.heads;
  if (gw >= rows) return;
  const int h = gw % p.heads;
  const int i = (gw / p.heads) % p.seqlen_q;
  const int b = gw / ((int64_t)p.heads * p.seqlen_q);
  int n = p.num_splits;
  if (p.nsplit_per_seq) n = max(0, min(n, p.nsplit_per_seq[b]));
  const int64_t split_o = (int64_t)p.batch * p.seqlen_q * p.heads * p.dv;
  const int64_t split_l = (int64_t)p.batch * p.heads * p.seqlen_q;
  const int64_t orow = (((int64_t)b * p.seqlen_q + i) * p.heads + h) * p.dv;
  const int64_t lrow = ((int64_t)b * p.heads + h) * p.seqlen_q + i;
  OutT* dst = reinterpret_cast<OutT*>(p.out) + b * p.o_sb + i * p.o_ss + h * p.o_sh;
  const float lse = combine_row(
      n, p.dv, p.sink ? p.sink[h] : 0.f, p.sink != nullptr,
      [&](int k) { return p.lse_part[k * split_l + lrow]; },
      [&](int k) { return p.o_part + k * split_o + orow; },
      [&](int c, float v) { store_out(dst + c, v); });
  if (p.lse && (threadIdx.x & 31) == 0) p.lse[lrow] = lse;
}

}  // namespace attn
