// Host side of attn_fwd_varlen: argument checks, the Q/K/V tensor maps and
// the launch of the prefill kernel instantiation for the head dim, input
// type and mask path.
#pragma once

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "host.cuh"
#include "prefill_sm100.cuh"

namespace attn {
namespace {

// ---------------------------------------------------------------------------
// attn_fwd_varlen
// ---------------------------------------------------------------------------
template <int D, int kType, bool kMask>
attn_status_t launch_prefill(int grid, const CUtensorMap& mq, const CUtensorMap& mk,
                             const CUtensorMap& mv, const CUtensorMap& mo, const PrefillParams& p,
                             cudaStream_t stream) {
  using C = PrefillCfg<D, kType>;
  auto kernel = prefill_kernel<D, kType, kMask>;
  static std::atomic<uint64_t> configured{0};
  const attn_status_t cst = configure_per_device(configured, [&]() -> attn_status_t {
    // The warpgroups trade registers with setmaxnreg out of the block's
    // launch allocation; that split is only valid at exactly this count.
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return ATTN_ERR_CUDA;
    if (fa.numRegs != kPrefillLaunchRegs) return ATTN_ERR_UNSUPPORTED;
    return launch_status(set_smem(kernel, C::kSmemBytes));
  });
  if (cst != ATTN_OK) return cst;
  if (p.work_counter &&
      cudaMemsetAsync(p.work_counter, 0, sizeof(int32_t), stream) != cudaSuccess)
    return ATTN_ERR_CUDA;
  kernel<<<grid, kPrefillThreads, C::kSmemBytes, stream>>>(mq, mk, mv, mo, p);
  return launch_status(cudaGetLastError());
}

template <int D, int kType>
attn_status_t run_prefill(const attn_varlen_args& a, cudaStream_t stream) {
  using C = PrefillCfg<D, kType>;
  const bool varlen = a.cu_seqlens_q != nullptr;
  const CUtensorMapDataType dt = kType >= 2   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : kType == 1 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                              : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int es = C::kInBytes;
  const uint32_t bx = C::kChunkElems;
  const uint64_t rows_q = varlen ? (uint64_t)a.total_q : (uint64_t)a.max_seqlen_q;
  const uint64_t rows_k = varlen ? (uint64_t)a.total_k : (uint64_t)a.max_seqlen_k;
  const uint64_t nb = varlen ? 1 : (uint64_t)a.batch;
  const uint64_t qsb = varlen ? rows_q * a.q_stride_s : a.q_stride_b;
  const uint64_t ksb = varlen ? rows_k * a.k_stride_s : a.k_stride_b;
  const uint64_t vsb = varlen ? rows_k * a.v_stride_s : a.v_stride_b;
  // The output (TMA stores of whole 128-row tiles): bf16, or fp16 for fp16
  // inputs; 64-column boxes.
  const CUtensorMapDataType dto =
      kType == 1 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t osb = varlen ? rows_q * a.o_stride_s : a.o_stride_b;
  CUtensorMap mq, mk, mv, mo;
  if (!encode_4d(&mq, a.q, dt, es, D, a.num_heads_q, rows_q, nb, a.q_stride_h, a.q_stride_s, qsb,
                 bx, 1, 128, 1) ||
      !encode_4d(&mk, a.k, dt, es, D, a.num_heads_kv, rows_k, nb, a.k_stride_h, a.k_stride_s, ksb,
                 bx, 1, kPrefillBN, 1) ||
      !encode_4d(&mv, a.v, dt, es, D, a.num_heads_kv, rows_k, nb, a.v_stride_h, a.v_stride_s, vsb,
                 bx, 1, kPrefillBN, 1) ||
      !encode_4d(&mo, a.out, dto, 2, D, a.num_heads_q, rows_q, nb, a.o_stride_h, a.o_stride_s, osb,
                 64, 1, kPrefillBM, 1))
    return ATTN_ERR_INVALID_ARG;

  PrefillParams p;
  memset(&p, 0, sizeof(p));
  p.out = a.out;
  p.lse = a.lse;
  p.cu_q = a.cu_seqlens_q;
  p.cu_k = a.cu_seqlens_k;
  p.sink = a.sink;
  p.seqused_q = a.seqused_q;
  p.seqused_k = a.seqused_k;
  p.mask = a.mask;
  p.m_sb = a.mask_stride_b;
  p.m_sh = a.mask_stride_h;
  p.m_ss = a.mask_stride_s;
  p.q_descale = a.q_descale;
  p.k_descale = a.k_descale;
  p.v_descale = a.v_descale;
  p.o_sb = a.o_stride_b;
  p.o_ss = a.o_stride_s;
  p.o_sh = a.o_stride_h;
  p.lse_sb = varlen ? 0 : a.lse_stride_b;
  p.lse_sh = a.lse_stride_h;
  p.batch = a.batch;
  p.seqlen_q = a.max_seqlen_q;
  p.seqlen_k = a.max_seqlen_k;
  p.num_units_q = (a.max_seqlen_q + kPrefillUnit - 1) / kPrefillUnit;
  p.num_heads_q = a.num_heads_q;
  p.num_heads_kv = a.num_heads_kv;
  p.group = a.num_heads_q / a.num_heads_kv;
  const int64_t total = (int64_t)p.num_units_q * a.batch * a.num_heads_q;
  if (total > INT32_MAX) return ATTN_ERR_UNSUPPORTED;
  p.total_units = (int32_t)total;
  p.scale_log2 = a.scale * kLog2e;
  p.causal = a.causal;
  p.window_left = a.window_left;
  p.window_right = a.window_right;
  p.work_counter = a.work_counter;

  const int sms = device_sm_count();
  if (sms <= 0) return ATTN_ERR_CUDA;
  const int grid = (int)std::min<int64_t>(total, sms);
  // The additive-mask path is a separate instantiation, so the common path
  // carries none of its registers.
  return a.mask ? launch_prefill<D, kType, true>(grid, mq, mk, mv, mo, p, stream)
                : launch_prefill<D, kType, false>(grid, mq, mk, mv, mo, p, stream);
}

attn_status_t check_varlen(const attn_varlen_args* a) {
  if (!a) return ATTN_ERR_INVALID_ARG;
  if (!a->q || !a->k || !a->v || !a->out) return ATTN_ERR_INVALID_ARG;
  const bool varlen = a->cu_seqlens_q != nullptr;
  if (varlen != (a->cu_seqlens_k != nullptr)) return ATTN_ERR_INVALID_ARG;
  if (a->batch <= 0 || a->max_seqlen_q <= 0 || a->max_seqlen_k <= 0) return ATTN_ERR_INVALID_ARG;
  if (varlen && (a->total_q <= 0 || a->total_k <= 0)) return ATTN_ERR_INVALID_ARG;
  if (a->num_heads_q <= 0 || a->num_heads_kv <= 0 || a->num_heads_q % a->num_heads_kv != 0)
    return ATTN_ERR_INVALID_ARG;
  if (a->head_dim_qk <= 0 || a->head_dim_v <= 0) return ATTN_ERR_INVALID_ARG;
  if (!(a->scale > 0.f) || !std::isfinite(a->scale)) return ATTN_ERR_INVALID_ARG;
  if (a->window_left < -1 || a->window_right < -1) return ATTN_ERR_INVALID_ARG;
  if (a->dtype < ATTN_DTYPE_BF16 || a->dtype > ATTN_DTYPE_E5M2) return ATTN_ERR_INVALID_ARG;
  const bool fp8 = a->dtype == ATTN_DTYPE_E4M3 || a->dtype == ATTN_DTYPE_E5M2;
  if (fp8 && (!a->q_descale || !a->k_descale || !a->v_descale)) return ATTN_ERR_INVALID_ARG;
  const int es = fp8 ? 1 : 2;
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->out))
    return ATTN_ERR_INVALID_ARG;
  if (!stride_ok(a->q_stride_s, es) || !stride_ok(a->q_stride_h, es) ||
      !stride_ok(a->k_stride_s, es) || !stride_ok(a->k_stride_h, es) ||
      !stride_ok(a->v_stride_s, es) || !stride_ok(a->v_stride_h, es) ||
      !stride_ok(a->o_stride_s, 2) || !stride_ok(a->o_stride_h, 2))
    return ATTN_ERR_INVALID_ARG;
  if (!varlen && (!stride_ok(a->q_stride_b, es) || !stride_ok(a->k_stride_b, es) ||
                  !stride_ok(a->v_stride_b, es) || !stride_ok(a->o_stride_b, 2)))
    return ATTN_ERR_INVALID_ARG;
  if (a->head_dim_qk != a->head_dim_v) return ATTN_ERR_UNSUPPORTED;
  if (a->head_dim_qk != 64 && a->head_dim_qk != 128) return ATTN_ERR_UNSUPPORTED;
  if (fp8 && a->head_dim_qk != 128) return ATTN_ERR_UNSUPPORTED;
  if (varlen && (a->seqused_q || a->seqused_k)) return ATTN_ERR_INVALID_ARG;  // padded only
  if (reinterpret_cast<uintptr_t>(a->work_counter) & 3u) return ATTN_ERR_INVALID_ARG;
  if (a->mask) {
    if (a->mask_stride_b < 0 || a->mask_stride_h < 0 || a->mask_stride_s < 0)
      return ATTN_ERR_INVALID_ARG;
    // mask rows are read as 16-byte vectors
    if (!aligned16(a->mask) || a->mask_stride_s % 4 || a->mask_stride_h % 4 ||
        a->mask_stride_b % 4)
      return ATTN_ERR_INVALID_ARG;
  }
  return ATTN_OK;
}

attn_status_t varlen_entry(const attn_varlen_args* args, void* stream) {
  const attn_status_t st = check_varlen(args);
  if (st != ATTN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = args->head_dim_qk;
  switch (args->dtype) {
    case ATTN_DTYPE_BF16:
      return D == 64 ? run_prefill<64, 0>(*args, s) : run_prefill<128, 0>(*args, s);
    case ATTN_DTYPE_FP16:
      return D == 64 ? run_prefill<64, 1>(*args, s) : run_prefill<128, 1>(*args, s);
    case ATTN_DTYPE_E4M3:
      return run_prefill<128, 2>(*args, s);
    case ATTN_DTYPE_E5M2:
      return run_prefill<128, 3>(*args, s);
    default:
      return ATTN_ERR_UNSUPPORTED;
  }
}

}  // namespace
}  // namespace attn
