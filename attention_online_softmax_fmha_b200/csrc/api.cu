// libattn C ABI: argument validation, TMA descriptor encoding and kernel
// launches. Declarations and the contract of every entry point are in
// include/libattn.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/libattn.h"
#include "common.cuh"
#include "prefill_sm100.cuh"

namespace attn {
namespace {

// ---------------------------------------------------------------------------
// Driver entry point for cuTensorMapEncodeTiled (fetched through the runtime
// so the library does not link libcuda directly).
// ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A 4-D tiled map over (dim0 = D contiguous, dim1, dim2, dim3) with strides
// in bytes for dims 1..3, a box of (box0, box1, box2, box3) and 128-byte
// swizzle. Out-of-range elements of a box read as zero.
bool encode_4d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int esize,
               uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3, uint64_t s1, uint64_t s2,
               uint64_t s3, uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {d0, d1, d2, d3};
  cuuint64_t strides[3] = {s1 * esize, s2 * esize, s3 * esize};
  cuuint32_t box[4] = {b0, b1, b2, b3};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool stride_ok(int64_t s, int esize) { return s > 0 && ((s * esize) % 16) == 0; }

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

attn_status_t launch_status(cudaError_t e) {
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// attn_fwd_varlen
// ---------------------------------------------------------------------------
template <int D, bool kFp16>
attn_status_t run_prefill(const attn_varlen_args& a, cudaStream_t stream) {
  using C = PrefillCfg<D>;
  const bool varlen = a.cu_seqlens_q != nullptr;
  const CUtensorMapDataType dt =
      kFp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t rows_q = varlen ? (uint64_t)a.total_q : (uint64_t)a.max_seqlen_q;
  const uint64_t rows_k = varlen ? (uint64_t)a.total_k : (uint64_t)a.max_seqlen_k;
  const uint64_t nb = varlen ? 1 : (uint64_t)a.batch;
  const uint64_t qsb = varlen ? rows_q * a.q_stride_s : a.q_stride_b;
  const uint64_t ksb = varlen ? rows_k * a.k_stride_s : a.k_stride_b;
  const uint64_t vsb = varlen ? rows_k * a.v_stride_s : a.v_stride_b;
  CUtensorMap mq, mk, mv;
  if (!encode_4d(&mq, a.q, dt, 2, D, a.num_heads_q, rows_q, nb, a.q_stride_h, a.q_stride_s, qsb,
                 64, 1, 128, 1) ||
      !encode_4d(&mk, a.k, dt, 2, D, a.num_heads_kv, rows_k, nb, a.k_stride_h, a.k_stride_s, ksb,
                 64, 1, 128, 1) ||
      !encode_4d(&mv, a.v, dt, 2, D, a.num_heads_kv, rows_k, nb, a.v_stride_h, a.v_stride_s, vsb,
                 64, 1, 128, 1))
    return ATTN_ERR_INVALID_ARG;

  PrefillParams p;
  memset(&p, 0, sizeof(p));
  p.out = a.out;
  p.lse = a.lse;
  p.cu_q = a.cu_seqlens_q;
  p.cu_k = a.cu_seqlens_k;
  p.sink = a.sink;
  p.o_sb = a.o_stride_b;
  p.o_ss = a.o_stride_s;
  p.o_sh = a.o_stride_h;
  p.lse_sb = varlen ? 0 : a.lse_stride_b;
  p.lse_sh = a.lse_stride_h;
  p.batch = a.batch;
  p.seqlen_q = a.max_seqlen_q;
  p.seqlen_k = a.max_seqlen_k;
  p.num_q_tiles = (a.max_seqlen_q + kPrefillBM - 1) / kPrefillBM;
  p.num_heads_q = a.num_heads_q;
  p.num_heads_kv = a.num_heads_kv;
  p.group = a.num_heads_q / a.num_heads_kv;
  const int64_t total = (int64_t)p.num_q_tiles * a.batch * a.num_heads_q;
  if (total > INT32_MAX) return ATTN_ERR_UNSUPPORTED;
  p.total_tiles = (int32_t)total;
  p.scale_log2 = a.scale * kLog2e;
  p.causal = a.causal;
  p.window_left = a.window_left;
  p.window_right = a.window_right;

  auto kernel = prefill_kernel<D, kFp16>;
  static bool configured = false;
  if (!configured) {
    if (set_smem(kernel, C::kSmemBytes) != cudaSuccess) return ATTN_ERR_CUDA;
    configured = true;
  }
  const int sms = device_sm_count();
  if (sms <= 0) return ATTN_ERR_CUDA;
  const int grid = (int)std::min<int64_t>(total, sms);
  kernel<<<grid, 192, C::kSmemBytes, stream>>>(mq, mk, mv, p);
  return launch_status(cudaGetLastError());
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
  if (a->dtype == ATTN_DTYPE_E5M2) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

}  // namespace
}  // namespace attn

using namespace attn;

extern "C" {

attn_status_t attn_fwd_varlen(const attn_varlen_args* args, void* stream) {
  const attn_status_t st = check_varlen(args);
  if (st != ATTN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = args->head_dim_qk;
  switch (args->dtype) {
    case ATTN_DTYPE_BF16:
      return D == 64 ? run_prefill<64, false>(*args, s) : run_prefill<128, false>(*args, s);
    case ATTN_DTYPE_FP16:
      return D == 64 ? run_prefill<64, true>(*args, s) : run_prefill<128, true>(*args, s);
    default:
      return ATTN_ERR_UNSUPPORTED;
  }
}

size_t attn_sched_metadata_size(const attn_sched_args*) { return 0; }
attn_status_t attn_sched_metadata(const attn_sched_args* a, void*) {
  return a ? ATTN_ERR_UNSUPPORTED : ATTN_ERR_INVALID_ARG;
}
size_t attn_paged_workspace_size(const attn_paged_args*, const attn_sched_args*) { return 0; }
attn_status_t attn_fwd_paged_kvcache(const attn_paged_args* a, void*) {
  return a ? ATTN_ERR_UNSUPPORTED : ATTN_ERR_INVALID_ARG;
}
attn_status_t attn_combine(const attn_combine_args* a, void*) {
  return a ? ATTN_ERR_UNSUPPORTED : ATTN_ERR_INVALID_ARG;
}
size_t mla_workspace_size(const mla_args*, const attn_sched_args*) { return 0; }
attn_status_t mla_fwd_paged(const mla_args* a, void*) {
  return a ? ATTN_ERR_UNSUPPORTED : ATTN_ERR_INVALID_ARG;
}
attn_status_t mla_sparse_fwd(const mla_args* a, void*) {
  return a ? ATTN_ERR_UNSUPPORTED : ATTN_ERR_INVALID_ARG;
}

attn_status_t attn_get_device_error(int32_t* code, void* stream) {
  if (!code) return ATTN_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t v = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_error_word, sizeof(v), 0, cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaMemcpyToSymbolAsync(g_error_word, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return ATTN_ERR_CUDA;
  *code = v;
  return v ? ATTN_ERR_DEVICE : ATTN_OK;
}

const char* attn_status_str(int32_t status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case ATTN_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case ATTN_ERR_CUDA: return "CUDA error";
    case ATTN_ERR_DEVICE: return "device error reported by a kernel";
    default: return "unknown status";
  }
}

size_t attn_args_sizeof(int32_t which) {
  switch (which) {
    case 0: return sizeof(attn_varlen_args);
    case 1: return sizeof(attn_sched_args);
    case 2: return sizeof(attn_paged_args);
    case 3: return sizeof(attn_combine_args);
    case 4: return sizeof(mla_args);
    default: return 0;
  }
}

}  // extern "C"
