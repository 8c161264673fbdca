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
#include "combine.cuh"
#include "common.cuh"
#include "decode_paged.cuh"
#include "host.cuh"
#include "mla_sm100.cuh"
#include "mla_host.cuh"
#include "prefill_host.cuh"
#include "sched.cuh"
#include "sched_host.cuh"

namespace attn {
namespace {

// ---------------------------------------------------------------------------
// Scheduler metadata / paged decode / combine
// ---------------------------------------------------------------------------

// The failure-detection self-test: one thread waits, with the kernels' own
// bounded wait, on a barrier nothing arrives on (phase 0 never completes),
// so the wait runs out, raises ATTN_DEVERR_TIMEOUT and the kernel returns.
__global__ void __launch_bounds__(32, 1) selftest_wait_timeout_kernel() {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, ATTN_SELFTEST_SITE);
}

attn_status_t check_paged(const attn_paged_args* a) {
  if (!a) return ATTN_ERR_INVALID_ARG;
  if (!a->q || !a->k_cache || !a->v_cache || !a->block_table || !a->cache_seqlens || !a->out)
    return ATTN_ERR_INVALID_ARG;
  if (a->batch <= 0 || a->seqlen_q <= 0 || a->num_heads_q <= 0 || a->num_heads_kv <= 0 ||
      a->num_heads_q % a->num_heads_kv != 0 || a->head_dim <= 0 || a->num_blocks <= 0 ||
      a->max_pages_per_seq <= 0 || a->page_size <= 0)
    return ATTN_ERR_INVALID_ARG;
  if (a->block_table_stride < a->max_pages_per_seq) return ATTN_ERR_INVALID_ARG;
  if (!(a->scale > 0.f) || !std::isfinite(a->scale)) return ATTN_ERR_INVALID_ARG;
  if (a->window_left < -1 || a->window_right < -1 || a->num_ctas < 0) return ATTN_ERR_INVALID_ARG;
  if (a->dtype < ATTN_DTYPE_BF16 || a->dtype > ATTN_DTYPE_E5M2) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(a->q) || !aligned16(a->k_cache) || !aligned16(a->v_cache) || !aligned16(a->out))
    return ATTN_ERR_INVALID_ARG;
  const bool fp8 = a->dtype == ATTN_DTYPE_E4M3 || a->dtype == ATTN_DTYPE_E5M2;
  if (fp8 && (!a->q_descale || !a->k_descale || !a->v_descale)) return ATTN_ERR_INVALID_ARG;
  const int es = fp8 ? 1 : 2;
  if (!stride_ok(a->q_stride_b, es) || !stride_ok(a->q_stride_s, es) ||
      !stride_ok(a->q_stride_h, es) || !stride_ok(a->kc_stride_blk, es) ||
      !stride_ok(a->kc_stride_tok, es) || !stride_ok(a->kc_stride_h, es) ||
      !stride_ok(a->vc_stride_blk, es) || !stride_ok(a->vc_stride_tok, es) ||
      !stride_ok(a->vc_stride_h, es) || !stride_ok(a->o_stride_b, 2) ||
      !stride_ok(a->o_stride_s, 2) || !stride_ok(a->o_stride_h, 2))
    return ATTN_ERR_INVALID_ARG;
  if ((a->k_new == nullptr) != (a->v_new == nullptr)) return ATTN_ERR_INVALID_ARG;
  if (a->k_new) {
    if (a->seqlen_new < 1 || !aligned16(a->k_new) || !aligned16(a->v_new))
      return ATTN_ERR_INVALID_ARG;
    if (!stride_ok(a->kn_stride_b, es) || !stride_ok(a->kn_stride_s, es) ||
        !stride_ok(a->kn_stride_h, es) || !stride_ok(a->vn_stride_b, es) ||
        !stride_ok(a->vn_stride_s, es) || !stride_ok(a->vn_stride_h, es))
      return ATTN_ERR_INVALID_ARG;
  } else if (a->seqlen_new != 0) {
    return ATTN_ERR_INVALID_ARG;
  }
  if (a->head_dim != 64 && a->head_dim != 128) return ATTN_ERR_UNSUPPORTED;
  if (fp8 && a->head_dim != 128) return ATTN_ERR_UNSUPPORTED;
  if (!pow2_in(a->page_size, 16, 256)) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

size_t paged_ws_bytes(const attn_paged_args* a, const DecodeShape& ds) {
  const size_t slots = (size_t)ds.S + ds.G;
  return slots * kDecRows * a->head_dim * sizeof(float) + slots * kDecRows * sizeof(float) + 256;
}

// kType: 0 bf16, 1 fp16, 2 e4m3, 3 e5m2 (q and both caches).
template <int D, int kType>
attn_status_t run_decode(const attn_paged_args& a, const DecodeShape& ds, cudaStream_t stream) {
  using C = DecodeCfg<D, (kType >= 2)>;
  const CUtensorMapDataType dt = kType >= 2   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : kType == 1 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                              : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint32_t box_rows = a.page_size >= kDecTileKeys ? kDecTileKeys : a.page_size;
  CUtensorMap mk, mv;
  if (!encode_4d(&mk, a.k_cache, dt, C::kElt, D, a.num_heads_kv, a.page_size, a.num_blocks,
                 a.kc_stride_h, a.kc_stride_tok, a.kc_stride_blk, C::kChunkCols, 1, box_rows,
                 1) ||
      !encode_4d(&mv, a.v_cache, dt, C::kElt, D, a.num_heads_kv, a.page_size, a.num_blocks,
                 a.vc_stride_h, a.vc_stride_tok, a.vc_stride_blk, C::kChunkCols, 1, box_rows,
                 1))
    return ATTN_ERR_INVALID_ARG;
  // appended keys: (D, H_kv, seqlen_new, B) with 64-row boxes; without them
  // the kernel never reads these maps and gets the cache maps in their place
  CUtensorMap mkn = mk, mvn = mv;
  if (a.k_new &&
      (!encode_4d(&mkn, a.k_new, dt, C::kElt, D, a.num_heads_kv, a.seqlen_new, a.batch,
                  a.kn_stride_h, a.kn_stride_s, a.kn_stride_b, C::kChunkCols, 1, kDecTileKeys,
                  1) ||
       !encode_4d(&mvn, a.v_new, dt, C::kElt, D, a.num_heads_kv, a.seqlen_new, a.batch,
                  a.vn_stride_h, a.vn_stride_s, a.vn_stride_b, C::kChunkCols, 1, kDecTileKeys,
                  1)))
    return ATTN_ERR_INVALID_ARG;
  DecodeParams p;
  memset(&p, 0, sizeof(p));
  p.q = a.q;
  p.out = a.out;
  p.lse = a.lse;
  p.block_table = a.block_table;
  p.cache_seqlens = a.cache_seqlens;
  p.meta = a.meta;
  p.sink = a.sink;
  p.q_descale = a.q_descale;
  p.k_descale = a.k_descale;
  p.v_descale = a.v_descale;
  p.bt_stride = a.block_table_stride;
  p.q_sb = a.q_stride_b;
  p.q_ss = a.q_stride_s;
  p.q_sh = a.q_stride_h;
  p.o_sb = a.o_stride_b;
  p.o_ss = a.o_stride_s;
  p.o_sh = a.o_stride_h;
  p.batch = a.batch;
  p.seqlen_q = a.seqlen_q;
  p.heads_q = a.num_heads_q;
  p.heads_kv = a.num_heads_kv;
  p.group = ds.group;
  p.rows = ds.rows;
  p.n_rsub = ds.n_rsub;
  p.segs_per_seq = ds.sh.segs_per_seq;
  p.num_segs = ds.S;
  p.page_size = a.page_size;
  p.num_ctas = ds.G;
  p.scale_log2 = a.scale * kLog2e;
  p.causal = a.causal;
  p.window_left = a.window_left;
  p.window_right = a.window_right;
  p.seqlen_new = a.k_new ? a.seqlen_new : 0;
  if (a.meta) {
    const size_t slots = (size_t)ds.S + ds.G;
    p.ws_o = reinterpret_cast<float*>(a.workspace);
    p.ws_lse = p.ws_o + slots * kDecRows * D;
  }
  auto kernel = decode_kernel<D, kType>;
  static std::atomic<uint64_t> configured{0};
  const attn_status_t cst = configure_per_device(configured, [&] {
    return launch_status(set_smem(kernel, C::kSmemBytes));
  });
  if (cst != ATTN_OK) return cst;
  const int grid = a.meta ? ds.G : ds.S;
  kernel<<<grid, kDecThreads, C::kSmemBytes, stream>>>(mk, mv, mkn, mvn, p);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  if (a.meta) {
    const int64_t warps = (int64_t)ds.S * kDecRows;
    const int blocks = (int)((warps + 7) / 8);
    decode_combine_kernel<D, kType == 1><<<blocks, 256, 0, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

}  // namespace
}  // namespace attn

using namespace attn;

extern "C" {

attn_status_t attn_fwd_varlen(const attn_varlen_args* args, void* stream) {
  return varlen_entry(args, stream);
}

size_t attn_sched_metadata_size(const attn_sched_args* a) {
  if (!a) return 0;
  DecodeShape ds;
  if (!sbs_ok(a->sparse_block_size)) return 0;
  if (decode_shape(a->mode, a->batch, a->seqlen_q, a->num_heads_q, a->num_heads_kv,
                   sparse_positions(a->mode, a->topk, a->sparse_block_size),
                   a->num_ctas, ds) != ATTN_OK)
    return 0;
  return meta_bytes_for(ds);
}

attn_status_t attn_sched_metadata(const attn_sched_args* a, void* stream) {
  if (!a || !a->cache_seqlens || !a->meta) return ATTN_ERR_INVALID_ARG;
  if (a->page_size <= 0 || a->head_dim_qk <= 0 || a->head_dim_v <= 0 || a->num_ctas < 0)
    return ATTN_ERR_INVALID_ARG;
  if (a->mode < ATTN_SCHED_MHA || a->mode > ATTN_SCHED_MLA_SPARSE) return ATTN_ERR_INVALID_ARG;
  if (!sbs_ok(a->sparse_block_size)) return ATTN_ERR_INVALID_ARG;
  // appended keys exist for the GQA decode only
  if (a->seqlen_new < 0 || (a->seqlen_new > 0 && a->mode != ATTN_SCHED_MHA))
    return ATTN_ERR_INVALID_ARG;
  DecodeShape ds;
  const attn_status_t st =
      decode_shape(a->mode, a->batch, a->seqlen_q, a->num_heads_q, a->num_heads_kv,
                   sparse_positions(a->mode, a->topk, a->sparse_block_size), a->num_ctas, ds);
  if (st != ATTN_OK) return st;
  ds.sh.new_keys = a->seqlen_new;
  if (a->meta_bytes < meta_bytes_for(ds)) return ATTN_ERR_WORKSPACE_TOO_SMALL;
  SchedParams p;
  memset(&p, 0, sizeof(p));
  p.cache_seqlens = a->cache_seqlens;
  p.meta = a->meta;
  p.sh = ds.sh;
  p.batch = a->batch;
  p.seqlen_q = a->seqlen_q;
  p.heads_q = a->num_heads_q;
  p.heads_kv = a->num_heads_kv;
  p.page_size = a->page_size;
  p.G = ds.G;
  p.S = ds.S;
  p.dim_qk = a->head_dim_qk;
  p.dim_v = a->head_dim_v;
  sched_kernel<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return launch_status(cudaGetLastError());
}

size_t attn_paged_workspace_size(const attn_paged_args* a) {
  if (!a || !a->meta || check_paged(a) != ATTN_OK) return 0;
  DecodeShape ds;
  if (decode_shape(ATTN_SCHED_MHA, a->batch, a->seqlen_q, a->num_heads_q, a->num_heads_kv, 0,
                   a->num_ctas, ds) != ATTN_OK)
    return 0;
  return paged_ws_bytes(a, ds);
}

attn_status_t attn_fwd_paged_kvcache(const attn_paged_args* a, void* stream) {
  attn_status_t st = check_paged(a);
  if (st != ATTN_OK) return st;
  DecodeShape ds;
  st = decode_shape(ATTN_SCHED_MHA, a->batch, a->seqlen_q, a->num_heads_q, a->num_heads_kv, 0,
                    a->num_ctas, ds);
  if (st != ATTN_OK) return st;
  if (a->meta) {
    if (a->meta_bytes < meta_bytes_for(ds)) return ATTN_ERR_INVALID_ARG;
    if (!a->workspace || a->workspace_bytes < paged_ws_bytes(a, ds))
      return ATTN_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(a->workspace)) return ATTN_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (a->dtype) {
    case ATTN_DTYPE_BF16:
      return a->head_dim == 64 ? run_decode<64, 0>(*a, ds, s) : run_decode<128, 0>(*a, ds, s);
    case ATTN_DTYPE_FP16:
      return a->head_dim == 64 ? run_decode<64, 1>(*a, ds, s) : run_decode<128, 1>(*a, ds, s);
    case ATTN_DTYPE_E4M3:
      return run_decode<128, 2>(*a, ds, s);
    case ATTN_DTYPE_E5M2:
      return run_decode<128, 3>(*a, ds, s);
    default:
      return ATTN_ERR_UNSUPPORTED;
  }
}

attn_status_t attn_combine(const attn_combine_args* a, void* stream) {
  if (!a || !a->out_partial || !a->lse_partial || !a->out) return ATTN_ERR_INVALID_ARG;
  if (a->num_splits <= 0 || a->batch <= 0 || a->seqlen_q <= 0 || a->num_heads <= 0 ||
      a->head_dim_v <= 0)
    return ATTN_ERR_INVALID_ARG;
  if (a->out_dtype != ATTN_DTYPE_BF16 && a->out_dtype != ATTN_DTYPE_FP16)
    return ATTN_ERR_INVALID_ARG;
  if (a->num_splits > kCombineMaxSplits || a->head_dim_v % 8 || a->head_dim_v > 1024)
    return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(a->out_partial) || !aligned16(a->out)) return ATTN_ERR_INVALID_ARG;
  if (!stride_ok(a->o_stride_b, 2) || !stride_ok(a->o_stride_s, 2) || !stride_ok(a->o_stride_h, 2))
    return ATTN_ERR_INVALID_ARG;
  CombineParams p;
  p.o_part = a->out_partial;
  p.lse_part = a->lse_partial;
  p.out = a->out;
  p.lse = a->lse;
  p.nsplit_per_seq = a->num_splits_per_seq;
  p.sink = a->sink;
  p.num_splits = a->num_splits;
  p.batch = a->batch;
  p.seqlen_q = a->seqlen_q;
  p.heads = a->num_heads;
  p.dv = a->head_dim_v;
  p.o_sb = a->o_stride_b;
  p.o_ss = a->o_stride_s;
  p.o_sh = a->o_stride_h;
  const int64_t rows = (int64_t)a->batch * a->seqlen_q * a->num_heads;
  const int64_t blocks = (rows + 7) / 8;
  if (blocks > INT32_MAX) return ATTN_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (a->out_dtype == ATTN_DTYPE_FP16)
    combine_kernel<true><<<(int)blocks, 256, 0, s>>>(p);
  else
    combine_kernel<false><<<(int)blocks, 256, 0, s>>>(p);
  return launch_status(cudaGetLastError());
}

size_t mla_workspace_size(const mla_args* a) {
  if (!a || !a->meta) return 0;
  const bool sparse = a->indices != nullptr;
  if (check_mla(a, sparse) != ATTN_OK) return 0;
  DecodeShape ds;
  const int mode = sparse ? ATTN_SCHED_MLA_SPARSE : ATTN_SCHED_MLA;
  if (decode_shape(mode, a->cu_seqlens_q ? 1 : a->batch, a->seqlen_q, a->num_heads_q,
                   a->num_heads_kv,
                   sparse_positions(mode, a->topk, a->sparse_block_size), a->num_ctas,
                   ds) != ATTN_OK)
    return 0;
  return mla_ws_bytes(ds);
}
attn_status_t mla_fwd_paged(const mla_args* a, void* stream) {
  if (a && a->indices) return ATTN_ERR_INVALID_ARG;  // indices belong to mla_sparse_fwd
  return mla_entry(a, stream, false);
}
attn_status_t mla_sparse_fwd(const mla_args* a, void* stream) {
  return mla_entry(a, stream, true);
}

attn_status_t attn_selftest_wait_timeout(void* stream) {
  selftest_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return launch_status(cudaGetLastError());
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

// ---------------------------------------------------------------------------
// attn_fwd_paged_kvcache_static: the paged decode with built-in scratch.
//
// The regular entry point needs two caller-provided device buffers (the
// scheduler metadata and the split-KV partials). This variant keeps both in
// one file-scope device array instead, so a caller that cannot allocate
// device memory can still run the split-KV decode. The array is part of the
// library image: every GPU on which the library is used holds it until the
// process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_paged_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

// The driver's cuCtxGetCurrent, fetched through the runtime (the library does
// not link libcuda directly).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of the scratch array on the current device (host code must
// not use the array's name as an address). It is looked up once per device
// and context: after a device reset the runtime creates a new primary context
// and loads the library's module again, so the array moves, and the address
// is looked up anew.
void* static_scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  if (get_ctx == nullptr) return nullptr;
  // null until the runtime has made the device's context current on this thread
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr || ctx == nullptr || g_scratch_ctx[dev] != ctx) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress((void**)&ptr, g_paged_scratch) != cudaSuccess) return nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return nullptr;
    g_scratch_addr[dev] = ptr;
    g_scratch_ctx[dev] = ctx;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" attn_status_t attn_fwd_paged_kvcache_static(const attn_paged_args* args,
                                                       void* stream) {
  if (!args) return ATTN_ERR_INVALID_ARG;
  // This entry point brings its own scratch; caller buffers are a usage error.
  if (args->meta != nullptr || args->workspace != nullptr) return ATTN_ERR_INVALID_ARG;
  attn_status_t st = check_paged(args);
  if (st != ATTN_OK) return st;
  DecodeShape ds;
  st = decode_shape(ATTN_SCHED_MHA, args->batch, args->seqlen_q, args->num_heads_q,
                    args->num_heads_kv, 0, args->num_ctas, ds);
  if (st != ATTN_OK) return st;
  // metadata first (256-byte aligned), the split-KV partials after it
  const size_t meta_bytes = (meta_bytes_for(ds) + 255) & ~size_t(255);
  const size_t ws_bytes = paged_ws_bytes(args, ds);
  if (meta_bytes + ws_bytes > kStaticScratchBytes) return ATTN_ERR_WORKSPACE_TOO_SMALL;
  unsigned char* base = static_cast<unsigned char*>(static_scratch_address());
  if (base == nullptr) return ATTN_ERR_CUDA;

  // Nothing in the scratch has to start at zero: the metadata kernel writes
  // every word the decode and combine kernels read, and every partial slot the
  // combine reads is written by the decode kernel first.
  attn_sched_args sa;
  memset(&sa, 0, sizeof(sa));
  sa.cache_seqlens = args->cache_seqlens;
  sa.batch = args->batch;
  sa.seqlen_q = args->seqlen_q;
  sa.num_heads_q = args->num_heads_q;
  sa.num_heads_kv = args->num_heads_kv;
  sa.head_dim_qk = args->head_dim;
  sa.head_dim_v = args->head_dim;
  sa.page_size = args->page_size;
  sa.mode = ATTN_SCHED_MHA;
  sa.num_ctas = args->num_ctas;
  sa.seqlen_new = args->k_new ? args->seqlen_new : 0;
  sa.meta = reinterpret_cast<int32_t*>(base);
  sa.meta_bytes = meta_bytes;
  st = attn_sched_metadata(&sa, stream);
  if (st != ATTN_OK) return st;
  attn_paged_args a = *args;
  a.meta = reinterpret_cast<const int32_t*>(base);
  a.meta_bytes = meta_bytes;
  a.workspace = base + meta_bytes;
  a.workspace_bytes = ws_bytes;
  return attn_fwd_paged_kvcache(&a, stream);
}
