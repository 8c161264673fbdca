// Host-side helpers shared by the launch code: tensor-map encoding through
// the driver entry point, device queries and argument checks.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>

#include "../../include/libattn.h"

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

// Runs `configure` (a kernel's function attributes) once per device: the
// attributes belong to the current device's context, so every device needs
// its own call. Devices past 63 configure on every launch. Safe under
// concurrent callers (a repeated call is harmless).
template <typename F>
attn_status_t configure_per_device(std::atomic<uint64_t>& done, F&& configure) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  const uint64_t bit = dev < 64 ? uint64_t(1) << dev : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return ATTN_OK;
  const attn_status_t st = configure();
  if (st == ATTN_OK && bit) done.fetch_or(bit, std::memory_order_release);
  return st;
}

bool pow2_in(int v, int lo, int hi) { return v >= lo && v <= hi && (v & (v - 1)) == 0; }

}  // namespace
}  // namespace attn
