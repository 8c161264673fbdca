// Device helpers shared by the libattn kernels: mbarriers with bounded waits,
// TMA tile loads, tcgen05 (TMEM allocation, MMA, loads/stores) and the device
// error word. sm_100a only.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/libattn.h"

#define DEVI __device__ __forceinline__

namespace attn {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// Online softmax: after the first key tile, the running max of a row is
// raised (and O rescaled) only when it grows by more than this many log2
// units; P then stays below 2^8 and the result is exact after the final
// division by the row sum.
constexpr float kRescaleThreshold = 8.0f;

// ---------------------------------------------------------------------------
// Device error word: the first error wins. Low 8 bits = ATTN_DEVERR_* code,
// bits 8.. = reporting site. Read and cleared by attn_get_device_error.
// ---------------------------------------------------------------------------
__device__ int32_t g_error_word;

DEVI void raise_error(int code, int site) {
  atomicCAS(&g_error_word, 0, (site << 8) | code);
}

DEVI uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// A pipeline wait gives up after this long (ns). Waits in these kernels are
// microseconds in normal operation; a timeout means a protocol bug, and the
// kernel then unwinds (see each kernel's teardown) instead of hanging.
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;

DEVI uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
DEVI void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
DEVI void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
DEVI void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
DEVI void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
DEVI bool mbar_test(uint32_t addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits until the phase with the given parity has completed. Returns false
// (after raising ATTN_DEVERR_TIMEOUT) if that takes longer than the timeout
// or if *abort is set by another thread of the CTA.
DEVI bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int site) {
  const uint32_t a = smem_u32(bar);
  if (mbar_test(a, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_test(a, parity)) return true;
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

// Warp-collective form: every lane waits, and the warp proceeds only if all
// lanes succeeded, so warp-collective (.sync.aligned) instructions after it
// are never reached by part of a warp.
DEVI bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int site) {
  const bool ok = mbar_wait(bar, parity, abort, site);
  return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------------------
// TMA (tiled tensor loads, no multicast)
// ---------------------------------------------------------------------------
DEVI void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
DEVI void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}
DEVI void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}
DEVI void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2,
                      int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(smem_u32(bar))
      : "memory");
}

// Generic-proxy writes to shared memory must be made visible to the async
// proxy (TMA, tcgen05.mma) before they are consumed there.
DEVI void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory and the 5th-generation MMA
// ---------------------------------------------------------------------------
DEVI void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {  // one full warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
DEVI void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
DEVI void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // the allocating warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
DEVI void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
DEVI void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrive once on `bar` when every tcgen05 operation issued so far by this
// thread has completed.
DEVI void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// D(tmem) (+)= A(smem) * B(smem), kind::f16 (bf16/fp16 in, fp32 accumulate).
DEVI void mma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                     uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D(tmem) (+)= A(tmem) * B(smem), kind::f16.
DEVI void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                     uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D(tmem) (+)= A(smem) * B(smem), kind::f8f6f4 (FP8 in, fp32 accumulate).
DEVI void mma_f8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                    uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D(tmem) (+)= A(tmem) * B(smem), kind::f8f6f4.
DEVI void mma_f8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                    uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor (kind::f16 and kind::f8f6f4, dense, fp32 D):
//   [4,6) D format (1 = f32); [7,10) A format; [10,13) B format
//   (kind::f16: 0 = f16, 1 = bf16; kind::f8f6f4: 0 = e4m3, 1 = e5m2);
//   bit 15 A major, bit 16 B major (0 = K-major, 1 = MN-major);
//   [17,23) N >> 3; [24,29) M >> 4.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N, int ab_format, int a_mn_major,
                                                  int b_mn_major) {
  return (1u << 4) | (uint32_t(ab_format) << 7) | (uint32_t(ab_format) << 10) |
         (uint32_t(a_mn_major) << 15) | (uint32_t(b_mn_major) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Shared-memory matrix descriptor for a 128-byte-swizzled tile (the layout a
// TMA load with CU_TENSOR_MAP_SWIZZLE_128B writes: rows of 128 bytes, 8-row
// atoms of 1024 bytes, 16-byte chunks XOR-ed with the row index mod 8).
//   [0,14) start >> 4; [16,30) leading byte offset >> 4; [32,46) stride byte
//   offset >> 4; [46,48) = 1 (sm_100 descriptor version); [61,64) = 2
//   (128-byte swizzle).
DEVI uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo_bytes >> 4) << 16) |
         ((uint64_t)(sbo_bytes >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// 32 lanes x 32-bit: thread t of the warp gets lane (taddr.lane + t), columns
// [taddr.col, taddr.col + N). Load and wait in one statement so the outputs
// are valid when it returns.
template <int N>
DEVI void tmem_load(uint32_t taddr, uint32_t* r);

#define ATTN_R4(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3])
#define ATTN_R16(i) ATTN_R4(i), ATTN_R4(i + 4), ATTN_R4(i + 8), ATTN_R4(i + 12)
#define ATTN_W4(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3])
#define ATTN_W16(i) ATTN_W4(i), ATTN_W4(i + 4), ATTN_W4(i + 8), ATTN_W4(i + 12)

template <>
DEVI void tmem_load<16>(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];\n\ttcgen05.wait::ld.sync.aligned;"
      : ATTN_R16(0)
      : "r"(taddr)
      : "memory");
}
template <>
DEVI void tmem_load<32>(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : ATTN_R16(0), ATTN_R16(16)
      : "r"(taddr)
      : "memory");
}

template <int N>
DEVI void tmem_store(uint32_t taddr, const uint32_t* r);
template <>
DEVI void tmem_store<16>(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16};" ::"r"(taddr),
      ATTN_W16(0)
      : "memory");
}
template <>
DEVI void tmem_store<32>(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(
          taddr),
      ATTN_W16(0), ATTN_W16(16)
      : "memory");
}
DEVI void tmem_store_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Small math helpers
// ---------------------------------------------------------------------------
DEVI float ex2(float x) {  // hardware 2^x (MUFU), flushes subnormals
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
DEVI uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half), .y = hi
  return *reinterpret_cast<uint32_t*>(&v);
}
DEVI uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
template <bool kFp16>
DEVI uint32_t pack2(float lo, float hi) {
  return kFp16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
}

// Sum of the two 16-bit floats packed in a 32-bit word.
template <bool kFp16>
DEVI float sum2(uint32_t packed) {
  if (kFp16) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&packed));
    return f.x + f.y;
  }
  return __uint_as_float(packed << 16) + __uint_as_float(packed & 0xffff0000u);
}

// Two FP8 values (low byte first) to two fp16 values, exactly (every e4m3
// and every e5m2 value is an fp16 value). kType: 2 = e4m3, 3 = e5m2.
template <int kType>
DEVI uint32_t fp8x2_to_f16x2(unsigned short v) {
  uint32_t h;
  if constexpr (kType == 3)
    asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h) : "h"(v));
  else
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(v));
  return h;
}

DEVI void store_out(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
DEVI void store_out(__half* p, float v) { *p = __float2half_rn(v); }

DEVI int elect_lane0() { return (threadIdx.x & 31) == 0; }

}  // namespace attn

namespace attn {

// ---------------------------------------------------------------------------
// Packed fp32x2 arithmetic (sm_100: two fp32 lanes per instruction)
// ---------------------------------------------------------------------------
DEVI uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
DEVI void f2unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
DEVI uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
DEVI uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
DEVI uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// max(a, b, c) in one instruction (sm_100).
DEVI float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Adds the two 16-bit floats of a packed word to two fp32 accumulators with
// the sm_100 mixed-precision add (the 16-bit operand is widened exactly).
template <bool kFp16>
DEVI void acc_packed(float& lo, float& hi, uint32_t packed) {
  if constexpr (kFp16) {
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
        "add.rn.f32.f16 %0, l, %0;\n\tadd.rn.f32.f16 %1, h, %1;\n\t}"
        : "+f"(lo), "+f"(hi) : "r"(packed));
  } else {
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
        "add.rn.f32.bf16 %0, l, %0;\n\tadd.rn.f32.bf16 %1, h, %1;\n\t}"
        : "+f"(lo), "+f"(hi) : "r"(packed));
  }
}

// The two 16-bit floats of a packed word, widened to fp32 (exact).
template <bool kFp16>
DEVI uint64_t widen2(uint32_t packed) {
  if (kFp16) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&packed));
    return f2pack(f.x, f.y);
  }
  return f2pack(__uint_as_float(packed << 16), __uint_as_float(packed & 0xffff0000u));
}

// Register reallocation between warpgroups (all warps of a warpgroup execute it).
template <uint32_t N>
DEVI void regs_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }
template <uint32_t N>
DEVI void regs_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }

// 32 lanes x 64 columns of 32 bits in one load (outputs valid on return).
DEVI void tmem_load64(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {"
      "%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : ATTN_R16(0), ATTN_R16(16), ATTN_R16(32), ATTN_R16(48)
      : "r"(taddr)
      : "memory");
}

// ---------------------------------------------------------------------------
// Thread-block clusters: rank, distributed shared memory, remote mbarriers
// ---------------------------------------------------------------------------
DEVI uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The shared::cluster address of the same shared-memory offset in CTA `rank`.
DEVI uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
DEVI void st_cluster_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b),
               "r"(c), "r"(d)
               : "memory");
}
// Arrive on an mbarrier of another CTA of the cluster, ordering this thread's
// earlier (distributed) shared-memory writes before the arrival.
DEVI void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
DEVI bool mbar_test_cluster(uint32_t addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(addr), "r"(parity)
      : "memory");
  return ok != 0;
}
// As warp_wait, with cluster-scope acquire (the arrivals come from another
// CTA of the cluster).
DEVI bool warp_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort, int site) {
  const uint32_t a = smem_u32(bar);
  bool ok = mbar_test_cluster(a, parity);
  if (!ok) {
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
      if (mbar_test_cluster(a, parity)) {
        ok = true;
        break;
      }
      if ((it & 255u) == 0) {
        if (*abort) break;
        if (globaltimer() - t0 > kWaitTimeoutNs) {
          raise_error(ATTN_DEVERR_TIMEOUT, site);
          *abort = 1;
          break;
        }
      }
    }
  }
  return __all_sync(0xffffffffu, ok);
}
// Arrive on another CTA's mbarrier and add `bytes` to the transaction count
// its phase waits for.
DEVI void mbar_arrive_expect_tx_remote(uint32_t cluster_addr, uint32_t bytes) {
  asm volatile(
      "mbarrier.arrive.expect_tx.release.cluster.shared::cluster.b64 _, [%0], %1;" ::"r"(
          cluster_addr),
      "r"(bytes)
      : "memory");
}
// Bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned) from
// this CTA's shared memory into another CTA's, completing on that CTA's
// mbarrier (no multicast).
DEVI void bulk_copy_to_cluster(uint32_t dst_cluster, uint32_t src, uint32_t bytes,
                               uint32_t mbar_cluster) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst_cluster),
      "r"(src), "r"(bytes), "r"(mbar_cluster)
      : "memory");
}
DEVI void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until at most N of this thread's committed bulk copies may still be
// reading their source.
template <int N>
DEVI void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory"); }
// Waits until this thread's committed bulk copies have completed.
DEVI void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// All threads of every CTA of the cluster.
DEVI void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// Named barrier over `count` threads (a multiple of 32).
DEVI void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// 32 lanes x 128 columns of 32 bits in one load (outputs valid on return).
DEVI void tmem_load128(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 {"
      "%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,"
      "%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,"
      "%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,"
      "%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,"
      "%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127},"
      " [%128];\n\ttcgen05.wait::ld.sync.aligned;"
      : ATTN_R16(0), ATTN_R16(16), ATTN_R16(32), ATTN_R16(48), ATTN_R16(64), ATTN_R16(80),
        ATTN_R16(96), ATTN_R16(112)
      : "r"(taddr)
      : "memory");
}

}  // namespace attn

namespace attn {

// 2^x for a pair of fp32 values on the FMA pipe (no MUFU), for x <= 64.
// Range reduction x = j + f with j = rint(x) (adding 1.5 * 2^23 rounds to an
// integer in the low mantissa bits), f in [-0.5, 0.5]; 2^f by a degree-3
// polynomial whose coefficients minimise the maximum relative error on
// [-0.5, 0.5] (a linear-programming minimax fit, max relative error 7.5e-5);
// 2^j is added to the exponent field with an integer multiply-add. Inputs
// below -126 are clamped: the result is then a tiny positive number
// (<= 2^-125), not 0.
DEVI uint64_t exp2_poly_x2(float x0, float x1) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  const uint64_t x = f2pack(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
  const uint64_t t = add2(x, f2pack(kMagic, kMagic));
  const uint64_t jf = add2(t, f2pack(-kMagic, -kMagic));
  const uint64_t f = fma2(jf, f2pack(-1.f, -1.f), x);
  uint64_t p = fma2(f2pack(0.05517222f, 0.05517222f), f, f2pack(0.24261115f, 0.24261115f));
  p = fma2(p, f, f2pack(0.69326085f, 0.69326085f));
  p = fma2(p, f, f2pack(0.99992806f, 0.99992806f));
  float p0, p1, t0, t1;
  f2unpack(p, p0, p1);
  f2unpack(t, t0, t1);
  uint32_t r0, r1;
  asm("mad.lo.u32 %0, %1, 8388608, %2;" : "=r"(r0) : "r"(__float_as_uint(t0)), "r"(__float_as_uint(p0)));
  asm("mad.lo.u32 %0, %1, 8388608, %2;" : "=r"(r1) : "r"(__float_as_uint(t1)), "r"(__float_as_uint(p1)));
  return f2pack(__uint_as_float(r0), __uint_as_float(r1));
}

}  // namespace attn

namespace attn {

// Warp-wide forms of the MMA issue: the whole warp runs the issuing loop (its
// values stay warp-uniform, so descriptors live in uniform registers) and
// one elected lane issues each tcgen05 instruction.
DEVI void mma_f16_ss_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
DEVI void mma_f16_ts_w(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
DEVI void mma_f8_ss_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                      uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
DEVI void mma_f8_ts_w(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                      uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
DEVI void tc_commit_w(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}

}  // namespace attn
