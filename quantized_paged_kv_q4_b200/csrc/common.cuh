// Shared constants and device helpers of libkvattn (sm_100a only).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kvattn.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ != 1000)
#error "libkvattn is built for sm_100a only"
#endif

namespace kvattn {

constexpr int kHeadDim = 256;
constexpr int kPageTokens = 128;
constexpr int kBlocks = kHeadDim / 32;  // quantisation blocks per row
constexpr int kKPageBytes = 34816;      // Q8_0: 128 x 8 x (32 + 2)
constexpr int kK4PageBytes = 18432;     // Q4_0 keys: 128 x 8 x (16 + 2)
constexpr int kK4ScaleOffset = 16384;
constexpr int kK5PageBytes = 24576;     // Q5_1 keys: 128 x 8 x (20 + 2 + 2)
constexpr int kK5HighOffset = 16384;    // fifth code bits, after the low nibbles
constexpr int kK5ScaleOffset = 20480;
constexpr int kK5MinOffset = 22528;
constexpr int kK50PageBytes = 22528;    // Q5_0 keys: 128 x 8 x (20 + 2); nibbles and fifth bits as Q5_1
// key and value formats as kernel template / flag values
constexpr int kKeyQ8 = 0, kKeyQ4 = 1, kKeyQ51 = 2, kKeyQ50 = 3;
constexpr int kValQ4 = 0, kValQ8 = 1, kValQ41 = 2;
constexpr int kV4PageBytes = 18432;     // Q4_0: 128 x 8 x (16 + 2)
constexpr int kV41PageBytes = 20480;    // Q4_1 values: 128 x 8 x (16 + 2 + 2)
constexpr int kV41MinOffset = 18432;    // Q4_1 minima, after the scales
constexpr int kV8PageBytes = 34816;     // Q8_0 values
constexpr int kKScaleOffset = 32768;    // K page: codes first, then fp16 scales
constexpr int kV4ScaleOffset = 16384;
constexpr int kV8ScaleOffset = 32768;
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // bounded in-kernel waits: 2 s

// ---- per-device error word (page-id checks, bounded waits) ----------------------------
// Defined here: the library is one translation unit (kvattn_unity.cu).
__device__ int g_error_word = 0;

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_error_word, 0, code); }

// ---- PTX wrappers ----------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait that lets the hardware suspend the thread until the phase completes or about
// `hint_ns` nanoseconds pass, so waiting warps do not spin on the issue slots.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Waits for the phase of `parity` to complete; gives up after kWaitTimeoutNs, records
// KVATTN_ERR_TIMEOUT and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  while (!mbar_try_wait_sleep(bar, parity, 1000000u)) {
    if (global_timer_ns() - t0 > kWaitTimeoutNs) {
      record_error(KVATTN_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Waits until a shared-memory word written by another warp equals `want`; gives up after
// kWaitTimeoutNs, records KVATTN_ERR_TIMEOUT and returns false.
__device__ __forceinline__ bool wait_tag(const int* tag, int want) {
  const volatile int* v = tag;
  if (*v == want) return true;
  const unsigned long long t0 = global_timer_ns();
  while (*v != want) {
    if (global_timer_ns() - t0 > kWaitTimeoutNs) {
      record_error(KVATTN_ERR_TIMEOUT);
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

// One contiguous global -> shared bulk copy (TMA engine), completion counted on `bar`.
// dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// D = A(16x16 f16, row) * B(16x8 f16, col), fp32 accumulate, starting from zero.
__device__ __forceinline__ void mma_f16_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}

// D += A(16x16 f16, row) * B(16x8 f16, col), fp32 accumulate.
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose of an 8x8 b16 matrix spread over the warp in mma fragment order.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// (x & mask) | orv in one LOP3.
__device__ __forceinline__ uint32_t and_or(uint32_t x, uint32_t mask, uint32_t orv) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "r"(mask), "r"(orv));
  return r;
}

// x | (y & mask)
__device__ __forceinline__ uint32_t or_and(uint32_t x, uint32_t y, uint32_t mask) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xF8;" : "=r"(r) : "r"(x), "r"(y), "r"(mask));
  return r;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Two fp32 -> packed f16x2 (lo in the low half), round to nearest.
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float half_lo(uint32_t h2) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFF)));
}
__device__ __forceinline__ float half_hi(uint32_t h2) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16)));
}

// Hardware base-2 exponential (MUFU); exp2(-inf) = 0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace kvattn
