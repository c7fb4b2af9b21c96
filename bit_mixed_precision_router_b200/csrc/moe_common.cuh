// Shared device helpers for the sm_100a kernels: bf16 bit helpers, mbarrier and
// bulk-copy (TMA engine, non-tensor form) wrappers with bounded waits, and the
// warp-level tensor-core MMA used by the weight-streaming GEMV path.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

#define MOE_DEVICE __device__ __forceinline__

namespace moe {

// ---------------------------------------------------------------- bf16 bits
MOE_DEVICE float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
MOE_DEVICE float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
MOE_DEVICE float bf16_bits_to_float(uint16_t v) { return __uint_as_float(uint32_t(v) << 16); }
MOE_DEVICE uint16_t float_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// ---------------------------------------------------------------- shared memory
MOE_DEVICE uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
MOE_DEVICE void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
MOE_DEVICE void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
MOE_DEVICE void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}
MOE_DEVICE bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
MOE_DEVICE uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bit in the device error word set by a wait that ran out.
constexpr unsigned kErrWaitTimeout = 1u;
// A wait gives up after this many nanoseconds of wall time.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Waits for phase `parity` of `bar` to complete.  Never spins forever: after
// kWaitLimitNs it records kErrWaitTimeout in *err and returns false.
MOE_DEVICE bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      atomicOr(err, kErrWaitTimeout);
      return false;
    }
  }
}

// One bulk (non-tensor) global -> shared copy on the TMA engine, completing on
// `bar` with `bytes` of transaction count.  src, dst 16-byte aligned; bytes % 16 == 0.
MOE_DEVICE void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// ---------------------------------------------------------------- warp MMA
// D += A * B, m16n8k16, A row-major 16x16, B column-major 16x8, fp32 accumulate.
// Fragment layout (lane = 4*g + c):
//   A: a[0] = (row g,   k 2c..2c+1), a[1] = (row g+8, k 2c..2c+1),
//      a[2] = (row g,   k 2c+8..2c+9), a[3] = (row g+8, k 2c+8..2c+9)
//   B: b[0] = (k 2c..2c+1, col g), b[1] = (k 2c+8..2c+9, col g)
//   D: d[0..1] = (row g, cols 2c..2c+1), d[2..3] = (row g+8, cols 2c..2c+1)
MOE_DEVICE void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
MOE_DEVICE void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                        uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

MOE_DEVICE uint4 ldg_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

MOE_DEVICE float silu(float g) { return g / (1.0f + expf(-g)); }

// ---------------------------------------------------------------- NVFP4 element conversions
// byte = two E2M1 codes (element 2i in the low nibble) -> fp16x2 (low half = element 2i)
MOE_DEVICE uint32_t e2m1x2_to_h2(uint32_t byte) {
  const __half2_raw r = __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(byte), __NV_E2M1);
  return uint32_t(r.x) | (uint32_t(r.y) << 16);
}
// E4M3 code -> fp16x2 (the value in both halves)
MOE_DEVICE uint32_t e4m3_to_h2(uint32_t byte) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(byte), __NV_E4M3);
  return uint32_t(h.x) | (uint32_t(h.x) << 16);
}
MOE_DEVICE uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

}  // namespace moe

// ---------------------------------------------------------------- host side
namespace moe {
// Device error word of the current device (see moe_check_device_errors).
unsigned* device_error_word();
}  // namespace moe
