// Device-side building blocks for the sm_100a kernels of libpagedkv:
// TMA tensor/bulk copies into shared memory tracked by mbarriers, bounded
// waits, warp-level tensor-core fragments (ldmatrix, mma.sync, movmatrix)
// and the library's device status word.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "../../include/pagedkv.h"

namespace pkv {

// OR of PKV_DEV_* bits raised by kernels of this library on this device.
__device__ unsigned int g_status;

__device__ __forceinline__ void raise_status(unsigned int bit) { atomicOr(&g_status, bit); }

// A wait on a copy barrier gives up after this many nanoseconds of wall time
// (copies complete in microseconds; this only bounds a broken launch).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier --
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// Waits until phase `parity` of the barrier completes; false on timeout
// (after raising PKV_DEV_TIMEOUT).  Never spins without bound.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      raise_status(PKV_DEV_TIMEOUT);
      return false;
    }
  }
  return true;
}

// ------------------------------------------------------------- TMA copies --
// 2-D tiled tensor load (no multicast) into this CTA's shared memory,
// completing `bytes` on the barrier.  x is the innermost coordinate.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Untiled bulk copy global -> shared (16-byte aligned addresses, size a
// multiple of 16), completing on the barrier.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// ------------------------------------------------- warp-level tensor cores --
// Shared-memory fragment loads.  Not volatile, so the compiler may schedule
// them early among register-only work, but with a memory clobber, so they stay
// between the mbarrier wait that makes a stage valid and the copy that
// refills it (both are volatile asm with memory clobbers).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
      : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
      : "r"(addr)
      : "memory");
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
      : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
      : "r"(addr)
      : "memory");
}

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
  uint32_t d;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

// D(16x8, fp32) += A(16x16) * B(16x8); A row-major, B column-major fragments.
template <bool kBF16>
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  if constexpr (kBF16) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

// ----------------------------------------------------------- conversions --
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <bool kBF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (kBF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}

// Two signed int8 codes sitting in bytes (i, j) of w -> fp16x2 (byte i in the
// low half), exactly.  u = w ^ 0x80808080 turns code x into x + 128; placing
// that byte under the fp16 pattern 0x64 gives 1024 + (x + 128); subtracting
// 1152 leaves x.  `sel` picks the two bytes (see callers).
__device__ __forceinline__ uint32_t i8pair_to_h2(uint32_t u, uint32_t sel) {
  uint32_t t = prmt(u, 0x64646464u, sel);
  __half2 h = *reinterpret_cast<__half2*>(&t);
  h = __hsub2(h, __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480)));
  return *reinterpret_cast<uint32_t*>(&h);
}

// Two uint8 codes in bytes (i, j) of w, minus their zero points, -> fp16x2
// (byte i in the low half), exactly.  Placing code c under the fp16 pattern
// 0x64 gives 1024 + c; `zz` holds the fp16 pair (1024 + z_i, 1024 + z_j), so
// the difference is c - z, an integer in [-255, 255].
__device__ __forceinline__ uint32_t u8pair_minus_zero(uint32_t w, uint32_t sel, uint32_t zz) {
  uint32_t t = prmt(w, 0x64646464u, sel);
  __half2 h = __hsub2(*reinterpret_cast<__half2*>(&t), *reinterpret_cast<__half2*>(&zz));
  return *reinterpret_cast<uint32_t*>(&h);
}

// (a & b) ^ c in one instruction.
__device__ __forceinline__ uint32_t and_xor(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Eight signed INT4 codes n0..n7 of w (n0 in the lowest nibble) -> four
// fp16x2 pairs placed under the fp16 pattern 0x6400, exactly:
// x[k] = (1032 + n_k, 1032 + n_{k+4}) for even k (a nibble x + 8 in bits
// 0-3 reads as 1024 + x + 8) and (1152 + 16 n_k, 1152 + 16 n_{k+4}) for odd
// k (a nibble in bits 4-7, no shift, reads as 1024 + 16 (x + 8)).  Flipping
// the nibble's top bit turns x into x + 8; since the masks and 0x6400 share
// no bits, mask, flip and exponent pattern are one three-input operation,
// so five operations per eight codes.  For a dot product whose other operand
// is pre-divided by 16 at the odd positions, the biases add 1032 (even) and
// 72 (odd) times that operand's sum, a constant the caller subtracts.
__device__ __forceinline__ void i4x8_to_h2x4_biased(uint32_t w, uint32_t (&x)[4]) {
  const uint32_t v = w >> 8;
  x[0] = and_xor(w, 0x000F000Fu, 0x64086408u);
  x[1] = and_xor(w, 0x00F000F0u, 0x64806480u);
  x[2] = and_xor(v, 0x000F000Fu, 0x64086408u);
  x[3] = and_xor(v, 0x00F000F0u, 0x64806480u);
}

// Eight E2M1 codes of w (two per byte, low nibble first) -> four fp16x2
// pairs q[k] = (n_2k, n_2k+1) with the hardware converter (exact: every
// E2M1 value is an fp16 value).
__device__ __forceinline__ void e2m1x8_to_h2x4(uint32_t w, uint32_t (&q)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(q[0]), "=r"(q[1]), "=r"(q[2]), "=r"(q[3])
      : "r"(w));
}

// Four E4M3 codes [b0 b1 b2 b3] of v -> fp16x2 (b0, b1) and (b2, b3), low
// byte in the low half, with the hardware converter (exact: e4m3 values are
// all representable in fp16).
__device__ __forceinline__ void e4m3x4_to_h2x2(uint32_t v, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\t"
      "mov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(v));
}

}  // namespace pkv
