// Slot-mapped KV write and physical block copy.
//
// Write ("大模型推理的KV Cache管理…优化实战" §二 append_slot; "LLM 推理优化深度解析"
// §KV Cache 的本质): row t of k / v [T, Hkv, D] goes to
// cache[slot / 16][h][slot % 16][:], slot = slot_mapping[t]; -1 skips.
// Quantised caches store per-(token, head) absmax codes (ascendai.csdn.net
// article §三 1. KV Cache量化; "KV Cache 与 PagedAttention" §三个直接推论):
// a = max|x|, s = a / 127 or a / 448, code = RNE(x / s) clamped, with IEEE
// fp32 divisions (this translation unit is compiled without fast-math).
// The asymmetric uint8 format ("大模型推理的KV Cache管理…优化实战" §四
// quantize_key, per-channel statistics over head_dim) stores, per (token,
// head), s = (max - min) / 255, z = RNE(-min / s) and code = RNE((x - min) / s),
// both clamped to [0, 255]; s = 0 stores zeros.
//
// Copy (ascendai.csdn.net article §二 写时复制): block dst := block src for K,
// V, scales and zero points.
#pragma once

#include "pkv_device.cuh"

namespace pkv {

constexpr int kBlockTokens = 16;

// 16-bit caches: a bit copy, one thread per 16-byte chunk of a (token, head)
// row; consecutive threads touch consecutive chunks of the same row.
template <int kChunks>
__global__ void __launch_bounds__(256) kv_write_copy_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                                            uint4* __restrict__ kc, uint4* __restrict__ vc,
                                                            const int64_t* __restrict__ slots, int num_tokens,
                                                            int num_kv_heads, int num_blocks) {
  // a decode launched behind this write may start its prologue now; it waits
  // for this grid to finish before it reads the cache
  asm volatile("griddepcontrol.launch_dependents;");
  const long long total = static_cast<long long>(num_tokens) * num_kv_heads * kChunks;
  const long long slot_limit = static_cast<long long>(num_blocks) * kBlockTokens;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(i % kChunks);
    const long long row = i / kChunks;  // t * Hkv + h
    const int h = static_cast<int>(row % num_kv_heads);
    const long long t = row / num_kv_heads;
    const long long slot = slots[t];
    if (slot < 0) continue;
    if (slot >= slot_limit) {
      if (c == 0) raise_status(PKV_DEV_BAD_SLOT);
      continue;
    }
    const long long blk = slot / kBlockTokens;
    const int off = static_cast<int>(slot % kBlockTokens);
    const long long dst = ((blk * num_kv_heads + h) * kBlockTokens + off) * kChunks + c;
    const uint4 kv = __ldg(k + i);
    const uint4 vv = __ldg(v + i);
    kc[dst] = kv;
    vc[dst] = vv;
  }
}

template <bool kInBF16>
__device__ __forceinline__ float load_in(const void* p, long long idx) {
  if constexpr (kInBF16) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[idx]);
  } else {
    return __half2float(reinterpret_cast<const __half*>(p)[idx]);
  }
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

__device__ __forceinline__ float warp_min(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fminf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// RNE of y clamped to [0, 255] (y >= 0 or +inf for codes; any sign for the
// zero point).
__device__ __forceinline__ uint32_t round_u8(float y) {
  return static_cast<uint32_t>(fminf(fmaxf(rintf(y), 0.0f), 255.0f));
}

// E2M1 code of y (|y| <= 6), round to nearest, ties to the even code
// (mantissa bit 0), sign of zero kept.  Magnitude codes 0..7 stand for
// 0, 0.5, 1, 1.5, 2, 3, 4, 6; the code is the number of decision points
// below |y|, where a tie counts when the upper neighbour is the even code.
__device__ __forceinline__ uint32_t e2m1_code(float y) {
  const float a = fabsf(y);
  const uint32_t m = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) + (a >= 3.5f) +
                     (a > 5.0f);
  return m | (signbit(y) ? 8u : 0u);
}

// One quantised code from x given scale s (s > 0).
template <bool kFP8>
__device__ __forceinline__ uint32_t quantize_one(float x, float s) {
  const float y = __fdiv_rn(x, s);
  if constexpr (kFP8) {
    const float yc = fminf(fmaxf(y, -448.0f), 448.0f);
    return static_cast<uint32_t>(__nv_cvt_float_to_fp8(yc, __NV_SATFINITE, __NV_E4M3));
  } else {
    int q = __float2int_rn(y);
    q = max(-127, min(127, q));
    return static_cast<uint32_t>(q) & 0xFFu;
  }
}

// Quantising write: one warp per (token, head) row, D / 32 elements per lane.
// kFmt: PKV_I8 or PKV_FP8E4M3 (symmetric absmax) or PKV_U8ASYM (min/max with
// a zero point; kz / vz receive the zero points) or PKV_I4 / PKV_FP4E2M1
// (symmetric absmax, two codes per byte, element 2k in the low nibble).
template <int kD, int kFmt, bool kInBF16>
__global__ void __launch_bounds__(256) kv_write_quant_kernel(const void* __restrict__ k, const void* __restrict__ v,
                                                             uint8_t* __restrict__ kc, uint8_t* __restrict__ vc,
                                                             float* __restrict__ ks, float* __restrict__ vs,
                                                             uint8_t* __restrict__ kz, uint8_t* __restrict__ vz,
                                                             const int64_t* __restrict__ slots, int num_tokens,
                                                             int num_kv_heads, int num_blocks) {
  constexpr int kE = kD / 32;
  constexpr bool kFP8 = kFmt == PKV_FP8E4M3;
  constexpr bool kAsym = kFmt == PKV_U8ASYM;
  constexpr bool k4 = kFmt == PKV_I4 || kFmt == PKV_FP4E2M1;
  constexpr int kRowBytes = k4 ? kD / 2 : kD;
  asm volatile("griddepcontrol.launch_dependents;");  // see kv_write_copy_kernel
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(num_tokens) * num_kv_heads;
  const long long slot_limit = static_cast<long long>(num_blocks) * kBlockTokens;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long row = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5; row < rows;
       row += warps) {
    const long long t = row / num_kv_heads;
    const int h = static_cast<int>(row % num_kv_heads);
    const long long slot = slots[t];
    if (slot < 0) continue;
    if (slot >= slot_limit) {
      if (lane == 0) raise_status(PKV_DEV_BAD_SLOT);
      continue;
    }
    const long long blk = slot / kBlockTokens;
    const int off = static_cast<int>(slot % kBlockTokens);
    const long long dst_row = (blk * num_kv_heads + h) * kBlockTokens + off;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const void* src = which == 0 ? k : v;
      uint8_t* cache = which == 0 ? kc : vc;
      float* scales = which == 0 ? ks : vs;
      float x[kE];
#pragma unroll
      for (int e = 0; e < kE; ++e) x[e] = load_in<kInBF16>(src, row * kD + lane * kE + e);
      float s;
      uint32_t packed = 0;
      if constexpr (kAsym) {
        float lo = x[0], hi = x[0];
#pragma unroll
        for (int e = 1; e < kE; ++e) {
          lo = fminf(lo, x[e]);
          hi = fmaxf(hi, x[e]);
        }
        lo = warp_min(lo);
        hi = warp_max(hi);
        s = __fdiv_rn(__fsub_rn(hi, lo), 255.0f);
        uint32_t z = 0;
        if (s > 0.0f) {
          z = round_u8(__fdiv_rn(-lo, s));
#pragma unroll
          for (int e = 0; e < kE; ++e) packed |= round_u8(__fdiv_rn(__fsub_rn(x[e], lo), s)) << (8 * e);
        }
        if (lane == 0) (which == 0 ? kz : vz)[dst_row] = static_cast<uint8_t>(z);
      } else if constexpr (k4) {
        float a = 0.0f;
#pragma unroll
        for (int e = 0; e < kE; ++e) a = fmaxf(a, fabsf(x[e]));
        a = warp_max(a);
        constexpr bool kF4 = kFmt == PKV_FP4E2M1;
        s = __fdiv_rn(a, kF4 ? 6.0f : 7.0f);
        if (a > 0.0f) {
#pragma unroll
          for (int e = 0; e < kE; ++e) {
            const float y = __fdiv_rn(x[e], s);
            uint32_t c;
            if constexpr (kF4) {
              c = e2m1_code(fminf(fmaxf(y, -6.0f), 6.0f));
            } else {
              c = static_cast<uint32_t>(max(-7, min(7, __float2int_rn(y)))) & 0xFu;
            }
            packed |= c << (4 * e);
          }
        }
      } else {
        float a = 0.0f;
#pragma unroll
        for (int e = 0; e < kE; ++e) a = fmaxf(a, fabsf(x[e]));
        a = warp_max(a);
        s = __fdiv_rn(a, kFP8 ? 448.0f : 127.0f);
        if (a > 0.0f) {
#pragma unroll
          for (int e = 0; e < kE; ++e) packed |= quantize_one<kFP8>(x[e], s) << (8 * e);
        }
      }
      // a lane's kE codes are contiguous: kE bytes, or kE / 2 bytes of nibbles
      if constexpr (k4 && kE == 2) {
        (cache + dst_row * kRowBytes)[lane] = static_cast<uint8_t>(packed);
      } else if constexpr ((k4 && kE == 4) || (!k4 && kE == 2)) {
        reinterpret_cast<uint16_t*>(cache + dst_row * kRowBytes)[lane] = static_cast<uint16_t>(packed);
      } else {
        reinterpret_cast<uint32_t*>(cache + dst_row * kRowBytes)[lane] = packed;
      }
      if (lane == 0) scales[dst_row] = s;
    }
  }
}

// Block copy: grid.x walks pairs, each CTA copies whole blocks with 16-byte
// vectors.  `words` = 16-byte units per block of one cache; `swords` = 16-byte
// units of one block's scales (0 for 16-bit caches); `zwords` those of its
// zero points (0 unless the format has them).
__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4* __restrict__ kc, uint4* __restrict__ vc,
                                                          uint4* __restrict__ ks, uint4* __restrict__ vs,
                                                          uint4* __restrict__ kz, uint4* __restrict__ vz,
                                                          const int32_t* __restrict__ pairs, int num_pairs,
                                                          int num_blocks, long long words, int swords, int zwords) {
  for (int p = blockIdx.x; p < num_pairs; p += gridDim.x) {
    const int src = pairs[2 * p];
    const int dst = pairs[2 * p + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
      if (threadIdx.x == 0) raise_status(PKV_DEV_BAD_PAIR);
      continue;
    }
    const uint4* ks_src = kc + src * words;
    const uint4* vs_src = vc + src * words;
    uint4* kd = kc + dst * words;
    uint4* vd = vc + dst * words;
    for (long long i = threadIdx.x; i < words; i += blockDim.x) {
      const uint4 a = ks_src[i];
      const uint4 b = vs_src[i];
      kd[i] = a;
      vd[i] = b;
    }
    for (int i = threadIdx.x; i < swords; i += blockDim.x) {
      ks[static_cast<long long>(dst) * swords + i] = ks[static_cast<long long>(src) * swords + i];
      vs[static_cast<long long>(dst) * swords + i] = vs[static_cast<long long>(src) * swords + i];
    }
    for (int i = threadIdx.x; i < zwords; i += blockDim.x) {
      kz[static_cast<long long>(dst) * zwords + i] = kz[static_cast<long long>(src) * zwords + i];
      vz[static_cast<long long>(dst) * zwords + i] = vz[static_cast<long long>(src) * zwords + i];
    }
  }
}

}  // namespace pkv
