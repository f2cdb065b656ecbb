// Single-query GQA decode attention over a block-table-indexed KV cache.
//
// Method ("LLM 推理优化深度解析" §KV Cache 的本质, §MQA 与 GQA, §PagedAttention；
// ascendai.csdn.net article §二 Fig. 2): every sequence's one new query per
// head attends to all of its cached keys/values; the cache lives in 16-token
// physical blocks reached through the sequence's block table; query head i
// reads KV head i / G.
//
// Design for sm_100a (HBM-bound: every K/V byte is read once):
//   * grid = (partition, kv_head, sequence); one CTA serves the whole GQA
//     group of a KV head, so the group's G queries share one read of K/V;
//   * each warp owns a ring of kR shared-memory stages fed by TMA: per
//     16-token block, 2-D tiled tensor copies of the K and V rows (128-byte
//     swizzle, so ldmatrix reads are bank-conflict free) plus untiled bulk
//     copies of the per-token scales of quantised caches, completing on one
//     mbarrier per stage; waits are bounded;
//   * both contractions run on the tensor cores with the block's 16 tokens
//     as the M dimension and the (zero-padded) query group as N = 8:
//       S^T[16 tok x 8 g]  = K[16 x D] . Q^T[D x 8]         (mma.m16n8k16)
//       O^T[D x 8 g]      += V^T[D x 16 tok] . P^T[16 x 8]
//     P^T is built from the S^T accumulators in registers with movmatrix;
//     8-bit codes are widened to fp16 in registers (int8 exactly through the
//     0x6400 exponent trick, e4m3 with the hardware converter) and their
//     per-token scales fold into S (keys) and P (values);
//   * online softmax in fp32 (base-2 exponentials), per warp; warps merge
//     through shared memory with a log-sum-exp rule; long contexts split into
//     token partitions whose (m, l, o) partials a reduce kernel merges.
#pragma once

#include "pkv_device.cuh"

namespace pkv {

enum CacheType : int { kF16 = PKV_F16, kBF16 = PKV_BF16, kI8 = PKV_I8, kFP8 = PKV_FP8E4M3 };

constexpr int round_up_c(int x, int m) { return (x + m - 1) / m * m; }

template <int kD, int kCT>
struct DecodeTraits {
  static constexpr bool k8bit = (kCT == kI8 || kCT == kFP8);
  static constexpr int kElt = k8bit ? 1 : 2;
  static constexpr int kRowBytes = kD * kElt;                       // one token's K (or V) row
  static constexpr int kTileBytes = kRowBytes < 128 ? kRowBytes : 128;  // TMA box width == swizzle span
  static constexpr int kNumColTiles = kRowBytes / kTileBytes;
  static constexpr int kColTileBytes = 16 * kTileBytes;             // 16 tokens x one column tile
  static constexpr int kChunksPerTileRow = kTileBytes / 16;
  static constexpr int kKVBytes = 16 * kRowBytes;                   // one block of one head, K or V
  static constexpr int kScaleBytes = k8bit ? 64 : 0;                // 16 fp32 scales
  static constexpr int kStageTx = 2 * kKVBytes + 2 * kScaleBytes;   // bytes landing per stage
  static constexpr int kStageBytes = round_up_c(kStageTx, 1024);    // keeps every tile 1024-aligned
  static constexpr int kWarps = 4;
  static constexpr int kRing = (24 * 1024) / kStageBytes < 2 ? 2 : (24 * 1024) / kStageBytes;
};

struct DecodeParams {
  void* out;
  const void* q;
  const float* k_scale;
  const float* v_scale;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* part_m;   // [B, Hq, NP]   (split only)
  float* part_l;   // [B, Hq, NP]
  float* part_o;   // [B, Hq, NP, D]
  int num_q_heads;
  int num_kv_heads;
  int group;
  int max_blocks_per_seq;
  int num_blocks;
  int partition_blocks;
  int num_partitions;
  int max_context_len;
  float qk_scale_log2;  // softmax scale * log2(e)
};

// Context length of sequence s as the kernels use it: clamped to what the
// grid and the block table can cover (an out-of-range value raises a bit).
__device__ __forceinline__ int clamp_context(int ctx, int max_ctx, int max_blocks, bool report) {
  const int cap = min(max_ctx, max_blocks * 16);
  if (ctx < 0 || ctx > cap) {
    if (report) raise_status(PKV_DEV_BAD_CONTEXT);
    ctx = ctx < 0 ? 0 : cap;
  }
  return ctx;
}

// Byte offset, inside one K (or V) block region of a stage, of 16-byte chunk
// `c` (counted along the whole row) of token row `t`, as TMA wrote it with
// the 128-byte (or, for 64-byte rows, 64-byte) swizzle.
template <class Tr>
__device__ __forceinline__ uint32_t swz(int t, int c) {
  const int ct = c / Tr::kChunksPerTileRow;
  const int cc = c % Tr::kChunksPerTileRow;
  int x;
  if constexpr (Tr::kTileBytes == 128) {
    x = cc ^ (t & 7);
  } else {
    x = cc ^ ((t >> 1) & 3);
  }
  return static_cast<uint32_t>(ct * Tr::kColTileBytes + t * Tr::kTileBytes + (x << 4));
}

template <bool kOutBF16>
__device__ __forceinline__ void store_out(void* out, long long idx, float v) {
  if constexpr (kOutBF16) {
    reinterpret_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
  } else {
    reinterpret_cast<__half*>(out)[idx] = __float2half_rn(v);
  }
}

// Loads two consecutive query elements (d, d+1) as the mma B operand type.
template <int kCT, bool kQBF16>
__device__ __forceinline__ uint32_t load_q_pair(const void* q, long long idx) {
  const uint32_t raw = *reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint16_t*>(q) + idx);
  if constexpr (kCT == kI8 || kCT == kFP8) {
    if constexpr (kQBF16) {
      const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&raw);
      const __half2 h = __float22half2_rn(__bfloat1622float2(b));
      return *reinterpret_cast<const uint32_t*>(&h);
    }
  }
  return raw;
}

template <int kD, int kCT, int kNT, bool kQBF16>
__global__ void __launch_bounds__(DecodeTraits<kD, kCT>::kWarps * 32)
    paged_decode_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                        const DecodeParams p) {
  using Tr = DecodeTraits<kD, kCT>;
  constexpr bool k8 = Tr::k8bit;
  constexpr bool kMmaBF16 = (kCT == kBF16);
  constexpr bool kOutBF16 = k8 ? kQBF16 : (kCT == kBF16);
  constexpr int kW = Tr::kWarps;
  constexpr int kR = Tr::kRing;
  constexpr int kKS = kD / 16;  // k-steps of S^T = K Q^T
  constexpr int kMT = kD / 16;  // m-tiles of O^T = V^T P^T
  constexpr int kGP = 8 * kNT;  // padded group
  static_assert(kR * Tr::kStageBytes >= (2 * kGP + kGP * kD) * 4, "warp ring too small for the merge");

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw_addr);
  const uint32_t bar_base = base + kW * kR * Tr::kStageBytes;
  int32_t* const blk_ids = reinterpret_cast<int32_t*>(base_ptr + kW * kR * Tr::kStageBytes + kW * kR * 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int r = lane >> 2;
  const int q4 = lane & 3;
  const int part = blockIdx.x;
  const int h = blockIdx.y;
  const int s = blockIdx.z;
  const int G = p.group;
  const int Hq = p.num_q_heads;
  const bool split = p.num_partitions > 1;

  const int ctx = clamp_context(p.context_lens[s], p.max_context_len, p.max_blocks_per_seq,
                                threadIdx.x == 0 && part == 0 && h == 0);
  const int tok_begin = part * p.partition_blocks * 16;
  const int tok_end = min(ctx, tok_begin + p.partition_blocks * 16);
  const int nblk = tok_end > tok_begin ? (tok_end - tok_begin + 15) / 16 : 0;
  const long long head_row0 = static_cast<long long>(s) * Hq + static_cast<long long>(h) * G;

  if (nblk == 0) {
    if (!split) {  // empty sequence: zero output rows
      for (int idx = threadIdx.x; idx < G * kD; idx += blockDim.x)
        store_out<kOutBF16>(p.out, head_row0 * kD + idx, 0.0f);
    }
    return;
  }

  // ---- block ids of this partition, barriers ----
  const int32_t* bt = p.block_tables + static_cast<long long>(s) * p.max_blocks_per_seq +
                      static_cast<long long>(part) * p.partition_blocks;
  for (int i = threadIdx.x; i < nblk; i += blockDim.x) {
    int id = bt[i];
    if (static_cast<unsigned>(id) >= static_cast<unsigned>(p.num_blocks)) {
      raise_status(PKV_DEV_BAD_BLOCK);
      id = 0;
    }
    blk_ids[i] = id;
  }
  if (lane == 0) {
#pragma unroll
    for (int j = 0; j < kR; ++j) mbar_init(bar_base + (warp * kR + j) * 8, 1);
    fence_barrier_init();
  }
  __syncthreads();

  const int count = nblk > warp ? (nblk - warp + kW - 1) / kW : 0;  // blocks of this warp
  const uint32_t ring = base + warp * kR * Tr::kStageBytes;
  const uint32_t bars = bar_base + warp * kR * 8;

  auto issue = [&](int k) {
    const int stage = k % kR;
    const uint32_t st = ring + stage * Tr::kStageBytes;
    const uint32_t bar = bars + stage * 8;
    const int phys = blk_ids[warp + k * kW];
    const int row0 = (phys * p.num_kv_heads + h) * 16;
    mbar_arrive_expect_tx(bar, Tr::kStageTx);
#pragma unroll
    for (int ct = 0; ct < Tr::kNumColTiles; ++ct) {
      const int x = ct * (Tr::kTileBytes / Tr::kElt);
      tma_load_2d(st + ct * Tr::kColTileBytes, &kmap, x, row0, bar);
      tma_load_2d(st + Tr::kKVBytes + ct * Tr::kColTileBytes, &vmap, x, row0, bar);
    }
    if constexpr (k8) {
      const long long so = static_cast<long long>(row0);
      bulk_load(st + 2 * Tr::kKVBytes, p.k_scale + so, 64, bar);
      bulk_load(st + 2 * Tr::kKVBytes + 64, p.v_scale + so, 64, bar);
    }
  };

  if (lane == 0) {
    const int pre = count < kR ? count : kR;
    for (int k = 0; k < pre; ++k) issue(k);
  }

  // ---- query fragments: B operand of S^T = K Q^T (Q^T is D x 8 per n-tile) ----
  uint32_t qf[kNT][kKS][2];
#pragma unroll
  for (int nt = 0; nt < kNT; ++nt) {
    const int g = nt * 8 + r;
    const bool valid = g < G;
    const long long qrow = (head_row0 + (valid ? g : 0)) * kD;
#pragma unroll
    for (int j = 0; j < kKS; ++j) {
      // 16-bit K: k-index 2q,2q+1 -> d 16j+2q.. ; 2q+8.. -> d 16j+8+2q..
      // 8-bit K:  k-index 2q,2q+1 -> d 16j+4q.. ; 2q+8.. -> d 16j+4q+2..
      const int da = k8 ? 16 * j + 4 * q4 : 16 * j + 2 * q4;
      const int db = k8 ? da + 2 : da + 8;
      qf[nt][j][0] = valid ? load_q_pair<kCT, kQBF16>(p.q, qrow + da) : 0u;
      qf[nt][j][1] = valid ? load_q_pair<kCT, kQBF16>(p.q, qrow + db) : 0u;
    }
  }

  float o[kMT][kNT][4];
  float m_run[kNT][2], l_run[kNT][2];
#pragma unroll
  for (int nt = 0; nt < kNT; ++nt) {
    m_run[nt][0] = m_run[nt][1] = -INFINITY;
    l_run[nt][0] = l_run[nt][1] = 0.0f;
#pragma unroll
    for (int i = 0; i < kMT; ++i) o[i][nt][0] = o[i][nt][1] = o[i][nt][2] = o[i][nt][3] = 0.0f;
  }

  bool timed_out = false;
  for (int k = 0; k < count; ++k) {
    const int stage = k % kR;
    const uint32_t st = ring + stage * Tr::kStageBytes;
    const bool landed = mbar_wait(bars + stage * 8, (k / kR) & 1);
    if (__any_sync(0xffffffffu, !landed)) {  // warp-uniform: never split the warp before ldmatrix/mma
      timed_out = true;
      break;
    }
    const int tok0 = tok_begin + (warp + k * kW) * 16;
    const int valid = tok_end - tok0;  // >= 1 tokens of this block count

    // ---- S^T = K . Q^T ----
    float sacc[kNT][4];
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.0f;
    if constexpr (!k8) {
      const int t = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int j = 0; j < kKS; ++j) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(st + swz<Tr>(t, 2 * j + (lane >> 4)), a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) mma_16816<kMmaBF16>(sacc[nt], a0, a1, a2, a3, qf[nt][j][0], qf[nt][j][1]);
      }
    } else {
      const int t = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int j = 0; j < kKS; j += 2) {
        uint32_t w[4];
        ldsm_x4(st + swz<Tr>(t, j + (lane >> 4)), w[0], w[1], w[2], w[3]);
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          uint32_t lo_r, hi_r, lo_r8, hi_r8;  // (d 4q,4q+1) and (d 4q+2,4q+3) of tokens r and r+8
          if constexpr (kCT == kI8) {
            const uint32_t u0 = w[2 * jj] ^ 0x80808080u, u1 = w[2 * jj + 1] ^ 0x80808080u;
            lo_r = i8pair_to_h2(u0, 0x4140u);
            hi_r = i8pair_to_h2(u0, 0x4342u);
            lo_r8 = i8pair_to_h2(u1, 0x4140u);
            hi_r8 = i8pair_to_h2(u1, 0x4342u);
          } else {
            lo_r = e4m3pair_to_h2(w[2 * jj]);
            hi_r = e4m3pair_to_h2(w[2 * jj] >> 16);
            lo_r8 = e4m3pair_to_h2(w[2 * jj + 1]);
            hi_r8 = e4m3pair_to_h2(w[2 * jj + 1] >> 16);
          }
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt)
            mma_16816<false>(sacc[nt], lo_r, lo_r8, hi_r, hi_r8, qf[nt][j + jj][0], qf[nt][j + jj][1]);
        }
      }
    }

    // ---- scale, mask, online softmax (base 2) ----
    float f_r = p.qk_scale_log2, f_r8 = p.qk_scale_log2;
    float vs_r = 1.0f, vs_r8 = 1.0f;
    if constexpr (k8) {
      const float* sc = reinterpret_cast<const float*>(base_ptr + (st - base) + 2 * Tr::kKVBytes);
      f_r *= sc[r];
      f_r8 *= sc[r + 8];
      vs_r = sc[16 + r];
      vs_r8 = sc[16 + r + 8];
    }
    const bool ok_r = r < valid;
    const bool ok_r8 = r + 8 < valid;
    uint32_t pb[kNT][2];
    bool grow = false;
    float alpha[kNT][2];
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
      const float s0 = ok_r ? sacc[nt][0] * f_r : -INFINITY;
      const float s1 = ok_r ? sacc[nt][1] * f_r : -INFINITY;
      const float s2 = ok_r8 ? sacc[nt][2] * f_r8 : -INFINITY;
      const float s3 = ok_r8 ? sacc[nt][3] * f_r8 : -INFINITY;
      float mx_a = fmaxf(s0, s2), mx_b = fmaxf(s1, s3);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, off));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, off));
      }
      const float mn_a = fmaxf(m_run[nt][0], mx_a);
      const float mn_b = fmaxf(m_run[nt][1], mx_b);
      grow |= (mn_a > m_run[nt][0]) || (mn_b > m_run[nt][1]);
      alpha[nt][0] = mn_a == m_run[nt][0] ? 1.0f : fast_exp2(m_run[nt][0] - mn_a);
      alpha[nt][1] = mn_b == m_run[nt][1] ? 1.0f : fast_exp2(m_run[nt][1] - mn_b);
      m_run[nt][0] = mn_a;
      m_run[nt][1] = mn_b;
      const float p0 = fast_exp2(s0 - mn_a), p1 = fast_exp2(s1 - mn_b);
      const float p2 = fast_exp2(s2 - mn_a), p3 = fast_exp2(s3 - mn_b);
      l_run[nt][0] = l_run[nt][0] * alpha[nt][0] + (p0 + p2);
      l_run[nt][1] = l_run[nt][1] * alpha[nt][1] + (p1 + p3);
      // P^T operand: rows = tokens of the block, columns = query heads
      pb[nt][0] = movmatrix_t(pack2<kMmaBF16>(p0 * vs_r, p1 * vs_r));
      pb[nt][1] = movmatrix_t(pack2<kMmaBF16>(p2 * vs_r8, p3 * vs_r8));
    }
    if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
      for (int i = 0; i < kMT; ++i)
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
          o[i][nt][0] *= alpha[nt][0];
          o[i][nt][1] *= alpha[nt][1];
          o[i][nt][2] *= alpha[nt][0];
          o[i][nt][3] *= alpha[nt][1];
        }
    }

    // ---- O^T += V^T . P^T ----
    const uint32_t vt = st + Tr::kKVBytes;
    if constexpr (!k8) {
      const int t = (lane & 7) + (lane >> 4) * 8;
#pragma unroll
      for (int i = 0; i < kMT; ++i) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(vt + swz<Tr>(t, 2 * i + ((lane >> 3) & 1)), a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) mma_16816<kMmaBF16>(o[i][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
      }
    } else {
      const int t = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int i = 0; i < kMT; i += 2) {
        uint32_t w[4];
        ldsm_x4_t(vt + swz<Tr>(t, i + (lane >> 4)), w[0], w[1], w[2], w[3]);
#pragma unroll
        for (int ii = 0; ii < 2; ++ii) {
          // w = [A0 A1 B0 B1]: tokens 2q (A) and 2q+1 (B) at d 16(i+ii)+2r (0) and +1 (1)
          uint32_t x0, x1, y0, y1;  // x: tokens 0-7 of the block, y: tokens 8-15
          if constexpr (kCT == kI8) {
            const uint32_t u0 = w[2 * ii] ^ 0x80808080u, u1 = w[2 * ii + 1] ^ 0x80808080u;
            x0 = i8pair_to_h2(u0, 0x4240u);
            x1 = i8pair_to_h2(u0, 0x4341u);
            y0 = i8pair_to_h2(u1, 0x4240u);
            y1 = i8pair_to_h2(u1, 0x4341u);
          } else {
            const uint32_t t0 = prmt(w[2 * ii], w[2 * ii], 0x3120u);
            const uint32_t t1 = prmt(w[2 * ii + 1], w[2 * ii + 1], 0x3120u);
            x0 = e4m3pair_to_h2(t0);
            x1 = e4m3pair_to_h2(t0 >> 16);
            y0 = e4m3pair_to_h2(t1);
            y1 = e4m3pair_to_h2(t1 >> 16);
          }
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt) mma_16816<false>(o[i + ii][nt], x0, x1, y0, y1, pb[nt][0], pb[nt][1]);
        }
      }
    }

    __syncwarp();
    if (lane == 0 && k + kR < count) issue(k + kR);
  }

  // ---- merge the warps of this CTA (log-sum-exp), then write ----
  const bool any_timeout = __syncthreads_or(timed_out) != 0;
  float* const wbase = reinterpret_cast<float*>(base_ptr);
  const int region = kR * Tr::kStageBytes / 4;  // floats per warp region
  if (!any_timeout) {
    float* mw = wbase + warp * region;
    float* lw = mw + kGP;
    float* ow = lw + kGP;
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
      float la = l_run[nt][0], lb = l_run[nt][1];
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        la += __shfl_xor_sync(0xffffffffu, la, off);
        lb += __shfl_xor_sync(0xffffffffu, lb, off);
      }
      const int ga = nt * 8 + 2 * q4;
      if (r == 0) {
        mw[ga] = m_run[nt][0];
        mw[ga + 1] = m_run[nt][1];
        lw[ga] = la;
        lw[ga + 1] = lb;
      }
#pragma unroll
      for (int i = 0; i < kMT; ++i) {
        // output row d of the C fragment halves (c0,c1) and (c2,c3)
        const int d0 = k8 ? 16 * i + 2 * r : 16 * i + r;
        const int d1 = k8 ? d0 + 1 : d0 + 8;
        ow[ga * kD + d0] = o[i][nt][0];
        ow[(ga + 1) * kD + d0] = o[i][nt][1];
        ow[ga * kD + d1] = o[i][nt][2];
        ow[(ga + 1) * kD + d1] = o[i][nt][3];
      }
    }
  }
  __syncthreads();

  const long long np = p.num_partitions;
  for (int idx = threadIdx.x; idx < G * kD; idx += blockDim.x) {
    const int g = idx / kD;
    const int d = idx - g * kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kW; ++w) {
      const float* mw = wbase + w * region;
      if (w < nblk && !any_timeout) M = fmaxf(M, mw[g]);
    }
    float L = 0.0f, O = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kW; ++w) {
        if (w >= nblk) continue;
        const float* mw = wbase + w * region;
        const float e = fast_exp2(mw[g] - M);
        L += e * mw[kGP + g];
        O += e * mw[2 * kGP + g * kD + d];
      }
    }
    const float val = L > 0.0f ? O / L : 0.0f;
    const long long hrow = head_row0 + g;
    if (!split) {
      store_out<kOutBF16>(p.out, hrow * kD + d, val);
    } else {
      p.part_o[(hrow * np + part) * kD + d] = val;
      if (d == 0) {
        p.part_m[hrow * np + part] = M;
        p.part_l[hrow * np + part] = L;
      }
    }
  }
}

// Merges the partitions of each (sequence, query head):
//   M = max_p m_p, w_p = 2^(m_p - M) l_p, out = sum_p w_p o_p / sum_p w_p.
template <int kD, bool kOutBF16>
__global__ void __launch_bounds__(kD) paged_reduce_kernel(DecodeParams p) {
  const int i = blockIdx.x;
  const int s = blockIdx.y;
  const int d = threadIdx.x;
  const int ctx = clamp_context(p.context_lens[s], p.max_context_len, p.max_blocks_per_seq, false);
  const int ptok = p.partition_blocks * 16;
  const int n = (ctx + ptok - 1) / ptok;
  const long long hrow = static_cast<long long>(s) * p.num_q_heads + i;
  const long long np = p.num_partitions;
  const float* m = p.part_m + hrow * np;
  const float* l = p.part_l + hrow * np;
  const float* o = p.part_o + hrow * np * kD + d;
  float M = -INFINITY;
  for (int j = 0; j < n; ++j) M = fmaxf(M, m[j]);
  float W = 0.0f, O = 0.0f;
  if (M != -INFINITY) {
    for (int j = 0; j < n; ++j) {
      const float w = fast_exp2(m[j] - M) * l[j];
      W += w;
      O += w * o[j * kD];
    }
  }
  store_out<kOutBF16>(p.out, hrow * kD + d, W > 0.0f ? O / W : 0.0f);
}

}  // namespace pkv
