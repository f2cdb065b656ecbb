// Single-query GQA decode attention over a block-table-indexed KV cache.
//
// Method ("LLM 推理优化深度解析" §KV Cache 的本质, §MQA 与 GQA, §PagedAttention;
// ascendai.csdn.net article §二 Fig. 2): every sequence's one new query per
// head attends to all of its cached keys/values; the cache lives in 16-token
// physical blocks reached through the sequence's block table; query head i
// reads KV head i / G.
//
// Design for sm_100a (HBM-bound: every K/V byte is read once):
//   * Work list.  All (sequence, KV head, block) triples form one ordered
//     list (sequence-major).  Each warp of a persistent grid (one CTA per SM:
//     8 warps for 16-bit caches, 12 for quantised ones) owns an equal contiguous
//     share of it and streams
//     through that share, crossing (sequence, head) boundaries without
//     stopping its copy pipeline.  The G query heads of a KV head are served
//     together, so the group shares one read of K/V.
//   * Copies.  Each warp owns a ring of shared-memory stages fed by TMA: per
//     block, 2-D tiled tensor copies of the 16-token K and V tiles (128-byte
//     swizzle, 64-byte for 64-byte rows, so ldmatrix reads are bank-conflict
//     free) plus untiled bulk copies of the per-token scales of quantised
//     caches, completing on one mbarrier per stage.  Block ids and copy
//     coordinates for the next 32-block chunk are computed ahead by the lanes.
//     Waits are bounded.
//   * Math.  Both contractions run on the tensor cores with the block's 16
//     tokens as M and the zero-padded query group as N = 8:
//       S^T[16 tok x 8 g]  = K[16 x D] . Q^T[D x 8]         (mma.m16n8k16)
//       O^T[D x 8 g]      += V^T[D x 16 tok] . P^T[16 x 8]
//     P^T comes from the S^T accumulators through movmatrix.  8-bit codes
//     are widened to fp16 in registers (int8 and uint8 exactly through the
//     0x6400 exponent trick, e4m3 with the hardware converter); a uint8
//     code's zero point is subtracted in that same fp16 step (exact: the
//     difference is an integer in [-255, 255]); per-token scales fold into
//     S (keys) and P (values).  Online softmax in fp32, base 2.
//   * Merge.  A warp that saw a whole (sequence, head) writes the output
//     directly.  A pair split across warps gets one fp32 partial (m, l, o/l)
//     per contributing warp; the last contributor to arrive (an epoch-tagged
//     counter per pair, so nothing needs zeroing between calls) merges them
//     with the log-sum-exp rule.  No warp ever waits for another.  Each warp
//     processes the pair at the end of its share first (it is the one shared
//     with the next warp), so merges happen early, not at the kernel's end.
//   * The kernel may launch while the preceding KV write kernel still runs
//     (programmatic dependent launch): it scans the context lengths, reads the
//     block tables and q, and waits for the write only before its first copy
//     from the cache.
//   * Multi-query mode (kMQ: several new tokens per sequence, for chunked
//     prefill and speculative verification, "LLM 推理优化深度解析"
//     §Continuous Batching and §投机解码): the N columns of a pair are
//     (new token, query head) pairs of one KV head, up to 8 * kNT of them per
//     "tile"; a sequence with n new tokens has ceil(n * G / (8 * kNT)) tiles
//     per KV head, each a pair of its own in the work list.  New token t of n
//     sees keys up to position ctx - n + t, so the mask is per column; a
//     column can meet a block that is wholly masked for it, so its running
//     max may still be -inf and the exponentials use a finite base.
#pragma once

#include "pkv_device.cuh"

namespace pkv {

enum CacheType : int {
  kF16 = PKV_F16, kBF16 = PKV_BF16, kI8 = PKV_I8, kFP8 = PKV_FP8E4M3, kU8 = PKV_U8ASYM, kI4 = PKV_I4, kFP4 = PKV_FP4E2M1
};

constexpr int round_up_c(int x, int m) { return (x + m - 1) / m * m; }

// A compile-time int carried as a value (selects a generic lambda's instance).
template <int N>
struct IntC {
  static constexpr int value = N;
};

template <int kD, int kCT>
struct DecodeTraits {
  static constexpr bool k8bit = (kCT == kI8 || kCT == kFP8 || kCT == kU8);
  static constexpr bool k4bit = (kCT == kI4 || kCT == kFP4);
  static constexpr bool kQuant = k8bit || k4bit;                    // per-token scales, fp16 math
  static constexpr int kElt = kQuant ? 1 : 2;                       // bytes per tensor-map element
  static constexpr int kRowBytes = k4bit ? kD / 2 : kD * kElt;      // one token's K (or V) row
  static constexpr int kTileBytes = kRowBytes < 128 ? kRowBytes : 128;  // TMA box width == swizzle span
  static constexpr int kNumColTiles = kRowBytes / kTileBytes;
  static constexpr int kColTileBytes = 16 * kTileBytes;             // 16 tokens x one column tile
  static constexpr int kChunksPerTileRow = kTileBytes / 16;
  static constexpr int kKVBytes = 16 * kRowBytes;                   // one block of one head, K or V
  static constexpr int kScaleBytes = kQuant ? 64 : 0;               // 16 fp32 scales
  static constexpr int kZeroBytes = kCT == kU8 ? 16 : 0;            // 16 uint8 zero points
  // stage layout: K tile, V tile, K scales, V scales, K zero points, V zero points
  static constexpr int kStageTx = 2 * kKVBytes + 2 * kScaleBytes + 2 * kZeroBytes;  // bytes landing per stage
  static constexpr int kStageBytes = round_up_c(kStageTx, 1024);    // keeps every tile 1024-aligned
  // Quantised caches with up to 8 columns per pair run 12 warps per CTA
  // (registers capped at 168 by the launch bounds, three warps per SM
  // sub-partition): their per-block instruction stream, not HBM, sets the
  // pace, so more warps hide more of its latency.  16-bit caches run 8 (up
  // to 8 are supported), and so do 16-column pairs, whose accumulators do not
  // fit 168 registers.
  static constexpr int max_warps(int nt) { return kQuant && nt == 1 ? 12 : 8; }
  // One CTA per SM.  Its warps (chosen per call) share up to this many bytes
  // of copy ring: 8 warps x 2 stages of 8 KiB for bf16 / fp16 at head_dim
  // 128 (measured: 3 stages lose 2-5 %), or 6 stages for a launch of 4
  // warps (the plan's choice for batches whose scan leaves no room for 8);
  // quantised caches 12 warps x 3 stages of 5 KiB (8-bit) or x 5 stages of
  // 3 KiB (4-bit).  The host trims the depth when a large batch's
  // context-length scan needs the shared memory.
  static constexpr int ring_budget(int warps) { return kQuant ? 180 * 1024 : (warps <= 4 ? 192 : 128) * 1024; }
};

// Epoch-tagged arrival counters: bits 63..24 hold the epoch of the call that
// last touched the counter, bits 23..0 the arrivals of that call.
constexpr int kEpochShift = 24;
constexpr unsigned long long kCountMask = (1ull << kEpochShift) - 1;

struct DecodeParams {
  void* out;
  const void* q;
  const float* k_scale;
  const float* v_scale;
  const uint8_t* k_zero;
  const uint8_t* v_zero;
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* query_start_loc;  // [B + 1] (multi-query mode only)
  unsigned long long* counters;  // [B * Hkv * max_tiles] arrival counters (workspace)
  float* slots;                  // [2 * num_streams][slot_floats] partials (workspace)
  int num_seqs;
  int num_q_heads;
  int num_kv_heads;
  int group;
  int max_blocks_per_seq;
  int num_blocks;
  int max_context_len;
  int num_streams;   // warps sharing the work list
  int ring;          // copy stages per warp (set at launch from ring_warps)
  int ring_warps;    // warps per CTA
  int slot_floats;   // ml + C * D: m[C], l[C] padded to ml = round_up(2C, 4), then o[C][D];
                     // C = G (decode) or tile_cols (multi-query)
  int tile_cols;     // multi-query: columns per tile (8 * kNT)
  int max_tiles;     // multi-query: tiles per KV head of the longest query run (1 for decode)
  int num_q_tokens;  // multi-query: rows of q and out
  int window;        // sliding window: a query at position P sees keys P - window + 1 .. P (0: all)
  int max_query_len; // multi-query: host bound of new tokens per sequence (sizes the counters)
  unsigned long long epoch;  // this call's epoch, nonzero, < 2^40
  float qk_scale_log2;       // softmax scale * log2(e)
};

// Context length of sequence s as the kernels use it: clamped to what the
// block table can hold (an out-of-range value raises a status bit).
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
  } else if constexpr (Tr::kTileBytes == 64) {
    x = cc ^ ((t >> 1) & 3);
  } else {  // 32-byte rows, 32-byte swizzle
    x = cc ^ ((t >> 2) & 1);
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
  if constexpr (DecodeTraits<64, kCT>::kQuant) {
    if constexpr (kQBF16) {
      const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&raw);
      const __half2 h = __float22half2_rn(__bfloat1622float2(b));
      return *reinterpret_cast<const uint32_t*>(&h);
    }
  }
  return raw;
}

// Two query elements (d0, d1), not adjacent, as an fp16x2 B operand pair
// (4-bit caches; the mma runs in fp16).
template <bool kQBF16>
__device__ __forceinline__ uint32_t load_q_two(const void* q, long long i0, long long i1) {
  const uint16_t* p = reinterpret_cast<const uint16_t*>(q);
  const uint16_t a = p[i0], b = p[i1];
  __half2 h;
  if constexpr (kQBF16) {
    h = __floats2half2_rn(__bfloat162float(__ushort_as_bfloat16(a)), __bfloat162float(__ushort_as_bfloat16(b)));
  } else {
    h = __halves2half2(__ushort_as_half(a), __ushort_as_half(b));
  }
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void query_range(const DecodeParams& p, int s, int ctx, int& q0, int& q1, int& n,
                                            bool report);

// First block any query of a sequence can see under the sliding window: its
// earliest new token (position ctx - n) sees keys from ctx - n + 1 - window.
// Blocks before it are never read (their table entries may be stale).
__device__ __forceinline__ int window_first_block(const DecodeParams& p, int ctx, int n) {
  if (p.window <= 0) return 0;
  const int lo = ctx - n + 1 - p.window;
  return lo > 0 ? (lo >> 4) : 0;
}

// Work items of sequence s: its blocks from the window's first block on,
// times Hkv, times (multi-query mode) the column tiles of its new tokens.
template <bool kMQ>
__device__ __forceinline__ int items_of(const DecodeParams& p, int s, bool report) {
  const int ctx = clamp_context(p.context_lens[s], p.max_context_len, p.max_blocks_per_seq, report);
  if constexpr (kMQ) {
    int q0, q1, n;
    query_range(p, s, ctx, q0, q1, n, report);
    const int tiles = (n * p.group + p.tile_cols - 1) / p.tile_cols;
    return (((ctx + 15) >> 4) - window_first_block(p, ctx, n)) * p.num_kv_heads * tiles;
  } else {
    return (((ctx + 15) >> 4) - window_first_block(p, ctx, 1)) * p.num_kv_heads;
  }
}

// cum[s] = sum over sequences s' < s of their work items, for s = 0..B; one
// entry per (sequence, KV head[, tile], block) work item before sequence s.
template <bool kMQ>
__device__ __forceinline__ void scan_work(const DecodeParams& p, int32_t* cum) {
  __shared__ int warp_sums[32];
  const int B = p.num_seqs;
  const int nthreads = blockDim.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int per = (B + nthreads - 1) / nthreads;
  const int s0 = min(tid * per, B);
  const int s1 = min(s0 + per, B);
  const bool report = blockIdx.x == 0;
  int local = 0;
  for (int s = s0; s < s1; ++s) local += items_of<kMQ>(p, s, report);
  int x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  int run = x - local;
  for (int w = 0; w < warp; ++w) run += warp_sums[w];
  if (tid == 0) cum[0] = 0;
  for (int s = s0; s < s1; ++s) {
    run += items_of<kMQ>(p, s, false);
    cum[s + 1] = run;
  }
  __syncthreads();
}

// Largest s with cum[s] <= g (g < cum[B]); never lands on an empty sequence.
__device__ __forceinline__ int find_seq(const int32_t* cum, int B, int g) {
  int lo = 0, hi = B;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cum[mid] <= g) lo = mid; else hi = mid;
  }
  return lo;
}

// Blocks per pair of sequence s (a sequence with work has at least one) and
// the first of them (nonzero only under a sliding window).
template <bool kMQ>
__device__ __forceinline__ int pair_blocks(const DecodeParams& p, const int32_t* cum, int s, int& jb) {
  if constexpr (kMQ) {
    const int ctx = clamp_context(p.context_lens[s], p.max_context_len, p.max_blocks_per_seq, false);
    int q0, q1, n;
    query_range(p, s, ctx, q0, q1, n, false);
    jb = window_first_block(p, ctx, n);
    return ((ctx + 15) >> 4) - jb;
  } else {
    jb = p.window > 0
             ? window_first_block(p, clamp_context(p.context_lens[s], p.max_context_len, p.max_blocks_per_seq,
                                                   false), 1)
             : 0;
    return (cum[s + 1] - cum[s]) / p.num_kv_heads;
  }
}

// TMA row coordinate (block * Hkv + head) * 16 of work item g.
template <bool kMQ>
__device__ __forceinline__ int item_row(const DecodeParams& p, const int32_t* cum, int g) {
  const int s = find_seq(cum, p.num_seqs, g);
  int jb;
  const int nb = pair_blocks<kMQ>(p, cum, s, jb);
  const int off = g - cum[s];
  const int pr = off / nb;
  const int j = off - pr * nb;
  // pairs of a sequence run KV head by KV head, tiles innermost
  const int h = kMQ ? pr / ((cum[s + 1] - cum[s]) / (nb * p.num_kv_heads)) : pr;
  int id = p.block_tables[static_cast<long long>(s) * p.max_blocks_per_seq + jb + j];
  if (static_cast<unsigned>(id) >= static_cast<unsigned>(p.num_blocks)) {
    raise_status(PKV_DEV_BAD_BLOCK);
    id = 0;
  }
  return (id * p.num_kv_heads + h) * 16;
}

// Rows [q0, q0 + n) of q / out hold the new tokens of sequence s in
// multi-query mode: query_start_loc clamped to [0, num_q_tokens] and n to
// the context and to max_query_len (an inconsistent entry raises a status
// bit when `report`; rows [q0 + n, q1) are then written as zeros).
__device__ __forceinline__ void query_range(const DecodeParams& p, int s, int ctx, int& q0, int& q1, int& n,
                                            bool report) {
  const int a = p.query_start_loc[s], b = p.query_start_loc[s + 1];
  q0 = min(max(a, 0), p.num_q_tokens);
  q1 = min(max(b, q0), p.num_q_tokens);
  n = min(min(q1 - q0, ctx), p.max_query_len);
  if (report && (a != q0 || b != q1 || q1 - q0 != n)) raise_status(PKV_DEV_BAD_CONTEXT);
}

// First work item of stream w among T items split over nw streams.
__device__ __forceinline__ int stream_start(long long T, long long w, long long nw) {
  return static_cast<int>(T * w / nw);
}

// Stream holding work item g.
__device__ __forceinline__ int stream_of(long long T, long long g, long long nw) {
  return static_cast<int>(((g + 1) * nw - 1) / T);
}

template <int kD, int kCT, int kNT, bool kQBF16, bool kMQ>
__global__ void __launch_bounds__(DecodeTraits<kD, kCT>::max_warps(kNT) * 32)
    paged_decode_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                        const DecodeParams p) {
  using Tr = DecodeTraits<kD, kCT>;
  constexpr bool k8 = Tr::k8bit;
  constexpr bool k4 = Tr::k4bit;
  constexpr bool kQt = Tr::kQuant;
  constexpr bool kMmaBF16 = (kCT == kBF16);
  constexpr bool kOutBF16 = kQt ? kQBF16 : (kCT == kBF16);
  const int kW = blockDim.x >> 5;  // warps of this CTA
  const int kR = p.ring;           // stages per warp (<= 8)
  constexpr int kKS = kD / 16;  // k-steps of S^T = K Q^T
  constexpr int kMT = kD / 16;  // m-tiles of O^T = V^T P^T

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t smem_base = (raw_addr + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (smem_base - raw_addr);
  const uint32_t bar_base = smem_base + kW * kR * Tr::kStageBytes;
  int32_t* const cum = reinterpret_cast<int32_t*>(base_ptr + kW * kR * Tr::kStageBytes + kW * kR * 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int r = lane >> 2;
  const int q4 = lane & 3;
  const int G = p.group;
  const int Hq = p.num_q_heads;
  const int Hkv = p.num_kv_heads;
  const int B = p.num_seqs;

  if (lane == 0) {
    for (int j = 0; j < kR; ++j) mbar_init(bar_base + (warp * kR + j) * 8, 1);
    fence_barrier_init();
  }
  scan_work<kMQ>(p, cum);  // ends with __syncthreads (barrier init visible too)

  // Sequences without context get zero rows (multi-query: rows of new tokens
  // beyond the context).  (Only the caches and scales can still be in flight
  // from a KV write launched just before this kernel; the wait for it comes
  // right before the first copy is issued.)
  for (int s = blockIdx.x; s < B; s += gridDim.x) {
    if constexpr (kMQ) {
      int q0, q1, n;
      query_range(p, s, clamp_context(p.context_lens[s], p.max_context_len, p.max_blocks_per_seq, false), q0, q1,
                  n, false);
      for (long long idx = threadIdx.x; idx < static_cast<long long>(q1 - q0 - n) * Hq * kD; idx += blockDim.x)
        store_out<kOutBF16>(p.out, static_cast<long long>(q0 + n) * Hq * kD + idx, 0.0f);
    } else {
      if (cum[s + 1] == cum[s]) {
        for (int idx = threadIdx.x; idx < Hq * kD; idx += blockDim.x)
          store_out<kOutBF16>(p.out, static_cast<long long>(s) * Hq * kD + idx, 0.0f);
      }
    }
  }

  const long long T = cum[B];
  const long long nw = min(static_cast<long long>(p.num_streams), T);
  const int gw = blockIdx.x * kW + warp;
  if (gw >= nw) return;  // warps are independent from here on
  const int g0 = stream_start(T, gw, nw);
  const int g1 = stream_start(T, gw + 1, nw);
  const int count = g1 - g0;
  // The stream's last pair is usually shared with the next stream: process it
  // first (then wrap to g0), so shared pairs finish early and their merges
  // stay off the end of the kernel.  `offset` = local position of the start
  // of the pair holding item g1 - 1 (0 if that pair began before g0).
  int offset;
  {
    const int sl = find_seq(cum, B, g1 - 1);
    int jbl;
    const int nbl = pair_blocks<kMQ>(p, cum, sl, jbl);
    const int gpl = cum[sl] + ((g1 - 1 - cum[sl]) / nbl) * nbl;
    offset = gpl > g0 ? gpl - g0 : 0;
  }
  auto item_of = [&](int k) { return g0 + (k + offset < count ? k + offset : k + offset - count); };

  const uint32_t ring = smem_base + warp * kR * Tr::kStageBytes;
  const uint32_t bars = bar_base + warp * kR * 8;

  // Copy coordinates of this warp's items, 32 at a time, two chunks ahead.
  int pre0 = lane < count ? item_row<kMQ>(p, cum, item_of(lane)) : 0;
  int pre1 = 32 + lane < count ? item_row<kMQ>(p, cum, item_of(32 + lane)) : 0;

  int istage = 0;  // ring stage of the next item to issue (only lane 0 issues)
  auto issue = [&](int row0) {
    const int stage = istage;
    istage = istage + 1 == kR ? 0 : istage + 1;
    const uint32_t st = ring + stage * Tr::kStageBytes;
    const uint32_t bar = bars + stage * 8;
    mbar_arrive_expect_tx(bar, Tr::kStageTx);
#pragma unroll
    for (int ct = 0; ct < Tr::kNumColTiles; ++ct) {
      const int x = ct * (Tr::kTileBytes / Tr::kElt);
      tma_load_2d(st + ct * Tr::kColTileBytes, &kmap, x, row0, bar);
      tma_load_2d(st + Tr::kKVBytes + ct * Tr::kColTileBytes, &vmap, x, row0, bar);
    }
    if constexpr (kQt) {
      bulk_load(st + 2 * Tr::kKVBytes, p.k_scale + row0, 64, bar);
      bulk_load(st + 2 * Tr::kKVBytes + 64, p.v_scale + row0, 64, bar);
    }
    if constexpr (Tr::kZeroBytes > 0) {
      bulk_load(st + 2 * Tr::kKVBytes + 128, p.k_zero + row0, 16, bar);
      bulk_load(st + 2 * Tr::kKVBytes + 144, p.v_zero + row0, 16, bar);
    }
  };

  // the caches may still be being written by the preceding kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");
#pragma unroll 1
  for (int k = 0; k < kR && k < count; ++k) {
    const int row0 = __shfl_sync(0xffffffffu, pre0, k);
    if (lane == 0) issue(row0);
  }

  // ---- cursor over (sequence, pair, block), in processing order; a pair is
  // a KV head (decode) or a (KV head, column tile) (multi-query) ----
  int s, nb, pr, h, j, ctx;
  int jb = 0;  // first block read (sliding window)
  int ntile = 1, tile = 0, q0 = 0, n_new = 1;  // multi-query only
  auto set_pair = [&]() {
    if constexpr (kMQ) {
      h = pr / ntile;
      tile = pr - h * ntile;
    } else {
      h = pr;
    }
  };
  auto enter_seq = [&]() {
    nb = pair_blocks<kMQ>(p, cum, s, jb);
    ctx = clamp_context(p.context_lens[s], p.max_context_len, p.max_blocks_per_seq, false);
    if constexpr (kMQ) {
      int q1;
      query_range(p, s, ctx, q0, q1, n_new, false);
      ntile = (cum[s + 1] - cum[s]) / (nb * Hkv);
    }
  };
  auto locate = [&](int g) {
    s = find_seq(cum, B, g);
    enter_seq();
    pr = (g - cum[s]) / nb;
    j = (g - cum[s]) - pr * nb;
    set_pair();
  };
  locate(item_of(0));

  // Multi-query: column c of tile `tile` is (new token t, head g) with
  // tile * C + c = t * G + g; its keys are positions < ctx - n_new + t + 1.
  auto col_token = [&](int c) { return (tile * p.tile_cols + c) / G; };
  auto col_head = [&](int c) { return (tile * p.tile_cols + c) % G; };

  // Integer K codes (INT8, uint8, INT4) are widened with their bias left in
  // (e.g. 1152 + c for INT8); the bias times the sum of the query elements
  // it multiplies is subtracted when the block's scores start.  kqs holds,
  // for this lane's two accumulator columns, that sum (uint8: the plain
  // query sum, scaled per token row by 1024 + its zero point).
  constexpr bool kBiasK = (kCT == kI8 || kCT == kU8 || kCT == kI4);
  uint32_t qf[kNT][kKS][2];
  float kqs[kNT][2];
  float o[kMT][kNT][4];
  // Integer V codes are widened with their bias left in as well (INT8
  // 1152 + c, uint8 1024 + c, INT4 1032 + c at even d and 1152 + 16c at odd
  // d).  One more MMA per block accumulates, per column, the weight that
  // bias carries into O^T (wacc = sum over tokens of bias x P), and it is
  // taken out of O^T every kFoldBlocks blocks and when the pair ends; so the
  // bias never builds up over a long context (the cancellation stays within
  // 128 tokens), and O^T is exact up to that rounding.
  constexpr bool kBiasV = kBiasK;
  constexpr int kFoldBlocks = 8;
  float wacc[kNT][4];
  int since_fold = 0;
  float m_run[kNT][2], l_run[kNT][2];
  int colv[kNT][2];  // multi-query: visible keys of the lane's accumulator columns

  auto begin_pair = [&]() {
    since_fold = 0;
    const long long head_row0 = static_cast<long long>(s) * Hq + static_cast<long long>(h) * G;
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
      const int g = nt * 8 + r;
      bool valid;
      long long qrow;
      if constexpr (kMQ) {
        const int t = col_token(g);
        valid = t < n_new;
        qrow = valid ? (static_cast<long long>(q0 + t) * Hq + static_cast<long long>(h) * G + col_head(g)) * kD : 0;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int tc = col_token(nt * 8 + 2 * q4 + c);
          colv[nt][c] = tc < n_new ? ctx - n_new + tc + 1 : ctx;
        }
      } else {
        valid = g < G;
        qrow = (head_row0 + (valid ? g : 0)) * kD;
      }
#pragma unroll
      for (int jj = 0; jj < kKS; ++jj) {
        if constexpr (k4) {
          // 4-bit K: k-step jj is half (jj & 1) of 32-code chunk jj / 2; a
          // lane's word holds d = 32(jj/2) + 8q .. + 7 and the widening
          // pairs them as (0,4)(1,5)(2,6)(3,7) for INT4, (0,1)(2,3)(4,5)(6,7)
          // for E2M1; k-slots 2q,2q+1 take the first pair of the step,
          // 2q+8,2q+9 the second
          const long long b8 = qrow + 32 * (jj >> 1) + 8 * q4;
          int e0, e1, e2, e3;  // d offsets of slots 2q, 2q+1, 2q+8, 2q+9
          if constexpr (kCT == kI4) {
            e0 = 2 * (jj & 1); e1 = e0 + 4; e2 = e0 + 1; e3 = e0 + 5;
          } else {
            e0 = 4 * (jj & 1); e1 = e0 + 1; e2 = e0 + 2; e3 = e0 + 3;
          }
          qf[nt][jj][0] = valid ? load_q_two<kQBF16>(p.q, b8 + e0, b8 + e1) : 0u;
          qf[nt][jj][1] = valid ? load_q_two<kQBF16>(p.q, b8 + e2, b8 + e3) : 0u;
          if constexpr (kCT == kI4) {
            // slots 2q+8, 2q+9 meet odd nibbles, widened at 16x: q / 16 (exact)
            const __half2 h = __hmul2(*reinterpret_cast<const __half2*>(&qf[nt][jj][1]),
                                      __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00)));
            qf[nt][jj][1] = *reinterpret_cast<const uint32_t*>(&h);
          }
        } else {
          // 16-bit K: k-index 2q,2q+1 -> d 16jj+2q.. ; 2q+8.. -> d 16jj+8+2q..
          // 8-bit K:  k-index 2q,2q+1 -> d 16jj+4q.. ; 2q+8.. -> d 16jj+4q+2..
          const int da = k8 ? 16 * jj + 4 * q4 : 16 * jj + 2 * q4;
          const int db = k8 ? da + 2 : da + 8;
          qf[nt][jj][0] = valid ? load_q_pair<kCT, kQBF16>(p.q, qrow + da) : 0u;
          qf[nt][jj][1] = valid ? load_q_pair<kCT, kQBF16>(p.q, qrow + db) : 0u;
        }
      }
      m_run[nt][0] = m_run[nt][1] = -INFINITY;
      l_run[nt][0] = l_run[nt][1] = 0.0f;
#pragma unroll
      for (int i = 0; i < kMT; ++i) o[i][nt][0] = o[i][nt][1] = o[i][nt][2] = o[i][nt][3] = 0.0f;
      wacc[nt][0] = wacc[nt][1] = wacc[nt][2] = wacc[nt][3] = 0.0f;
      if constexpr (kBiasK) {
        // this lane holds column r's query elements at its k-slots: sum them
        // in the weights the biases give them, over the four lanes of the
        // column, then fetch the sums of the lane's accumulator columns
        // 2q and 2q+1 (held by lanes 8q and 8q + 4)
        float sb = 0.0f;
#pragma unroll
        for (int jj = 0; jj < kKS; ++jj) {
          const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&qf[nt][jj][0]));
          const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&qf[nt][jj][1]));
          if constexpr (kCT == kI4) {
            sb += 1032.0f * (a.x + a.y) + 1152.0f * (b.x + b.y);
          } else {
            sb += (a.x + a.y) + (b.x + b.y);
          }
        }
        sb += __shfl_xor_sync(0xffffffffu, sb, 1);
        sb += __shfl_xor_sync(0xffffffffu, sb, 2);
        const float s0 = __shfl_sync(0xffffffffu, sb, 8 * q4);
        const float s1 = __shfl_sync(0xffffffffu, sb, 8 * q4 + 4);
        kqs[nt][0] = kCT == kI8 ? 1152.0f * s0 : s0;
        kqs[nt][1] = kCT == kI8 ? 1152.0f * s1 : s1;
      }
    }
  };
  begin_pair();

  int cstage = 0;        // ring stage of the next item
  uint32_t cphase = 0;   // its barrier phase

  // Scores S^T = K . Q^T of the block in stage `st`: even k-steps accumulate
  // into `ae`, odd ones into `ao` (the same array for one chain per block).
  auto scores = [&](uint32_t st, float (&ae)[kNT][4], float (&ao)[kNT][4]) {
    if constexpr (!kQt) {
      const int t = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int jj = 0; jj < kKS; ++jj) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(st + swz<Tr>(t, 2 * jj + (lane >> 4)), a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt)
          mma_16816<kMmaBF16>((jj & 1) ? ao[nt] : ae[nt], a0, a1, a2, a3, qf[nt][jj][0], qf[nt][jj][1]);
      }
    } else if constexpr (k4) {
      // one ldmatrix.x4 = tokens 0-7 / 8-15 of two 32-code chunks (4 k-steps)
      const int t = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int c = 0; c < kD / 32; c += 2) {
        uint32_t w[4];
        ldsm_x4(st + swz<Tr>(t, c + (lane >> 4)), w[0], w[1], w[2], w[3]);
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          uint32_t x[4], y[4];  // fp16 pairs of token r (x) and token r + 8 (y)
          if constexpr (kCT == kI4) {
            i4x8_to_h2x4_biased(w[2 * c2], x);
            i4x8_to_h2x4_biased(w[2 * c2 + 1], y);
          } else {
            e2m1x8_to_h2x4(w[2 * c2], x);
            e2m1x8_to_h2x4(w[2 * c2 + 1], y);
          }
          const int jj = 2 * (c + c2);
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt) {
            mma_16816<false>(ae[nt], x[0], y[0], x[1], y[1], qf[nt][jj][0], qf[nt][jj][1]);
            mma_16816<false>(ao[nt], x[2], y[2], x[3], y[3], qf[nt][jj + 1][0], qf[nt][jj + 1][1]);
          }
        }
      }
    } else {
      const int t = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int jj = 0; jj < kKS; jj += 2) {
        uint32_t w[4];
        ldsm_x4(st + swz<Tr>(t, jj + (lane >> 4)), w[0], w[1], w[2], w[3]);
#pragma unroll
        for (int j2 = 0; j2 < 2; ++j2) {
          uint32_t lo_r, hi_r, lo_r8, hi_r8;  // (d 4q,4q+1) and (d 4q+2,4q+3) of tokens r and r+8
          if constexpr (kCT == kI8) {
            // fp16 1152 + c (the bias is taken out through kqs)
            const uint32_t u0 = w[2 * j2] ^ 0x80808080u, u1 = w[2 * j2 + 1] ^ 0x80808080u;
            lo_r = prmt(u0, 0x64646464u, 0x4140u);
            hi_r = prmt(u0, 0x64646464u, 0x4342u);
            lo_r8 = prmt(u1, 0x64646464u, 0x4140u);
            hi_r8 = prmt(u1, 0x64646464u, 0x4342u);
          } else if constexpr (kCT == kU8) {
            // fp16 1024 + c (the bias 1024 + z is taken out through kqs)
            lo_r = prmt(w[2 * j2], 0x64646464u, 0x4140u);
            hi_r = prmt(w[2 * j2], 0x64646464u, 0x4342u);
            lo_r8 = prmt(w[2 * j2 + 1], 0x64646464u, 0x4140u);
            hi_r8 = prmt(w[2 * j2 + 1], 0x64646464u, 0x4342u);
          } else {
            e4m3x4_to_h2x2(w[2 * j2], lo_r, hi_r);
            e4m3x4_to_h2x2(w[2 * j2 + 1], lo_r8, hi_r8);
          }
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt)
            mma_16816<false>(j2 ? ao[nt] : ae[nt], lo_r, lo_r8, hi_r, hi_r8, qf[nt][jj + j2][0], qf[nt][jj + j2][1]);
        }
      }
    }
  };

  // O^T += V^T . P^T for the block in stage `st`.
  auto values = [&](uint32_t st, const uint32_t (&pb)[kNT][2]) {
    const uint32_t vt = st + Tr::kKVBytes;
    if constexpr (!kQt) {
      const int t = (lane & 7) + (lane >> 4) * 8;
#pragma unroll
      for (int i = 0; i < kMT; ++i) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(vt + swz<Tr>(t, 2 * i + ((lane >> 3) & 1)), a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) mma_16816<kMmaBF16>(o[i][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
      }
    } else if constexpr (k4) {
      // transposed load: a lane's word holds tokens 2q (bytes 0-1) and 2q+1
      // (bytes 2-3) at d = 32c + 4r .. + 3; pairs (token 2q, token 2q+1) at
      // one d are (n0,n4) (n1,n5) (n2,n6) (n3,n7): m-tile 2c takes d offsets
      // 0 / 1 as rows r / r + 8, m-tile 2c + 1 offsets 2 / 3
      const int t = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int c = 0; c < kD / 32; c += 2) {
        uint32_t w[4];
        ldsm_x4_t(vt + swz<Tr>(t, c + (lane >> 4)), w[0], w[1], w[2], w[3]);
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          uint32_t x[4], y[4];  // x: tokens 0-7 of the block, y: tokens 8-15
          if constexpr (kCT == kI4) {
            // rows r (even d) read 1032 + c, rows r + 8 (odd d) 1152 + 16c
            i4x8_to_h2x4_biased(w[2 * c2], x);
            i4x8_to_h2x4_biased(w[2 * c2 + 1], y);
          } else {
            uint32_t a[4], b[4];
            e2m1x8_to_h2x4(w[2 * c2], a);
            e2m1x8_to_h2x4(w[2 * c2 + 1], b);
            x[0] = prmt(a[0], a[2], 0x5410u);
            x[1] = prmt(a[0], a[2], 0x7632u);
            x[2] = prmt(a[1], a[3], 0x5410u);
            x[3] = prmt(a[1], a[3], 0x7632u);
            y[0] = prmt(b[0], b[2], 0x5410u);
            y[1] = prmt(b[0], b[2], 0x7632u);
            y[2] = prmt(b[1], b[3], 0x5410u);
            y[3] = prmt(b[1], b[3], 0x7632u);
          }
          const int i = 2 * (c + c2);
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt) {
            mma_16816<false>(o[i][nt], x[0], x[1], y[0], y[1], pb[nt][0], pb[nt][1]);
            mma_16816<false>(o[i + 1][nt], x[2], x[3], y[2], y[3], pb[nt][0], pb[nt][1]);
          }
        }
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
            // fp16 1152 + c (the bias leaves through wacc)
            const uint32_t u0 = w[2 * ii] ^ 0x80808080u, u1 = w[2 * ii + 1] ^ 0x80808080u;
            x0 = prmt(u0, 0x64646464u, 0x4240u);
            x1 = prmt(u0, 0x64646464u, 0x4341u);
            y0 = prmt(u1, 0x64646464u, 0x4240u);
            y1 = prmt(u1, 0x64646464u, 0x4341u);
          } else if constexpr (kCT == kU8) {
            // fp16 1024 + c (the bias 1024 + z leaves through wacc)
            x0 = prmt(w[2 * ii], 0x64646464u, 0x4240u);
            x1 = prmt(w[2 * ii], 0x64646464u, 0x4341u);
            y0 = prmt(w[2 * ii + 1], 0x64646464u, 0x4240u);
            y1 = prmt(w[2 * ii + 1], 0x64646464u, 0x4341u);
          } else {
            e4m3x4_to_h2x2(prmt(w[2 * ii], w[2 * ii], 0x3120u), x0, x1);
            e4m3x4_to_h2x2(prmt(w[2 * ii + 1], w[2 * ii + 1], 0x3120u), y0, y1);
          }
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt) mma_16816<false>(o[i + ii][nt], x0, x1, y0, y1, pb[nt][0], pb[nt][1]);
        }
      }
    }
    if constexpr (kBiasV) {
      // every row of the A operand holds the bias of each token: INT8 1152,
      // uint8 1024 + z, INT4 1 (its two row biases are applied at the fold)
      uint32_t ax = 0x3C003C00u, ay = 0x3C003C00u;
      if constexpr (kCT == kI8) {
        ax = ay = 0x64806480u;
      } else if constexpr (kCT == kU8) {
        const uint8_t* zv = base_ptr + (st - smem_base) + 2 * Tr::kKVBytes + 144;
        ax = (0x6400u + zv[2 * q4]) | ((0x6400u + zv[2 * q4 + 1]) << 16);
        ay = (0x6400u + zv[2 * q4 + 8]) | ((0x6400u + zv[2 * q4 + 9]) << 16);
      }
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt) mma_16816<false>(wacc[nt], ax, ax, ay, ay, pb[nt][0], pb[nt][1]);
    }
  };

  // Takes the accumulated bias weight out of O^T (integer V codes).
  auto fold_v = [&]() {
    if constexpr (kBiasV) {
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt) {
#pragma unroll
        for (int i = 0; i < kMT; ++i)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if constexpr (kCT == kI4) {
              o[i][nt][e] -= (e < 2 ? 1032.0f : 1152.0f) * wacc[nt][e];
            } else {
              o[i][nt][e] -= wacc[nt][e];
            }
          }
        wacc[nt][0] = wacc[nt][1] = wacc[nt][2] = wacc[nt][3] = 0.0f;
      }
      since_fold = 0;
    }
  };

  // Items k .. k + NB - 1: NB consecutive blocks of the current pair (NB = 2
  // only when both belong to it), whose scores share one softmax update.
  // False when a copy wait timed out (the warp then leaves).
  auto blocks = [&](int k, auto nb_tag) -> bool {
    constexpr int NB = decltype(nb_tag)::value;
    uint32_t stb[NB];
    bool landed = true;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      stb[b] = ring + cstage * Tr::kStageBytes;
      landed = mbar_wait(bars + cstage * 8, cphase) && landed;
      if (++cstage == kR) {
        cstage = 0;
        cphase ^= 1u;
      }
    }
    if (__any_sync(0xffffffffu, !landed)) {  // warp-uniform: never split the warp before ldmatrix/mma
      // let copies already in flight land (bounded) before the warp leaves
      for (int kk = k + NB; kk < count && kk < k + kR; ++kk) mbar_wait(bars + (kk % kR) * 8, (kk / kR) & 1);
      return false;
    }
    const int kpos0 = (jb + j) * 16;  // position of the first block's first token
    const int valid = ctx - kpos0;    // >= 1 tokens of these blocks count
    // sliding window: tokens before position ctx - window are not seen
    const int lowv = p.window > 0 ? ctx - p.window - kpos0 : -32;
    // Rows of a sequence's last block at or beyond its context were never
    // written and may hold anything, NaN included; P is 0 there, but 0 * NaN
    // is not, so those V rows are zeroed in the stage first (and their
    // scales replaced by 0 below).  Only the last block of a pair can have
    // such rows.
    bool any_tail = false;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int vb = valid - 16 * b;
      if (vb < 16) {
        any_tail = true;
        uint8_t* vrow = base_ptr + (stb[b] - smem_base) + Tr::kKVBytes;
        constexpr int kChunks = Tr::kNumColTiles * Tr::kChunksPerTileRow;  // 16-byte chunks per row
        for (int e = lane; e < (16 - vb) * kChunks; e += 32) {
          const int t = vb + e / kChunks, c = e % kChunks;
          *reinterpret_cast<uint4*>(vrow + (c / Tr::kChunksPerTileRow) * Tr::kColTileBytes + t * Tr::kTileBytes +
                                    (c % Tr::kChunksPerTileRow) * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
    }
    if (any_tail) __syncwarp();

    // ---- S^T = K . Q^T: two independent accumulation chains (one per block
    // when NB = 2, even and odd k-steps of the one block otherwise) ----
    float sacc[NB][kNT][4];
    float sacc2[kNT][4];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if constexpr (kBiasK) {
        // uint8: the bias of token row r (r + 8) is 1024 + its zero point
        float zb_r = 1.0f, zb_r8 = 1.0f;
        if constexpr (kCT == kU8) {
          const uint8_t* zk = base_ptr + (stb[b] - smem_base) + 2 * Tr::kKVBytes + 128;
          zb_r = 1024.0f + static_cast<float>(zk[r]);
          zb_r8 = 1024.0f + static_cast<float>(zk[r + 8]);
        }
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sacc[b][nt][e] = -kqs[nt][e & 1] * (e < 2 ? zb_r : zb_r8);
      } else {
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sacc[b][nt][e] = 0.0f;
      }
    }
    if constexpr (NB == 1) {
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc2[nt][e] = 0.0f;
      scores(stb[0], sacc[0], sacc2);
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[0][nt][e] += sacc2[nt][e];
    } else {
#pragma unroll
      for (int b = 0; b < NB; ++b) scores(stb[b], sacc[b], sacc[b]);
    }

    // ---- scale, mask, online softmax (base 2) over the NB blocks ----
    float f_r[NB], f_r8[NB], vs_r[NB], vs_r8[NB];
    bool ok_r[NB], ok_r8[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int vb = valid - 16 * b, lb = lowv - 16 * b;
      f_r[b] = p.qk_scale_log2;
      f_r8[b] = p.qk_scale_log2;
      vs_r[b] = 1.0f;
      vs_r8[b] = 1.0f;
      if constexpr (kQt) {
        const float* sc = reinterpret_cast<const float*>(base_ptr + (stb[b] - smem_base) + 2 * Tr::kKVBytes);
        f_r[b] *= sc[r];
        f_r8[b] *= sc[r + 8];
        vs_r[b] = r < vb ? sc[16 + r] : 0.0f;
        vs_r8[b] = r + 8 < vb ? sc[16 + r + 8] : 0.0f;
      }
      ok_r[b] = r < vb && r >= lb;
      ok_r8[b] = r + 8 < vb && r + 8 >= lb;
    }
    // Lazy exponent base: a column's base m_run moves only when one of its
    // scores exceeds it by more than 8 (log2 units), so p = 2^(s - m_run)
    // stays below 256 and the common block needs no cross-lane maximum and
    // no rescale, only one warp vote.  When a column's base must move, the
    // whole warp takes the block maximum and rescales (the first block of a
    // pair always does: its base starts at -inf).
    float sv[NB][kNT][4];
    bool up = false;
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        bool ok0 = ok_r[b], ok1 = ok_r[b], ok2 = ok_r8[b], ok3 = ok_r8[b];
        if constexpr (kMQ) {
          const int va = colv[nt][0] - kpos0 - 16 * b, vb = colv[nt][1] - kpos0 - 16 * b;
          const int la = p.window > 0 ? va - p.window : -32, lb = p.window > 0 ? vb - p.window : -32;
          ok0 = r < va && r >= la;
          ok1 = r < vb && r >= lb;
          ok2 = r + 8 < va && r + 8 >= la;
          ok3 = r + 8 < vb && r + 8 >= lb;
        }
        sv[b][nt][0] = ok0 ? sacc[b][nt][0] * f_r[b] : -INFINITY;
        sv[b][nt][1] = ok1 ? sacc[b][nt][1] * f_r[b] : -INFINITY;
        sv[b][nt][2] = ok2 ? sacc[b][nt][2] * f_r8[b] : -INFINITY;
        sv[b][nt][3] = ok3 ? sacc[b][nt][3] * f_r8[b] : -INFINITY;
        up |= fmaxf(sv[b][nt][0], sv[b][nt][2]) > m_run[nt][0] + 8.0f;
        up |= fmaxf(sv[b][nt][1], sv[b][nt][3]) > m_run[nt][1] + 8.0f;
      }
    // P enters the MMA as p x (value scale) in fp16: with p up to 2^8 a
    // value scale above 128 could overflow it, so such blocks move the base
    // to their maximum (p <= 1 there, as with an exact running maximum)
#pragma unroll
    for (int b = 0; b < NB; ++b) up |= fmaxf(vs_r[b], vs_r8[b]) > 128.0f;
    if (__any_sync(0xffffffffu, up)) {
      float alpha[kNT][2];
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt) {
        float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          mx_a = fmaxf(mx_a, fmaxf(sv[b][nt][0], sv[b][nt][2]));
          mx_b = fmaxf(mx_b, fmaxf(sv[b][nt][1], sv[b][nt][3]));
        }
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, off));
          mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, off));
        }
        const float mn_a = fmaxf(m_run[nt][0], mx_a);
        const float mn_b = fmaxf(m_run[nt][1], mx_b);
        alpha[nt][0] = mn_a == m_run[nt][0] ? 1.0f : fast_exp2(m_run[nt][0] - mn_a);
        alpha[nt][1] = mn_b == m_run[nt][1] ? 1.0f : fast_exp2(m_run[nt][1] - mn_b);
        m_run[nt][0] = mn_a;
        m_run[nt][1] = mn_b;
        l_run[nt][0] *= alpha[nt][0];
        l_run[nt][1] *= alpha[nt][1];
      }
#pragma unroll
      for (int i = 0; i < kMT; ++i)
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
          o[i][nt][0] *= alpha[nt][0];
          o[i][nt][1] *= alpha[nt][1];
          o[i][nt][2] *= alpha[nt][0];
          o[i][nt][3] *= alpha[nt][1];
        }
      if constexpr (kBiasV) {
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
          wacc[nt][0] *= alpha[nt][0];
          wacc[nt][1] *= alpha[nt][1];
          wacc[nt][2] *= alpha[nt][0];
          wacc[nt][3] *= alpha[nt][1];
        }
      }
    }
    uint32_t pb[NB][kNT][2];
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
      // a column with no visible key yet keeps m = -inf: exponentiate
      // against 0 instead, which gives p = 0 for its masked entries
      const float b_a = m_run[nt][0] == -INFINITY ? 0.0f : m_run[nt][0];
      const float b_b = m_run[nt][1] == -INFINITY ? 0.0f : m_run[nt][1];
      float la = 0.0f, lbs = 0.0f;
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const float p0 = fast_exp2(sv[b][nt][0] - b_a), p1 = fast_exp2(sv[b][nt][1] - b_b);
        const float p2 = fast_exp2(sv[b][nt][2] - b_a), p3 = fast_exp2(sv[b][nt][3] - b_b);
        la += p0 + p2;
        lbs += p1 + p3;
        // P^T operand: rows = tokens of the block, columns = query heads
        pb[b][nt][0] = movmatrix_t(pack2<kMmaBF16>(p0 * vs_r[b], p1 * vs_r[b]));
        pb[b][nt][1] = movmatrix_t(pack2<kMmaBF16>(p2 * vs_r8[b], p3 * vs_r8[b]));
      }
      l_run[nt][0] += la;
      l_run[nt][1] += lbs;
    }

    // ---- O^T += V^T . P^T ----
#pragma unroll
    for (int b = 0; b < NB; ++b) values(stb[b], pb[b]);
    if constexpr (kBiasV) {
      since_fold += NB;
      if (since_fold >= kFoldBlocks) fold_v();
    }

    // ---- refill these stages with items k + kR .. ----
    __syncwarp();
    // the zeroed rows were generic-proxy writes; order them before the TMA
    // (async-proxy) refill of the same stage
    if (any_tail) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int kn = k + b + kR;
      if (kn < count) {
        const int chunk = kn >> 5;
        if ((kn & 31) == 0) {
          // entering chunk `chunk` (held in pre[chunk & 1]); chunk - 1 is
          // spent, so its register takes chunk + 1
          const int ki = (chunk + 1) * 32 + lane;
          const int nxt = ki < count ? item_row<kMQ>(p, cum, item_of(ki)) : 0;
          if (chunk & 1) pre0 = nxt; else pre1 = nxt;
        }
        const int row0 = __shfl_sync(0xffffffffu, (chunk & 1) ? pre1 : pre0, kn & 31);
        if (lane == 0) issue(row0);
      }
    }
    return true;
  };

  constexpr bool kPairBlocks = kQt;
  if constexpr (kPairBlocks) {
    // Quantised caches take two blocks of a pair per iteration: their
    // per-block bookkeeping (softmax reduction and update, rescale test, loop
    // and pair tests) is shared, and the two blocks' independent work
    // interleaves.
#pragma unroll 1
    for (int k = 0; k < count;) {
      const int nbk = (k + 1 < count && j + 1 < nb && !(offset > 0 && k + 1 == count - offset)) ? 2 : 1;
      if (!(nbk == 2 ? blocks(k, IntC<2>{}) : blocks(k, IntC<1>{}))) return;
      k += nbk;
      const int kl = k - 1;  // the last item processed

      // ---- advance; finish the (sequence, head) pair at its end or the stream's ----
      j += nbk;
      const bool wrap_next = offset > 0 && kl + 1 == count - offset;  // next item is g0
      if (j == nb || wrap_next || kl == count - 1) {
        fold_v();
        if constexpr (kCT == kI4) {
          // rows r + 8 (odd d) were widened at 16x
#pragma unroll
          for (int i = 0; i < kMT; ++i)
#pragma unroll
            for (int nt = 0; nt < kNT; ++nt) {
              o[i][nt][2] *= 0.0625f;
              o[i][nt][3] *= 0.0625f;
            }
        }
        float lsum[kNT][2];
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
          float la = l_run[nt][0], lb = l_run[nt][1];
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) {
            la += __shfl_xor_sync(0xffffffffu, la, off);
            lb += __shfl_xor_sync(0xffffffffu, lb, off);
          }
          lsum[nt][0] = la;
          lsum[nt][1] = lb;
        }
        const long long head_row0 = static_cast<long long>(s) * Hq + static_cast<long long>(h) * G;
        // columns of this pair: G heads (decode) or a tile of (token, head)
        const int C = kMQ ? p.tile_cols : G;
        const int ncols = kMQ ? min(p.tile_cols, n_new * G - tile * p.tile_cols) : G;
        auto out_row = [&](int c) -> long long {
          if constexpr (kMQ) {
            return static_cast<long long>(q0 + col_token(c)) * Hq + static_cast<long long>(h) * G + col_head(c);
          } else {
            return head_row0 + c;
          }
        };
        const int gp0 = cum[s] + pr * nb;  // the pair's first and last items
        const int gpe = gp0 + nb - 1;
        if (gp0 >= g0 && gpe < g1) {
          // the whole pair went through this warp: write the output
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const int g = nt * 8 + 2 * q4 + c;
              if (g >= ncols) continue;
              const float inv = 1.0f / lsum[nt][c];
              const long long row = out_row(g);
#pragma unroll
              for (int i = 0; i < kMT; ++i) {
                const int d0 = k4 ? 32 * (i >> 1) + 4 * r + 2 * (i & 1) : (k8 ? 16 * i + 2 * r : 16 * i + r);
                const int d1 = kQt ? d0 + 1 : d0 + 8;
                store_out<kOutBF16>(p.out, row * kD + d0, o[i][nt][c] * inv);
                store_out<kOutBF16>(p.out, row * kD + d1, o[i][nt][2 + c] * inv);
              }
            }
        } else {
          // a share of a split pair: publish (m, l, o / l), then count arrivals
          const int ml = p.slot_floats - C * kD;
          float* slot = p.slots + static_cast<long long>(2 * gw + (gp0 <= g0 && g0 <= gpe ? 0 : 1)) * p.slot_floats;
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const int g = nt * 8 + 2 * q4 + c;
              if (g >= ncols) continue;
              // multi-query: a share may hold no visible key of a column (l = 0)
              const float inv = (kMQ && lsum[nt][c] == 0.0f) ? 0.0f : 1.0f / lsum[nt][c];
              if (r == 0) {
                slot[g] = m_run[nt][c];
                slot[C + g] = lsum[nt][c];
              }
              float* og = slot + ml + g * kD;
#pragma unroll
              for (int i = 0; i < kMT; ++i) {
                const int d0 = k4 ? 32 * (i >> 1) + 4 * r + 2 * (i & 1) : (k8 ? 16 * i + 2 * r : 16 * i + r);
                const int d1 = kQt ? d0 + 1 : d0 + 8;
                og[d0] = o[i][nt][c] * inv;
                og[d1] = o[i][nt][2 + c] * inv;
              }
            }
          __threadfence();
          __syncwarp();
          const int w_first = stream_of(T, gp0, nw);
          const int n_c = stream_of(T, gpe, nw) - w_first + 1;
          int last = 0;
          if (lane == 0) {
            unsigned long long* ctr =
                p.counters + (static_cast<long long>(s) * Hkv + h) * (kMQ ? p.max_tiles : 1) + (kMQ ? tile : 0);
            const unsigned long long E = p.epoch;
            unsigned long long old = atomicAdd(ctr, 0ull), assumed, next;
            do {
              assumed = old;
              next = ((assumed >> kEpochShift) == E) ? assumed + 1 : ((E << kEpochShift) | 1ull);
              old = atomicCAS(ctr, assumed, next);
            } while (old != assumed);
            last = static_cast<int>(next & kCountMask) == n_c;
          }
          last = __shfl_sync(0xffffffffu, last, 0);
          if (last) {
            __threadfence();
            // contributor c = w_first + c keeps its share in slot 2w (the pair
            // holds the stream's first item) or 2w + 1 (it does not)
            auto slot_of = [&](int c) -> const float* {
              const int w = w_first + c;
              const int idx = 2 * w + (stream_start(T, w, nw) >= gp0 ? 0 : 1);
              return p.slots + static_cast<long long>(idx) * p.slot_floats;
            };
            // One pass over the contributors per group of kMG heads, with a
            // running max per head: every load of a contributor is independent
            // of the others, and two contributors are in flight at once.  Each
            // lane owns kD / 32 output columns of every head.  (Groups of 4 for
            // quantised caches keep this rarely run code within their 168
            // registers.)
            constexpr int kV = kD / 32;
            constexpr int kMG = kQt ? 4 : 8;
#pragma unroll 1
            for (int c0 = 0; c0 < ncols; c0 += kMG) {
              float Mg[kMG], Lg[kMG], acc[kMG][kV];
#pragma unroll
              for (int gg = 0; gg < kMG; ++gg) {
                Mg[gg] = -INFINITY;
                Lg[gg] = 0.0f;
#pragma unroll
                for (int e = 0; e < kV; ++e) acc[gg][e] = 0.0f;
              }
#pragma unroll 2
              for (int c = 0; c < n_c; ++c) {
                const float* sl = slot_of(c);
                float mc[kMG], lc[kMG], ov[kMG][kV];
#pragma unroll
                for (int gg = 0; gg < kMG; ++gg) {
                  const int g = c0 + gg;
                  if (g < ncols) {
                    mc[gg] = __ldcg(sl + g);
                    lc[gg] = __ldcg(sl + C + g);
                    const float* og = sl + ml + g * kD + lane * kV;
                    if constexpr (kV == 4) {
                      const float4 v = __ldcg(reinterpret_cast<const float4*>(og));
                      ov[gg][0] = v.x;
                      ov[gg][1] = v.y;
                      ov[gg][2] = v.z;
                      ov[gg][3] = v.w;
                    } else {
                      const float2 v = __ldcg(reinterpret_cast<const float2*>(og));
                      ov[gg][0] = v.x;
                      ov[gg][1] = v.y;
                    }
                  }
                }
#pragma unroll
                for (int gg = 0; gg < kMG; ++gg) {
                  // multi-query: skip a share that saw no visible key of the column
                  if (c0 + gg < ncols && (!kMQ || mc[gg] != -INFINITY)) {
                    const float mn = fmaxf(Mg[gg], mc[gg]);
                    const float a = fast_exp2(Mg[gg] - mn);  // 0 for the first contributor
                    const float w = fast_exp2(mc[gg] - mn) * lc[gg];
                    Lg[gg] = Lg[gg] * a + w;
#pragma unroll
                    for (int e = 0; e < kV; ++e) acc[gg][e] = acc[gg][e] * a + w * ov[gg][e];
                    Mg[gg] = mn;
                  }
                }
              }
#pragma unroll
              for (int gg = 0; gg < kMG; ++gg) {
                const int g = c0 + gg;
                if (g < ncols) {
                  const float inv = Lg[gg] > 0.0f ? 1.0f / Lg[gg] : 0.0f;
                  const long long row = out_row(g);
#pragma unroll
                  for (int e = 0; e < kV; ++e)
                    store_out<kOutBF16>(p.out, row * kD + lane * kV + e, acc[gg][e] * inv);
                }
              }
            }
          }
        }
        if (kl + 1 < count) {  // the stream continues: back to g0, or the next non-empty pair
          if (wrap_next) {
            locate(g0);
          } else {
            j = 0;
            if (++pr == Hkv * ntile) {
              pr = 0;
              do {
                ++s;
              } while (cum[s + 1] == cum[s]);
              enter_seq();
            }
            set_pair();
          }
          begin_pair();
        }
      }
    }
  } else {
    // 16-bit caches: one block per iteration (this loop is kept as it is:
    // with one warp per SM sub-partition the HBM stream is sensitive to the
    // instruction schedule, and a shared body with the quantised path
    // measured 7 % slower on the long-context workload)
#pragma unroll 1
    for (int k = 0; k < count; ++k) {
      const int stage = cstage;
      const uint32_t st = ring + stage * Tr::kStageBytes;
      const bool landed = mbar_wait(bars + stage * 8, cphase);
      if (++cstage == kR) {
        cstage = 0;
        cphase ^= 1u;
      }
      if (__any_sync(0xffffffffu, !landed)) {  // warp-uniform: never split the warp before ldmatrix/mma
        // let copies already in flight land (bounded) before the warp leaves
        for (int kk = k + 1; kk < count && kk < k + kR; ++kk) mbar_wait(bars + (kk % kR) * 8, (kk / kR) & 1);
        return;
      }
      const int kpos0 = (jb + j) * 16;  // position of the block's first token
      const int valid = ctx - kpos0;    // >= 1 tokens of this block count
      // sliding window: tokens before position ctx - window are not seen
      const int lowv = p.window > 0 ? ctx - p.window - kpos0 : -32;
      // Rows of a sequence's last block at or beyond its context were never
      // written and may hold anything, NaN included; P is 0 there, but 0 * NaN
      // is not, so those V rows are zeroed in the stage first.
      const bool tail = valid < 16;
      if (tail) {
        uint8_t* vrow = base_ptr + (st - smem_base) + Tr::kKVBytes;
        constexpr int kChunks = Tr::kNumColTiles * Tr::kChunksPerTileRow;  // 16-byte chunks per row
        for (int e = lane; e < (16 - valid) * kChunks; e += 32) {
          const int t = valid + e / kChunks, c = e % kChunks;
          *reinterpret_cast<uint4*>(vrow + (c / Tr::kChunksPerTileRow) * Tr::kColTileBytes + t * Tr::kTileBytes +
                                    (c % Tr::kChunksPerTileRow) * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
      }

      // ---- S^T = K . Q^T (two independent accumulation chains, summed) ----
      float sacc[kNT][4], sacc2[kNT][4];
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[nt][e] = sacc2[nt][e] = 0.0f;
      {
        const int t = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int jj = 0; jj < kKS; ++jj) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(st + swz<Tr>(t, 2 * jj + (lane >> 4)), a0, a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt)
            mma_16816<kMmaBF16>((jj & 1) ? sacc2[nt] : sacc[nt], a0, a1, a2, a3, qf[nt][jj][0], qf[nt][jj][1]);
        }
      }
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[nt][e] += sacc2[nt][e];

      // ---- scale, mask, online softmax (base 2) ----
      const float f_r = p.qk_scale_log2, f_r8 = p.qk_scale_log2;
      const float vs_r = 1.0f, vs_r8 = 1.0f;
      const bool ok_r = r < valid && r >= lowv;
      const bool ok_r8 = r + 8 < valid && r + 8 >= lowv;
      uint32_t pb[kNT][2];
      bool grow = false;
      float alpha[kNT][2];
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt) {
        bool ok0 = ok_r, ok1 = ok_r, ok2 = ok_r8, ok3 = ok_r8;
        if constexpr (kMQ) {
          const int va = colv[nt][0] - kpos0, vb = colv[nt][1] - kpos0;
          const int la = p.window > 0 ? va - p.window : -32, lb = p.window > 0 ? vb - p.window : -32;
          ok0 = r < va && r >= la;
          ok1 = r < vb && r >= lb;
          ok2 = r + 8 < va && r + 8 >= la;
          ok3 = r + 8 < vb && r + 8 >= lb;
        }
        const float s0 = ok0 ? sacc[nt][0] * f_r : -INFINITY;
        const float s1 = ok1 ? sacc[nt][1] * f_r : -INFINITY;
        const float s2 = ok2 ? sacc[nt][2] * f_r8 : -INFINITY;
        const float s3 = ok3 ? sacc[nt][3] * f_r8 : -INFINITY;
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
        // a column with no visible key yet keeps m = -inf: exponentiate
        // against 0 instead, which gives p = 0 for its masked entries
        const float b_a = (kMQ && mn_a == -INFINITY) ? 0.0f : mn_a;
        const float b_b = (kMQ && mn_b == -INFINITY) ? 0.0f : mn_b;
        const float p0 = fast_exp2(s0 - b_a), p1 = fast_exp2(s1 - b_b);
        const float p2 = fast_exp2(s2 - b_a), p3 = fast_exp2(s3 - b_b);
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
      {
        const int t = (lane & 7) + (lane >> 4) * 8;
#pragma unroll
        for (int i = 0; i < kMT; ++i) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(vt + swz<Tr>(t, 2 * i + ((lane >> 3) & 1)), a0, a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt) mma_16816<kMmaBF16>(o[i][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
        }
      }

      // ---- refill this stage with item k + kR ----
      __syncwarp();
      // the zeroed rows were generic-proxy writes; order them before the TMA
      // (async-proxy) refill of the same stage
      if (tail) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      const int kn = k + kR;
      if (kn < count) {
        const int chunk = kn >> 5;
        if ((kn & 31) == 0) {
          // entering chunk `chunk` (held in pre[chunk & 1]); chunk - 1 is spent,
          // so its register takes chunk + 1
          const int ki = (chunk + 1) * 32 + lane;
          const int nxt = ki < count ? item_row<kMQ>(p, cum, item_of(ki)) : 0;
          if (chunk & 1) pre0 = nxt; else pre1 = nxt;
        }
        const int row0 = __shfl_sync(0xffffffffu, (chunk & 1) ? pre1 : pre0, kn & 31);
        if (lane == 0) issue(row0);
      }

      // ---- advance; finish the (sequence, head) pair at its end or the stream's ----
      ++j;
      const bool wrap_next = offset > 0 && k + 1 == count - offset;  // next item is g0
      if (j == nb || wrap_next || k == count - 1) {
        float lsum[kNT][2];
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
          float la = l_run[nt][0], lb = l_run[nt][1];
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) {
            la += __shfl_xor_sync(0xffffffffu, la, off);
            lb += __shfl_xor_sync(0xffffffffu, lb, off);
          }
          lsum[nt][0] = la;
          lsum[nt][1] = lb;
        }
        const long long head_row0 = static_cast<long long>(s) * Hq + static_cast<long long>(h) * G;
        // columns of this pair: G heads (decode) or a tile of (token, head)
        const int C = kMQ ? p.tile_cols : G;
        const int ncols = kMQ ? min(p.tile_cols, n_new * G - tile * p.tile_cols) : G;
        auto out_row = [&](int c) -> long long {
          if constexpr (kMQ) {
            return static_cast<long long>(q0 + col_token(c)) * Hq + static_cast<long long>(h) * G + col_head(c);
          } else {
            return head_row0 + c;
          }
        };
        const int gp0 = cum[s] + pr * nb;  // the pair's first and last items
        const int gpe = gp0 + nb - 1;
        if (gp0 >= g0 && gpe < g1) {
          // the whole pair went through this warp: write the output
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const int g = nt * 8 + 2 * q4 + c;
              if (g >= ncols) continue;
              const float inv = 1.0f / lsum[nt][c];
              const long long row = out_row(g);
#pragma unroll
              for (int i = 0; i < kMT; ++i) {
                const int d0 = k4 ? 32 * (i >> 1) + 4 * r + 2 * (i & 1) : (k8 ? 16 * i + 2 * r : 16 * i + r);
                const int d1 = kQt ? d0 + 1 : d0 + 8;
                store_out<kOutBF16>(p.out, row * kD + d0, o[i][nt][c] * inv);
                store_out<kOutBF16>(p.out, row * kD + d1, o[i][nt][2 + c] * inv);
              }
            }
        } else {
          // a share of a split pair: publish (m, l, o / l), then count arrivals
          const int ml = p.slot_floats - C * kD;
          float* slot = p.slots + static_cast<long long>(2 * gw + (gp0 <= g0 && g0 <= gpe ? 0 : 1)) * p.slot_floats;
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const int g = nt * 8 + 2 * q4 + c;
              if (g >= ncols) continue;
              // multi-query: a share may hold no visible key of a column (l = 0)
              const float inv = (kMQ && lsum[nt][c] == 0.0f) ? 0.0f : 1.0f / lsum[nt][c];
              if (r == 0) {
                slot[g] = m_run[nt][c];
                slot[C + g] = lsum[nt][c];
              }
              float* og = slot + ml + g * kD;
#pragma unroll
              for (int i = 0; i < kMT; ++i) {
                const int d0 = k4 ? 32 * (i >> 1) + 4 * r + 2 * (i & 1) : (k8 ? 16 * i + 2 * r : 16 * i + r);
                const int d1 = kQt ? d0 + 1 : d0 + 8;
                og[d0] = o[i][nt][c] * inv;
                og[d1] = o[i][nt][2 + c] * inv;
              }
            }
          __threadfence();
          __syncwarp();
          const int w_first = stream_of(T, gp0, nw);
          const int n_c = stream_of(T, gpe, nw) - w_first + 1;
          int last = 0;
          if (lane == 0) {
            unsigned long long* ctr =
                p.counters + (static_cast<long long>(s) * Hkv + h) * (kMQ ? p.max_tiles : 1) + (kMQ ? tile : 0);
            const unsigned long long E = p.epoch;
            unsigned long long old = atomicAdd(ctr, 0ull), assumed, next;
            do {
              assumed = old;
              next = ((assumed >> kEpochShift) == E) ? assumed + 1 : ((E << kEpochShift) | 1ull);
              old = atomicCAS(ctr, assumed, next);
            } while (old != assumed);
            last = static_cast<int>(next & kCountMask) == n_c;
          }
          last = __shfl_sync(0xffffffffu, last, 0);
          if (last) {
            __threadfence();
            // contributor c = w_first + c keeps its share in slot 2w (the pair
            // holds the stream's first item) or 2w + 1 (it does not)
            auto slot_of = [&](int c) -> const float* {
              const int w = w_first + c;
              const int idx = 2 * w + (stream_start(T, w, nw) >= gp0 ? 0 : 1);
              return p.slots + static_cast<long long>(idx) * p.slot_floats;
            };
            // One pass over the contributors per group of kMG heads, with a
            // running max per head: every load of a contributor is independent
            // of the others, and two contributors are in flight at once.  Each
            // lane owns kD / 32 output columns of every head.  (Groups of 4 for
            // quantised caches keep this rarely run code within their 168
            // registers.)
            constexpr int kV = kD / 32;
            constexpr int kMG = kQt ? 4 : 8;
#pragma unroll 1
            for (int c0 = 0; c0 < ncols; c0 += kMG) {
              float Mg[kMG], Lg[kMG], acc[kMG][kV];
#pragma unroll
              for (int gg = 0; gg < kMG; ++gg) {
                Mg[gg] = -INFINITY;
                Lg[gg] = 0.0f;
#pragma unroll
                for (int e = 0; e < kV; ++e) acc[gg][e] = 0.0f;
              }
#pragma unroll 2
              for (int c = 0; c < n_c; ++c) {
                const float* sl = slot_of(c);
                float mc[kMG], lc[kMG], ov[kMG][kV];
#pragma unroll
                for (int gg = 0; gg < kMG; ++gg) {
                  const int g = c0 + gg;
                  if (g < ncols) {
                    mc[gg] = __ldcg(sl + g);
                    lc[gg] = __ldcg(sl + C + g);
                    const float* og = sl + ml + g * kD + lane * kV;
                    if constexpr (kV == 4) {
                      const float4 v = __ldcg(reinterpret_cast<const float4*>(og));
                      ov[gg][0] = v.x;
                      ov[gg][1] = v.y;
                      ov[gg][2] = v.z;
                      ov[gg][3] = v.w;
                    } else {
                      const float2 v = __ldcg(reinterpret_cast<const float2*>(og));
                      ov[gg][0] = v.x;
                      ov[gg][1] = v.y;
                    }
                  }
                }
#pragma unroll
                for (int gg = 0; gg < kMG; ++gg) {
                  // multi-query: skip a share that saw no visible key of the column
                  if (c0 + gg < ncols && (!kMQ || mc[gg] != -INFINITY)) {
                    const float mn = fmaxf(Mg[gg], mc[gg]);
                    const float a = fast_exp2(Mg[gg] - mn);  // 0 for the first contributor
                    const float w = fast_exp2(mc[gg] - mn) * lc[gg];
                    Lg[gg] = Lg[gg] * a + w;
#pragma unroll
                    for (int e = 0; e < kV; ++e) acc[gg][e] = acc[gg][e] * a + w * ov[gg][e];
                    Mg[gg] = mn;
                  }
                }
              }
#pragma unroll
              for (int gg = 0; gg < kMG; ++gg) {
                const int g = c0 + gg;
                if (g < ncols) {
                  const float inv = Lg[gg] > 0.0f ? 1.0f / Lg[gg] : 0.0f;
                  const long long row = out_row(g);
#pragma unroll
                  for (int e = 0; e < kV; ++e)
                    store_out<kOutBF16>(p.out, row * kD + lane * kV + e, acc[gg][e] * inv);
                }
              }
            }
          }
        }
        if (k + 1 < count) {  // the stream continues: back to g0, or the next non-empty pair
          if (wrap_next) {
            locate(g0);
          } else {
            j = 0;
            if (++pr == Hkv * ntile) {
              pr = 0;
              do {
                ++s;
              } while (cum[s + 1] == cum[s]);
              enter_seq();
            }
            set_pair();
          }
          begin_pair();
        }
      }
    }
  }
}

}  // namespace pkv
