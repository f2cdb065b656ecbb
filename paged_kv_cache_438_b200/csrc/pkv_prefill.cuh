// Query-major paged attention for long runs of new tokens (chunked prefill),
// on the 5th-generation tensor cores (tcgen05, accumulators in TMEM).
//
// Method ("LLM 推理优化深度解析" §Continuous Batching and §调优心法: a long
// prompt is cut into chunks interleaved with decode steps): the n new tokens
// of a sequence are the last n of its context; token t attends keys
// 0 .. ctx - n + t (and, under a sliding window, only the last `window` of
// them).  Same result as the multi-query mode of the decode kernel; this
// kernel is the one that suits chunks of many tokens, where the work is a
// real matrix product.
//
// Design (sm_100a):
//   * One CTA of 4 warps per (sequence, KV head, tile of 128 query rows); a
//     row is a (new token, query head of the group) pair, row = t * G + g,
//     so the GQA group shares every K/V tile.  Thread i owns row i: TMEM lane
//     i holds its scores and its output accumulator, and the whole softmax of
//     a row runs in one thread (no shuffles).
//   * Keys stream in tiles of 64 (four 16-token cache blocks found through
//     the block table) by TMA into a 2-stage ring (128-byte swizzle); K tiles
//     are K-major B operands, V tiles MN-major B operands of the same layout.
//   * S = Q K^T: tcgen05.mma M=128, N=64, K=16 steps over head_dim into TMEM
//     (fp32); P = exp2(S - m) in bf16/fp16 written to shared memory
//     (K-major, swizzled; at head_dim 128 over the stage's K tile, which S
//     no longer needs) as the A operand of O += P V (M=128, N=head_dim).
//     One thread issues the MMAs; completion is signalled by tcgen05.commit
//     on an mbarrier; every wait is bounded.
//   * Online softmax with a lazy rescale: the running max used for the
//     exponentials only moves when a row's max grows by more than 8 (log2
//     units), and only then is that row's O rescaled in TMEM.  Two CTAs fit
//     on an SM, so one CTA's softmax overlaps the other's MMAs.
//   * Tokens of a sequence's last block beyond its context were never
//     written: their V rows are zeroed in the stage, blocks past the context
//     are loaded from outside the tensor (TMA fills zeros).
#pragma once

#include "pkv_device.cuh"

namespace pkv {

// ------------------------------------------------------------- tcgen05 --
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// D[tmem] (+)= A[smem] . B[smem]^T, kind::f16 (fp32 accumulate); one thread.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the mbarrier when every MMA this thread issued so far is done.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// 32 consecutive fp32 columns of the calling thread's TMEM lane (warp-wide).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle (rows of 128 bytes in
// 8-row, 1024-byte atoms; every region used here starts 1024-aligned).
//   K-major operand: `lead` unused (1); the stride between 8-row groups is
//   1024 bytes.
//   MN-major operand: rows are the K index; `lead` = bytes between groups of
//   64 MN elements; 8-row K groups 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lead_bytes) {
  uint64_t d = static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lead_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // descriptor version of sm_100
  d |= static_cast<uint64_t>(2) << 61;  // 128-byte swizzle
  return d;
}

// Instruction descriptor of kind::f16 with fp32 accumulation, A K-major.
__host__ __device__ constexpr uint32_t umma_idesc(int m, int n, bool bf16, bool b_mn_major) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

struct PrefillParams {
  void* out;
  const void* q;
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* query_start_loc;
  int num_seqs;
  int num_q_tokens;
  int max_query_len;
  int num_q_heads;
  int num_kv_heads;
  int group;
  int max_blocks_per_seq;
  int num_blocks;
  int max_context_len;
  int window;
  int max_tiles;   // tiles of 128 rows of the longest query run (grid.x)
  int oob_row;     // a TMA row coordinate past the cache (zero fill)
  float qk_scale_log2;
};

template <int kD>
struct PrefillTraits {
  static constexpr int kRows = 128;                    // query rows per CTA (M)
  static constexpr int kKeys = 64;                     // keys per tile (N of S)
  static constexpr int kRegions = kD / 64;             // 128-byte column regions of a row
  static constexpr int kQBytes = kRegions * kRows * 128;
  static constexpr int kKVRegion = kKeys * 128;        // 64 rows x 128 B
  static constexpr int kStageBytes = 2 * kRegions * kKVRegion;  // K regions, then V regions
  static constexpr int kStages = 2;
  static constexpr int kPBytes = kRows * 128;          // 128 rows x 64 keys x 2 B
  // at head_dim 128 the stage's K tile (16 KB) holds P once S is computed;
  // otherwise P has its own buffer
  static constexpr bool kPInK = kRegions * kKVRegion >= kPBytes;
  static constexpr int kTmemCols = 256;                // S: columns [0, 64); O: [128, 128 + kD)
  // two CTAs per SM (TMEM: 2 x 256 columns of 512), never three: the smem
  // request is padded above a third of the SM's 228 KB
  static constexpr int kSmemUsed = 1024 + kQBytes + kStages * kStageBytes + (kPInK ? 0 : kPBytes) + 128;
  static constexpr int kSmem = kSmemUsed > 80 * 1024 ? kSmemUsed : 80 * 1024;
};

template <bool kBF16>
__device__ __forceinline__ uint32_t pack_p2(float a, float b) {
  if constexpr (kBF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}

template <bool kBF16>
__device__ __forceinline__ float2 unpack_p2(uint32_t u) {
  if constexpr (kBF16) {
    return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u));
  } else {
    return __half22float2(*reinterpret_cast<__half2*>(&u));
  }
}

template <int kD, bool kBF16>
__global__ void __launch_bounds__(128, 2)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                         const PrefillParams p) {
  using Tr = PrefillTraits<kD>;
  constexpr int kR = Tr::kRegions;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int s = blockIdx.z;
  const int h = blockIdx.y;
  const int G = p.group;

  // ---- this CTA's rows: tile qt of sequence s's new tokens ----
  int ctx = p.context_lens[s];
  {
    const int cap = min(p.max_context_len, p.max_blocks_per_seq * 16);
    if (ctx < 0 || ctx > cap) {
      if (tid == 0 && h == 0 && blockIdx.x == 0) raise_status(PKV_DEV_BAD_CONTEXT);
      ctx = ctx < 0 ? 0 : cap;
    }
  }
  const int qa = p.query_start_loc[s], qb = p.query_start_loc[s + 1];
  const int q0 = min(max(qa, 0), p.num_q_tokens);
  const int q1 = min(max(qb, q0), p.num_q_tokens);
  const int n = min(min(q1 - q0, ctx), p.max_query_len);
  const int toks = Tr::kRows / G;                  // new tokens per tile
  const int ntiles = (n * G + Tr::kRows - 1) / Tr::kRows;
  if (blockIdx.x >= ntiles) return;                // whole CTA, before any TMEM use
  const int qt = ntiles - 1 - blockIdx.x;          // longest (latest) tiles start first
  const int t0 = qt * toks;
  const int nt = min(toks, n - t0);
  // keys: row of token t (0-based in the run) sees positions < ctx - n + t + 1
  const int klim = ctx - n + t0 + nt;              // exclusive bound of the tile's last token
  const int kfirst = p.window > 0 ? max(0, ctx - n + t0 + 1 - p.window) : 0;
  const int kbeg = kfirst & ~15;
  const int nk = (klim - kbeg + Tr::kKeys - 1) / Tr::kKeys;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* const sptr = smem_raw + (sbase - raw);
  const uint32_t q_s = sbase;
  const uint32_t kv_s = q_s + Tr::kQBytes;
  const uint32_t p_own = kv_s + Tr::kStages * Tr::kStageBytes;        // P buffer when not in the K tile
  const uint32_t bars = p_own + (Tr::kPInK ? 0 : Tr::kPBytes);  // full[0], full[1], s_done, o_done
  const uint32_t bar_sdone = bars + 16, bar_odone = bars + 24;
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(sptr + (bars - sbase) + 32);
  int* const abort_flag = reinterpret_cast<int*>(sptr + (bars - sbase) + 36);

  if (warp == 0) {
    tmem_alloc(smem_addr(tmem_slot), Tr::kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(bars + 8 * i, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }

  // ---- Q tile -> shared memory, K-major with the 128-byte swizzle ----
  const int row = tid;
  const int rt = row / G, rg = row - (row / G) * G;
  const bool row_ok = rt < nt;
  {
    const uint4* src = reinterpret_cast<const uint4*>(
        reinterpret_cast<const uint16_t*>(p.q) +
        (static_cast<long long>(q0 + t0 + (row_ok ? rt : 0)) * p.num_q_heads + static_cast<long long>(h) * G +
         rg) * kD);
#pragma unroll
    for (int c = 0; c < kD / 8; ++c) {
      const uint4 v = row_ok ? src[c] : make_uint4(0u, 0u, 0u, 0u);
      const int reg = c >> 3, cc = c & 7;
      *reinterpret_cast<uint4*>(sptr + (q_s - sbase) + reg * (Tr::kRows * 128) + row * 128 +
                                ((cc ^ (row & 7)) << 4)) = v;
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;          // 64 columns of scores
  const uint32_t tO = tmem + 128;    // kD columns of output accumulator
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;

  // ---- K/V tile producer (thread 0) ----
  int issued = 0;  // tiles whose loads thread 0 has issued
  auto load_tile = [&](int j) {
    ++issued;
    const int stage = j & 1;
    const uint32_t st = kv_s + stage * Tr::kStageBytes;
    const uint32_t bar = bars + 8 * stage;
    mbar_arrive_expect_tx(bar, Tr::kStageBytes);
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int kb = (kbeg >> 4) + 4 * j + b;  // logical block
      int row0 = p.oob_row;                    // past the context: zero fill
      if (kb * 16 < ctx) {
        int id = p.block_tables[static_cast<long long>(s) * p.max_blocks_per_seq + kb];
        if (static_cast<unsigned>(id) >= static_cast<unsigned>(p.num_blocks)) {
          raise_status(PKV_DEV_BAD_BLOCK);
          id = 0;
        }
        row0 = (id * p.num_kv_heads + h) * 16;
      }
#pragma unroll
      for (int r = 0; r < kR; ++r) {
        tma_load_2d(st + r * Tr::kKVRegion + b * 2048, &kmap, r * 64, row0, bar);
        tma_load_2d(st + (kR + r) * Tr::kKVRegion + b * 2048, &vmap, r * 64, row0, bar);
      }
    }
  };

  // the cache may still be being written by the preceding kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0) {
    load_tile(0);
    if (nk > 1) load_tile(1);
  }

  constexpr uint32_t kIdescS = umma_idesc(128, Tr::kKeys, kBF16, false);
  constexpr uint32_t kIdescO = umma_idesc(128, kD, kBF16, true);
  const int lim = row_ok ? ctx - n + t0 + rt + 1 : kbeg + 1;  // exclusive key bound of this row
  const int lo = p.window > 0 ? lim - p.window : -1;          // keys < lo are outside the window
  float m_used = -INFINITY, l = 0.0f;
  uint32_t ph_s = 0, ph_o = 0;
  int consumed = 0;  // tiles whose loads were waited for

#pragma unroll 1
  for (int j = 0; j < nk; ++j) {
    const int stage = j & 1;
    const uint32_t st = kv_s + stage * Tr::kStageBytes;
    const uint32_t p_s = Tr::kPInK ? st : p_own;
    const int kt0 = kbeg + j * Tr::kKeys;  // first key of the tile
    if (!mbar_wait(bars + 8 * stage, (j >> 1) & 1)) atomicExch(abort_flag, 1);
    consumed = j + 1;
    // keys of the tile at or past the context: zero their V rows (never
    // written, or zero-filled already)
    if (kt0 + Tr::kKeys > ctx) {
      const int r0 = max(ctx - kt0, 0);
      for (int e = tid; e < (Tr::kKeys - r0) * kR * 8; e += 128) {
        const int rr = r0 + e / (kR * 8), reg = (e / 8) % kR, c = e % 8;
        *reinterpret_cast<uint4*>(sptr + (st - sbase) + (kR + reg) * Tr::kKVRegion + rr * 128 + c * 16) =
            make_uint4(0u, 0u, 0u, 0u);
      }
      fence_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    if (*reinterpret_cast<volatile int*>(abort_flag)) break;

    // ---- S = Q K^T ----
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < kD / 16; ++ks) {
        const int reg = ks >> 2, off = (ks & 3) * 32;
        umma_f16(tS, smem_desc_sw128(q_s + reg * (Tr::kRows * 128) + off, 16),
                 smem_desc_sw128(st + reg * Tr::kKVRegion + off, 16), kIdescS, ks > 0 ? 1u : 0u);
      }
      umma_commit(bar_sdone);
    }
    if (!mbar_wait(bar_sdone, ph_s)) atomicExch(abort_flag, 1);
    ph_s ^= 1u;
    tc_fence_after();

    // ---- scores of this row, mask, online softmax ----
    float sv[64];
    {
      float a[32], b[32];
      tmem_ld32(tS + lane_off, a);
      tmem_ld32(tS + lane_off + 32, b);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        sv[c] = a[c];
        sv[32 + c] = b[c];
      }
    }
    float mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < 64; ++c) {
      const int key = kt0 + c;
      const bool ok = key < lim && key >= lo;
      sv[c] = ok ? sv[c] * p.qk_scale_log2 : -INFINITY;
      mx = fmaxf(mx, sv[c]);
    }
    float factor = 1.0f;
    bool rescale = false;
    if (mx > m_used + 8.0f) {
      // the base moves; O and l were accumulated against the old one
      factor = m_used == -INFINITY ? 0.0f : fast_exp2(m_used - mx);
      rescale = m_used != -INFINITY;
      m_used = mx;
    }
    const float base = m_used == -INFINITY ? 0.0f : m_used;
    float sum = 0.0f;
#pragma unroll
    for (int c8 = 0; c8 < 8; ++c8) {
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        w[k] = pack_p2<kBF16>(fast_exp2(sv[8 * c8 + 2 * k] - base), fast_exp2(sv[8 * c8 + 2 * k + 1] - base));
        const float2 f = unpack_p2<kBF16>(w[k]);  // sum what the MMA multiplies
        sum += f.x + f.y;
      }
      *reinterpret_cast<uint4*>(sptr + (p_s - sbase) + row * 128 + ((c8 ^ (row & 7)) << 4)) =
          make_uint4(w[0], w[1], w[2], w[3]);
    }
    l = l * factor + sum;
    if (__any_sync(0xffffffffu, rescale)) {
      // O of the previous tiles is complete (waited below); rescale this
      // warp's rows in TMEM
      const float f = rescale ? factor : 1.0f;
#pragma unroll 1
      for (int cb = 0; cb < kD / 32; ++cb) {
        float o[32];
        tmem_ld32(tO + lane_off + 32 * cb, o);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] *= f;
        tmem_st32(tO + lane_off + 32 * cb, o);
      }
      tmem_wait_st();
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- O += P V ----
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < Tr::kKeys / 16; ++ks) {
        umma_f16(tO, smem_desc_sw128(p_s + ks * 32, 16),
                 smem_desc_sw128(st + kR * Tr::kKVRegion + ks * 2048, Tr::kKVRegion), kIdescO,
                 (j > 0 || ks > 0) ? 1u : 0u);
      }
      umma_commit(bar_odone);
    }
    if (!mbar_wait(bar_odone, ph_o)) atomicExch(abort_flag, 1);
    ph_o ^= 1u;
    tc_fence_after();
    // this stage is free again: prefetch tile j + 2 into it
    if (tid == 0 && j + 2 < nk) {
      fence_async_smem();
      load_tile(j + 2);
    }
  }

  // after an abort, let loads still in flight land (bounded) before exit
  if (tid == 0) {
    for (int j = consumed; j < issued; ++j) mbar_wait(bars + 8 * (j & 1), (j >> 1) & 1);
  }

  // ---- epilogue: O / l -> out ----
  if (!*reinterpret_cast<volatile int*>(abort_flag)) {
    const float inv = l > 0.0f ? 1.0f / l : 0.0f;
    uint16_t* dst = reinterpret_cast<uint16_t*>(p.out) +
                    (static_cast<long long>(q0 + t0 + (row_ok ? rt : 0)) * p.num_q_heads +
                     static_cast<long long>(h) * G + rg) * kD;
#pragma unroll 1
    for (int cb = 0; cb < kD / 32; ++cb) {
      float o[32];
      tmem_ld32(tO + lane_off + 32 * cb, o);
      tmem_wait_ld();
      if (row_ok) {
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          uint4 v;
          v.x = pack_p2<kBF16>(o[8 * c8 + 0] * inv, o[8 * c8 + 1] * inv);
          v.y = pack_p2<kBF16>(o[8 * c8 + 2] * inv, o[8 * c8 + 3] * inv);
          v.z = pack_p2<kBF16>(o[8 * c8 + 4] * inv, o[8 * c8 + 5] * inv);
          v.w = pack_p2<kBF16>(o[8 * c8 + 6] * inv, o[8 * c8 + 7] * inv);
          *reinterpret_cast<uint4*>(dst + 32 * cb + 8 * c8) = v;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, Tr::kTmemCols);
}

}  // namespace pkv
