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
//   * One CTA per (sequence, KV head, pair of tiles of 128 query rows); a row
//     is a (new token, query head of the group) pair, row = t * G + g, so the
//     GQA group shares every K/V tile, and so do the CTA's two query tiles.
//     Warpgroup A (warps 0-3) and B (warps 4-7) own one tile each; thread i
//     of a warpgroup owns row i, i.e. TMEM lane i: the whole online softmax of
//     a row runs in one thread.  Lane 0 of warp 8 issues every MMA; warp 9
//     loads K and V.  Sequences start in decreasing context length (the
//     hardware launches CTAs in blockIdx order), so long runs of key tiles do
//     not form the tail of the launch.
//   * Keys stream in tiles of 128 (eight 16-token cache blocks found through
//     the block table) by TMA into a ring of entries holding K_0, V_0, K_1,
//     V_1, ... (128-byte swizzle); K tiles are K-major B operands, V tiles
//     MN-major B operands of the same layout.
//   * S = Q K^T: tcgen05.mma M=128, N=128, K=16 steps over head_dim, both
//     operands in shared memory, into TMEM (fp32).  P = exp2(S - m) in
//     bf16/fp16 is written by the softmax threads over the upper half of S in
//     TMEM and read from there by O += P V (the TS form, M=128,
//     N=head_dim), so P never goes through shared memory.  After P_x(j) . V_j
//     the same thread issues S_x(j+1) into S's columns; the tensor core runs
//     one thread's MMAs in issue order, so P is read before it is
//     overwritten.  The two query tiles ping-pong: one warpgroup's softmax
//     overlaps the other tile's MMAs.  Completion is signalled by
//     tcgen05.commit on mbarriers; every wait is bounded.
//   * Online softmax with a lazy rescale: the exponent base of a row only
//     moves when its max grows by more than 8 (log2 units), and only then is
//     that row's O rescaled in TMEM.  With bf16 probabilities a tile is
//     first computed against the current base without taking its maximum
//     (the row sum bounds every probability; a sum above 2^20 takes the
//     maximum and writes P again).  Unmasked tiles skip the mask; the
//     softmax scale is folded into one FMA per score, two scores per packed
//     f32x2 instruction.  tcgen05.ld / st / wait are warp-wide, so every
//     branch around them is decided per warp.
//   * Tokens of a sequence's last block beyond its context were never
//     written: the load warp zeroes their V rows in the entry before P . V
//     reads them; blocks past the context are loaded from outside the tensor
//     (TMA fills zeros).
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

// D[tmem] (+)= A[tmem] . B[smem]^T: A (M rows = TMEM lanes, K along the
// columns, two 16-bit elements per column) is read from tensor memory.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
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

// 64 consecutive fp32 columns of the calling thread's TMEM lane (warp-wide).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float* v) {
  uint32_t r[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, "
      "%36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, "
      "%57, %58, %59, %60, %61, %62, %63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

// 16 consecutive 32-bit columns of the calling thread's TMEM lane (warp-wide).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&w)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]), "r"(w[8]), "r"(w[9]),
      "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])
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
  int max_tiles;   // tiles of 128 rows of the longest query run (grid.x = pairs of them)
  int oob_row;     // a TMA row coordinate past the cache (zero fill)
  float qk_scale_log2;
};

template <int kD>
struct PrefillTraits {
  static constexpr int kRows = 128;                    // query rows per tile (M)
  static constexpr int kTiles = 2;                     // query tiles per CTA (ping-pong)
  static constexpr int kKeys = 128;                    // keys per K/V tile (N of S, K of P . V)
  static constexpr int kBlocks = kKeys / 16;           // cache blocks per K/V tile
  static constexpr int kRegions = kD / 64;             // 128-byte column regions of a row
  static constexpr int kQBytes = kRegions * kRows * 128;
  static constexpr int kRegionBytes = kKeys * 128;     // 128 rows x 128 B
  static constexpr int kEntryBytes = kRegions * kRegionBytes;  // one K tile or one V tile
  static constexpr int kBarBytes = 256;
  static constexpr int kFit = (227 * 1024 - 1024 - kTiles * kQBytes - kBarBytes) / kEntryBytes;
  static constexpr int kEntries = kFit > 8 ? 8 : kFit;  // ring of K and V tiles: K0 V0 K1 V1 ...
  static constexpr int kThreads = 10 * 32;             // 2 softmax warpgroups, MMA warp, load warp
  static constexpr int kRankMax = 64;                  // sequences ranked by context length per launch
  // TMEM: S of tile x at 128 x (P of tile x, 16-bit, over its upper half at
  // 128 x + 64), O of tile x at 256 + 128 x
  static constexpr int kTmemCols = 512;
  static constexpr int kSmemUsed = 1024 + kTiles * kQBytes + kEntries * kEntryBytes + kBarBytes;
  // one CTA per SM (it holds all 512 TMEM columns): ask for more than half
  static constexpr int kSmem = kSmemUsed > 116 * 1024 ? kSmemUsed : 116 * 1024;
};

// Packed two-lane fp32 arithmetic: one instruction for two lanes (sm_100),
// each lane rounded once as its scalar form would be.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// Two output values, round to nearest.
template <bool kBF16>
__device__ __forceinline__ uint32_t pack_out(float a, float b) {
  if constexpr (kBF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}

// Two probabilities packed as the MMA's 16-bit operand pair (a in the low
// half).  bf16 keeps the top 16 bits (rounding toward zero: one byte permute
// instead of a conversion); the row sum is taken over the same packed values,
// so the normalisation matches what the MMA multiplies.
template <bool kBF16>
__device__ __forceinline__ uint32_t pack_p2(float a, float b) {
  if constexpr (kBF16) {
    return __byte_perm(__float_as_uint(a), __float_as_uint(b), 0x7632);
  } else {
    __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}

// Sum of the two 16-bit values packed in u, as the MMA will multiply them.
template <bool kBF16>
__device__ __forceinline__ float sum_p2(uint32_t u) {
  if constexpr (kBF16) {
    return __uint_as_float(u << 16) + __uint_as_float(u & 0xFFFF0000u);
  } else {
    const float2 f = __half22float2(*reinterpret_cast<__half2*>(&u));
    return f.x + f.y;
  }
}

// One CTA: two tiles of 128 (token, head) rows of one (sequence, KV head)
// ("A" = the later tokens, "B" = the 128 rows before them), warpgroup A
// (warps 0-3) and B (warps 4-7) each owning one tile's softmax, warp 8
// issuing every MMA and warp 9 loading K and V tiles into a ring of entries
// (an entry is refilled once the MMAs that read it are done).  For K/V tile
// j and x = A, B, once P_x(j) is in TMEM: O_x += P_x(j) . V_j, then
// S_x(j+1) = Q_x K_{j+1}^T into the same TMEM columns (the tensor core runs
// one thread's MMAs in issue order, so P_x(j) is read before it is
// overwritten), committed to s_full[x].  That commit also covers every
// earlier MMA, so a warpgroup that sees S_x(j+1) may rescale O_x and write
// P_x(j+1) without further waits.
template <int kD, bool kBF16>
__global__ void __launch_bounds__(PrefillTraits<kD>::kThreads, 1)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                         const PrefillParams p) {
  using Tr = PrefillTraits<kD>;
  constexpr int kR = Tr::kRegions;
  constexpr int kE = Tr::kEntries;
  constexpr int kN = Tr::kKeys;
  constexpr int kBlk = Tr::kBlocks;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int h = blockIdx.y;
  const int G = p.group;
  const int cap = min(p.max_context_len, p.max_blocks_per_seq * 16);

  // ---- sequence of this CTA ----
  // Sequences are taken in decreasing context length (ties by index): the
  // hardware starts CTAs in blockIdx order, so the longest runs of key tiles
  // start first and short pairs fill the tail.  Beyond kRankMax sequences the
  // launch order stays as it is (many sequences balance by themselves).
  int s = blockIdx.z;
  if (p.num_seqs <= Tr::kRankMax) {
    __shared__ int seq_of_rank;
    auto ctx_of = [&](int t) {
      const int c = p.context_lens[t];
      return c < 0 ? 0 : (c > cap ? cap : c);
    };
    for (int t = tid; t < p.num_seqs; t += blockDim.x) {
      const int ct = ctx_of(t);
      int r = 0;
      for (int u = 0; u < p.num_seqs; ++u) {
        const int cu = ctx_of(u);
        r += (cu > ct || (cu == ct && u < t)) ? 1 : 0;
      }
      if (r == static_cast<int>(blockIdx.z)) seq_of_rank = t;  // ranks are a permutation of 0 .. num_seqs - 1
    }
    __syncthreads();
    s = seq_of_rank;
  }

  // ---- rows of this CTA ----
  int ctx = p.context_lens[s];
  {
    if (ctx < 0 || ctx > cap) {
      if (tid == 0 && h == 0 && blockIdx.x == 0) raise_status(PKV_DEV_BAD_CONTEXT);
      ctx = ctx < 0 ? 0 : cap;
    }
  }
  const int qa = p.query_start_loc[s], qb = p.query_start_loc[s + 1];
  const int q0 = min(max(qa, 0), p.num_q_tokens);
  const int q1 = min(max(qb, q0), p.num_q_tokens);
  const int n = min(min(q1 - q0, ctx), p.max_query_len);
  const int toks = Tr::kRows / G;                    // new tokens per tile
  const int ntiles = (n * G + Tr::kRows - 1) / Tr::kRows;
  const int pairs = (ntiles + 1) / 2;
  if (static_cast<int>(blockIdx.x) >= pairs) return;  // whole CTA, before any TMEM use
  // tile A: the later one (more keys); tile B: the one before it (may not exist)
  const int tile_a = ntiles - 1 - 2 * static_cast<int>(blockIdx.x);
  const int tile_b = tile_a - 1;
  const int ta0 = tile_a * toks, nta = min(toks, n - ta0);
  const int tb0 = tile_b * toks, ntb = tile_b >= 0 ? min(toks, n - tb0) : 0;
  // keys: token t (0-based in the run) sees positions < ctx - n + t + 1
  const int klim = ctx - n + ta0 + nta;
  const int t_first = tile_b >= 0 ? tb0 : ta0;
  const int kfirst = p.window > 0 ? max(0, ctx - n + t_first + 1 - p.window) : 0;
  const int kbeg = kfirst & ~15;
  const int nk = (klim - kbeg + kN - 1) / kN;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* const sptr = smem_raw + (sbase - raw);
  const uint32_t q_s = sbase;                                  // Q_A, Q_B
  const uint32_t kv_s = q_s + Tr::kTiles * Tr::kQBytes;       // kE ring entries
  const uint32_t bars = kv_s + kE * Tr::kEntryBytes;
  // barriers: full[kE], empty[kE], s_full[2], p_full[2], o_full, v_tail
  const uint32_t b_full = bars, b_empty = bars + 8 * kE, b_sfull = bars + 16 * kE;
  const uint32_t b_pfull = b_sfull + 16, b_ofull = b_sfull + 32, b_vtail = b_sfull + 40;
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(sptr + (bars - sbase) + 16 * kE + 48);
  int* const abort_flag = reinterpret_cast<int*>(sptr + (bars - sbase) + 16 * kE + 52);
  auto aborted = [&]() { return *reinterpret_cast<volatile int*>(abort_flag) != 0; };
  auto wait_or_abort = [&](uint32_t bar, uint32_t parity) {
    if (!mbar_wait(bar, parity)) atomicExch(abort_flag, 1);
  };

  if (warp == 0) {
    tmem_alloc(smem_addr(tmem_slot), Tr::kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < kE; ++i) {
      mbar_init(b_full + 8 * i, 1);
      mbar_init(b_empty + 8 * i, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(b_sfull + 8 * x, 1);
      mbar_init(b_pfull + 8 * x, Tr::kRows / 32);  // one arrival per softmax warp
    }
    mbar_init(b_ofull, 1);
    mbar_init(b_vtail, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }

  // ---- Q tiles -> shared memory, K-major with the 128-byte swizzle ----
  const int wg = warp >> 2;          // 0: tile A, 1: tile B, 2: MMA warp (8) and load warp (9)
  const int row = tid & 127;         // row of the warpgroup's tile / TMEM lane
  const int t0x = wg == 0 ? ta0 : tb0;
  const int ntx = wg == 0 ? nta : ntb;
  const int rt = row / G, rg = row - (row / G) * G;
  const bool row_ok = wg < 2 && rt < ntx;
  if (wg < 2) {
    const uint4* src = reinterpret_cast<const uint4*>(
        reinterpret_cast<const uint16_t*>(p.q) +
        (static_cast<long long>(q0 + (row_ok ? t0x + rt : ta0)) * p.num_q_heads + static_cast<long long>(h) * G +
         rg) * kD);
    const uint32_t qx = q_s + wg * Tr::kQBytes;
#pragma unroll
    for (int c = 0; c < kD / 8; ++c) {
      const uint4 v = row_ok ? src[c] : make_uint4(0u, 0u, 0u, 0u);
      const int reg = c >> 3, cc = c & 7;
      *reinterpret_cast<uint4*>(sptr + (qx - sbase) + reg * (Tr::kRows * 128) + row * 128 + ((cc ^ (row & 7)) << 4)) =
          v;
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the cache may still be being written by the preceding kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");

  constexpr uint32_t kIdescS = umma_idesc(128, kN, kBF16, false);
  constexpr uint32_t kIdescO = umma_idesc(128, kD, kBF16, true);

  if (warp == 9) {
    // =================== load warp: K_0 V_0 K_1 V_1 ... through the ring ===================
    if (lane == 0) {
      // Block ids of K/V tile j; those of the next tile are read before the
      // waits for free entries, so their latency hides behind them.
      auto fetch_ids = [&](int j, int (&ids)[kBlk]) {
#pragma unroll
        for (int b = 0; b < kBlk; ++b) {
          const int kb = (kbeg >> 4) + kBlk * j + b;  // logical block
          ids[b] = kb * 16 < ctx ? p.block_tables[static_cast<long long>(s) * p.max_blocks_per_seq + kb] : -1;
        }
      };
      int issued = 0;
      int ids[kBlk], nxt[kBlk];
#pragma unroll
      for (int b = 0; b < kBlk; ++b) nxt[b] = -1;
      if (nk > 0) fetch_ids(0, ids);
#pragma unroll 1
      for (int i = 0; i < 2 * nk; ++i) {
        const int j = i >> 1;
        const bool is_v = (i & 1) != 0;
        if (!is_v && j + 1 < nk) fetch_ids(j + 1, nxt);
        const int slot = i % kE;
        if (i >= kE) {
          // the entry's previous tile (i - kE) has been read by its MMAs
          wait_or_abort(b_empty + 8 * slot, ((i - kE) / kE) & 1);
          if (aborted()) break;
          fence_async_smem();
        }
        const uint32_t dst = kv_s + slot * Tr::kEntryBytes;
        const uint32_t bar = b_full + 8 * slot;
        const CUtensorMap* map = is_v ? &vmap : &kmap;
        mbar_arrive_expect_tx(bar, Tr::kEntryBytes);
        ++issued;
#pragma unroll
        for (int b = 0; b < kBlk; ++b) {
          int row0 = p.oob_row;  // past the context: zero fill
          int id = ids[b];
          if (id != -1) {
            if (static_cast<unsigned>(id) >= static_cast<unsigned>(p.num_blocks)) {
              raise_status(PKV_DEV_BAD_BLOCK);
              id = 0;
            }
            row0 = (id * p.num_kv_heads + h) * 16;
          }
#pragma unroll
          for (int r = 0; r < kR; ++r) tma_load_2d(dst + r * Tr::kRegionBytes + b * 2048, map, r * 64, row0, bar);
        }
        if (is_v) {
#pragma unroll
          for (int b = 0; b < kBlk; ++b) ids[b] = nxt[b];
        }
      }
      // loads still in flight after an abort land (bounded) before exit; the
      // last tile of each entry is the only one that can still be pending
      for (int i = max(issued - kE, 0); i < issued; ++i) mbar_wait(b_full + 8 * (i % kE), (i / kE) & 1);
    }
    __syncwarp();
    // The last K/V tile may reach past the context: once it has landed, its V
    // rows there (never written, or zero-filled already) are zeroed before
    // any P . V reads them, and v_tail tells the MMA warp so.
    const int kt_last = kbeg + (nk - 1) * kN;
    if (nk > 0 && kt_last + kN > ctx) {
      const int vi = 2 * nk - 1, vslot = vi % kE;
      wait_or_abort(b_full + 8 * vslot, (vi / kE) & 1);
      if (!aborted()) {
        const int r0 = max(ctx - kt_last, 0);
        uint8_t* const ve = sptr + (kv_s + vslot * Tr::kEntryBytes - sbase);
        for (int e = lane; e < (kN - r0) * kR * 8; e += 32) {
          const int rr = r0 + e / (kR * 8), reg = (e / 8) % kR, c = e % 8;
          *reinterpret_cast<uint4*>(ve + reg * Tr::kRegionBytes + rr * 128 + c * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(b_vtail);
    }
  } else if (warp == 8) {
    // =================== MMA warp: every tcgen05.mma, issued by lane 0 ===================
    // Descriptors are computed once; a K-step or an entry moves only the
    // start-address field (bits 0-13, 16-byte units), so each MMA adds a
    // small constant instead of rebuilding its descriptors.
    const uint64_t dq0 = smem_desc_sw128(q_s, 16);
    const uint64_t dk0 = smem_desc_sw128(kv_s, 16);                  // K tiles: K-major
    const uint64_t dv0 = smem_desc_sw128(kv_s, Tr::kRegionBytes);    // V tiles: MN-major
    auto issue_s = [&](int x, int j) {  // S_x = Q_x K_j^T
      const uint64_t dq = dq0 + static_cast<uint32_t>(x * (Tr::kQBytes >> 4));
      const uint64_t dk = dk0 + static_cast<uint32_t>(((2 * j) % kE) * (Tr::kEntryBytes >> 4));
      const uint32_t d = tmem + 128 * x;
#pragma unroll
      for (int ks = 0; ks < kD / 16; ++ks) {
        constexpr int kQReg = Tr::kRows * 128 / 16, kKReg = Tr::kRegionBytes / 16;
        const uint32_t qo = (ks >> 2) * kQReg + (ks & 3) * 2, ko = (ks >> 2) * kKReg + (ks & 3) * 2;
        umma_f16(d, dq + qo, dk + ko, kIdescS, ks > 0 ? 1u : 0u);
      }
    };
    auto issue_pv = [&](int x, int j) {  // O_x += P_x V_j, P_x read from TMEM
      const uint64_t dv = dv0 + static_cast<uint32_t>(((2 * j + 1) % kE) * (Tr::kEntryBytes >> 4));
      const uint32_t a = tmem + 128 * x + 64;
      const uint32_t d = tmem + 256 + 128 * x;
#pragma unroll
      for (int ks = 0; ks < kN / 16; ++ks) {
        umma_f16_ts(d, a + 8 * ks, dv + static_cast<uint32_t>(ks * 128), kIdescO, (j > 0 || ks > 0) ? 1u : 0u);
      }
    };
    // lane 0 alone runs the loop (no warp-wide waits between tiles)
    if (lane == 0 && nk > 0) {
      wait_or_abort(b_full, 0);  // K_0 sits in entry 0
      tc_fence_after();
      issue_s(0, 0);
      umma_commit(b_sfull);
      issue_s(1, 0);
      umma_commit(b_sfull + 8);
      umma_commit(b_empty);
#pragma unroll 1
      for (int j = 0; j < nk; ++j) {
        const int vi = 2 * j + 1, vslot = vi % kE;
        const int kt0 = kbeg + j * kN;
        wait_or_abort(b_full + 8 * vslot, (vi / kE) & 1);
        // a tile past the context: its V rows there are zeroed by the load warp
        if (kt0 + kN > ctx) wait_or_abort(b_vtail, 0);
        if (aborted()) break;
        const bool more = j + 1 < nk;
        const int ki = 2 * (j + 1), kslot = ki % kE;
#pragma unroll 1
        for (int x = 0; x < 2; ++x) {
          wait_or_abort(b_pfull + 8 * x, j & 1);  // P_x(j) in TMEM, O_x rescaled
          tc_fence_after();
          issue_pv(x, j);
          if (x == 1) umma_commit(b_empty + 8 * vslot);  // V_j read by both P . V
          if (more) {
            if (x == 0) {
              wait_or_abort(b_full + 8 * kslot, (ki / kE) & 1);
              tc_fence_after();
            }
            issue_s(x, j + 1);
            umma_commit(b_sfull + 8 * x);
            if (x == 1) umma_commit(b_empty + 8 * kslot);  // K_{j+1} read by both S
          }
        }
        if (!more) umma_commit(b_ofull);  // every MMA of the CTA done
      }
    }
    __syncwarp();
  } else {
    // =================== softmax warpgroup x = wg ===================
    const int x = wg;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + 128 * x + lane_off;
    const uint32_t tP = tS + 64;
    const uint32_t tO = tmem + 256 + 128 * x + lane_off;
    // exclusive key bound and window start of this row; rows past the run
    // see one key so that their (discarded) math stays finite
    const int lim = row_ok ? ctx - n + t0x + rt + 1 : kbeg + 1;
    const int lo = p.window > 0 ? lim - p.window : -1;
    // a tile is unmasked for the whole warpgroup when it lies between the
    // largest window start and the smallest bound of the tile's rows
    const int wmin_lim = ctx - n + t0x + 1;
    const int wmax_lo = p.window > 0 ? ctx - n + t0x + max(ntx, 1) - p.window : -1;
    const float c = p.qk_scale_log2;  // > 0 (checked by the host)
    float m_used = -INFINITY, l = 0.0f;
#pragma unroll 1
    for (int j = 0; j < nk; ++j) {
      wait_or_abort(b_sfull + 8 * x, j & 1);
      if (__any_sync(0xFFFFFFFFu, aborted())) break;  // the warp leaves together
      tc_fence_after();
      float sv[kN];
#pragma unroll
      for (int q = 0; q < kN / 64; ++q) tmem_ld64(tS + 64 * q, sv + 64 * q);
      tmem_wait_ld();
      const int kt0 = kbeg + j * kN;
      const bool full = kt0 + kN <= wmin_lim && kt0 >= wmax_lo && row_ok;
      if (!full) {
#pragma unroll
        for (int k = 0; k < kN; ++k) {
          const int key = kt0 + k;
          sv[k] = (key < lim && key >= lo) ? sv[k] : -INFINITY;
        }
      }
      // P over the upper half of S (already read into registers) with the
      // exponent base -nb; returns the row sum of the packed values
      auto emit_p = [&](float nb) {
        if constexpr (kBF16) {
          // two scores per packed instruction: s * c + nb, and the row sum
          // over the packed (truncated) probabilities
          const float2 c2 = make_float2(c, c), nb2 = make_float2(nb, nb);
          float2 sp2[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
          for (int q = 0; q < kN / 32; ++q) {
            uint32_t w[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const int e = 32 * q + 2 * k;
              const float2 xy = fma2(make_float2(sv[e], sv[e + 1]), c2, nb2);
              w[k] = pack_p2<true>(fast_exp2(xy.x), fast_exp2(xy.y));
              sp2[k & 1] = add2(sp2[k & 1], make_float2(__uint_as_float(w[k] << 16),
                                                        __uint_as_float(w[k] & 0xFFFF0000u)));
            }
            tmem_st16(tP + 16 * q, w);
          }
          return (sp2[0].x + sp2[1].x) + (sp2[0].y + sp2[1].y);
        } else {
          float sp[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
          for (int q = 0; q < kN / 32; ++q) {
            uint32_t w[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const int e = 32 * q + 2 * k;
              w[k] = pack_p2<kBF16>(fast_exp2(fmaf(sv[e], c, nb)), fast_exp2(fmaf(sv[e + 1], c, nb)));
              sp[k & 3] += sum_p2<kBF16>(w[k]);
            }
            tmem_st16(tP + 16 * q, w);
          }
          return (sp[0] + sp[1]) + (sp[2] + sp[3]);
        }
      };
      // Common case (bf16): the base of the earlier tiles still serves.  The
      // row sum bounds every probability, so a sum of at most 2^20
      // (p <= 2^20, far from overflowing O or l) keeps the tile without ever
      // taking its maximum; a larger or non-finite sum (a score far above the base, or
      // no base yet) takes the maximum, moves the base and writes P again.
      // tcgen05.ld / st / wait are warp-wide instructions, so the choice is
      // made per warp: it takes the slow way when any of its rows needs it.
      // fp16 probabilities (largest value 65504) always take the maximum
      // first.
      float factor = 1.0f;
      bool rescale = false;
      float sum = 0.0f;
      bool need_max = !kBF16 || __any_sync(0xFFFFFFFFu, m_used == -INFINITY);
      if (!need_max) {
        sum = emit_p(-m_used);
        need_max = __any_sync(0xFFFFFFFFu, !(sum <= 1048576.0f));
        if (need_max) tmem_wait_st();  // the first try has landed before it is overwritten
      }
      if (need_max) {
        // independent partial maxima keep the dependency chains short
        float mp[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mp[k] = fmaxf(sv[k], sv[k + 8]);
#pragma unroll
        for (int k = 16; k < kN; ++k) mp[k & 7] = fmaxf(mp[k & 7], sv[k]);
        const float mr = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                               fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
        const float mx = mr * c;  // scores are used as s * c (log2 units)
        if (mx > m_used + 8.0f) {
          factor = m_used == -INFINITY ? 0.0f : fast_exp2(m_used - mx);
          rescale = m_used != -INFINITY;
          m_used = mx;
        }
        sum = emit_p(m_used == -INFINITY ? 0.0f : -m_used);
      }
      l = l * factor + sum;
      // O_x holds every P . V before this tile (S_x(j) was committed after
      // them); the warp rescales together, rows keeping their base by 1
      if (__any_sync(0xFFFFFFFFu, rescale)) {
        const float oscale = rescale ? factor : 1.0f;
#pragma unroll 1
        for (int cb = 0; cb < kD / 32; ++cb) {
          float o[32];
          tmem_ld32(tO + 32 * cb, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] *= oscale;
          tmem_st32(tO + 32 * cb, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_pfull + 8 * x);
    }
    // ---- epilogue: O / l -> out ----
    if (!__any_sync(0xFFFFFFFFu, aborted())) wait_or_abort(b_ofull, 0);
    tc_fence_after();
    if (!__any_sync(0xFFFFFFFFu, aborted())) {
      const float inv = l > 0.0f ? 1.0f / l : 0.0f;
      uint16_t* dst = reinterpret_cast<uint16_t*>(p.out) +
                      (static_cast<long long>(q0 + (row_ok ? t0x + rt : ta0)) * p.num_q_heads +
                       static_cast<long long>(h) * G + rg) * kD;
#pragma unroll 1
      for (int cb = 0; cb < kD / 32; ++cb) {
        float o[32];
        tmem_ld32(tO + 32 * cb, o);
        tmem_wait_ld();
        if (row_ok) {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            uint4 v;
            v.x = pack_out<kBF16>(o[8 * c8 + 0] * inv, o[8 * c8 + 1] * inv);
            v.y = pack_out<kBF16>(o[8 * c8 + 2] * inv, o[8 * c8 + 3] * inv);
            v.z = pack_out<kBF16>(o[8 * c8 + 4] * inv, o[8 * c8 + 5] * inv);
            v.w = pack_out<kBF16>(o[8 * c8 + 6] * inv, o[8 * c8 + 7] * inv);
            *reinterpret_cast<uint4*>(dst + 32 * cb + 8 * c8) = v;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, Tr::kTmemCols);
}

}  // namespace pkv
