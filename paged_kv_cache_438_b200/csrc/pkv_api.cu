// C-ABI entry points of libpagedkv: argument checks, launch planning, TMA
// tensor maps and kernel launches.  The single CUDA translation unit of the
// library (the kernels live in the included headers), so the device status
// word exists once per device.  Compiled without fast-math: the quantising
// write relies on IEEE fp32 division and round-to-nearest-even.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <map>
#include <mutex>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "pkv_decode.cuh"
#include "pkv_prefill.cuh"
#include "pkv_error.h"
#include "pkv_write.cuh"

using pkv::fail;
using pkv::ok;

namespace {

std::atomic<int> g_validate{0};

bool is16(int dt) { return dt == PKV_F16 || dt == PKV_BF16; }
bool is4(int dt) { return dt == PKV_I4 || dt == PKV_FP4E2M1; }
// quantised formats: per-token scales, 8 or 4 bits per element
bool isq(int dt) { return dt == PKV_I8 || dt == PKV_FP8E4M3 || dt == PKV_U8ASYM || is4(dt); }
bool has_zero(int dt) { return dt == PKV_U8ASYM; }
// bytes of one token's K (or V) row in the cache
int row_bytes(int dt, int head_dim) { return is16(dt) ? 2 * head_dim : (is4(dt) ? head_dim / 2 : head_dim); }
int elt_size(int dt) { return is16(dt) ? 2 : 1; }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int cuda_fail(cudaError_t e, const char* what) {
  return fail(PKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

// Copies a device array to the host (validation mode only; synchronous).
template <class T>
int fetch(std::vector<T>* dst, const T* src, size_t n, cudaStream_t st) {
  dst->resize(n);
  if (n == 0) return PKV_OK;
  cudaError_t e = cudaMemcpyAsync(dst->data(), src, n * sizeof(T), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  return e == cudaSuccess ? PKV_OK : cuda_fail(e, "validation copy");
}

// A driver API function by name and ABI version (nullptr if unavailable);
// the library links only the runtime.
void* driver_entry(const char* name, unsigned int version) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPointByVersion(name, &p, version, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return p;
}

// ---------------------------------------------------------- tensor maps --
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn =
      reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(driver_entry("cuTensorMapEncodeTiled", 12000));
  return fn;
}

// 2-D view of a cache: one row of row_bytes per (block, head, token), in
// elements of elt bytes (2 for 16-bit caches, else bytes); box = one 16-token
// block x (128 bytes or the whole row) with the matching swizzle.
int make_cache_map(CUtensorMap* map, const void* cache, int row_bytes, int elt, long long rows) {
  auto fn = encode_fn();
  if (!fn) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const int tile_bytes = row_bytes < 128 ? row_bytes : 128;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes / elt), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(tile_bytes / elt), 16u};
  cuuint32_t estr[2] = {1u, 1u};
  const CUtensorMapSwizzle swz = tile_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : tile_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                    : CU_TENSOR_MAP_SWIZZLE_32B;
  CUresult r = fn(map, elt == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                  const_cast<void*>(cache), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
  return PKV_OK;
}

// ------------------------------------------------------------ planning --
constexpr int kMaxCtaSmem = 227 * 1024;  // opt-in shared memory per CTA on sm_100

struct Plan {
  int warps;           // warps per CTA (one CTA per SM)
  int num_streams;     // warps that share the (sequence, head, block) work list
  int stream_tokens;   // upper bound of tokens one stream processes
  size_t workspace;    // arrival counters + partial slots
  size_t counter_bytes;
  int slot_floats;
  int tile_cols;       // columns per pair: G (decode) or 8 / 16 (multi-query)
  int max_tiles;       // pairs per KV head of the longest sequence (1 for decode)
};

// One partial: m[G] and l[G] padded to a multiple of 4 floats, then o[G][D];
// every slot and its o rows stay 16-byte aligned.
int slot_floats(int G, int D) { return (2 * G + 3) / 4 * 4 + G * D; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// The work list has at most B * Hkv * tiles * ceil(max_ctx / 16) items
// (tiles = 1 for decode; multi-query mode (max_q > 0) cuts the max_q * G
// (token, head) columns of a KV head into tiles of 8 or 16).  By default it
// is spread over the warps of the resident CTAs (one CTA per SM: a
// persistent grid) but never thinner than 16 blocks per warp;
// partition_tokens > 0 instead caps the items per warp at partition_tokens / 16.
int decode_warps(int cache_dtype, int D, bool wide, int B);

int make_plan(int B, int Hq, int Hkv, int D, int max_ctx, int cache_dtype, int req_tokens, Plan* out,
              int max_q = 0) {
  const int G = Hq / Hkv;
  int tile_cols = G, max_tiles = 1;
  if (max_q > 0) {
    const long long cols = static_cast<long long>(max_q) * G;
    tile_cols = cols > 8 ? 16 : 8;
    max_tiles = static_cast<int>((cols + tile_cols - 1) / tile_cols);
  }
  const long long blocks_max = std::max(1, (max_ctx + 15) / 16);
  const long long t_max = static_cast<long long>(std::max(B, 1)) * Hkv * max_tiles * blocks_max;
  if (t_max >= (1LL << 31)) return fail(PKV_ERR_UNSUPPORTED, "more than 2^31 (sequence, head, block) items");
  // One CTA per SM.  Quantised caches use 12 warps (8 when a pair has more
  // than 8 columns): their conversion work per byte, not HBM, sets the pace
  // and more warps hide its latency.  16-bit caches use 8 warps.  (Measured
  // on 32 sequences of 32k tokens: 4 warps with twice the ring depth match 8
  // warps within 0.5 % at the full SM clock, but under the power cap's lower
  // clocks the longer per-warp chains slow a step by ~10 % for a 6 % lower
  // clock, where 8 warps lose under 2 % for 9 %.)  Fewer warps take a
  // batch whose context-length scan would not fit beside their smallest
  // rings (decode_warps).
  const long long sms = sm_count();
  const bool wide = tile_cols > 8;
  const int warps = decode_warps(cache_dtype, D, wide, B);
  long long nw;
  if (req_tokens > 0) {
    if (req_tokens % 16 != 0) return fail(PKV_ERR_INVALID_ARG, "partition_tokens %d is not a multiple of 16", req_tokens);
    const long long per = req_tokens / 16;
    nw = (t_max + per - 1) / per;
  } else {
    // Streams of at least 16 blocks (a merge contributor costs about one
    // block) while the work fills a wave of warps; below that the warps'
    // copy rings, not HBM, set the time (each stream waits for its copies one
    // after another), so shorter streams of at least 4 blocks spread a small
    // batch over more SMs.
    const long long wave = static_cast<long long>(warps) * sms;
    nw = std::min(wave, (t_max + 15) / 16);
    if (nw < wave) nw = std::min(wave, (t_max + 3) / 4);
    if (max_tiles > 1) {
      // Several column tiles per KV head re-read the same K/V blocks: one
      // stream per (sequence, head, tile) bound makes the warps of a CTA (and
      // neighbouring CTAs) walk the same blocks of one head at the same time,
      // so the re-reads hit L2 instead of HBM.  The grid then runs in waves.
      nw = static_cast<long long>(std::max(B, 1)) * Hkv * max_tiles;
    }
  }
  nw = std::max(1LL, std::min(nw, t_max));
  if (nw > (1LL << 24)) return fail(PKV_ERR_UNSUPPORTED, "more than 2^24 decode streams");
  out->warps = warps;
  out->num_streams = static_cast<int>(nw);
  out->stream_tokens = static_cast<int>((t_max + nw - 1) / nw * 16);
  out->counter_bytes = align_up(static_cast<size_t>(std::max(B, 1)) * Hkv * max_tiles * 8, 256);
  out->slot_floats = slot_floats(tile_cols, D);
  out->tile_cols = tile_cols;
  out->max_tiles = max_tiles;
  out->workspace = out->counter_bytes + 2 * static_cast<size_t>(nw) * out->slot_floats * 4;
  return PKV_OK;
}

// Multi-query calls whose runs of new tokens fill at least one tile of 128
// (token, head) rows, on 16-bit caches, with the automatic plan, go to the
// query-major tcgen05 kernel (paged_prefill_kernel); the rest stay on the
// decode kernel's multi-query mode.
bool prefill_eligible(int cache_dtype, int head_dim, int G, int max_q, int num_seqs, int partition_tokens) {
  return is16(cache_dtype) && (head_dim == 64 || head_dim == 128) && G >= 1 && 128 % G == 0 &&
         static_cast<long long>(max_q) * G >= 128 && num_seqs <= 65535 && partition_tokens == 0;
}

int prefill_tiles(int max_q, int G) { return static_cast<int>((static_cast<long long>(max_q) * G + 127) / 128); }

// Monotonic epoch of decode calls (40 bits, never 0): tags the arrival
// counters so a workspace needs zeroing only before its first use.
unsigned long long next_epoch() {
  static std::atomic<unsigned long long> epoch{0};
  unsigned long long e;
  do {
    e = (epoch.fetch_add(1) + 1) & ((1ull << 40) - 1);
  } while (e == 0);
  return e;
}

// A workspace holds the arrival counters at its head and the partials after
// them, and the boundary moves with the call's shape (sequences x KV heads x
// column tiles).  Bytes that an earlier call used for partials may hold any
// float pair, and a float pair can read as a counter of the current epoch.
// So the library records, per (device, workspace address), how many leading
// bytes hold counters or zeros since the last call, and clears the rest of a
// call's counter area (an asynchronous memset on the call's stream, not an
// allocation) before the launch.  A workspace the record does not know has
// its whole counter area cleared on its first use.
int prepare_counters(void* ws, size_t counter_bytes, cudaStream_t st) {
  static std::mutex mu;
  static std::map<std::pair<int, uintptr_t>, size_t> clean;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  const auto key = std::make_pair(dev, reinterpret_cast<uintptr_t>(ws));
  std::lock_guard<std::mutex> lk(mu);
  auto it = clean.find(key);
  const size_t have = it == clean.end() ? 0 : it->second;
  if (counter_bytes > have) {
    e = cudaMemsetAsync(static_cast<uint8_t*>(ws) + have, 0, counter_bytes - have, st);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the workspace's arrival counters");
  }
  // bounded: a workspace dropped from the record is cleared again on its next use
  if (it == clean.end() && clean.size() >= 4096) clean.clear();
  clean[key] = counter_bytes;  // this call's partials start right after its counters
  return PKV_OK;
}

template <class T>
int set_smem(T* kernel, size_t bytes) {
  // cudaFuncSetAttribute is per device; remember the largest value set for
  // each (device, kernel).
  static std::mutex mu;
  static std::unordered_map<unsigned long long, size_t> done;
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned long long key = (reinterpret_cast<uintptr_t>(kernel) << 8) ^ static_cast<unsigned>(dev);
  std::lock_guard<std::mutex> lk(mu);
  auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return PKV_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  done[key] = bytes;
  return PKV_OK;
}

// Shared memory of a decode CTA: alignment slack, the warps' copy rings and
// their barriers, and the context-length scan (num_seqs + 1 entries).
template <int kD, int kCT>
size_t decode_smem_bytes(int num_seqs, int warps, int ring) {
  using Tr = pkv::DecodeTraits<kD, kCT>;
  return 1024 + static_cast<size_t>(warps) * ring * (Tr::kStageBytes + 8) + (static_cast<size_t>(num_seqs) + 1) * 4;
}

// Copy stages per warp: as many as the ring budget holds (2 to 8), fewer
// when the scan of a large batch would not leave room for them.
template <int kD, int kCT>
int decode_ring(int num_seqs, int warps) {
  using Tr = pkv::DecodeTraits<kD, kCT>;
  int r = std::max(2, std::min(8, Tr::ring_budget(warps) / (warps * Tr::kStageBytes)));
  while (r > 2 && decode_smem_bytes<kD, kCT>(num_seqs, warps, r) > static_cast<size_t>(kMaxCtaSmem)) --r;
  return r;
}

// Shared memory of a CTA of `warps` warps with two-stage rings (the fewest
// the kernel runs with) beside the scan of B sequences.
template <int kD>
size_t min_decode_smem(int cache_dtype, int warps, int B) {
  switch (cache_dtype) {
    case PKV_F16: return decode_smem_bytes<kD, PKV_F16>(B, warps, 2);
    case PKV_BF16: return decode_smem_bytes<kD, PKV_BF16>(B, warps, 2);
    case PKV_I8: return decode_smem_bytes<kD, PKV_I8>(B, warps, 2);
    case PKV_FP8E4M3: return decode_smem_bytes<kD, PKV_FP8E4M3>(B, warps, 2);
    case PKV_U8ASYM: return decode_smem_bytes<kD, PKV_U8ASYM>(B, warps, 2);
    case PKV_I4: return decode_smem_bytes<kD, PKV_I4>(B, warps, 2);
    case PKV_FP4E2M1: return decode_smem_bytes<kD, PKV_FP4E2M1>(B, warps, 2);
    default: return 0;
  }
}

// Warps per decode CTA: 12 for quantised caches (8 when a pair has more than
// 8 columns), 8 for 16-bit ones; 4 fewer at a time while the context-length
// scan of a very large batch would not fit beside those warps' two-stage
// rings (16-bit caches at head_dim 128: above ~25,000 sequences with 8 warps,
// ~41,000 with 4).
int decode_warps(int cache_dtype, int D, bool wide, int B) {
  int w = isq(cache_dtype) ? (wide ? 8 : 12) : 8;
  while (w > 4) {
    const size_t need = D == 128 ? min_decode_smem<128>(cache_dtype, w, std::max(B, 1))
                                 : min_decode_smem<64>(cache_dtype, w, std::max(B, 1));
    if (need <= static_cast<size_t>(kMaxCtaSmem)) break;
    w -= 4;
  }
  return w;
}

template <int kD, int kCT, int kNT, bool kQBF16, bool kMQ>
int launch_decode(const CUtensorMap& km, const CUtensorMap& vm, const pkv::DecodeParams& p, cudaStream_t st) {
  using Tr = pkv::DecodeTraits<kD, kCT>;
  auto kernel = pkv::paged_decode_kernel<kD, kCT, kNT, kQBF16, kMQ>;
  const int warps = p.ring_warps;
  if (warps < 1 || warps > Tr::max_warps(kNT)) return fail(PKV_ERR_INVALID_ARG, "bad warp count %d", warps);
  pkv::DecodeParams q = p;
  q.ring = decode_ring<kD, kCT>(p.num_seqs, warps);
  const size_t smem = decode_smem_bytes<kD, kCT>(p.num_seqs, warps, q.ring);
  if (smem > static_cast<size_t>(kMaxCtaSmem))
    return fail(PKV_ERR_UNSUPPORTED, "batch of %d sequences needs %zu bytes of shared memory", p.num_seqs, smem);
  int rc = set_smem(kernel, smem);
  if (rc != PKV_OK) return rc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((p.num_streams + warps - 1) / warps);
  cfg.blockDim = dim3(warps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  // may start while the preceding kernel (the KV write) finishes; the kernel
  // waits for it (griddepcontrol.wait) before reading the cache
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, km, vm, q);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return PKV_OK;
}

// kNT = 2 (16 columns per pair) when the group (decode) or the tile
// (multi-query) is wider than 8.
template <int kD, int kCT, bool kMQ>
int dispatch_nt_q(const CUtensorMap& km, const CUtensorMap& vm, const pkv::DecodeParams& p, bool q_bf16,
                  cudaStream_t st) {
  const bool nt2 = (kMQ ? p.tile_cols : p.group) > 8;
  if constexpr (pkv::DecodeTraits<kD, kCT>::kQuant) {
    if (q_bf16)
      return nt2 ? launch_decode<kD, kCT, 2, true, kMQ>(km, vm, p, st)
                 : launch_decode<kD, kCT, 1, true, kMQ>(km, vm, p, st);
    return nt2 ? launch_decode<kD, kCT, 2, false, kMQ>(km, vm, p, st)
               : launch_decode<kD, kCT, 1, false, kMQ>(km, vm, p, st);
  } else {
    (void)q_bf16;
    constexpr bool kQ = (kCT == pkv::kBF16);
    return nt2 ? launch_decode<kD, kCT, 2, kQ, kMQ>(km, vm, p, st)
               : launch_decode<kD, kCT, 1, kQ, kMQ>(km, vm, p, st);
  }
}

template <int kD, bool kBF16>
int launch_prefill(const CUtensorMap& km, const CUtensorMap& vm, const pkv::PrefillParams& p, cudaStream_t st) {
  auto kernel = pkv::paged_prefill_kernel<kD, kBF16>;
  const size_t smem = pkv::PrefillTraits<kD>::kSmem;
  int rc = set_smem(kernel, smem);
  if (rc != PKV_OK) return rc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((p.max_tiles + 1) / 2, p.num_kv_heads, p.num_seqs);  // two tiles per CTA
  cfg.blockDim = dim3(pkv::PrefillTraits<kD>::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, km, vm, p);
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
  return PKV_OK;
}

template <int kD, bool kMQ>
int dispatch_ct(int ct, const CUtensorMap& km, const CUtensorMap& vm, const pkv::DecodeParams& p, bool q_bf16,
                cudaStream_t st) {
  switch (ct) {
    case PKV_F16: return dispatch_nt_q<kD, pkv::kF16, kMQ>(km, vm, p, q_bf16, st);
    case PKV_BF16: return dispatch_nt_q<kD, pkv::kBF16, kMQ>(km, vm, p, q_bf16, st);
    case PKV_I8: return dispatch_nt_q<kD, pkv::kI8, kMQ>(km, vm, p, q_bf16, st);
    case PKV_FP8E4M3: return dispatch_nt_q<kD, pkv::kFP8, kMQ>(km, vm, p, q_bf16, st);
    case PKV_U8ASYM: return dispatch_nt_q<kD, pkv::kU8, kMQ>(km, vm, p, q_bf16, st);
    case PKV_I4: return dispatch_nt_q<kD, pkv::kI4, kMQ>(km, vm, p, q_bf16, st);
    case PKV_FP4E2M1: return dispatch_nt_q<kD, pkv::kFP4, kMQ>(km, vm, p, q_bf16, st);
  }
  return fail(PKV_ERR_UNSUPPORTED, "cache dtype %d", ct);
}

int grid_for(long long work, int per_cta) {
  const long long ctas = (work + per_cta - 1) / per_cta;
  const long long cap = 16LL * sm_count();
  return static_cast<int>(std::max(1LL, std::min(ctas, cap)));
}

}  // namespace

extern "C" {

int pkv_set_validation(int on) {
  g_validate.store(on ? 1 : 0);
  return ok();
}

int pkv_device_status(unsigned int* status_out, int clear) {
  if (!status_out) return fail(PKV_ERR_INVALID_ARG, "status_out is NULL");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  e = cudaMemcpyFromSymbol(status_out, pkv::g_status, sizeof(unsigned int));
  if (e != cudaSuccess) return cuda_fail(e, "read status");
  if (clear) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(pkv::g_status, &zero, sizeof(unsigned int));
    if (e != cudaSuccess) return cuda_fail(e, "clear status");
  }
  return ok();
}

int pkv_kv_cache_write(const void* k, const void* v, void* k_cache, void* v_cache, float* k_scale, float* v_scale,
                       uint8_t* k_zero, uint8_t* v_zero, const int64_t* slot_mapping, int num_tokens, int num_kv_heads, int head_dim, int block_size,
                       int num_blocks, int in_dtype, int cache_dtype, void* stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0)
    return fail(PKV_ERR_INVALID_ARG, "bad sizes (num_tokens %d, num_kv_heads %d, num_blocks %d)", num_tokens,
                num_kv_heads, num_blocks);
  if (block_size != 16) return fail(PKV_ERR_UNSUPPORTED, "block_size must be 16 (got %d)", block_size);
  if (head_dim != 64 && head_dim != 128) return fail(PKV_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", head_dim);
  if (!is16(in_dtype)) return fail(PKV_ERR_UNSUPPORTED, "input dtype %d (need PKV_F16 or PKV_BF16)", in_dtype);
  if (is16(cache_dtype) && cache_dtype != in_dtype)
    return fail(PKV_ERR_UNSUPPORTED, "a 16-bit cache must have the input's dtype");
  if (!is16(cache_dtype) && !isq(cache_dtype)) return fail(PKV_ERR_UNSUPPORTED, "cache dtype %d", cache_dtype);
  if (num_tokens == 0) return ok();
  if (!k || !v || !k_cache || !v_cache || !slot_mapping) return fail(PKV_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
    return fail(PKV_ERR_INVALID_ARG, "k, v and caches must be 16-byte aligned");
  if (isq(cache_dtype) && (!k_scale || !v_scale || !aligned(k_scale, 4) || !aligned(v_scale, 4)))
    return fail(PKV_ERR_INVALID_ARG, "quantised caches need k_scale and v_scale");
  if (has_zero(cache_dtype) && (!k_zero || !v_zero))
    return fail(PKV_ERR_INVALID_ARG, "PKV_U8ASYM caches need k_zero and v_zero");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (g_validate.load()) {
    std::vector<int64_t> sl;
    int rc = fetch(&sl, slot_mapping, static_cast<size_t>(num_tokens), st);
    if (rc != PKV_OK) return rc;
    std::unordered_set<int64_t> seen;
    const int64_t lim = static_cast<int64_t>(num_blocks) * 16;
    for (int t = 0; t < num_tokens; ++t) {
      if (sl[t] == -1) continue;
      if (sl[t] < -1 || sl[t] >= lim) return fail(PKV_ERR_INVALID_ARG, "slot_mapping[%d] = %lld out of range", t, (long long)sl[t]);
      if (!seen.insert(sl[t]).second) return fail(PKV_ERR_INVALID_ARG, "slot %lld appears twice", (long long)sl[t]);
    }
  }
  const long long rows = static_cast<long long>(num_tokens) * num_kv_heads;
  if (is16(cache_dtype)) {
    const int chunks = head_dim * 2 / 16;
    const int grid = grid_for(rows * chunks, 256);
    if (chunks == 16)
      pkv::kv_write_copy_kernel<16><<<grid, 256, 0, st>>>(
          static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint4*>(k_cache),
          static_cast<uint4*>(v_cache), slot_mapping, num_tokens, num_kv_heads, num_blocks);
    else
      pkv::kv_write_copy_kernel<8><<<grid, 256, 0, st>>>(
          static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint4*>(k_cache),
          static_cast<uint4*>(v_cache), slot_mapping, num_tokens, num_kv_heads, num_blocks);
  } else {
    const int grid = grid_for(rows, 8);  // 8 warps per CTA, one row per warp
    const bool bf = in_dtype == PKV_BF16;
    auto* kc = static_cast<uint8_t*>(k_cache);
    auto* vc = static_cast<uint8_t*>(v_cache);
#define PKV_QW(D, F, B)                                                                                          \
  pkv::kv_write_quant_kernel<D, F, B><<<grid, 256, 0, st>>>(k, v, kc, vc, k_scale, v_scale, k_zero, v_zero, \
                                                             slot_mapping, num_tokens, num_kv_heads, num_blocks)
#define PKV_QW_FMT(D, F) \
  do { if (bf) PKV_QW(D, F, true); else PKV_QW(D, F, false); } while (0)
#define PKV_QW_D(D)                                                 \
  do {                                                              \
    if (cache_dtype == PKV_FP8E4M3) PKV_QW_FMT(D, PKV_FP8E4M3);     \
    else if (cache_dtype == PKV_U8ASYM) PKV_QW_FMT(D, PKV_U8ASYM);   \
    else if (cache_dtype == PKV_I4) PKV_QW_FMT(D, PKV_I4);           \
    else if (cache_dtype == PKV_FP4E2M1) PKV_QW_FMT(D, PKV_FP4E2M1); \
    else PKV_QW_FMT(D, PKV_I8);                                     \
  } while (0)
    if (head_dim == 128) PKV_QW_D(128);
    else PKV_QW_D(64);
#undef PKV_QW_D
#undef PKV_QW_FMT
#undef PKV_QW
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kv_cache_write launch");
  return ok();
}

int pkv_decode_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int max_context_len,
                    int cache_dtype, int partition_tokens, int* num_partitions_out, int* partition_tokens_out,
                    size_t* workspace_bytes_out) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_context_len < 0)
    return fail(PKV_ERR_INVALID_ARG, "bad sizes");
  if (head_dim != 64 && head_dim != 128) return fail(PKV_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (!is16(cache_dtype) && !isq(cache_dtype)) return fail(PKV_ERR_UNSUPPORTED, "cache dtype %d", cache_dtype);
  Plan pl{};
  int rc = make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, cache_dtype, partition_tokens, &pl);
  if (rc != PKV_OK) return rc;
  if (num_partitions_out) *num_partitions_out = pl.num_streams;
  if (partition_tokens_out) *partition_tokens_out = pl.stream_tokens;
  if (workspace_bytes_out) *workspace_bytes_out = pl.workspace;
  return ok();
}

int pkv_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int max_context_len,
                              int cache_dtype, size_t* bytes) {
  if (!bytes) return fail(PKV_ERR_INVALID_ARG, "bytes is NULL");
  return pkv_decode_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, cache_dtype, 0, nullptr,
                         nullptr, bytes);
}

}  // extern "C"

namespace {

// Shared body of the decode and multi-query entry points (mq: query_start_loc
// and the packed query rows are used; otherwise one query row per sequence).
int attention_call(void* out, const void* q, const void* k_cache, const void* v_cache, const float* k_scale,
                   const float* v_scale, const uint8_t* k_zero, const uint8_t* v_zero, const int32_t* block_tables,
                   const int32_t* context_lens, const int32_t* query_start_loc, int num_q_tokens, int max_query_len,
                   bool mq, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                   int num_blocks, int max_blocks_per_seq, int max_context_len, float scale, int sliding_window,
                   int q_dtype, int cache_dtype, int partition_tokens, void* workspace, size_t workspace_bytes,
                   void* stream) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0 ||
      max_context_len < 0)
    return fail(PKV_ERR_INVALID_ARG, "bad sizes");
  if (mq && (num_q_tokens < 0 || max_query_len < 0))
    return fail(PKV_ERR_INVALID_ARG, "bad query sizes (num_q_tokens %d, max_query_len %d)", num_q_tokens,
                max_query_len);
  if (block_size != 16) return fail(PKV_ERR_UNSUPPORTED, "block_size must be 16 (got %d)", block_size);
  if (head_dim != 64 && head_dim != 128) return fail(PKV_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", head_dim);
  if (num_q_heads % num_kv_heads != 0) return fail(PKV_ERR_INVALID_ARG, "num_q_heads %% num_kv_heads != 0");
  const int G = num_q_heads / num_kv_heads;
  if (G > 16) return fail(PKV_ERR_UNSUPPORTED, "query group %d > 16", G);
  if (!is16(q_dtype)) return fail(PKV_ERR_UNSUPPORTED, "q dtype %d", q_dtype);
  if (is16(cache_dtype) && q_dtype != cache_dtype) return fail(PKV_ERR_UNSUPPORTED, "q dtype must match a 16-bit cache");
  if (!is16(cache_dtype) && !isq(cache_dtype)) return fail(PKV_ERR_UNSUPPORTED, "cache dtype %d", cache_dtype);
  if (!std::isfinite(scale)) return fail(PKV_ERR_INVALID_ARG, "scale is not finite");
  if (sliding_window < 0) return fail(PKV_ERR_INVALID_ARG, "sliding_window %d < 0", sliding_window);
  if (static_cast<long long>(num_blocks) * num_kv_heads * 16 >= (1LL << 31))
    return fail(PKV_ERR_UNSUPPORTED, "pool too large for 32-bit copy coordinates");
  if (static_cast<long long>(max_context_len) > static_cast<long long>(max_blocks_per_seq) * 16)
    return fail(PKV_ERR_INVALID_ARG, "max_context_len %d exceeds max_blocks_per_seq * 16", max_context_len);
  if (num_seqs == 0 || (mq && (num_q_tokens == 0 || max_query_len == 0))) return ok();
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || (mq && !query_start_loc))
    return fail(PKV_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16)) return fail(PKV_ERR_INVALID_ARG, "caches must be 16-byte aligned");
  if (!aligned(q, 4) || !aligned(out, 4)) return fail(PKV_ERR_INVALID_ARG, "q and out must be 4-byte aligned");
  if (isq(cache_dtype) && (!k_scale || !v_scale || !aligned(k_scale, 16) || !aligned(v_scale, 16)))
    return fail(PKV_ERR_INVALID_ARG, "quantised caches need 16-byte aligned k_scale and v_scale");
  if (has_zero(cache_dtype) && (!k_zero || !v_zero || !aligned(k_zero, 16) || !aligned(v_zero, 16)))
    return fail(PKV_ERR_INVALID_ARG, "PKV_U8ASYM caches need 16-byte aligned k_zero and v_zero");
  Plan pl{};
  int rc = make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, cache_dtype, partition_tokens,
                     &pl, mq ? max_query_len : 0);
  if (rc != PKV_OK) return rc;
  const bool prefill = mq && prefill_eligible(cache_dtype, head_dim, G, max_query_len, num_seqs, partition_tokens) &&
                       aligned(q, 16) && aligned(out, 16) && scale > 0.0f;
  if (!prefill && pl.num_streams > 1 && (!workspace || workspace_bytes < pl.workspace || !aligned(workspace, 256)))
    return fail(PKV_ERR_INVALID_ARG, "workspace of %zu bytes (256-byte aligned) required, got %zu", pl.workspace,
                workspace ? workspace_bytes : 0);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (g_validate.load()) {
    std::vector<int32_t> ctx, bt, qsl;
    rc = fetch(&ctx, context_lens, static_cast<size_t>(num_seqs), st);
    if (rc == PKV_OK) rc = fetch(&bt, block_tables, static_cast<size_t>(num_seqs) * max_blocks_per_seq, st);
    if (rc == PKV_OK && mq) rc = fetch(&qsl, query_start_loc, static_cast<size_t>(num_seqs) + 1, st);
    if (rc != PKV_OK) return rc;
    for (int s = 0; s < num_seqs; ++s) {
      if (ctx[s] < 0 || ctx[s] > max_context_len)
        return fail(PKV_ERR_INVALID_ARG, "context_lens[%d] = %d outside [0, %d]", s, ctx[s], max_context_len);
      for (int j = 0; j < (ctx[s] + 15) / 16; ++j) {
        const int32_t b = bt[static_cast<size_t>(s) * max_blocks_per_seq + j];
        if (b < 0 || b >= num_blocks) return fail(PKV_ERR_INVALID_ARG, "block_tables[%d][%d] = %d out of range", s, j, b);
      }
    }
    if (mq) {
      if (qsl[0] != 0 || qsl[num_seqs] != num_q_tokens)
        return fail(PKV_ERR_INVALID_ARG, "query_start_loc must run from 0 to num_q_tokens (%d)", num_q_tokens);
      for (int s = 0; s < num_seqs; ++s) {
        const int n = qsl[s + 1] - qsl[s];
        if (n < 0 || n > max_query_len || n > ctx[s])
          return fail(PKV_ERR_INVALID_ARG, "sequence %d has %d new tokens (max_query_len %d, context %d)", s, n,
                      max_query_len, ctx[s]);
      }
    }
  }
  CUtensorMap km, vm;
  const long long rows = static_cast<long long>(num_blocks) * num_kv_heads * 16;
  rc = make_cache_map(&km, k_cache, row_bytes(cache_dtype, head_dim), elt_size(cache_dtype), rows);
  if (rc == PKV_OK) rc = make_cache_map(&vm, v_cache, row_bytes(cache_dtype, head_dim), elt_size(cache_dtype), rows);
  if (rc != PKV_OK) return rc;

  if (prefill) {
    pkv::PrefillParams pp{};
    pp.out = out;
    pp.q = q;
    pp.block_tables = block_tables;
    pp.context_lens = context_lens;
    pp.query_start_loc = query_start_loc;
    pp.num_seqs = num_seqs;
    pp.num_q_tokens = num_q_tokens;
    pp.max_query_len = max_query_len;
    pp.num_q_heads = num_q_heads;
    pp.num_kv_heads = num_kv_heads;
    pp.group = G;
    pp.max_blocks_per_seq = max_blocks_per_seq;
    pp.num_blocks = num_blocks;
    pp.max_context_len = max_context_len;
    pp.window = sliding_window;
    pp.max_tiles = prefill_tiles(max_query_len, G);
    pp.oob_row = static_cast<int>(rows);
    pp.qk_scale_log2 = scale * 1.4426950408889634f;
    const bool bf = cache_dtype == PKV_BF16;
    if (head_dim == 128)
      rc = bf ? launch_prefill<128, true>(km, vm, pp, st) : launch_prefill<128, false>(km, vm, pp, st);
    else
      rc = bf ? launch_prefill<64, true>(km, vm, pp, st) : launch_prefill<64, false>(km, vm, pp, st);
    if (rc != PKV_OK) return rc;
    return ok();
  }

  pkv::DecodeParams p{};
  p.out = out;
  p.q = q;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.k_zero = k_zero;
  p.v_zero = v_zero;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.query_start_loc = mq ? query_start_loc : nullptr;
  if (pl.num_streams > 1) {
    auto* ws = static_cast<uint8_t*>(workspace);
    rc = prepare_counters(workspace, pl.counter_bytes, st);
    if (rc != PKV_OK) return rc;
    p.counters = reinterpret_cast<unsigned long long*>(ws);
    p.slots = reinterpret_cast<float*>(ws + pl.counter_bytes);
  }
  p.num_seqs = num_seqs;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.group = G;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.num_blocks = num_blocks;
  p.max_context_len = max_context_len;
  p.num_streams = pl.num_streams;
  p.ring_warps = pl.warps;
  p.slot_floats = pl.slot_floats;
  p.tile_cols = pl.tile_cols;
  p.max_tiles = pl.max_tiles;
  p.num_q_tokens = mq ? num_q_tokens : num_seqs;
  p.max_query_len = mq ? max_query_len : 1;
  p.window = sliding_window;
  p.epoch = next_epoch();
  p.qk_scale_log2 = scale * 1.4426950408889634f;
  const bool q_bf16 = q_dtype == PKV_BF16;
  if (mq)
    rc = head_dim == 128 ? dispatch_ct<128, true>(cache_dtype, km, vm, p, q_bf16, st)
                         : dispatch_ct<64, true>(cache_dtype, km, vm, p, q_bf16, st);
  else
    rc = head_dim == 128 ? dispatch_ct<128, false>(cache_dtype, km, vm, p, q_bf16, st)
                         : dispatch_ct<64, false>(cache_dtype, km, vm, p, q_bf16, st);
  if (rc != PKV_OK) return rc;
  return ok();
}

}  // namespace

extern "C" {

int pkv_paged_attention_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                               const float* k_scale, const float* v_scale, const uint8_t* k_zero,
                               const uint8_t* v_zero, const int32_t* block_tables, const int32_t* context_lens,
                               int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                               int num_blocks, int max_blocks_per_seq, int max_context_len, float scale,
                               int sliding_window, int q_dtype, int cache_dtype, int partition_tokens,
                               void* workspace, size_t workspace_bytes, void* stream) {
  return attention_call(out, q, k_cache, v_cache, k_scale, v_scale, k_zero, v_zero, block_tables, context_lens,
                        nullptr, num_seqs, 1, false, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                        num_blocks, max_blocks_per_seq, max_context_len, scale, sliding_window, q_dtype,
                        cache_dtype, partition_tokens, workspace, workspace_bytes, stream);
}

int pkv_multi_query_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int max_context_len,
                         int max_query_len, int cache_dtype, int partition_tokens, int* num_streams_out,
                         int* partition_tokens_out, size_t* workspace_bytes_out) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_context_len < 0 || max_query_len < 0)
    return fail(PKV_ERR_INVALID_ARG, "bad sizes");
  if (num_q_heads % num_kv_heads != 0) return fail(PKV_ERR_INVALID_ARG, "num_q_heads %% num_kv_heads != 0");
  if (head_dim != 64 && head_dim != 128) return fail(PKV_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (!is16(cache_dtype) && !isq(cache_dtype)) return fail(PKV_ERR_UNSUPPORTED, "cache dtype %d", cache_dtype);
  Plan pl{};
  int rc = make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, cache_dtype, partition_tokens,
                     &pl, std::max(max_query_len, 1));
  if (rc != PKV_OK) return rc;
  const int G = num_q_heads / num_kv_heads;
  if (prefill_eligible(cache_dtype, head_dim, G, max_query_len, num_seqs, partition_tokens)) {
    // one CTA per (sequence, KV head, two 128-row tiles), each over all its
    // keys; the workspace of the other path is still reported (it is used
    // when q or out is not 16-byte aligned, or the scale is not positive)
    if (num_streams_out) *num_streams_out = num_seqs * num_kv_heads * ((prefill_tiles(max_query_len, G) + 1) / 2);
    if (partition_tokens_out) *partition_tokens_out = (max_context_len + 15) / 16 * 16;
  } else {
    if (num_streams_out) *num_streams_out = pl.num_streams;
    if (partition_tokens_out) *partition_tokens_out = pl.stream_tokens;
  }
  if (workspace_bytes_out) *workspace_bytes_out = pl.workspace;
  return ok();
}

int pkv_paged_attention_multi_query(void* out, const void* q, const void* k_cache, const void* v_cache,
                                    const float* k_scale, const float* v_scale, const uint8_t* k_zero,
                                    const uint8_t* v_zero, const int32_t* block_tables, const int32_t* context_lens,
                                    const int32_t* query_start_loc, int num_seqs, int num_q_tokens,
                                    int max_query_len, int num_q_heads, int num_kv_heads, int head_dim,
                                    int block_size, int num_blocks, int max_blocks_per_seq, int max_context_len,
                                    float scale, int sliding_window, int q_dtype, int cache_dtype,
                                    int partition_tokens, void* workspace, size_t workspace_bytes, void* stream) {
  return attention_call(out, q, k_cache, v_cache, k_scale, v_scale, k_zero, v_zero, block_tables, context_lens,
                        query_start_loc, num_q_tokens, max_query_len, true, num_seqs, num_q_heads, num_kv_heads,
                        head_dim, block_size, num_blocks, max_blocks_per_seq, max_context_len, scale,
                        sliding_window, q_dtype, cache_dtype, partition_tokens, workspace, workspace_bytes, stream);
}

int pkv_copy_blocks(void* k_cache, void* v_cache, float* k_scale, float* v_scale, uint8_t* k_zero, uint8_t* v_zero,
                    const int32_t* src_dst_pairs,
                    int num_pairs, int num_kv_heads, int head_dim, int block_size, int num_blocks, int cache_dtype,
                    void* stream) {
  if (num_pairs < 0 || num_kv_heads <= 0 || num_blocks <= 0) return fail(PKV_ERR_INVALID_ARG, "bad sizes");
  if (block_size != 16) return fail(PKV_ERR_UNSUPPORTED, "block_size must be 16 (got %d)", block_size);
  if (head_dim != 64 && head_dim != 128) return fail(PKV_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (!is16(cache_dtype) && !isq(cache_dtype)) return fail(PKV_ERR_UNSUPPORTED, "cache dtype %d", cache_dtype);
  if (num_pairs == 0) return ok();
  if (!k_cache || !v_cache || !src_dst_pairs) return fail(PKV_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16)) return fail(PKV_ERR_INVALID_ARG, "caches must be 16-byte aligned");
  const bool q8 = isq(cache_dtype);
  if (q8 && (!k_scale || !v_scale || !aligned(k_scale, 16) || !aligned(v_scale, 16)))
    return fail(PKV_ERR_INVALID_ARG, "quantised caches need 16-byte aligned k_scale and v_scale");
  const bool zp = has_zero(cache_dtype);
  if (zp && (!k_zero || !v_zero || !aligned(k_zero, 16) || !aligned(v_zero, 16)))
    return fail(PKV_ERR_INVALID_ARG, "PKV_U8ASYM caches need 16-byte aligned k_zero and v_zero");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (g_validate.load()) {
    std::vector<int32_t> pr;
    int rc = fetch(&pr, src_dst_pairs, static_cast<size_t>(num_pairs) * 2, st);
    if (rc != PKV_OK) return rc;
    std::unordered_set<int32_t> dsts, srcs;
    for (int i = 0; i < num_pairs; ++i) {
      const int32_t a = pr[2 * i], b = pr[2 * i + 1];
      if (a < 0 || a >= num_blocks || b < 0 || b >= num_blocks)
        return fail(PKV_ERR_INVALID_ARG, "pair %d (%d, %d) out of range", i, a, b);
      if (!dsts.insert(b).second) return fail(PKV_ERR_INVALID_ARG, "destination %d appears twice", b);
      srcs.insert(a);
    }
    for (int32_t b : dsts)
      if (srcs.count(b)) return fail(PKV_ERR_INVALID_ARG, "block %d is both a source and a destination", b);
  }
  const long long words = static_cast<long long>(num_kv_heads) * 16 * row_bytes(cache_dtype, head_dim) / 16;
  const int swords = q8 ? num_kv_heads * 4 : 0;
  const int zwords = zp ? num_kv_heads : 0;
  const int grid = std::min(num_pairs, 16 * sm_count());
  pkv::copy_blocks_kernel<<<grid, 256, 0, st>>>(static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
                                                reinterpret_cast<uint4*>(k_scale), reinterpret_cast<uint4*>(v_scale),
                                                reinterpret_cast<uint4*>(k_zero), reinterpret_cast<uint4*>(v_zero),
                                                src_dst_pairs, num_pairs, num_blocks, words, swords, zwords);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "copy_blocks launch");
  return ok();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free decode.  Some callers cannot allocate device memory at all:
// a plugin whose host framework owns every device allocation and hands it
// only its input and output buffers, or a latency-critical loop where a
// cudaMalloc could synchronise the device.  For them the split-KV partials
// live in one library-owned device array instead of a caller workspace.
// The array is file-scope, so every GPU that loads this library holds it
// (PKV_NOALLOC_SCRATCH_BYTES) until the process exits.  Host code must not
// use the array's name as a device address: it is a host-side stand-in, so
// its device address is fetched once per device with cudaGetSymbolAddress.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(PKV_NOALLOC_SCRATCH_BYTES);

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Unique ID of the calling thread's current CUDA context, or 0 when there is
// none or the driver cannot say.  A device reset ends the primary context
// (and the module holding the array); the next context has a new ID.
unsigned long long current_context_id() {
  static auto get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(driver_entry("cuCtxGetCurrent", 4000));
  static auto get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(driver_entry("cuCtxGetId", 12000));
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  return get_id(ctx, &id) == CUDA_SUCCESS ? id : 0;
}

// Device address of g_noalloc_scratch on the current device, looked up on
// the first call for that device (with that device current) and cached per
// (device, context): after a device reset the address is looked up again.
int noalloc_scratch_address(void** out) {
  static std::mutex mu;
  static std::vector<std::pair<unsigned long long, void*>> by_device;  // (context ID, address)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lk(mu);
  if (ctx != 0 && static_cast<size_t>(dev) < by_device.size() && by_device[dev].first == ctx &&
      by_device[dev].second != nullptr) {
    *out = by_device[dev].second;
    return PKV_OK;
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
  if (p == nullptr) return fail(PKV_ERR_CUDA, "cudaGetSymbolAddress returned NULL for the no-alloc scratch");
  if (by_device.size() <= static_cast<size_t>(dev)) by_device.resize(dev + 1, {0ull, nullptr});
  // with no context ID to check against, the address is looked up on every call
  by_device[dev] = {ctx, ctx != 0 ? p : nullptr};
  *out = p;
  return PKV_OK;
}

}  // namespace

extern "C" int pkv_paged_attention_decode_noalloc(void* out, const void* q, const void* k_cache,
                                                  const void* v_cache, const float* k_scale, const float* v_scale,
                                                  const uint8_t* k_zero, const uint8_t* v_zero,
                                                  const int32_t* block_tables, const int32_t* context_lens,
                                                  int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                                  int block_size, int num_blocks, int max_blocks_per_seq,
                                                  int max_context_len, float scale, int sliding_window,
                                                  int q_dtype, int cache_dtype, int partition_tokens, void* stream) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_context_len < 0)
    return fail(PKV_ERR_INVALID_ARG, "bad sizes");
  if (head_dim != 64 && head_dim != 128) return fail(PKV_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", head_dim);
  Plan pl{};
  int rc = make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, cache_dtype, partition_tokens, &pl);
  if (rc != PKV_OK) return rc;
  int pt = partition_tokens;
  if (pt == 0 && pl.num_streams > 1 && pl.workspace > kNoAllocScratchBytes &&
      pl.counter_bytes < kNoAllocScratchBytes) {
    // The automatic plan needs more partials than the array holds: the same
    // work in fewer, longer warp streams, as many as fit.
    const long long per_stream = 2LL * pl.slot_floats * 4;
    const long long fit = static_cast<long long>(kNoAllocScratchBytes - pl.counter_bytes) / per_stream;
    const long long blocks = static_cast<long long>(std::max(num_seqs, 1)) * num_kv_heads *
                             std::max(1, (max_context_len + 15) / 16);
    if (fit >= 1) {
      const long long per = (blocks + fit - 1) / fit;  // blocks per stream
      if (per * 16 <= (1LL << 30)) {
        pt = static_cast<int>(per * 16);
        rc = make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, cache_dtype, pt, &pl);
        if (rc != PKV_OK) return rc;
      }
    }
  }
  const bool needs_scratch = pl.num_streams > 1;
  if (needs_scratch && pl.workspace > kNoAllocScratchBytes)
    return fail(PKV_ERR_INVALID_ARG,
                "this decode needs %zu bytes of split-KV scratch but the built-in array holds %zu "
                "(PKV_NOALLOC_SCRATCH_BYTES); use fewer sequences per call, a larger partition_tokens, "
                "or pkv_paged_attention_decode with a caller workspace",
                pl.workspace, kNoAllocScratchBytes);
  void* scratch = nullptr;
  if (needs_scratch) {
    rc = noalloc_scratch_address(&scratch);
    if (rc != PKV_OK) return rc;
  }
  return pkv_paged_attention_decode(out, q, k_cache, v_cache, k_scale, v_scale, k_zero, v_zero, block_tables,
                                    context_lens,
                                    num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                                    max_blocks_per_seq, max_context_len, scale, sliding_window, q_dtype, cache_dtype,
                                    pt, scratch, needs_scratch ? kNoAllocScratchBytes : 0, stream);
}
