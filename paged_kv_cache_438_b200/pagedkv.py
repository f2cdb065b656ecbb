"""ctypes binding of libpagedkv.so (C ABI declared in include/pagedkv.h).

Argument marshalling only: every computation runs in the library's CUDA
kernels (or, for the block allocator, its C++ code).  torch provides device
memory and streams.  If the shared library is missing, every call raises.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedkv.so")

PKV_OK = 0
PKV_ERR_INVALID_ARG = -1
PKV_ERR_UNSUPPORTED = -2
PKV_ERR_NO_BLOCKS = -3
PKV_ERR_CUDA = -4
PKV_ERR_NOT_FOUND = -5
PKV_ERR_EXISTS = -6

PKV_F16, PKV_BF16, PKV_I8, PKV_FP8E4M3, PKV_U8ASYM, PKV_I4, PKV_FP4E2M1 = 0, 1, 2, 3, 4, 5, 6
QUANTISED = (PKV_I8, PKV_FP8E4M3, PKV_U8ASYM, PKV_I4, PKV_FP4E2M1)
FOUR_BIT = (PKV_I4, PKV_FP4E2M1)
KV_FORMATS = {"int8": PKV_I8, "fp8": PKV_FP8E4M3, "u8asym": PKV_U8ASYM, "int4": PKV_I4, "fp4": PKV_FP4E2M1}

DEV_BAD_SLOT, DEV_BAD_BLOCK, DEV_BAD_CONTEXT, DEV_TIMEOUT, DEV_BAD_PAIR = 1, 2, 4, 8, 16

EXPORTS = [
    "pkv_last_error", "pkv_version", "pkv_kv_cache_write", "pkv_decode_plan", "pkv_decode_workspace_size",
    "pkv_paged_attention_decode", "pkv_paged_attention_decode_noalloc", "pkv_multi_query_plan",
    "pkv_paged_attention_multi_query", "pkv_copy_blocks", "pkv_device_status", "pkv_set_validation",
    "pkv_alloc_create", "pkv_alloc_destroy", "pkv_seq_add", "pkv_seq_fork", "pkv_seq_append",
    "pkv_batch_append", "pkv_batch_tables", "pkv_seq_free", "pkv_seq_block_table", "pkv_seq_len",
    "pkv_block_refcount", "pkv_alloc_stats", "pkv_prefix_key", "pkv_prefix_cache_insert", "pkv_prefix_cache_match",
    "pkv_seq_add_cached", "pkv_prefix_cache_evict", "pkv_prefix_cache_stats",
]


class PagedKVError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"libpagedkv error {code}: {msg}")
        self.code = code


class NoBlocksError(PagedKVError):
    pass


_lib_handle = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_F = ctypes.c_float


def _signatures(lib):
    sig = {
        "pkv_last_error": ([], ctypes.c_char_p),
        "pkv_version": ([], _I),
        "pkv_kv_cache_write": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P], _I),
        "pkv_decode_plan": ([_I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I),
                             ctypes.POINTER(_SZ)], _I),
        "pkv_decode_workspace_size": ([_I, _I, _I, _I, _I, _I, ctypes.POINTER(_SZ)], _I),
        "pkv_paged_attention_decode": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I,
                                        _F, _I, _I, _I, _I, _P, _SZ, _P], _I),
        "pkv_paged_attention_decode_noalloc": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                                _I, _I, _F, _I, _I, _I, _I, _P], _I),
        "pkv_multi_query_plan": ([_I, _I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I),
                                  ctypes.POINTER(_SZ)], _I),
        "pkv_paged_attention_multi_query": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                             _I, _I, _I, _I, _F, _I, _I, _I, _I, _P, _SZ, _P], _I),
        "pkv_copy_blocks": ([_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P], _I),
        "pkv_device_status": ([ctypes.POINTER(ctypes.c_uint), _I], _I),
        "pkv_set_validation": ([_I], _I),
        "pkv_alloc_create": ([_I, _I, _P, ctypes.POINTER(_P)], _I),
        "pkv_alloc_destroy": ([_P], _I),
        "pkv_seq_add": ([_P, _I64], _I),
        "pkv_seq_fork": ([_P, _I64, _I64, _I], _I),
        "pkv_seq_append": ([_P, _I64, _I, _P, _P, _I, ctypes.POINTER(_I)], _I),
        "pkv_batch_append": ([_P, _P, _I, _P, _P, _I, ctypes.POINTER(_I)], _I),
        "pkv_batch_tables": ([_P, _P, _I, _P, _I, _P], _I),
        "pkv_seq_free": ([_P, _I64], _I),
        "pkv_seq_block_table": ([_P, _I64, _P, _I, ctypes.POINTER(_I)], _I),
        "pkv_seq_len": ([_P, _I64, ctypes.POINTER(_I)], _I),
        "pkv_block_refcount": ([_P, ctypes.c_int32, ctypes.POINTER(_I)], _I),
        "pkv_alloc_stats": ([_P, ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(_I)], _I),
        "pkv_prefix_key": ([_P, _I, _P], _I),
        "pkv_prefix_cache_insert": ([_P, _I64, _P, _I, ctypes.POINTER(_I)], _I),
        "pkv_prefix_cache_match": ([_P, _P, _I, ctypes.POINTER(_I), _P], _I),
        "pkv_seq_add_cached": ([_P, _I64, _P, _I, ctypes.POINTER(_I)], _I),
        "pkv_prefix_cache_evict": ([_P, _I, ctypes.POINTER(_I)], _I),
        "pkv_prefix_cache_stats": ([_P, ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(_I64),
                                    ctypes.POINTER(_I64), ctypes.POINTER(_I64)], _I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res


def lib():
    """The loaded library; raises if libpagedkv.so has not been built."""
    global _lib_handle
    if _lib_handle is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_438_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        _signatures(h)
        _lib_handle = h
    return _lib_handle


def _check(rc):
    if rc != PKV_OK:
        msg = lib().pkv_last_error().decode(errors="replace")
        if rc == PKV_ERR_NO_BLOCKS:
            raise NoBlocksError(rc, msg)
        raise PagedKVError(rc, msg)


# ------------------------------------------------------------------ helpers --

def dtype_code(t):
    d = t.dtype if isinstance(t, torch.Tensor) else t
    if d == torch.float16:
        return PKV_F16
    if d == torch.bfloat16:
        return PKV_BF16
    if d == torch.int8:
        return PKV_I8
    if d in (torch.uint8, torch.float8_e4m3fn):
        return PKV_FP8E4M3
    raise TypeError(f"unsupported dtype {d}")


def cache_code(cache, k_zero=None, kv_format=None):
    """Cache format code: ``kv_format`` when given ("int8", "fp8", "u8asym",
    "int4", "fp4"; the 4-bit caches are uint8 [NB, Hkv, 16, D / 2]), else the
    asymmetric uint8 format when zero points are given, else the cache
    tensor's dtype (uint8 alone means FP8-e4m3)."""
    if kv_format is not None:
        ct = KV_FORMATS[kv_format]
        if ct != PKV_I8 and cache.dtype != torch.uint8:
            raise TypeError(f"a {kv_format} cache must be uint8")
        return ct
    if k_zero is not None:
        if cache.dtype != torch.uint8:
            raise TypeError("a cache with zero points must be uint8")
        return PKV_U8ASYM
    return dtype_code(cache)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, device=None, dtype=None, contiguous=True):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# ---------------------------------------------------------------- kernels ----

def version():
    return lib().pkv_version()


def set_validation(on):
    _check(lib().pkv_set_validation(1 if on else 0))


def device_status(clear=True):
    v = ctypes.c_uint(0)
    _check(lib().pkv_device_status(ctypes.byref(v), 1 if clear else 0))
    return v.value


def _need_quant(ct, dev, k_scale, v_scale, k_zero, v_zero):
    if ct in QUANTISED:
        _need(k_scale, "k_scale", device=dev, dtype=torch.float32)
        _need(v_scale, "v_scale", device=dev, dtype=torch.float32)
    if ct == PKV_U8ASYM:
        _need(k_zero, "k_zero", device=dev, dtype=torch.uint8)
        _need(v_zero, "v_zero", device=dev, dtype=torch.uint8)


def _head_dim_of_cache(cache, ct):
    return cache.shape[3] * (2 if ct in FOUR_BIT else 1)


def kv_cache_write(k, v, k_cache, v_cache, slot_mapping, k_scale=None, v_scale=None, stream=None,
                   k_zero=None, v_zero=None, kv_format=None):
    """Writes rows k, v [T, Hkv, D] into the paged caches at slot_mapping [T]
    (int64, -1 skips).  Quantised caches (int8 / float8_e4m3fn, or uint8 with
    zero points) need the fp32 scale arrays [NB, Hkv, 16]; the asymmetric
    uint8 format also the uint8 zero-point arrays k_zero, v_zero [NB, Hkv, 16]."""
    for n, t in (("k", k), ("v", v), ("k_cache", k_cache), ("v_cache", v_cache)):
        _need(t, n, device=k.device)
    _need(slot_mapping, "slot_mapping", device=k.device, dtype=torch.int64)
    if k.dim() != 3 or v.shape != k.shape or k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("k, v must be [T, Hkv, D]; caches [NB, Hkv, 16, D]")
    T, hkv, d = k.shape
    nb = k_cache.shape[0]
    ct = cache_code(k_cache, k_zero, kv_format)
    if k_cache.shape[1] != hkv or _head_dim_of_cache(k_cache, ct) != d or slot_mapping.numel() != T:
        raise ValueError("shape mismatch between k and the caches")
    _need_quant(ct, k.device, k_scale, v_scale, k_zero, v_zero)
    _check(lib().pkv_kv_cache_write(_ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale),
                                    _ptr(k_zero), _ptr(v_zero), _ptr(slot_mapping), T, hkv, d, k_cache.shape[2], nb,
                                    dtype_code(k), ct, _stream(stream)))


def decode_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, cache_dtype, partition_tokens=0):
    """(num_streams, tokens_per_stream_bound, workspace_bytes) the decode call
    uses: the warps sharing the (sequence, head, block) work list, the most
    tokens one of them processes, and the workspace it needs."""
    npart, ptok, ws = _I(0), _I(0), _SZ(0)
    ct = cache_dtype if isinstance(cache_dtype, int) else dtype_code(cache_dtype)
    _check(lib().pkv_decode_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, ct,
                                 partition_tokens, ctypes.byref(npart), ctypes.byref(ptok), ctypes.byref(ws)))
    return npart.value, ptok.value, ws.value


_WORKSPACES = {}


def _cached_workspace(device, stream, nbytes):
    """A decode workspace for (device, stream), grown on demand (the library
    prepares its counter area itself).  One per stream, so calls on different
    streams never share one."""
    s = torch.cuda.current_stream(device) if stream is None else stream
    key = (device.index, s.cuda_stream)
    ws = _WORKSPACES.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
        _WORKSPACES[key] = ws
    return ws


def new_workspace(device, nbytes):
    """A decode workspace of at least ``nbytes`` (see decode_plan); the library
    clears its counter area itself, so the zero fill here is only tidiness."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def paged_attention_decode(q, k_cache, v_cache, block_tables, context_lens, scale, k_scale=None, v_scale=None,
                           max_context_len=None, out=None, workspace=None, partition_tokens=0, stream=None,
                           k_zero=None, v_zero=None, sliding_window=0, kv_format=None):
    """out[s, i] = softmax(scale * q[s, i] . K_s) V_s through block tables.

    q [B, Hq, D] fp16/bf16; caches [NB, Hkv, 16, D]; block_tables [B, MB]
    int32; context_lens [B] int32.  ``max_context_len`` is a host-side upper
    bound on context_lens (if None it is read from the device, which
    synchronises).  ``workspace`` (uint8, from ``new_workspace``) serves one
    call at a time and is written by nothing else between calls; when None
    a cached per-stream workspace is used.  A uint8 cache with ``k_zero`` /
    ``v_zero`` is the asymmetric format, read as (code - zero) * scale.
    ``sliding_window`` W > 0 limits each query to its W most recent keys.
    Returns ``out`` [B, Hq, D] in q's dtype."""
    dev = q.device
    for n, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _need(t, n, device=dev)
    _need(block_tables, "block_tables", device=dev, dtype=torch.int32)
    _need(context_lens, "context_lens", device=dev, dtype=torch.int32)
    if q.dim() != 3 or k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("q must be [B, Hq, D]; caches [NB, Hkv, 16, D]")
    B, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    ct = cache_code(k_cache, k_zero, kv_format)
    if _head_dim_of_cache(k_cache, ct) != d or block_tables.dim() != 2 or block_tables.shape[0] != B or \
            context_lens.numel() != B:
        raise ValueError("shape mismatch")
    _need_quant(ct, dev, k_scale, v_scale, k_zero, v_zero)
    if max_context_len is None:
        max_context_len = int(context_lens.max().item()) if B else 0
    if out is None:
        out = torch.empty_like(q)
    else:
        _need(out, "out", device=dev, dtype=q.dtype)
    nstreams, _, ws_bytes = decode_plan(B, hq, hkv, d, max_context_len, ct, partition_tokens)
    if nstreams > 1 and workspace is None:
        workspace = _cached_workspace(dev, stream, ws_bytes)
    ws_len = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().pkv_paged_attention_decode(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), _ptr(k_zero), _ptr(v_zero),
        _ptr(block_tables), _ptr(context_lens), B, hq, hkv, d, bs, nb, block_tables.shape[1], max_context_len,
        float(scale), int(sliding_window), dtype_code(q), ct, partition_tokens, _ptr(workspace), ws_len,
        _stream(stream)))
    return out


def multi_query_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, max_query_len, cache_dtype,
                     partition_tokens=0):
    """(num_streams, tokens_per_stream_bound, workspace_bytes) of a
    multi-query call (see decode_plan)."""
    nst, ptok, ws = _I(0), _I(0), _SZ(0)
    ct = cache_dtype if isinstance(cache_dtype, int) else dtype_code(cache_dtype)
    _check(lib().pkv_multi_query_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                      max_query_len, ct, partition_tokens, ctypes.byref(nst), ctypes.byref(ptok),
                                      ctypes.byref(ws)))
    return nst.value, ptok.value, ws.value


def paged_attention_multi_query(q, k_cache, v_cache, block_tables, context_lens, query_start_loc, scale,
                                max_query_len, max_context_len, k_scale=None, v_scale=None, k_zero=None,
                                v_zero=None, out=None, workspace=None, partition_tokens=0, stream=None,
                                sliding_window=0, kv_format=None):
    """Several new tokens per sequence (chunked prefill, speculative verify):
    q [T, Hq, D] packed by sequence with query_start_loc [B + 1] int32; the
    n_s new tokens of sequence s are the last n_s of its context_lens[s]
    tokens and attend causally.  max_query_len and max_context_len are
    host-side bounds.  Returns out [T, Hq, D] in q's dtype."""
    dev = q.device
    for n, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _need(t, n, device=dev)
    _need(block_tables, "block_tables", device=dev, dtype=torch.int32)
    _need(context_lens, "context_lens", device=dev, dtype=torch.int32)
    _need(query_start_loc, "query_start_loc", device=dev, dtype=torch.int32)
    if q.dim() != 3 or k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("q must be [T, Hq, D]; caches [NB, Hkv, 16, D]")
    T, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    B = context_lens.numel()
    ct = cache_code(k_cache, k_zero, kv_format)
    if _head_dim_of_cache(k_cache, ct) != d or block_tables.dim() != 2 or block_tables.shape[0] != B or \
            query_start_loc.numel() != B + 1:
        raise ValueError("shape mismatch")
    _need_quant(ct, dev, k_scale, v_scale, k_zero, v_zero)
    if out is None:
        out = torch.empty_like(q)
    else:
        _need(out, "out", device=dev, dtype=q.dtype)
    nstreams, _, ws_bytes = multi_query_plan(B, hq, hkv, d, max_context_len, max_query_len, ct, partition_tokens)
    if nstreams > 1 and workspace is None:
        workspace = _cached_workspace(dev, stream, ws_bytes)
    ws_len = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().pkv_paged_attention_multi_query(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), _ptr(k_zero), _ptr(v_zero),
        _ptr(block_tables), _ptr(context_lens), _ptr(query_start_loc), B, T, int(max_query_len), hq, hkv, d, bs, nb,
        block_tables.shape[1], int(max_context_len), float(scale), int(sliding_window), dtype_code(q), ct,
        partition_tokens, _ptr(workspace), ws_len, _stream(stream)))
    return out


NOALLOC_SCRATCH_BYTES = 16 << 20


def paged_attention_decode_noalloc(q, k_cache, v_cache, block_tables, context_lens, scale, max_context_len,
                                   out, k_scale=None, v_scale=None, partition_tokens=0, stream=None,
                                   k_zero=None, v_zero=None, sliding_window=0, kv_format=None):
    """paged_attention_decode for callers that cannot allocate device memory
    (for instance a plugin whose host framework owns every allocation and
    hands it only input and output buffers): ``out`` must be given, no
    workspace is taken, and the split-KV partials use the library's own
    device array of NOALLOC_SCRATCH_BYTES.  With partition_tokens 0 the work
    is cut into fewer, longer warp streams when the automatic plan needs more
    scratch; work that needs more even then, or whose explicit partition
    does, is rejected with an error.  Calls that overlap on the GPU share that array
    and race; keep them on one stream.  The first call on a device looks up
    the array's address, so make it before any stream capture."""
    dev = q.device
    for n, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("out", out)):
        _need(t, n, device=dev)
    _need(block_tables, "block_tables", device=dev, dtype=torch.int32)
    _need(context_lens, "context_lens", device=dev, dtype=torch.int32)
    B, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    ct = cache_code(k_cache, k_zero, kv_format)
    _need_quant(ct, dev, k_scale, v_scale, k_zero, v_zero)
    _check(lib().pkv_paged_attention_decode_noalloc(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), _ptr(k_zero), _ptr(v_zero),
        _ptr(block_tables), _ptr(context_lens), B, hq, hkv, d, bs, nb, block_tables.shape[1], int(max_context_len),
        float(scale), int(sliding_window), dtype_code(q), ct, partition_tokens, _stream(stream)))
    return out


def copy_blocks(k_cache, v_cache, src_dst_pairs, k_scale=None, v_scale=None, stream=None, k_zero=None,
                v_zero=None, kv_format=None):
    """Block dst := block src for every row (src, dst) of src_dst_pairs
    [N, 2] int32 (device), for K, V and the scales (and zero points) of
    quantised caches."""
    dev = k_cache.device
    _need(k_cache, "k_cache", device=dev)
    _need(v_cache, "v_cache", device=dev)
    _need(src_dst_pairs, "src_dst_pairs", device=dev, dtype=torch.int32)
    nb, hkv, bs, _ = k_cache.shape
    ct = cache_code(k_cache, k_zero, kv_format)
    d = _head_dim_of_cache(k_cache, ct)
    _need_quant(ct, dev, k_scale, v_scale, k_zero, v_zero)
    n = src_dst_pairs.numel() // 2
    _check(lib().pkv_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), _ptr(k_zero),
                                 _ptr(v_zero), _ptr(src_dst_pairs), n, hkv, d, bs, nb, ct, _stream(stream)))


# --------------------------------------------------------- block allocator --

class BlockAllocator:
    """Host block manager (C++): LIFO free list, reference counts, fork and
    copy-on-write, slot and block-table production."""

    def __init__(self, num_blocks, block_size=16, initial_free_order=None):
        self._h = ctypes.c_void_p()
        order = None
        if initial_free_order is not None:
            self._order = torch.as_tensor(initial_free_order, dtype=torch.int32).contiguous()
            order = ctypes.c_void_p(self._order.data_ptr())
        _check(lib().pkv_alloc_create(num_blocks, block_size, order, ctypes.byref(self._h)))
        self.num_blocks = num_blocks
        self.block_size = block_size

    def close(self):
        if self._h:
            lib().pkv_alloc_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add(self, seq_id):
        _check(lib().pkv_seq_add(self._h, seq_id))

    def fork(self, parent, child, prefix_len=-1):
        _check(lib().pkv_seq_fork(self._h, parent, child, prefix_len))

    def append(self, seq_id, n_tokens):
        """Returns (slots int64 tensor [n_tokens], cow pairs int32 tensor [k, 2])."""
        slots = torch.empty(n_tokens, dtype=torch.int64)
        pairs = torch.empty((max(n_tokens, 1), 2), dtype=torch.int32)
        npairs = _I(0)
        _check(lib().pkv_seq_append(self._h, seq_id, n_tokens, _ptr(slots), _ptr(pairs), pairs.shape[0],
                                    ctypes.byref(npairs)))
        return slots, pairs[:npairs.value].clone()

    def batch_append(self, seq_ids, slots_out=None, pairs_out=None):
        """One token for each sequence; returns (slots [n], cow pairs [k, 2]).
        ``slots_out`` (int64 [n]) and ``pairs_out`` (int32 [>= n, 2]) may be
        given (e.g. pinned host buffers); the pairs returned are then a view
        of ``pairs_out``."""
        ids = seq_ids if isinstance(seq_ids, torch.Tensor) and seq_ids.dtype == torch.int64 \
            else torch.as_tensor(seq_ids, dtype=torch.int64)
        ids = ids.contiguous()
        n = ids.numel()
        slots = torch.empty(n, dtype=torch.int64) if slots_out is None else slots_out
        pairs = torch.empty((max(n, 1), 2), dtype=torch.int32) if pairs_out is None else pairs_out
        npairs = _I(0)
        _check(lib().pkv_batch_append(self._h, _ptr(ids), n, _ptr(slots), _ptr(pairs), pairs.shape[0],
                                      ctypes.byref(npairs)))
        if pairs_out is not None:
            return slots, pairs[:npairs.value]
        return slots, pairs[:npairs.value].clone()

    def batch_tables(self, seq_ids, max_blocks, out_tables=None, out_lens=None):
        ids = seq_ids if isinstance(seq_ids, torch.Tensor) and seq_ids.dtype == torch.int64 \
            else torch.as_tensor(seq_ids, dtype=torch.int64)
        ids = ids.contiguous()
        n = ids.numel()
        bt = torch.empty((n, max_blocks), dtype=torch.int32) if out_tables is None else out_tables
        cl = torch.empty(n, dtype=torch.int32) if out_lens is None else out_lens
        _check(lib().pkv_batch_tables(self._h, _ptr(ids), n, _ptr(bt), max_blocks, _ptr(cl)))
        return bt, cl

    def free(self, seq_id):
        _check(lib().pkv_seq_free(self._h, seq_id))

    def block_table(self, seq_id):
        n = _I(0)
        length = self.seq_len(seq_id)
        cap = (length + self.block_size - 1) // self.block_size
        out = torch.empty(max(cap, 1), dtype=torch.int32)
        _check(lib().pkv_seq_block_table(self._h, seq_id, _ptr(out), out.numel(), ctypes.byref(n)))
        return out[:n.value].tolist()

    def seq_len(self, seq_id):
        n = _I(0)
        _check(lib().pkv_seq_len(self._h, seq_id, ctypes.byref(n)))
        return n.value

    def refcount(self, block):
        rc = _I(0)
        _check(lib().pkv_block_refcount(self._h, block, ctypes.byref(rc)))
        return rc.value

    def stats(self):
        a, b, c = _I(0), _I(0), _I(0)
        _check(lib().pkv_alloc_stats(self._h, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)))
        return a.value, b.value, c.value

    # -- automatic prefix caching --------------------------------------------
    def prefix_insert(self, seq_id, token_ids):
        """Cache the sequence's full blocks under their token prefix; returns
        how many blocks became newly cached."""
        t = _tokens(token_ids)
        n = _I(0)
        _check(lib().pkv_prefix_cache_insert(self._h, seq_id, _ptr(t), t.numel(), ctypes.byref(n)))
        return n.value

    def prefix_match(self, token_ids):
        """(hit tokens, 16-byte key of the hit prefix)."""
        t = _tokens(token_ids)
        hit = _I(0)
        key = (ctypes.c_uint8 * 16)()
        _check(lib().pkv_prefix_cache_match(self._h, _ptr(t), t.numel(), ctypes.byref(hit), key))
        return hit.value, bytes(key)

    def add_cached(self, seq_id, token_ids):
        """New sequence starting with its longest cached prefix; returns the hit."""
        t = _tokens(token_ids)
        hit = _I(0)
        _check(lib().pkv_seq_add_cached(self._h, seq_id, _ptr(t), t.numel(), ctypes.byref(hit)))
        return hit.value

    def prefix_evict(self, max_cached_blocks):
        n = _I(0)
        _check(lib().pkv_prefix_cache_evict(self._h, max_cached_blocks, ctypes.byref(n)))
        return n.value

    def prefix_stats(self):
        """(cached blocks, evictable now, lookups, hits, evictions)."""
        a, b = _I(0), _I(0)
        c, d, e = _I64(0), _I64(0), _I64(0)
        _check(lib().pkv_prefix_cache_stats(self._h, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c),
                                            ctypes.byref(d), ctypes.byref(e)))
        return a.value, b.value, c.value, d.value, e.value


def _tokens(token_ids):
    t = token_ids if isinstance(token_ids, torch.Tensor) and token_ids.dtype == torch.int32 \
        else torch.as_tensor(list(token_ids), dtype=torch.int32)
    return t.contiguous()


def prefix_key(token_ids):
    """BLAKE2b-128 of token ids as little-endian int32 (the prefix cache key)."""
    t = _tokens(token_ids)
    key = (ctypes.c_uint8 * 16)()
    _check(lib().pkv_prefix_key(_ptr(t) if t.numel() else None, t.numel(), key))
    return bytes(key)
