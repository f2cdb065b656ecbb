"""Benchmark of the paged-KV decode step on B200.

One step = one decode iteration of one layer for the whole batch: the host
block allocator appends one token per sequence (slots, copy-on-write pairs,
block tables), copy_blocks runs for any CoW pairs, kv_cache_write stores the
new K/V rows, and paged_attention_decode (split-KV + reduce when planned)
attends each sequence's query heads over its whole cache.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

The default workload is the long-context one (Llama-3-70B-shaped, 64 q / 8 KV
heads, batch 32, 32768 tokens each, bf16).  ``value`` is the effective
KV-read bandwidth (KV bytes the step's attention must read / device time of
the step, inputs resident in HBM); ``e2e`` is the same metric measured
through the Python API with host buffers (allocator on the host, pinned H2D
of the step's inputs, D2H and a host read of the output, every step,
pipelined over two buffer sets).  At N = 1 the line also carries
``other_workloads``: the decode-call roofline of every other workload and
cache format (and the oracle timed on the quantised ones).  Multi-GPU runs
are independent replicas (one batch per rank, weak scaling, no data-path
collective); time is the max over ranks.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_438_b200 import inputs as I  # noqa: E402

METRIC = "paged decode attention: effective KV-read GB/s (% of HBM peak), seq-steps/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 * 2 ** 20

WORKLOAD_TEXT = {
    "llama3_8b": "Llama-3-8B-shaped decode layer: 32 q / 8 KV heads, head_dim 128, block 16, batch 64, "
                 "context U[512,4096], bf16, shuffled pool 1.1x need",
    "llama3_70b_32k": "Llama-3-70B-shaped long context: 64 q / 8 KV heads, head_dim 128, block 16, batch 32, "
                      "context 32768, bf16, split-KV",
    "prefix_shared": "prefix-shared: Llama-3-8B heads, 128 seqs sharing one 2048-token prefix + suffix U[64,1024], bf16",
    "quant_mha": "quantised KV: Llama-2-7B MHA 32/32 heads, head_dim 128, batch 256, context log-uniform[128,8192]",
    "tiny": "tiny: batch 4, 8 q / 2 KV heads, head_dim 64, context U[1,256], fp16",
    "spec_verify": "speculative verify: Llama-3-8B heads (32 q / 8 KV), head_dim 128, batch 64, context U[512,4096] "
                   "incl. 4 new tokens per sequence, causal among them, bf16",
    "chunked_prefill": "chunked prefill: Llama-3-8B heads (32 q / 8 KV), head_dim 128, batch 8, context "
                       "U[1024,4096] whose last 512 tokens are one new chunk, causal, bf16",
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama3_70b_32k", choices=sorted(I.WORKLOADS))
    ap.add_argument("--cache", default=None, choices=[None, "int8", "fp8", "u8asym", "int4", "fp4"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the decode-call records of the other workloads (N = 1 only)")
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch (profiling)")
    return ap.parse_args()


# ------------------------------------------------------------------ peaks --

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Dense bf16 tensor TFLOP/s (burst) of MEASURED_PEAKS.json, else the
    fallback figure."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured"
    return FALLBACK_BF16_TFLOPS, "fallback"


DECODE_SOURCES = ("pkv_decode.cuh", "pkv_device.cuh")
PREFILL_SOURCES = ("pkv_prefill.cuh", "pkv_device.cuh")


def uses_prefill_kernel(workload):
    """True when the workload's calls go to the query-major tcgen05 kernel:
    runs of new tokens filling a tile of 128 (token, head) rows."""
    spec = I.WORKLOADS[workload]
    return spec.get("q_len", 1) * (spec["hq"] // spec["hkv"]) >= 128


def strip_comments(src):
    """C++ source without its comments (string literals kept) and with runs of
    whitespace collapsed: what the compiler sees of the code."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c == '"':
            j = i + 1
            while j < n and src[j] != '"':
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash(files=DECODE_SOURCES):
    """Hash of a kernel's device code, comments and layout aside (a traffic
    record is valid only for the kernel it was captured on)."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "paged_kv_cache_438_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(strip_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def traffic_record(workload, cache=None):
    """The committed ncu record of a workload's decode call, or None when
    absent or taken on a different kernel source."""
    p = os.path.join(ROOT, "profiles", "kernel_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload + ("" if cache is None else "_" + cache))
    files = PREFILL_SOURCES if uses_prefill_kernel(workload) else DECODE_SOURCES
    if not e or e.get("source_hash") != kernel_source_hash(files):
        return None
    return e


def recorded_traffic(workload, cache, alg_bytes):
    """DRAM bytes (read + write) per decode call from the committed ncu
    record, or None when absent or taken on a different kernel source.  A
    record captured on a smaller slice of the workload is scaled to this
    call by its algorithmic bytes (traffic grows in proportion)."""
    p = os.path.join(ROOT, "profiles", "kernel_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    key = workload + ("" if cache is None else "_" + cache)
    e = d.get(key)
    files = PREFILL_SOURCES if uses_prefill_kernel(workload) else DECODE_SOURCES
    if not e or e.get("source_hash") != kernel_source_hash(files) or not e.get("alg_bytes_per_call"):
        return None
    return int(e["dram_bytes_per_call"] * alg_bytes / e["alg_bytes_per_call"])


# ---------------------------------------------------------------- clocks --

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during timing."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.proc = None
        self.path = None
        try:
            # raw samples go to PKV_CLOCKS_DIR when set (to keep them), else
            # to the temporary directory; the JSON line carries the summary
            self.path = os.path.join(os.environ.get("PKV_CLOCKS_DIR") or tempfile.gettempdir(),
                                     f"pkv_clocks_{os.getpid()}.csv")
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def wait_ready(self, timeout_s=10.0):
        """Blocks until nvidia-smi has written its first sample (the sampler
        needs several hundred ms to start; that sample is dropped later)."""
        if self.proc is None:
            return
        t0 = time.time()
        while time.time() - t0 < timeout_s:
            self.fh.flush()
            if os.path.getsize(self.path) > 0:
                return
            time.sleep(0.02)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            lines = f.readlines()[1:]          # the first sample predates the busy window
            for line in lines:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    sm.append(float(parts[0]))
                    mx = float(parts[1])
                except ValueError:
                    continue
                for n, v in zip(names, parts[4:8]):
                    if v.lower() == "active":
                        reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------- workload --

def kv_bytes_per_token(hkv, d, cache):
    """Algorithmic cache bytes one token of context costs a decode read: K
    and V rows, plus per-(token, head) fp32 scales of quantised caches and
    uint8 zero points of the asymmetric format."""
    if cache is None:
        return hkv * d * 2 * 2
    codes = hkv * d * 2 // (2 if cache in ("int4", "fp4") else 1)
    return codes + hkv * 2 * 4 + (hkv * 2 if cache == "u8asym" else 0)


class DecodeWorkload:
    """A batch of sequences living in a paged cache on one GPU, advanced one
    decode step at a time through the library's public API."""

    def __init__(self, name, cache, device, seed_offset=0, batch=None):
        from paged_kv_cache_438_b200 import pagedkv as P
        self.P = P
        self.name = name
        spec = dict(I.WORKLOADS[name])
        if batch is not None:
            spec["batch"] = batch
        self.spec = spec
        self.dev = device
        seed = spec["seed"] + seed_offset
        gen = I.generator(seed)
        self.B, self.hq, self.hkv, self.d = spec["batch"], spec["hq"], spec["hkv"], spec["d"]
        self.dtype = I.TORCH_DTYPES[spec["dtype"]]
        self.cache_kind = cache
        ctx = I.context_lens(spec, gen)
        self.prefix = spec.get("prefix", 0)
        start = (ctx + self.prefix).tolist()
        self.max_steps_ahead = 256
        need = sum(I.blocks_for(c + self.max_steps_ahead) for c in start)
        if self.prefix:
            need -= (self.B - 1) * I.blocks_for(self.prefix)
        nb = I.pool_size(spec, need)
        self.nb = nb
        order = torch.randperm(nb, generator=gen).tolist()
        self.alloc = P.BlockAllocator(nb, initial_free_order=order)
        elt = 1 if cache else 2
        cdt = {None: self.dtype, "int8": torch.int8, "fp8": torch.uint8, "u8asym": torch.uint8, "int4": torch.uint8,
               "fp4": torch.uint8}[cache]
        self.kv_format = cache if cache in ("int4", "fp4") else None
        dc = self.d // 2 if self.kv_format else self.d
        self.k_cache = torch.empty((nb, self.hkv, 16, dc), dtype=cdt, device=device)
        self.v_cache = torch.empty_like(self.k_cache)
        self.k_scale = self.v_scale = self.k_zero = self.v_zero = None
        if cache:
            self.k_scale = torch.zeros((nb, self.hkv, 16), dtype=torch.float32, device=device)
            self.v_scale = torch.zeros_like(self.k_scale)
        if cache == "u8asym":
            self.k_zero = torch.zeros((nb, self.hkv, 16), dtype=torch.uint8, device=device)
            self.v_zero = torch.zeros_like(self.k_zero)
        self.elt = elt
        self.per_tok = kv_bytes_per_token(self.hkv, self.d, cache)
        self.dg = torch.Generator(device=device)
        self.dg.manual_seed(seed + 17)
        self.ids = list(range(self.B))
        # fill: every sequence holds its context minus the token the first step appends
        if self.prefix:
            self.alloc.add(0)
            slots, _ = self.alloc.append(0, self.prefix)
            self._fill(slots)
            for s in range(1, self.B):
                self.alloc.fork(0, s)
            lens = [c - self.prefix - 1 for c in start]
            # the suffix tokens (except the last) are written after the shared prefix
            for s in range(self.B):
                slots, pairs = self.alloc.append(s, lens[s])
                if pairs.shape[0]:
                    P.copy_blocks(self.k_cache, self.v_cache, pairs.to(device), self.k_scale, self.v_scale,
                                  k_zero=self.k_zero, v_zero=self.v_zero, kv_format=self.kv_format)
                self._fill(slots)
        else:
            for s in range(self.B):
                self.alloc.add(s)
                slots, _ = self.alloc.append(s, start[s] - 1)
                self._fill(slots)
        torch.cuda.synchronize(device)
        self.max_blocks = max(I.blocks_for(c + self.max_steps_ahead) for c in start)
        self.scale = 1.0 / math.sqrt(self.d)

    def _fill(self, slots, chunk=1 << 18):
        for i in range(0, slots.numel(), chunk):
            sl = slots[i:i + chunk].to(self.dev)
            n = sl.numel()
            k = torch.randn((n, self.hkv, self.d), generator=self.dg, device=self.dev, dtype=self.dtype)
            v = torch.randn((n, self.hkv, self.d), generator=self.dg, device=self.dev, dtype=self.dtype)
            self.P.kv_cache_write(k, v, self.k_cache, self.v_cache, sl, self.k_scale, self.v_scale,
                                  k_zero=self.k_zero, v_zero=self.v_zero, kv_format=self.kv_format)

    def host_step(self):
        """Allocator work of one step: slots and CoW pairs for one new token per
        sequence, then the block tables and context lengths."""
        slots, pairs = self.alloc.batch_append(self.ids)
        bt, cl = self.alloc.batch_tables(self.ids, self.max_blocks)
        return slots, pairs, bt, cl

    def kv_bytes(self, cl):
        return int(cl.sum()) * self.per_tok

    def new_rows(self):
        q = torch.randn((self.B, self.hq, self.d), generator=self.dg, device=self.dev, dtype=self.dtype)
        k = torch.randn((self.B, self.hkv, self.d), generator=self.dg, device=self.dev, dtype=self.dtype)
        v = torch.randn((self.B, self.hkv, self.d), generator=self.dg, device=self.dev, dtype=self.dtype)
        return q, k, v

    def device_step(self, q, k, v, slots, pairs, bt, cl, maxc, out, ws):
        """Launches of one step; returns the number of kernels launched.  No
        event sits between the write and the decode launch, so the decode may
        start its prologue while the write finishes."""
        P = self.P
        n = 0
        if pairs is not None and pairs.numel():
            P.copy_blocks(self.k_cache, self.v_cache, pairs, self.k_scale, self.v_scale, k_zero=self.k_zero,
                          v_zero=self.v_zero, kv_format=self.kv_format)
            n += 1
        P.kv_cache_write(k, v, self.k_cache, self.v_cache, slots, self.k_scale, self.v_scale, k_zero=self.k_zero,
                         v_zero=self.v_zero, kv_format=self.kv_format)
        self.decode(q, bt, cl, maxc, out, ws)
        return n + 2

    def decode(self, q, bt, cl, maxc, out, ws):
        self.P.paged_attention_decode(q, self.k_cache, self.v_cache, bt, cl, self.scale, self.k_scale,
                                      self.v_scale, max_context_len=maxc, out=out, workspace=ws,
                                      k_zero=self.k_zero, v_zero=self.v_zero, kv_format=self.kv_format)

    def cache_code(self):
        return self.P.cache_code(self.k_cache, self.k_zero, self.kv_format)

    # shapes and plan of one step (the multi-query workload overrides these)
    q_rows = property(lambda self: self.B)
    mq = False

    def plan(self, maxc):
        return self.P.decode_plan(self.B, self.hq, self.hkv, self.d, maxc, self.cache_code())

    def flops(self, cl):
        """Tensor-core FLOPs of the step's attention (2 per multiply-add, QK
        and PV) for each (query, key) pair a query head sees."""
        return 4 * self.d * self.hq * int(cl.sum())


class MultiQueryWorkload(DecodeWorkload):
    """Sequences whose last n tokens are new (speculative verify, one prefill
    chunk).  The cache holds every sequence's full context; a step writes the
    n new K/V rows of every sequence into their slots and runs multi-query
    attention over the whole context.  The state does not advance between
    steps (each step re-scores the same new tokens), so every step does the
    same work."""

    mq = True

    def __init__(self, name, cache, device, seed_offset=0, batch=None):
        from paged_kv_cache_438_b200 import pagedkv as P
        self.P = P
        self.name = name
        spec = dict(I.WORKLOADS[name])
        if batch is not None:
            spec["batch"] = batch
        self.spec = spec
        self.dev = device
        seed = spec["seed"] + seed_offset
        gen = I.generator(seed)
        self.B, self.hq, self.hkv, self.d = spec["batch"], spec["hq"], spec["hkv"], spec["d"]
        self.dtype = I.TORCH_DTYPES[spec["dtype"]]
        self.cache_kind = cache
        ctx = I.context_lens(spec, gen)
        self.n = torch.clamp(torch.full_like(ctx, spec["q_len"]), max=ctx)
        need = sum(I.blocks_for(c) for c in ctx.tolist())
        nb = I.pool_size(spec, need)
        self.nb = nb
        order = torch.randperm(nb, generator=gen).tolist()
        self.alloc = P.BlockAllocator(nb, initial_free_order=order)
        cdt = {None: self.dtype, "int8": torch.int8, "fp8": torch.uint8, "u8asym": torch.uint8, "int4": torch.uint8,
               "fp4": torch.uint8}[cache]
        self.kv_format = cache if cache in ("int4", "fp4") else None
        dc = self.d // 2 if self.kv_format else self.d
        self.k_cache = torch.empty((nb, self.hkv, 16, dc), dtype=cdt, device=device)
        self.v_cache = torch.empty_like(self.k_cache)
        self.k_scale = self.v_scale = self.k_zero = self.v_zero = None
        if cache:
            self.k_scale = torch.zeros((nb, self.hkv, 16), dtype=torch.float32, device=device)
            self.v_scale = torch.zeros_like(self.k_scale)
        if cache == "u8asym":
            self.k_zero = torch.zeros((nb, self.hkv, 16), dtype=torch.uint8, device=device)
            self.v_zero = torch.zeros_like(self.k_zero)
        self.elt = 1 if cache else 2
        self.per_tok = kv_bytes_per_token(self.hkv, self.d, cache)
        self.dg = torch.Generator(device=device)
        self.dg.manual_seed(seed + 17)
        self.ids = list(range(self.B))
        new_slots = []
        for s in range(self.B):
            self.alloc.add(s)
            slots, _ = self.alloc.append(s, int(ctx[s] - self.n[s]))
            self._fill(slots)
            slots, _ = self.alloc.append(s, int(self.n[s]))
            self._fill(slots)
            new_slots.append(slots)
        self.new_slots = torch.cat(new_slots)
        self.max_blocks = max(I.blocks_for(c) for c in ctx.tolist())
        self.qsl = torch.zeros(self.B + 1, dtype=torch.int32)
        self.qsl[1:] = torch.cumsum(self.n, 0)
        self.max_q = int(self.n.max())
        self.qsl_dev = self.qsl.to(device)
        torch.cuda.synchronize(device)
        self.scale = 1.0 / math.sqrt(self.d)

    q_rows = property(lambda self: int(self.qsl[-1]))

    def host_step(self):
        bt, cl = self.alloc.batch_tables(self.ids, self.max_blocks)
        return self.new_slots, torch.empty((0, 2), dtype=torch.int32), bt, cl

    def new_rows(self):
        T = self.q_rows
        q = torch.randn((T, self.hq, self.d), generator=self.dg, device=self.dev, dtype=self.dtype)
        k = torch.randn((T, self.hkv, self.d), generator=self.dg, device=self.dev, dtype=self.dtype)
        v = torch.randn((T, self.hkv, self.d), generator=self.dg, device=self.dev, dtype=self.dtype)
        return q, k, v

    def decode(self, q, bt, cl, maxc, out, ws):
        self.P.paged_attention_multi_query(q, self.k_cache, self.v_cache, bt, cl, self.qsl_dev, self.scale,
                                           max_query_len=self.max_q, max_context_len=maxc, k_scale=self.k_scale,
                                           v_scale=self.v_scale, k_zero=self.k_zero, v_zero=self.v_zero, out=out,
                                           workspace=ws, kv_format=self.kv_format)

    def plan(self, maxc):
        return self.P.multi_query_plan(self.B, self.hq, self.hkv, self.d, maxc, self.max_q, self.cache_code())

    def flops(self, cl):
        # new token t of n sees ctx - n + t + 1 keys
        n = self.n.long()
        seen = (cl.long() - n) * n + n * (n + 1) // 2
        return 4 * self.d * self.hq * int(seen.sum())


def make_workload(name, cache, device, seed_offset=0, batch=None):
    cls = MultiQueryWorkload if "q_len" in I.WORKLOADS[name] else DecodeWorkload
    return cls(name, cache, device, seed_offset=seed_offset, batch=batch)


# ------------------------------------------------------------------ ours --

def run_ours(args, rank, world, device):
    from paged_kv_cache_438_b200 import build
    from paged_kv_cache_438_b200 import pagedkv as P
    build.build()
    P.lib()
    wl = make_workload(args.workload, args.cache, device, seed_offset=replica_seed_offset(rank), batch=args.batch)
    K, W = args.steps, args.warmup
    # host allocator outputs of every step, staged in HBM before timing
    staged = []
    for _ in range(W + K):
        slots, pairs, bt, cl = wl.host_step()
        q, k, v = wl.new_rows()
        staged.append(dict(slots=slots.to(device), pairs=pairs.to(device) if pairs.numel() else None,
                           bt=bt.to(device), cl=cl.to(device), maxc=int(cl.max()), q=q, k=k, v=v,
                           kv=wl.kv_bytes(cl), flops=wl.flops(cl)))
    maxc_all = max(s["maxc"] for s in staged)
    _, _, ws_bytes = wl.plan(maxc_all)
    ws = P.new_workspace(device, ws_bytes)
    out = torch.empty((wl.q_rows, wl.hq, wl.d), dtype=wl.dtype, device=device)
    kv_step = staged[0]["kv"]
    flush = kv_step < 4 * L2_BYTES
    scrub = torch.empty(512 * 2 ** 20, dtype=torch.uint8, device=device) if flush else None
    stream = torch.cuda.current_stream(device)
    P.device_status(clear=True)

    for i in range(W):
        st = staged[i]
        wl.device_step(st["q"], st["k"], st["v"], st["slots"], st["pairs"], st["bt"], st["cl"], st["maxc"], out, ws)
        if flush:
            scrub_l2(scrub)
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()

    sampler = ClockSampler(device.index if device.index is not None else 0)
    sampler.wait_ready()
    roll(wl, staged[:W], out, ws, flush, scrub, device, seconds=0.4)   # busy window before the timed steps
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    launches = 0
    kv_total = 0
    torch.cuda.synchronize(device)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(K):
        st = staged[W + i]
        step_ev[i][0].record(stream)
        launches += wl.device_step(st["q"], st["k"], st["v"], st["slots"], st["pairs"], st["bt"], st["cl"],
                                   st["maxc"], out, ws)
        step_ev[i][1].record(stream)
        kv_total += st["kv"]
        if flush:
            scrub_l2(scrub)
    t1.record(stream)
    torch.cuda.synchronize(device)
    roll(wl, staged[:W], out, ws, flush, scrub, device, seconds=0.3)   # and after them
    clocks = sampler.stop()
    wall_ms = t0.elapsed_time(t1)
    step_ms = sum(a.elapsed_time(b) for a, b in step_ev)       # excludes L2 scrubs
    # the decode kernel alone, for its roofline: the timed steps' decode calls
    # again, each bracketed by events on the launching stream
    dec_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i in range(K):
        st = staged[W + i]
        if flush:
            scrub_l2(scrub)
        dec_ev[i][0].record(stream)
        wl.decode(st["q"], st["bt"], st["cl"], st["maxc"], out, ws)
        dec_ev[i][1].record(stream)
    torch.cuda.synchronize(device)
    dec_ms = sum(a.elapsed_time(b) for a, b in dec_ev)
    timed_ms = step_ms if flush else wall_ms
    status = P.device_status(clear=True)
    if status:
        raise RuntimeError(f"device status {status} raised during the bench")

    timed_ms, kv_all, seqsteps_all = aggregate_ranks(timed_ms, kv_total, wl.B * K, world, device)

    res = dict(wl=wl, K=K, W=W, timed_ms=timed_ms, dec_ms=dec_ms, kv_all=kv_all, kv_rank=kv_total,
               flops_call=staged[W]["flops"],
               seqsteps_all=seqsteps_all, launches=launches, clocks=clocks, flush=flush, kv_step=kv_step,
               maxc=maxc_all, staged=staged)
    if not args.no_e2e:
        res["e2e"] = run_e2e(wl, K, W, device, world)
    return res


def aggregate_ranks(ms, kv_bytes, seq_steps, world, device):
    """Whole-job numbers of independent replicas: the time is the slowest
    rank's, the bytes and sequence-steps are summed over ranks.  The only
    collective of a multi-GPU run (no data moves between ranks)."""
    if world <= 1:
        return float(ms), float(kv_bytes), float(seq_steps)
    t = torch.tensor([float(ms)], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    tot = torch.tensor([float(kv_bytes), float(seq_steps)], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(tot)
    return float(t.item()), float(tot[0]), float(tot[1])


def replica_seed_offset(rank):
    """Each rank draws its own batch (weak scaling: per-GPU work is fixed)."""
    return 1000 * rank


def roll(wl, steps, out, ws, flush, scrub, device, seconds):
    """Replays already-run warm-up steps (same slots, same values) for about
    ``seconds`` so the clock sampler sees the GPU under this load."""
    if not steps:
        return
    t0 = time.time()
    while time.time() - t0 < seconds:
        for st in steps:
            wl.device_step(st["q"], st["k"], st["v"], st["slots"], None, st["bt"], st["cl"], st["maxc"], out, ws)
            if flush:
                scrub_l2(scrub)
        torch.cuda.synchronize(device)


def run_e2e(wl, K, W, device, world):
    """The same steps through the public API with host buffers, pipelined the
    way a serving loop runs them.  Every step: the C++ allocator appends one
    token per sequence on the host (slots, CoW pairs, block tables, context
    lengths written into pinned buffers), the step's inputs (q, new K/V rows,
    slots, tables, lengths, pairs) are copied host-to-device on a copy stream,
    the kernels run on the compute stream, and the output is copied back on a
    second copy stream and read on the host.  Two sets of pinned and device
    buffers alternate, so step i+1's allocator work and input copies overlap
    step i's kernels, and step i's output is read while step i+1 runs; events
    (not a device synchronisation) guard each buffer before it is reused."""
    P = wl.P
    B, MB, T = wl.B, wl.max_blocks, wl.q_rows
    g = I.generator(4242)

    def pinned_set():
        pin = dict(q=torch.empty((T, wl.hq, wl.d), dtype=wl.dtype).pin_memory(),
                   k=torch.empty((T, wl.hkv, wl.d), dtype=wl.dtype).pin_memory(),
                   v=torch.empty((T, wl.hkv, wl.d), dtype=wl.dtype).pin_memory(),
                   out=torch.empty((T, wl.hq, wl.d), dtype=wl.dtype).pin_memory(),
                   slots=torch.empty(T, dtype=torch.int64).pin_memory(),
                   pairs=torch.empty((B, 2), dtype=torch.int32).pin_memory(),
                   bt=torch.empty((B, MB), dtype=torch.int32).pin_memory(),
                   cl=torch.empty(B, dtype=torch.int32).pin_memory())
        for key in ("q", "k", "v"):
            pin[key].copy_(torch.randn(pin[key].shape, generator=g).to(wl.dtype))
        if wl.mq:
            # the new tokens' slots are fixed; the query layout travels every step
            pin["qsl"] = wl.qsl.clone().pin_memory()
            pin["slots"].copy_(wl.new_slots)
        return pin

    pins = [pinned_set(), pinned_set()]
    devs = [{k: torch.empty_like(v, device=device) for k, v in pin.items() if k != "out"} for pin in pins]
    outs = [torch.empty((T, wl.hq, wl.d), dtype=wl.dtype, device=device) for _ in range(2)]
    ids = torch.arange(B, dtype=torch.int64)
    _, _, wsb = wl.plan(MB * 16)
    ws = P.new_workspace(device, wsb)
    comp = torch.cuda.current_stream(device)
    h2d_stream = torch.cuda.Stream(device)
    d2h_stream = torch.cuda.Stream(device)
    keys = ("q", "k", "v", "slots", "bt", "cl") + (("qsl",) if wl.mq else ())
    fixed = sum(pins[0][k].numel() * pins[0][k].element_size() for k in keys)
    d2h = pins[0]["out"].numel() * pins[0]["out"].element_size()
    h2d_done = [None, None]    # the H2D copies that read pins[b] have finished
    comp_done = [None, None]   # the kernels that read devs[b] and wrote outs[b] have finished
    d2h_done = [None, None]    # outs[b] has reached pins[b]["out"]
    checksum = [0.0]

    def consume(b):
        """Waits for buffer b's output on the host and reads it."""
        if d2h_done[b] is not None:
            d2h_done[b].synchronize()
            checksum[0] += float(pins[b]["out"][0, 0, 0])
            d2h_done[b] = None

    def one(i):
        b = i & 1
        pin, dev, out = pins[b], devs[b], outs[b]
        if h2d_done[b] is not None:
            h2d_done[b].synchronize()          # pins[b] is free to be rewritten
        consume(b)                             # (and its last output has been read)
        if wl.mq:
            npairs = 0
        else:
            _, pairs = wl.alloc.batch_append(ids, slots_out=pin["slots"], pairs_out=pin["pairs"])
            npairs = pairs.shape[0]
        wl.alloc.batch_tables(ids, MB, out_tables=pin["bt"], out_lens=pin["cl"])
        maxc = int(pin["cl"].max())
        with torch.cuda.stream(h2d_stream):
            if comp_done[b] is not None:
                h2d_stream.wait_event(comp_done[b])   # the kernels of step i-2 no longer read devs[b]
            for key in keys:
                dev[key].copy_(pin[key], non_blocking=True)
            gp = None
            if npairs:
                gp = dev["pairs"][:npairs]
                gp.copy_(pin["pairs"][:npairs], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(h2d_stream)
            h2d_done[b] = ev
        comp.wait_event(ev)
        if wl.mq:
            wl.qsl_dev = dev["qsl"]
        wl.device_step(dev["q"], dev["k"], dev["v"], dev["slots"], gp, dev["bt"], dev["cl"], maxc, out, ws)
        ev = torch.cuda.Event()
        ev.record(comp)
        comp_done[b] = ev
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(ev)
            pin["out"].copy_(out, non_blocking=True)
            ev2 = torch.cuda.Event()
            ev2.record(d2h_stream)
            d2h_done[b] = ev2
        consume(b ^ 1)                         # the previous step's output, read while this one runs
        return fixed + npairs * 8, wl.kv_bytes(pin["cl"])

    for i in range(W):
        one(i)
    consume(0)
    consume(1)
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    h2d = kv = 0
    t0 = time.perf_counter()
    for i in range(W, W + K):
        a, c = one(i)
        h2d += a
        kv += c
    consume(0)
    consume(1)
    ms = (time.perf_counter() - t0) * 1e3
    torch.cuda.synchronize(device)
    ms, kv, _ = aggregate_ranks(ms, kv, 0, world, device)
    return {"value": round(kv / (ms * 1e-3) / 1e9, 2), "unit": "GB/s", "ms_per_step": round(ms / K, 4),
            "h2d_bytes_per_step": h2d // K, "d2h_bytes_per_step": d2h,
            "timing": "host wall clock over the steps: allocator + H2D + kernels + D2H + host read of every "
                      "step's output; two buffer sets, step i+1's host work and copies overlap step i's kernels"}


# ------------------------------------------------- the other workloads --

EXTRA_WORKLOADS = (("llama3_8b", None), ("prefix_shared", None), ("quant_mha", "int8"), ("quant_mha", "fp8"),
                   ("quant_mha", "u8asym"), ("quant_mha", "int4"), ("quant_mha", "fp4"), ("spec_verify", None),
                   ("chunked_prefill", None), ("tiny", None))
# quantised workloads whose oracle is also timed on the host cores
EXTRA_ORACLE = (("quant_mha", "int8"), ("quant_mha", "fp8"))


def scrub_l2(scrub):
    """Evicts L2 by reading a buffer four times its size (a read leaves no
    dirty lines whose write-back would land on the next kernel)."""
    return scrub.view(torch.int64).sum()


def decode_call_ms(wl, staged, out, ws, flush, scrub, stream, device, reps=3):
    """Mean CUDA-event time of decode-only calls over the staged inputs
    (``reps`` passes), with an L2 scrub before each call when ``flush``."""
    ev = []
    for _ in range(reps):
        for st in staged:
            if flush:
                scrub_l2(scrub)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            wl.decode(st["q"], st["bt"], st["cl"], st["maxc"], out, ws)
            b.record(stream)
            ev.append((a, b))
    torch.cuda.synchronize(device)
    return sum(a.elapsed_time(b) for a, b in ev) / len(ev)


def extra_record(name, cache, device, peak, tflops_peak, steps=8, warmup=3):
    """Decode-call roofline of one more workload at N = 1: the workload is
    built through the public API, ``warmup + steps`` whole steps run (write +
    decode), then the staged steps' decode calls are timed alone."""
    from paged_kv_cache_438_b200 import pagedkv as P
    wl = make_workload(name, cache, device)
    staged = []
    for _ in range(warmup + steps):
        slots, pairs, bt, cl = wl.host_step()
        q, k, v = wl.new_rows()
        staged.append(dict(slots=slots.to(device), pairs=pairs.to(device) if pairs.numel() else None,
                           bt=bt.to(device), cl=cl.to(device), maxc=int(cl.max()), q=q, k=k, v=v,
                           kv=wl.kv_bytes(cl), flops=wl.flops(cl)))
    maxc_all = max(st["maxc"] for st in staged)
    _, _, ws_bytes = wl.plan(maxc_all)
    ws = P.new_workspace(device, ws_bytes)
    out = torch.empty((wl.q_rows, wl.hq, wl.d), dtype=wl.dtype, device=device)
    stream = torch.cuda.current_stream(device)
    scrub = torch.empty(512 * 2 ** 20, dtype=torch.uint8, device=device)
    step_ev = []
    for st in staged:
        scrub_l2(scrub)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        wl.device_step(st["q"], st["k"], st["v"], st["slots"], st["pairs"], st["bt"], st["cl"], st["maxc"], out, ws)
        b.record(stream)
        step_ev.append((a, b))
    torch.cuda.synchronize(device)
    step_ms = sum(a.elapsed_time(b) for a, b in step_ev[warmup:]) / steps
    timed = staged[warmup:]
    kv_call = sum(st["kv"] for st in timed) / steps
    flops_call = sum(st["flops"] for st in timed) / steps
    small = wl.q_rows * wl.hq * wl.d * 2 * 2 + (kv_call // (wl.per_tok * 16)) * 4
    alg = kv_call + small
    # as for the main line: calls back to back when the call reads more than
    # 4 x L2, else with L2 scrubbed before every call (the prefix workload
    # reports both)
    flush = kv_call < 4 * L2_BYTES or name == "prefix_shared"
    call_ms = decode_call_ms(wl, timed, out, ws, flush, scrub, stream, device)
    rec = {"workload": name, "cache": cache or ("bf16" if wl.dtype == torch.bfloat16 else "f16"),
           "batch": wl.B, "kv_bytes_per_call": int(kv_call), "algorithmic_bytes_per_call": int(alg),
           "ms_per_call": round(call_ms, 4),
           "l2": ("scrubbed (reading 512 MiB) before every call" if flush
                  else "calls back to back, inputs larger than L2 (KV read per call > 4 x 126 MB)"),
           "achieved_gbs": round(alg / (call_ms * 1e-3) / 1e9, 1),
           "frac_of_hbm": round(alg / (call_ms * 1e-3) / 1e9 / peak, 4),
           "ms_per_step": round(step_ms, 4), "seq_steps_per_s": round(wl.B / (step_ms * 1e-3), 1),
           "traffic": recorded_traffic(name, cache, alg)}
    if flops_call / (tflops_peak * 1e12) > alg / (peak * 1e9):
        rec["bound"] = "tensor"
        rec["achieved_tflops"] = round(flops_call / (call_ms * 1e-3) / 1e12, 2)
        rec["frac_of_tensor"] = round(flops_call / (call_ms * 1e-3) / 1e12 / tflops_peak, 4)
    else:
        rec["bound"] = "hbm"
    if wl.mq:
        rec["query_tokens_per_s"] = round(wl.q_rows / (step_ms * 1e-3), 1)
    if name == "prefix_shared":
        # every sequence reads the shared prefix; its blocks are stored once
        unique = sum((int(st["cl"].sum()) - (wl.B - 1) * wl.prefix) * wl.per_tok for st in timed) / steps
        warm_ms = decode_call_ms(wl, timed, out, ws, False, scrub, stream, device)
        rec.update({"unique_kv_bytes_per_call": int(unique),
                    "unique_gbs": round(unique / (call_ms * 1e-3) / 1e9, 1),
                    "unflushed": {"ms_per_call": round(warm_ms, 4), "l2": "calls back to back, no scrub",
                                  "achieved_gbs": round(alg / (warm_ms * 1e-3) / 1e9, 1),
                                  "unique_gbs": round(unique / (warm_ms * 1e-3) / 1e9, 1)},
                    "note": "achieved_gbs counts logical bytes (the prefix once per sequence); the repeats "
                            "of the 8 MiB prefix are L2 hits, so it may exceed the HBM figure"})
        e = traffic_record(name)
        if e is not None:
            rec["ncu"] = {"dram_bytes_per_call": e["dram_bytes_per_call"],
                          "l2_sector_hit_pct": e.get("l2_sector_hit_pct"),
                          "capture": "one launch, caches flushed by ncu before it"}
    status = P.device_status(clear=True)
    if status:
        raise RuntimeError(f"device status {status} raised during the {name} record")
    if (name, cache) in EXTRA_ORACLE:
        sec, kvb, seqs = oracle_sample(name, cache, budget_s=6.0)
        rec["cpu_baseline"] = {"value": round(kvb / sec / 1e9, 4), "unit": "GB/s", "cores": oracle_threads(),
                               "kind": "oracle", "sample": f"{seqs} of {wl.B} sequences of one step "
                                                           f"(fp64 numpy oracle, ~6 s, inputs drawn on the CPU)"}
    del wl, staged, ws, out, scrub
    torch.cuda.empty_cache()
    return rec


# ----------------------------------------------------------- oracle (CPU) --

def oracle_sample(name, cache, budget_s=10.0, seed_offset=0):
    """Times the fp64 CPU oracle on sequences of the workload until about
    ``budget_s`` seconds of oracle work; inputs are drawn on the CPU from the
    seeded generators (one sequence at a time, its blocks in a shuffled
    pool).  Returns (seconds, kv_bytes, seqs)."""
    from oracle import attention as OA
    from oracle import quant as OQ
    spec = I.WORKLOADS[name]
    gen = I.generator(spec["seed"] + seed_offset + 555)
    ctx = (I.context_lens(spec, gen) + spec.get("prefix", 0)).tolist()
    hq, hkv, d = spec["hq"], spec["hkv"], spec["d"]
    per_tok = kv_bytes_per_token(hkv, d, cache)
    spent, kvb, seqs = 0.0, 0, 0
    for c in ctx:
        nblk = I.blocks_for(c)
        if "q_len" in spec:
            case = I.multi_query_case(name, seed=int(gen.initial_seed()) + seqs, ctx_override=[c],
                                      q_lens=[min(spec["q_len"], c)], cache_kind=cache, num_blocks=nblk)
        else:
            case = I.decode_case(name, seed=int(gen.initial_seed()) + seqs, ctx_override=[c], cache_kind=cache,
                                 num_blocks=nblk)
        kind = case["cache_kind"]
        if kind == "fp8":
            kc, vc = OQ.e4m3_decode(case["k_cache"].numpy()), OQ.e4m3_decode(case["v_cache"].numpy())
        elif kind in ("int4", "fp4"):
            dec = OQ.int4_values if kind == "int4" else OQ.fp4_values
            kc, vc = dec(case["k_cache"].numpy()), dec(case["v_cache"].numpy())
        else:
            kc = case["k_cache"].to(torch.float64).numpy()
            vc = case["v_cache"].to(torch.float64).numpy()
        side = {key: case[key].numpy() for key in ("k_scale", "v_scale", "k_zero", "v_zero") if key in case}
        q = case["q"].to(torch.float64).numpy()
        t0 = time.perf_counter()
        if "q_len" in spec:
            OA.paged_multi_query_attention(q, kc, vc, case["block_tables"].numpy(), [c],
                                           case["query_start_loc"].numpy(), case["scale"], side.get("k_scale"),
                                           side.get("v_scale"), side.get("k_zero"), side.get("v_zero"))
        else:
            OA.paged_decode_attention(q, kc, vc, case["block_tables"].numpy(), [c], case["scale"],
                                      side.get("k_scale"), side.get("v_scale"), k_zero=side.get("k_zero"),
                                      v_zero=side.get("v_zero"))
        spent += time.perf_counter() - t0
        kvb += c * per_tok
        seqs += 1
        if spent >= budget_s:
            break
    return spent, kvb, seqs


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def run_reference(args, rank, world):
    """The oracle as the reference arm: each step a bounded sample of the
    workload on the host cores; rank 0 only."""
    if rank != 0:
        return None
    budget = max(1.0, 120.0 / max(1, args.warmup + args.steps))
    for i in range(args.warmup):
        oracle_sample(args.workload, args.cache, budget_s=budget, seed_offset=i)
    sec = kvb = seqs = 0
    for i in range(args.steps):
        a, b, c = oracle_sample(args.workload, args.cache, budget_s=budget, seed_offset=args.warmup + i)
        sec += a
        kvb += b
        seqs += c
    gbs = kvb / sec / 1e9
    return {"impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD_TEXT[args.workload], "name": args.workload,
                       "cache": args.cache or "bf16"},
            "seq_steps_per_s": seqs / sec,
            "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": oracle_threads(), "kind": "oracle",
                             "sample": f"{seqs} sequences over {args.steps} steps, ~{budget:.1f} s of oracle "
                                       f"work per step"},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


# ------------------------------------------------------------------ main --

def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    r = run_ours(args, rank, world, device)
    wl = r["wl"]
    peak, peak_kind = peaks()
    ms_step = r["timed_ms"] / r["K"]
    value = r["kv_all"] / (r["timed_ms"] * 1e-3) / 1e9
    seqsteps = r["seqsteps_all"] / (r["timed_ms"] * 1e-3)
    # roofline of the decode call (decode kernel + reduce when split) on this rank
    dec_ms = r["dec_ms"] / r["K"]
    nstreams, stream_tokens, ws_bytes = wl.plan(r["maxc"])
    kv_call = r["kv_rank"] / r["K"]
    # q read + out written + the block-table entries the step reads
    small = wl.q_rows * wl.hq * wl.d * 2 * 2 + (kv_call // (wl.per_tok * 16)) * 4
    alg_bytes = kv_call + small
    achieved = alg_bytes / (dec_ms * 1e-3) / 1e9
    traffic = recorded_traffic(args.workload, args.cache, alg_bytes)
    tflops_peak, tflops_kind = tensor_peak()
    flops_call = r["flops_call"]
    # the bound is whichever floor is higher: bytes at the copy bandwidth or
    # FLOPs at the dense bf16 tensor rate
    tensor_bound = flops_call / (tflops_peak * 1e12) > alg_bytes / (peak * 1e9)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": r["K"],
        "warmup": r["W"], "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": {None: "bf16" if wl.dtype == torch.bfloat16 else "f16",
                                       "int8": "int8 KV / fp16 mma", "fp8": "fp8e4m3 KV / fp16 mma",
                                       "u8asym": "u8 KV with zero point / fp16 mma",
                                       "int4": "int4 KV / fp16 mma", "fp4": "fp4e2m1 KV / fp16 mma"}[args.cache],
        "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[args.workload], "name": args.workload, "batch": wl.B,
                   "q_heads": wl.hq, "kv_heads": wl.hkv, "head_dim": wl.d, "block_size": 16,
                   "cache": args.cache or ("bf16" if wl.dtype == torch.bfloat16 else "f16"),
                   "kv_bytes_per_step": r["kv_step"], "decode_warp_streams": nstreams,
                   "l2": "L2 scrubbed (reading 512 MiB) between steps, outside the step events" if r["flush"]
                   else "inputs larger than L2 (KV read per step > 4 x 126 MB)",
                   "parallelism": f"replicas x{world} (independent batches)"},
        "seq_steps_per_s": round(seqsteps, 1),
        "pct_of_hbm_measured": round(100 * value / (peak * world), 2),
        "pct_of_hbm_nominal_8tbs": round(100 * value / (NOMINAL_HBM_GBS * world), 2),
        "roofline": ({"kernel": "paged_decode_kernel (one launch per decode call)", "bound": "hbm",
                      "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                      "frac": round(achieved / peak, 4), "peak_source": f"{peak_kind} hbm_gbs (copy, burst)"}
                     if not tensor_bound else
                     {"kernel": ("paged_prefill_kernel (query-major, tcgen05; one launch per call)"
                                 if uses_prefill_kernel(args.workload) else
                                 "paged_decode_kernel, multi-query mode (one launch per call)"), "bound": "tensor",
                      "achieved": round(flops_call / (dec_ms * 1e-3) / 1e12, 2), "peak": tflops_peak,
                      "unit": "TFLOP/s", "frac": round(flops_call / (dec_ms * 1e-3) / 1e12 / tflops_peak, 4),
                      "peak_source": f"{tflops_kind} bf16_tflops (cuBLAS, burst)",
                      "hbm_achieved_gbs": round(achieved, 1)}),
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
    }
    line["roofline"].update({
        "timing": "decode-only launches of the timed steps' inputs, CUDA events on the launching stream",
        "traffic": traffic, "algorithmic_bytes_per_call": int(alg_bytes), "flops_per_call": int(flops_call),
        "ms_per_call": round(dec_ms, 4)})
    if wl.mq:
        line["query_tokens_per_s"] = round(wl.q_rows * r["K"] * world / (r["timed_ms"] * 1e-3), 1)
        line["config"]["new_tokens_per_sequence"] = wl.spec["q_len"]
    if "e2e" in r:
        line["e2e"] = r["e2e"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sec, kvb, seqs = oracle_sample(args.workload, args.cache, budget_s=12.0)
        line["cpu_baseline"] = {"value": round(kvb / sec / 1e9, 4), "unit": "GB/s", "cores": oracle_threads(),
                                "kind": "oracle",
                                "sample": f"{seqs} of {wl.B} sequences of one step (fp64 numpy oracle, ~12 s, "
                                          f"inputs drawn on the CPU)",
                                "seq_steps_per_s": round(seqs / sec, 3)}
    if world == 1 and not args.no_extra:
        del r, wl
        torch.cuda.empty_cache()
        others = []
        for name, cache in EXTRA_WORKLOADS:
            if (name, cache) == (args.workload, args.cache):
                continue
            try:
                others.append(extra_record(name, cache, device, peak, tflops_peak))
            except Exception as e:  # the headline line must still print; the failure is recorded
                others.append({"workload": name, "cache": cache, "error": f"{type(e).__name__}: {e}"[:300]})
                torch.cuda.synchronize(device)
                torch.cuda.empty_cache()
        line["other_workloads"] = others
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
