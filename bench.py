"""Benchmark: attention over a paged KV cache on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the CPU oracle on this host's cores

A step is one pass of the hot path over one batch.  Default workload (`gqa70b`): the
70B-class GQA decode -- 80 layers, 64 query heads, 8 KV heads, head dim 128, bf16 K/V,
170 sequences with contexts ~ N(3000, 400) clipped to [1024, 4096], block tables
permuted over a pool of 170 x 256 blocks per layer; per layer, kv_append of every
sequence's new token, then paged_decode_attn over its whole cached context.

Other workloads (one JSON line each): `llama8b` (1 layer, B 64, H_q 32, ctx U[512, 4096]);
`quant_int8` / `quant_fp8` / `quant_int4` / `quant_bf16` (1 layer, B 16, H_q 64, H_kv 8,
ctx U[32768, 131072], K/V stored quantized with one fp32 scale per (block, head), bf16
N(0,1) source with 1% outlier channels x8; `quant_bf16` is the unquantized control);
`prefix_chunk` (1 layer of the 70B shape: 256 decodes sharing a 4,000-token prefix plus
private 200-token suffixes and 0-300 decoded tokens, and one 512-token prefill chunk of
a new request over the same prefix, in every step).

Prints ONE JSON line (rank 0).  `value` is KV GB/s: the K/V bytes the step's attention
calls read (logically, per sequence) / the max-over-ranks device time of the K timed
steps.  With --gpus N > 1 (torchrun), every rank runs an independent replica (the path
has no data exchange), so there is no collective beyond the timing barrier.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
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

from paged_kv_cache_431_b200 import workloads as wl  # noqa: E402

METRIC = "paged GQA decode: KV HBM GB/s (% of ~8 TB/s peak); seq-tokens/s per layer"
PROFILES = os.path.join(ROOT, "profiles")
# the sources each kernel's DRAM-byte capture depends on (kernel, shared device code, launch setup)
DECODE16_SRCS = ["paged_kv_cache_431_b200/csrc/decode.cu", "paged_kv_cache_431_b200/csrc/decode_common.cuh",
                 "paged_kv_cache_431_b200/csrc/common.cuh", "paged_kv_cache_431_b200/csrc/api.cu"]
DECODETC_SRCS = ["paged_kv_cache_431_b200/csrc/decode_tc.cu", "paged_kv_cache_431_b200/csrc/tcgen05.cuh",
                 "paged_kv_cache_431_b200/csrc/decode.cu", "paged_kv_cache_431_b200/csrc/decode_common.cuh",
                 "paged_kv_cache_431_b200/csrc/common.cuh", "paged_kv_cache_431_b200/csrc/api.cu"]
DECODETCK_SRCS = ["paged_kv_cache_431_b200/csrc/decode_tc_keys.cu", "paged_kv_cache_431_b200/csrc/tcgen05.cuh",
                  "paged_kv_cache_431_b200/csrc/decode.cu", "paged_kv_cache_431_b200/csrc/decode_common.cuh",
                  "paged_kv_cache_431_b200/csrc/common.cuh", "paged_kv_cache_431_b200/csrc/api.cu"]
DECODEQ8TC_SRCS = ["paged_kv_cache_431_b200/csrc/decode_tc_fp8.cu", "paged_kv_cache_431_b200/csrc/tcgen05.cuh",
                   "paged_kv_cache_431_b200/csrc/decode.cu", "paged_kv_cache_431_b200/csrc/decode_common.cuh",
                   "paged_kv_cache_431_b200/csrc/common.cuh", "paged_kv_cache_431_b200/csrc/api.cu"]
DECODEQ_SRCS = ["paged_kv_cache_431_b200/csrc/decode_quant.cu", "paged_kv_cache_431_b200/csrc/decode_common.cuh",
                "paged_kv_cache_431_b200/csrc/common.cuh", "paged_kv_cache_431_b200/csrc/api.cu"]
PREFILL_SRCS = ["paged_kv_cache_431_b200/csrc/prefill_tc.cu", "paged_kv_cache_431_b200/csrc/common.cuh"]
BLOCKS_SRCS = ["paged_kv_cache_431_b200/csrc/blocks.cu", "paged_kv_cache_431_b200/csrc/common.cuh"]


# ------------------------------------------------------------------ utils --

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"pkv_clocks_{os.getpid()}_gpu{gpu_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        with open(self.path) as f:
            return summarize_clocks(f)


def summarize_clocks(lines):
    """Median SM clock, max SM clock and the throttle reasons seen in nvidia-smi CSV rows
    (ClockSampler.FIELDS, no header, no units); None if no row parses."""
    sm, mx, reasons = [], 0.0, set()
    for line in lines:
        parts = [x.strip() for x in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            mx = max(mx, float(parts[2]))
        except ValueError:
            continue
        for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                             parts[5:9]):
            if val.lower() == "active":
                reasons.add(name)
    if not sm:
        return None
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def source_hash(src_files):
    h = hashlib.sha256()
    for s in src_files:
        with open(os.path.join(ROOT, s), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def scaled(v, f):
    """v * f rounded to an integer, None stays None (traffic records are per full launch)."""
    return None if v is None else int(round(v * f))


def kernel_traffic(key: str, src_files):
    """DRAM bytes per launch from a committed ncu summary, used only while the kernel
    sources still hash to the version that was captured."""
    try:
        with open(os.path.join(PROFILES, "traffic.json")) as f:
            rec = json.load(f).get(key)
    except Exception:
        return None
    if not rec or rec.get("src_sha256") != source_hash(src_files):
        return None
    return rec.get("bytes_per_launch")


# -------------------------------------------------------------- workloads --

QUANT_DESC = ("quantized long-context decode, 1 layer: H_q 64, H_kv 8, d 128, B 16, ctx ~ U[32768, 131072], "
              "bf16 N(0,1) source with 1% outlier channels x8, stored as {}, one fp32 scale per (block, kv head)")
WORKLOADS = {
    "gqa70b": dict(kind="decode", layers=80, B=170, H_q=64, H_kv=8, d=128, dtype=wl.BF16, width=256,
                   lens="gqa70b", pool_blocks=170 * 256,
                   desc="70B-class GQA decode: 80 layers, H_q 64, H_kv 8, d 128, bf16, B 170, "
                        "ctx ~ N(3000, 400) clipped to [1024, 4096], pool 170 x 256 blocks per layer"),
    "llama8b": dict(kind="decode", layers=1, B=64, H_q=32, H_kv=8, d=128, dtype=wl.BF16, width=256,
                    lens="llama8b", pool_blocks=64 * 256,
                    desc="Llama-3-8B-shaped decode, 1 layer: H_q 32, H_kv 8, d 128, bf16, B 64, "
                         "ctx ~ U[512, 4096], pool for 64 x 4096 tokens"),
    "quant_int8": dict(kind="decode", layers=1, B=16, H_q=64, H_kv=8, d=128, dtype=wl.INT8, width=8192,
                       lens="quant", pool_blocks=16 * 8192, desc=QUANT_DESC.format("int8")),
    "quant_fp8": dict(kind="decode", layers=1, B=16, H_q=64, H_kv=8, d=128, dtype=wl.FP8, width=8192,
                      lens="quant", pool_blocks=16 * 8192, desc=QUANT_DESC.format("fp8 e4m3")),
    "quant_int4": dict(kind="decode", layers=1, B=16, H_q=64, H_kv=8, d=128, dtype=wl.INT4, width=8192,
                       lens="quant", pool_blocks=16 * 8192, desc=QUANT_DESC.format("packed int4")),
    "quant_bf16": dict(kind="decode", layers=1, B=16, H_q=64, H_kv=8, d=128, dtype=wl.BF16, width=8192,
                       lens="quant", pool_blocks=16 * 8192, desc=QUANT_DESC.format("bf16 (control)")),
    "mha": dict(kind="decode", layers=1, B=32, H_q=64, H_kv=64, d=128, dtype=wl.BF16, width=256,
                lens="gqa70b", pool_blocks=32 * 256,
                desc="MHA decode (one KV head per query head, G = 1), 1 layer, H 64, d 128, bf16, B 32, "
                     "ctx ~ N(3000, 400) clipped to [1024, 4096]"),
    "mqa": dict(kind="decode", layers=1, B=256, H_q=64, H_kv=1, d=128, dtype=wl.BF16, width=256,
                lens="gqa70b", pool_blocks=256 * 256,
                desc="MQA decode (one KV head for all 64 query heads, G = 64), 1 layer, d 128, bf16, B 256, "
                     "ctx ~ N(3000, 400) clipped to [1024, 4096]"),
    "window": dict(kind="decode", layers=1, B=64, H_q=64, H_kv=8, d=128, dtype=wl.BF16, width=2048,
                   lens="long", pool_blocks=64 * 2048, window=4096,
                   desc="sliding-window decode, 1 layer of the 70B shape (H_q 64, H_kv 8, d 128, bf16), B 64, "
                        "ctx ~ U[16384, 32768], window 4,096 tokens: only the window's K/V is read"),
    "blocks": dict(kind="blocks", layers=80, H_kv=8, d=128, dtype=wl.BF16, pool_blocks=4096, copies=512, swaps=16,
                   desc="whole-block moves on the 80-layer 70B-class bf16 pool (a block = 80 layers x K and V of 8 "
                        "heads, 5.24 MB): copy-on-write of 512 blocks, swap-out of 16 blocks to pinned host memory "
                        "and swap-in of 16"),
    "prefix_chunk": dict(kind="prefix", layers=1, B=256, H_q=64, H_kv=8, d=128, dtype=wl.BF16,
                         desc="prefix sharing + chunked prefill, 1 layer of the 70B shape, bf16: 256 decodes "
                              "share a 4,000-token prefix (250 blocks) + private 200-token suffixes + U{0..300} "
                              "decoded tokens; plus one 512-token causal prefill chunk of a new request over "
                              "the prefix"),
}
ELEM_BYTES = {wl.F16: 2.0, wl.BF16: 2.0, wl.INT8: 1.0, wl.FP8: 1.0, wl.INT4: 0.5}
DTYPE_NAME = {wl.F16: "f16", wl.BF16: "bf16", wl.INT8: "int8", wl.FP8: "fp8e4m3", wl.INT4: "int4"}


def make_lens(kind, gen, B):
    if kind == "long":
        return torch.randint(16384, 32769, (B,), generator=gen, dtype=torch.int32)
    return {"gqa70b": wl.gqa70b_lens, "llama8b": wl.llama8b_lens, "quant": wl.quant_long_lens}[kind](gen, B)


def decode_bytes(ctx_lens, B, H_q, H_kv, d, dt, window=0):
    """(K/V bytes, all algorithmic bytes) of one decode call: every visible cached K and V
    element once (and its block's scales), plus q, out, used table entries, lengths.  With a
    sliding window only the last `window` tokens of each context are visible."""
    if window:
        ctx_lens = torch.clamp(ctx_lens, max=window)
    sum_ctx = int(ctx_lens.sum())
    blocks = int(sum(wl.ceil_div(int(n), 16) for n in ctx_lens))
    kv = int(sum_ctx * 2 * H_kv * d * ELEM_BYTES[dt])
    scales = blocks * H_kv * 2 * 4 if dt in (wl.INT8, wl.FP8, wl.INT4) else 0
    other = B * H_q * d * 2 + B * H_q * d * 4 + blocks * 4 + B * 4
    return kv, kv + scales + other


# ------------------------------------------------------------- GPU arm --

class Timed:
    """Device timing of the K steps plus per-call events around the dominant calls.  With
    `external`, the events can be recorded inside a CUDA-graph capture: they become event-record
    nodes that take their timestamps at every replay."""

    def __init__(self, steps, per_step, external=False):
        mk = lambda: torch.cuda.Event(enable_timing=True, external=external)  # noqa: E731
        self.ev = [[(mk(), mk()) for _ in range(per_step)] for _ in range(steps)]

    def call_ms(self):
        return [a.elapsed_time(b) for st in self.ev for (a, b) in st]


def build_decode(args, cfg, dev, rank):
    from paged_kv_cache_431_b200 import pkv

    L, H_q, H_kv, d, dt = cfg["layers"], cfg["H_q"], cfg["H_kv"], cfg["d"], cfg["dtype"]
    B = args.batch or cfg["B"]
    gen = wl.generator(431 + 3 + rank)
    ctx = make_lens(cfg["lens"], gen, B)
    N = cfg["pool_blocks"] * B // cfg["B"]   # the pool scales with a --batch override
    paging = wl.allocate(ctx, N, cfg["width"], gen)
    quant = dt in (wl.INT8, wl.FP8, wl.INT4)
    per_layer_pool = 2 * N * H_kv * 16 * d * ELEM_BYTES[dt]
    free, _ = torch.cuda.mem_get_info(dev)
    L_phys = max(1, min(L, int(args.pool_fraction * free // per_layer_pool)))
    gd = wl.generator(431 + 100 + rank, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    if not quant:
        tdt = wl.TORCH_DTYPE[dt]
        k_pool = torch.empty(L_phys, N, H_kv, 16, d, dtype=tdt, device=dev)
        v_pool = torch.empty_like(k_pool)
        for l in range(L_phys):
            k_pool[l] = wl.normal((N, H_kv, 16, d), tdt, gd, dev)
            v_pool[l] = wl.normal((N, H_kv, 16, d), tdt, gd, dev)
        pool = pkv.KVPool(k_pool, v_pool, dt, d, device_status=status)
        src_dtype = tdt
    else:
        pool = pkv.KVPool.allocate(L_phys, N, H_kv, d, dt)
        out_ch = wl.outlier_channels(gen, H_kv, d)
        for l in range(L_phys):           # bulk fill through kv_append (untimed)
            for b in range(B):
                n = int(ctx[b])
                k, v = wl.kv_source(n, H_kv, d, gd, dev, outliers=out_ch)
                pkv.kv_append(pool, l, k, v, wl.slots_for(paging.tables, [b] * n, torch.arange(n)).to(dev))
                del k, v
        src_dtype = torch.bfloat16
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()

    tables = paging.tables.to(dev)
    ctx_d = ctx.to(dev)
    max_ctx = int(ctx.max())
    slots = wl.slots_for(paging.tables, range(B), (ctx - 1).long()).to(dev)   # each step's new token
    q = wl.normal((L, B, H_q, d), src_dtype, gd, dev)
    k_new = wl.normal((L, B, H_kv, d), src_dtype, gd, dev)
    v_new = wl.normal((L, B, H_kv, d), src_dtype, gd, dev)
    out = torch.empty(L, B, H_q, d, dtype=torch.float32, device=dev)
    window = cfg.get("window", 0)
    # paged_decode_attn's default engine takes the tcgen05 kernel for 64 or 128 query heads
    # per KV head (16-bit pool, head dim 128, no window)
    wide = not quant and d == 128 and H_q // H_kv in (64, 128) and not window and args.engine == 0
    keys_on_m = wide and H_q // H_kv == 64   # 64 heads: the keys-on-M form of that kernel
    # fp8 pools with 8 query heads per KV head: the tcgen05 kernel that multiplies the e4m3 codes
    fp8_tc = dt == wl.FP8 and d == 128 and H_q // H_kv == 8 and not window and args.engine == 0
    ws = torch.empty(max(pkv.paged_decode_workspace_bytes(pool, B, H_q, max_ctx, partition_tokens=args.partition,
                                                          sliding_window=window), 16),
                     dtype=torch.uint8, device=dev)
    aws = torch.empty(max(pkv.kv_append_workspace_bytes(pool, B), 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    scale = d ** -0.5

    def step(ev=None):
        for l in range(L):
            lp = l % L_phys
            pkv.kv_append(pool, lp, k_new[l], v_new[l], slots, workspace=aws)
            if ev is not None:
                ev[l][0].record()
            pkv.paged_decode_attn(pool, lp, q[l], tables, ctx_d, scale, max_ctx, out=out[l], workspace=ws,
                                  engine=args.engine, partition_tokens=args.partition, sliding_window=window)
            if ev is not None:
                ev[l][1].record()

    kv, alg = decode_bytes(ctx, B, H_q, H_kv, d, dt, window)
    # this library's kernels per layer: the append (3 for quantized pools), the decode and, when a
    # context spans several partitions, the split-K merge
    parts = pkv.paged_decode_workspace_bytes(pool, B, H_q, max_ctx, partition_tokens=args.partition,
                                             sliding_window=window) > 0
    launches = L * ((3 if quant else 1) + 1 + (1 if parts else 0))

    # host-buffer (e2e) step: inputs from pinned memory, every layer's output read back
    g = wl.generator(999)
    hq = wl.normal((L, B, H_q, d), src_dtype, g).pin_memory()
    hk = wl.normal((L, B, H_kv, d), src_dtype, g).pin_memory()
    hv = wl.normal((L, B, H_kv, d), src_dtype, g).pin_memory()
    htab = paging.tables.clone().pin_memory()
    hctx = ctx.clone().pin_memory()
    hslots = wl.slots_for(paging.tables, range(B), (ctx - 1).long()).pin_memory()
    hout = torch.empty(L, B, H_q, d, dtype=torch.float32).pin_memory()
    dq, dk, dv = (torch.empty(t.shape, dtype=t.dtype, device=dev) for t in (hq, hk, hv))
    dtab, dctx, dslots = (torch.empty(t.shape, dtype=t.dtype, device=dev) for t in (htab, hctx, hslots))
    dout = torch.empty(hout.shape, dtype=torch.float32, device=dev)
    h2d = torch.cuda.Stream(dev)
    d2h = torch.cuda.Stream(dev)

    def e2e_step():
        start = torch.cuda.Event()
        start.record(stream)
        h2d.wait_event(start)
        ready = []
        with torch.cuda.stream(h2d):
            dtab.copy_(htab, non_blocking=True)
            dctx.copy_(hctx, non_blocking=True)
            dslots.copy_(hslots, non_blocking=True)
            for l in range(L):
                dq[l].copy_(hq[l], non_blocking=True)
                dk[l].copy_(hk[l], non_blocking=True)
                dv[l].copy_(hv[l], non_blocking=True)
                e = torch.cuda.Event()
                e.record(h2d)
                ready.append(e)
        done = []
        for l in range(L):
            stream.wait_event(ready[l])
            pkv.kv_append(pool, l % L_phys, dk[l], dv[l], dslots, workspace=aws)
            pkv.paged_decode_attn(pool, l % L_phys, dq[l], dtab, dctx, scale, max_ctx, out=dout[l], workspace=ws,
                                  engine=args.engine, partition_tokens=args.partition, sliding_window=window)
            e = torch.cuda.Event()
            e.record(stream)
            done.append(e)
        with torch.cuda.stream(d2h):
            for l in range(L):
                d2h.wait_event(done[l])
                hout[l].copy_(dout[l], non_blocking=True)
        fin = torch.cuda.Event()
        fin.record(d2h)
        stream.wait_event(fin)

    h2d_bytes = sum(t.numel() * t.element_size() for t in (hq, hk, hv, htab, hctx, hslots))
    d2h_bytes = hout.numel() * hout.element_size()
    peaks, kind = measured_peaks()
    info = dict(
        config={"workload": args.workload if B == cfg["B"] else f"{args.workload} (batch {B})",
                "description": cfg["desc"], "layers": L, "batch": B, "q_heads": H_q,
                "kv_heads": H_kv, "head_dim": d, "kv_dtype": DTYPE_NAME[dt], "sum_ctx": int(ctx.sum()),
                "physical_layer_pools": L_phys, "parallelism": "replicas",
                "l2": (f"inputs larger than L2: each decode call reads {kv / 1e9:.2f} GB of K/V from one of "
                       f"{L_phys} layer pools" if L > 1 else
                       f"L2 flushed between timed steps (a 256 MiB write, then a read of it, outside the timed "
                       f"events); each decode "
                       f"call reads {kv / 1e9:.2f} GB of K/V"),
                "partition_tokens": args.partition or "auto", "sliding_window": window or None,
                "decode_engine": {0: ("tensor cores (tcgen05, keys on the MMA's M side)" if keys_on_m else
                                      "tensor cores (tcgen05)") if wide else
                                     "tensor cores (tcgen05 kind::f8f6f4 on the e4m3 codes)" if fp8_tc else
                                     "tensor cores (mma.sync)",
                                  1: "tensor cores (mma.sync)", 2: "CUDA cores, packed fp32x2 FMA",
                                  3: "CUDA cores, fp32 FMA"}[args.engine]},
        kv_bytes_per_step=kv * L, layers=L,
        seq_tokens_per_step=int((torch.clamp(ctx, max=window) if window else ctx).sum()) * L,
        roofline=dict(bound="hbm", kernel="paged_decode_attn (main + split-K merge)", alg_bytes=alg,
                      peak=float(peaks["hbm_gbs"]), unit="GB/s",
                      peak_source=f"{kind} (MEASURED_PEAKS.json hbm_gbs)",
                      traffic=kernel_traffic(f"decode_{args.workload}",
                                             DECODEQ8TC_SRCS if fp8_tc else
                                             DECODEQ_SRCS if quant else DECODETCK_SRCS if keys_on_m else
                                             DECODETC_SRCS if wide else DECODE16_SRCS)),
        launches_per_step=launches, dtype=DTYPE_NAME[dt] if quant else "bf16",
        h2d=h2d_bytes, d2h=d2h_bytes, calls_per_step=L, flush_l2=L == 1)
    return step, e2e_step, info, pool


def build_prefix_chunk(args, cfg, dev, rank):
    """Config 4: one step = 256 decode appends + decode over prefix-sharing tables, then
    the new request's 512-token chunk append + chunked prefill over the same prefix."""
    from paged_kv_cache_431_b200 import pkv

    B, H_q, H_kv, d = cfg["B"], cfg["H_q"], cfg["H_kv"], cfg["d"]
    P0, C, pre_blocks = 4000, 512, 250
    gen = wl.generator(431 + 4 + rank)
    n_dec = torch.randint(0, 301, (B,), generator=gen, dtype=torch.int32)
    ctx = (P0 + 200 + n_dec + 1).to(torch.int32)           # includes this step's token
    lens_all = torch.cat([ctx, torch.tensor([P0 + C], dtype=torch.int32)])
    N = pre_blocks + B * 32 + 32 + 64
    width = wl.ceil_div(int(lens_all.max()), 16)
    paging = wl.allocate(lens_all, N, width, gen, shared_prefix_blocks=pre_blocks)
    gd = wl.generator(431 + 200 + rank, dev)
    k_pool = wl.normal((1, N, H_kv, 16, d), torch.bfloat16, gd, dev)
    v_pool = wl.normal((1, N, H_kv, 16, d), torch.bfloat16, gd, dev)
    pool = pkv.KVPool(k_pool, v_pool, wl.BF16, d, device_status=torch.zeros(1, dtype=torch.int32, device=dev))
    tables = paging.tables[:B].contiguous().to(dev)
    ctx_d = ctx.to(dev)
    max_ctx = int(ctx.max())
    chunk_table = paging.tables[B].contiguous().to(dev)
    dec_slots = wl.slots_for(paging.tables, range(B), (ctx - 1).long()).to(dev)
    chunk_slots = wl.slots_for(paging.tables, [B] * C, torch.arange(P0, P0 + C)).to(dev)
    q_dec = wl.normal((B, H_q, d), torch.bfloat16, gd, dev)
    k_dec = wl.normal((B, H_kv, d), torch.bfloat16, gd, dev)
    v_dec = wl.normal((B, H_kv, d), torch.bfloat16, gd, dev)
    q_chunk = wl.normal((C, H_q, d), torch.bfloat16, gd, dev)
    k_chunk = wl.normal((C, H_kv, d), torch.bfloat16, gd, dev)
    v_chunk = wl.normal((C, H_kv, d), torch.bfloat16, gd, dev)
    out_dec = torch.empty(B, H_q, d, dtype=torch.float32, device=dev)
    out_chunk = torch.empty(C, H_q, d, dtype=torch.float32, device=dev)
    cascade = args.decode_form == "cascade"
    if cascade:
        ws_bytes = pkv.paged_decode_cascade_workspace_bytes(pool, B, H_q, max_ctx, P0)
    else:
        ws_bytes = pkv.paged_decode_workspace_bytes(pool, B, H_q, max_ctx)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    scale = d ** -0.5

    def decode(q, out):
        if cascade:   # the 4,000-token shared prompt once per KV group on the tensor cores
            pkv.paged_decode_attn_cascade(pool, 0, q, tables, ctx_d, scale, max_ctx, P0, out=out, workspace=ws)
        else:
            pkv.paged_decode_attn(pool, 0, q, tables, ctx_d, scale, max_ctx, out=out, workspace=ws)

    def step(ev=None):
        pkv.kv_append(pool, 0, k_dec, v_dec, dec_slots)
        if ev is not None:
            ev[0][0].record()
        decode(q_dec, out_dec)
        if ev is not None:
            ev[0][1].record()
        pkv.kv_append(pool, 0, k_chunk, v_chunk, chunk_slots)
        if ev is not None:
            ev[1][0].record()
        pkv.paged_prefill_chunk_attn(pool, 0, q_chunk, chunk_table, P0, scale, out=out_chunk)
        if ev is not None:
            ev[1][1].record()

    dec_kv, dec_alg = decode_bytes(ctx, B, H_q, H_kv, d, wl.BF16)
    pairs = sum(P0 + i + 1 for i in range(C))                      # causal (query, key) pairs per head
    flops = 4 * d * pairs * H_q
    chunk_kv = (P0 + C) * 2 * H_kv * d * 2
    unique_blocks = int(torch.unique(paging.tables[paging.tables >= 0]).numel())

    hq = torch.cat([q_dec, q_chunk]).cpu().pin_memory()
    hk = torch.cat([k_dec, k_chunk]).cpu().pin_memory()
    hv = torch.cat([v_dec, v_chunk]).cpu().pin_memory()
    hout = torch.empty(B + C, H_q, d, dtype=torch.float32).pin_memory()
    dq, dk, dv = (torch.empty(t.shape, dtype=t.dtype, device=dev) for t in (hq, hk, hv))
    dout = torch.empty(hout.shape, dtype=torch.float32, device=dev)

    def e2e_step():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        pkv.kv_append(pool, 0, dk[:B], dv[:B], dec_slots)
        decode(dq[:B], dout[:B])
        pkv.kv_append(pool, 0, dk[B:], dv[B:], chunk_slots)
        pkv.paged_prefill_chunk_attn(pool, 0, dq[B:], chunk_table, P0, scale, out=dout[B:])
        hout.copy_(dout, non_blocking=True)

    peaks, kind = measured_peaks()
    info = dict(
        config={"workload": args.workload, "description": cfg["desc"], "decode_batch": B, "q_heads": H_q,
                "kv_heads": H_kv, "head_dim": d, "prefix_tokens": P0, "chunk_tokens": C,
                "sum_ctx_decode": int(ctx.sum()), "unique_kv_blocks": unique_blocks,
                "unique_kv_bytes": unique_blocks * H_kv * 16 * d * 2 * 2,
                "chunk_gflop": round(flops / 1e9, 2), "parallelism": "replicas",
                "decode_form": ("cascade: the shared prefix once per KV group on tensor cores + per-sequence "
                                "suffix split-K + merge") if cascade else "plain split-K decode",
                "l2": "steady state, no flush: the shared prefix stays in L2 across the 256 decodes (as in real "
                      "prefix reuse)"},
        kv_bytes_per_step=dec_kv + chunk_kv, seq_tokens_per_step=int(ctx.sum()), layers=1,
        roofline=dict(bound="tensor", kernel="paged_prefill_chunk_attn", alg_flops=flops,
                      peak=float(peaks["bf16_tflops"]), unit="TFLOP/s",
                      peak_source=f"{kind} (MEASURED_PEAKS.json bf16_tflops, burst: a short kernel)",
                      traffic=kernel_traffic("prefill_prefix_chunk", PREFILL_SRCS), call_index=1,
                      decode_alg_bytes=dec_alg),
        launches_per_step=(6 if cascade else 4 + (1 if ws.numel() > 16 else 0)), dtype="bf16",
        h2d=sum(t.numel() * t.element_size() for t in (hq, hk, hv)), d2h=hout.numel() * 4, calls_per_step=2)
    return step, e2e_step, info, pool


def build_blocks(args, cfg, dev, rank):
    """Whole-block moves on the 80-layer 70B-class pool: one step copies `copies` blocks
    (copy-on-write at divergence) and swaps `swaps` blocks out to pinned host memory and
    back in (preemption).  Block = all layers' K and V tiles of its 8 KV heads (5.24 MB)."""
    from paged_kv_cache_431_b200 import pkv

    L, H_kv, d, N = args.layers or cfg["layers"], cfg["H_kv"], cfg["d"], cfg["pool_blocks"]
    n_copy, n_swap = cfg["copies"], cfg["swaps"]
    gd = wl.generator(431 + 500 + rank, dev)
    k_pool = torch.empty(L, N, H_kv, 16, d, dtype=torch.bfloat16, device=dev)
    v_pool = torch.empty_like(k_pool)
    for l in range(L):
        k_pool[l] = wl.normal((N, H_kv, 16, d), torch.bfloat16, gd, dev)
        v_pool[l] = wl.normal((N, H_kv, 16, d), torch.bfloat16, gd, dev)
    pool = pkv.KVPool(k_pool, v_pool, wl.BF16, d, device_status=torch.zeros(1, dtype=torch.int32, device=dev))
    gen = wl.generator(431 + 6 + rank)
    perm = torch.randperm(N, generator=gen).to(torch.int32)
    src = perm[:n_copy].contiguous()
    dst = perm[n_copy:2 * n_copy].contiguous()
    out_ids = perm[2 * n_copy:2 * n_copy + n_swap].contiguous()
    in_ids = perm[2 * n_copy + n_swap:2 * n_copy + 2 * n_swap].contiguous()
    d_src, d_dst, d_out, d_in = (t.to(dev) for t in (src, dst, out_ids, in_ids))
    per_block = pkv.kv_swap_bytes_per_block(pool)
    host = torch.empty(n_swap, per_block, dtype=torch.uint8).pin_memory()
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0][0].record()
        pkv.kv_copy_blocks(pool, d_src, d_dst)
        if ev is not None:
            ev[0][1].record()
            ev[1][0].record()
        pkv.kv_swap_out(pool, d_out, host)
        if ev is not None:
            ev[1][1].record()
            ev[2][0].record()
        pkv.kv_swap_in(pool, d_in, host)
        if ev is not None:
            ev[2][1].record()

    # end to end: the block ids come from pinned host memory every step
    h_ids = torch.cat([src, dst, out_ids, in_ids]).pin_memory()
    d_ids = torch.empty_like(h_ids, device=dev)

    def e2e_step():
        d_ids.copy_(h_ids, non_blocking=True)
        pkv.kv_copy_blocks(pool, d_ids[:n_copy], d_ids[n_copy:2 * n_copy])
        pkv.kv_swap_out(pool, d_ids[2 * n_copy:2 * n_copy + n_swap], host)
        pkv.kv_swap_in(pool, d_ids[2 * n_copy + n_swap:], host)

    copied = n_copy * per_block
    swapped = n_swap * per_block
    peaks, kind = measured_peaks()
    info = dict(
        config={"workload": args.workload if L == cfg["layers"] else f"{args.workload} ({L} layers)",
                "description": cfg["desc"], "layers": L, "kv_heads": H_kv, "head_dim": d,
                "kv_dtype": "bf16", "pool_blocks_per_layer": N, "copy_pairs": n_copy, "swapped_blocks": n_swap,
                "bytes_per_block": per_block, "parallelism": "replicas",
                "l2": f"inputs larger than L2: each copy call moves {copied / 1e9:.2f} GB"},
        kv_bytes_per_step=copied + 2 * swapped, seq_tokens_per_step=(n_copy + 2 * n_swap) * 16 * L, layers=L,
        roofline=dict(bound="hbm", kernel="kv_copy_blocks", alg_bytes=2 * copied, call_index=0,
                      peak=float(peaks["hbm_gbs"]), unit="GB/s",
                      peak_source=f"{kind} (MEASURED_PEAKS.json hbm_gbs; a copy reads and writes each byte)",
                      traffic=scaled(kernel_traffic("copy_blocks", BLOCKS_SRCS), L / cfg["layers"]),
                      swap_bytes=swapped),
        launches_per_step=3, dtype="u8", h2d=h_ids.numel() * 4 + swapped, d2h=swapped, calls_per_step=3)
    return step, e2e_step, info, pool


def max_over_ranks(value: float, device) -> float:
    """The largest `value` over all ranks: the slowest replica bounds the whole job.  The
    identity without a process group (one GPU)."""
    if not torch.distributed.is_available() or not torch.distributed.is_initialized():
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_step: float, steps: int, world: int, elapsed_ms: float) -> float:
    """Whole-job units per second: every rank processes units_per_step each step (weak
    scaling, independent replicas), all ranks within elapsed_ms (the max over ranks)."""
    return units_per_step * steps * world / (elapsed_ms * 1e-3)


def time_steps(step, n_steps, per_step_calls, dev, world, flush=None):
    """Device time of n_steps steps (CUDA events on the launching stream).  With `flush`, it
    runs before every step outside the timed events (an L2 flush), and the time is the sum of
    the steps' own event intervals."""
    timed = Timed(n_steps, per_step_calls)
    stream = torch.cuda.current_stream(dev)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    if flush is None:
        t0, t1 = mk(), mk()
        t0.record(stream)
        for s in range(n_steps):
            step(timed.ev[s])
        t1.record(stream)
        torch.cuda.synchronize(dev)
        ms = t0.elapsed_time(t1)
    else:
        marks = [(mk(), mk()) for _ in range(n_steps)]
        for s in range(n_steps):
            flush()
            marks[s][0].record(stream)
            step(timed.ev[s])
            marks[s][1].record(stream)
        torch.cuda.synchronize(dev)
        ms = sum(a.elapsed_time(b) for a, b in marks)
    if world > 1:
        torch.distributed.barrier()
        ms = max_over_ranks(ms, dev)
    return ms, timed


class L2Flush:
    """Writes a buffer twice the size of the L2 (126 MB on B200), so no input of the next step
    is still cached, then reads it back: the L2 is left holding clean lines, so the timed step
    does not also pay for writing the flush's dirty lines back to HBM."""

    def __init__(self, dev, nbytes=256 << 20):
        self.buf = torch.empty(nbytes // 4, dtype=torch.int32, device=dev)
        self.sink = None
        self.n = 0

    def __call__(self):
        self.n += 1
        self.buf.fill_(self.n)
        self.sink = self.buf.sum(dtype=torch.int64)


def run_gpu(args):
    from paged_kv_cache_431_b200 import pkv

    rank, local_rank, world = dist_env()
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local_rank if world > 1 else 0)
    torch.cuda.set_device(dev)
    cfg = WORKLOADS[args.workload]
    builder = {"prefix": build_prefix_chunk, "blocks": build_blocks}.get(cfg["kind"], build_decode)
    step, e2e_step, info, pool = builder(args, cfg, dev, rank)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if pkv.read_device_status(pool):
        raise RuntimeError("device status set during warm-up")
    graph = tgraph = None
    gtimed = Timed(1, info["calls_per_step"], external=True)
    if args.graph:   # the whole step (every layer's append and attention) as one CUDA graph; a
        # second capture adds event nodes around the dominant calls, for their durations only
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        tgraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(tgraph):
            step(gtimed.ev[0])
        for _ in range(args.warmup):
            graph.replay()
            tgraph.replay()
        torch.cuda.synchronize(dev)

    # single-layer decode workloads re-read inputs that could still sit in L2 from the step
    # before: flush it between timed steps (the 80-layer step cycles over pools >> L2)
    flush = L2Flush(dev) if info.get("flush_l2") else None
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    # per-call durations (the roofline): events around each call of eager steps; with a graph,
    # also the event nodes of a second, evented capture of the step (one replay at a time, read
    # after each), reported beside them
    eager_ms, timed = time_steps(step, args.steps, info["calls_per_step"], dev, world, flush)
    call_ms = timed.call_ms()
    graph_call_ms = None
    elapsed_ms = eager_ms
    if graph is not None:
        elapsed_ms, _ = time_steps(lambda ev=None: graph.replay(), args.steps, 1, dev, world, flush)
        graph_call_ms = []
        for _ in range(args.steps):
            if flush is not None:
                flush()
            tgraph.replay()
            torch.cuda.synchronize(dev)
            graph_call_ms += gtimed.call_ms()
    clk = clocks.stop()
    if pkv.read_device_status(pool):
        raise RuntimeError("device status set during timing")
    info["config"]["step_timing"] = ("CUDA-graph replays of one captured step" if graph is not None
                                     else "eager launches") + f"; eager steps {eager_ms / args.steps:.4f} ms"
    info["config"]["call_timing"] = ("events around each call of eager steps; graph_launch_us: event nodes "
                                     "around each call in a second, evented capture of the step (the graph "
                                     "timed for `value` has none)" if graph is not None
                                     else "events around each call of eager steps")

    # end to end through the same calls with host buffers
    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize(dev)
    e2e_ms, _ = time_steps(lambda ev=None: e2e_step(), args.steps, 1, dev, world, flush)

    ms_per_step = elapsed_ms / args.steps
    value = job_throughput(info["kv_bytes_per_step"], args.steps, world, elapsed_ms) / 1e9
    e2e_value = job_throughput(info["kv_bytes_per_step"], args.steps, world, e2e_ms) / 1e9
    rf = info["roofline"]
    if rf["bound"] == "hbm":
        cpk = info["calls_per_step"]
        sel = call_ms if "call_index" not in rf else call_ms[rf["call_index"]::cpk]
        avg_s = statistics.mean(sel) * 1e-3
        achieved = rf["alg_bytes"] / avg_s / 1e9
        roofline = {"bound": "hbm", "kernel": rf["kernel"], "achieved": round(achieved, 1), "peak": rf["peak"],
                    "unit": "GB/s", "frac": round(achieved / rf["peak"], 4), "peak_source": rf["peak_source"],
                    "traffic": rf["traffic"], "algorithmic_bytes_per_launch": rf["alg_bytes"],
                    "avg_launch_us": round(avg_s * 1e6, 2)}
        if graph_call_ms:
            gsel = graph_call_ms if "call_index" not in rf else graph_call_ms[rf["call_index"]::cpk]
            roofline["graph_launch_us"] = round(statistics.mean(gsel) * 1e3, 2)
        if "swap_bytes" in rf:   # host-link moves: swap-out then swap-in calls
            for name, i in (("swap_out_gbs", 1), ("swap_in_gbs", 2)):
                roofline[name] = round(rf["swap_bytes"] / (statistics.mean(call_ms[i::cpk]) * 1e-3) / 1e9, 2)
    else:
        ci = rf["call_index"]
        per_call = [call_ms[i] for i in range(ci, len(call_ms), info["calls_per_step"])]
        dec_calls = [call_ms[i] for i in range(0, len(call_ms), info["calls_per_step"])]
        avg_s = statistics.mean(per_call) * 1e-3
        achieved = rf["alg_flops"] / avg_s / 1e12
        dec_s = statistics.mean(dec_calls) * 1e-3
        roofline = {"bound": "tensor", "kernel": rf["kernel"], "achieved": round(achieved, 1), "peak": rf["peak"],
                    "unit": "TFLOP/s", "frac": round(achieved / rf["peak"], 4), "peak_source": rf["peak_source"],
                    "traffic": rf["traffic"], "algorithmic_flops_per_launch": rf["alg_flops"],
                    "avg_launch_us": round(avg_s * 1e6, 2),
                    "decode_call_us": round(dec_s * 1e6, 2),
                    "decode_logical_gbs": round(rf["decode_alg_bytes"] / dec_s / 1e9, 1)}
        if graph_call_ms:
            roofline["graph_launch_us"] = round(statistics.mean(graph_call_ms[ci::info["calls_per_step"]]) * 1e3, 2)

    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": info["dtype"], "data": "synthetic",
        "config": info["config"],
        "seq_tokens_per_s_per_layer": round(job_throughput(info["seq_tokens_per_step"] / info["layers"],
                                                           args.steps, world, elapsed_ms)),
        "pct_of_8tbs_nominal": round(100 * value / world / 8000.0, 1),
        "roofline": roofline,
        "e2e": {"value": round(e2e_value, 1), "unit": "GB/s", "ms_per_step": round(e2e_ms / args.steps, 4),
                "h2d_bytes_per_step": info["h2d"], "d2h_bytes_per_step": info["d2h"]},
        "gpu_launches": args.steps * info["launches_per_step"],
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_oracle(args.workload, budget_s=args.cpu_seconds)
        try:
            every = cpu_oracle_all_cores(args.workload, budget_s=args.cpu_seconds / 2)
        except Exception as e:   # the all-cores figure is extra; never lose the line over it
            every = {"error": repr(e)}
        if every is not None:
            res["cpu_baseline"]["all_cores"] = every
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


# ------------------------------------------------------ CPU oracle timing --

def cpu_oracle(workload, budget_s=12.0, per_step=None, steps=None, warmup=0):
    """The oracle as it stands (single-threaded C, fp64) on whole sequences of one layer of
    the same workload, generated on the host with the same recipe.  With `per_step` it
    runs warmup + steps steps of `per_step` sequences; otherwise sequences in order until
    about `budget_s` seconds.  Returns (result dict, list of per-step seconds)."""
    import oracle

    oracle.build()
    cfg = WORKLOADS[workload]
    if cfg["kind"] == "blocks":
        return cpu_oracle_blocks(cfg, workload, budget_s, per_step, steps, warmup)
    H_q, H_kv, d, dt = cfg["H_q"], cfg["H_kv"], cfg["d"], cfg["dtype"]
    gen = wl.generator(431 + 3)
    if cfg["kind"] == "prefix":
        ctx = (4000 + 200 + torch.randint(0, 301, (cfg["B"],), generator=gen, dtype=torch.int32) + 1)
    else:
        ctx = make_lens(cfg["lens"], gen, cfg["B"])
    gh = wl.generator(431 + 300)
    quant = dt in (wl.INT8, wl.FP8, wl.INT4)
    total_s, total_kv, total_tok, seqs, step_secs = 0.0, 0, 0, 0, []
    n_steps = (warmup + steps) if per_step else 10 ** 9
    b = 0
    for s in range(n_steps):
        ids = [(b + i) % len(ctx) for i in range(per_step or 1)]
        b += len(ids)
        step_s = 0.0
        for sid in ids:
            n = int(ctx[sid])
            nb = wl.ceil_div(n, 16)
            table = torch.arange(nb, dtype=torch.int32).view(1, nb)
            opool = oracle.Pool(nb, H_kv, d, dt if quant else dt)
            k, v = wl.kv_source(n, H_kv, d, gh) if quant else (wl.normal((n, H_kv, d), torch.bfloat16, gh),
                                                              wl.normal((n, H_kv, d), torch.bfloat16, gh))
            oracle.kv_append(opool, k, v, oracle.BF16, np.arange(n, dtype=np.int32))
            q = wl.normal((1, H_q, d), torch.bfloat16, gh)
            t0 = time.perf_counter()
            window = cfg.get("window", 0)
            oracle.paged_decode(opool, q, oracle.BF16, table, [n], np.float32(d ** -0.5), window=window)
            step_s += time.perf_counter() - t0
            if s >= warmup:
                seen = min(n, window) if window else n
                total_kv += int(seen * 2 * H_kv * d * ELEM_BYTES[dt])
                total_tok += seen
                seqs += 1
        if s >= warmup:
            total_s += step_s
            step_secs.append(step_s)
        if not per_step and total_s >= budget_s:
            break
    res = {"value": round(total_kv / total_s / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
           "seq_tokens_per_s_per_layer": round(total_tok / total_s),
           "sample": f"{seqs} whole sequence(s) of one layer of the {workload} workload ({total_tok} cached "
                     f"tokens), fp64 C oracle, single thread, {total_s:.1f} s"}
    return (res, step_secs) if per_step else res


def cpu_oracle_all_cores(workload, budget_s=6.0, max_threads=64, mem_budget=8e9):
    """The same oracle calls from T concurrent host threads (ctypes releases the GIL while the C
    oracle runs), one whole sequence of the workload per thread; T = the cores this process may
    run on, capped by `max_threads` and by a host-memory budget.  Aggregate K/V bytes of the
    completed calls over the wall time from the common start until the last call in flight at
    `budget_s` ends.
    Returns None for the block-move workload, or a dict with an "error" key if a thread failed."""
    import threading

    import oracle

    cfg = WORKLOADS[workload]
    if cfg["kind"] == "blocks":
        return None
    oracle.build()
    oracle.lib()
    H_q, H_kv, d, dt = cfg["H_q"], cfg["H_kv"], cfg["d"], cfg["dtype"]
    gen = wl.generator(431 + 3)
    if cfg["kind"] == "prefix":
        ctx = (4000 + 200 + torch.randint(0, 301, (cfg["B"],), generator=gen, dtype=torch.int32) + 1)
    else:
        ctx = make_lens(cfg["lens"], gen, cfg["B"])
    quant = dt in (wl.INT8, wl.FP8, wl.INT4)
    window = cfg.get("window", 0)
    # host bytes per thread: the oracle's pool plus the bf16 K and V source it is built from
    per_seq = float(ctx.float().max()) * H_kv * d * (2 * ELEM_BYTES[dt] + 4)
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    T = max(1, min(cores, max_threads, int(mem_budget // per_seq)))
    stop = threading.Event()
    start = threading.Barrier(T + 1, timeout=600)
    done_bytes = [0] * T
    errors = []

    def worker(i):
        try:
            n = int(ctx[i % len(ctx)])
            g = wl.generator(431 + 700 + i)
            nb = wl.ceil_div(n, 16)
            table = torch.arange(nb, dtype=torch.int32).view(1, nb)
            opool = oracle.Pool(nb, H_kv, d, dt)
            k, v = wl.kv_source(n, H_kv, d, g) if quant else (wl.normal((n, H_kv, d), torch.bfloat16, g),
                                                             wl.normal((n, H_kv, d), torch.bfloat16, g))
            oracle.kv_append(opool, k, v, oracle.BF16, np.arange(n, dtype=np.int32))
            del k, v
            q = wl.normal((1, H_q, d), torch.bfloat16, g)
            seen = min(n, window) if window else n
            start.wait()
            while not stop.is_set():
                oracle.paged_decode(opool, q, oracle.BF16, table, [n], np.float32(d ** -0.5), window=window)
                done_bytes[i] += seen * 2 * H_kv * d * ELEM_BYTES[dt]
        except Exception as e:   # a failed thread ends the measurement, not the bench
            errors.append(repr(e))
            start.abort()

    prev_threads = torch.get_num_threads()
    torch.set_num_threads(1)   # one host core per oracle thread, also while generating
    threads = [threading.Thread(target=worker, args=(i,), daemon=True) for i in range(T)]
    try:
        for t in threads:
            t.start()
        try:
            start.wait()
        except threading.BrokenBarrierError:
            stop.set()
            return {"error": errors[0] if errors else "threads did not start"}
        t0 = time.perf_counter()
        time.sleep(budget_s)
        stop.set()
        for t in threads:
            t.join(timeout=600)
        wall = time.perf_counter() - t0
    finally:
        stop.set()
        torch.set_num_threads(prev_threads)
    if errors or any(t.is_alive() for t in threads):
        return {"error": errors[0] if errors else "a thread did not finish"}
    total = sum(done_bytes)
    return {"value": round(total / wall / 1e9, 4), "unit": "GB/s", "cores": T,
            "sample": f"{T} threads, one whole sequence of one layer each, fp64 C oracle called concurrently; "
                      f"{total / 1e9:.2f} GB of K/V in {wall:.1f} s"}


def cpu_oracle_waves(workload, steps, warmup, max_threads=64, mem_budget=8e9):
    """--impl reference on the host's cores: each step is one wave of T whole sequences of one
    layer, one per host thread (T = the cores this process may run on, capped by `max_threads`
    and a host-memory budget), the C oracle called concurrently (ctypes releases the GIL).  A
    step's time runs from the moment every thread holds its generated sequence until the last
    call returns.  Returns (result dict, list of per-step seconds)."""
    import threading

    import oracle

    cfg = WORKLOADS[workload]
    oracle.build()
    oracle.lib()
    H_q, H_kv, d, dt = cfg["H_q"], cfg["H_kv"], cfg["d"], cfg["dtype"]
    gen = wl.generator(431 + 3)
    if cfg["kind"] == "prefix":
        ctx = (4000 + 200 + torch.randint(0, 301, (cfg["B"],), generator=gen, dtype=torch.int32) + 1)
    else:
        ctx = make_lens(cfg["lens"], gen, cfg["B"])
    quant = dt in (wl.INT8, wl.FP8, wl.INT4)
    window = cfg.get("window", 0)
    per_seq = float(ctx.float().max()) * H_kv * d * (2 * ELEM_BYTES[dt] + 4)
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    T = max(1, min(cores, max_threads, int(mem_budget // per_seq)))
    step_secs, total_kv, total_tok = [], 0, 0
    prev_threads = torch.get_num_threads()
    torch.set_num_threads(1)
    try:
        for s in range(warmup + steps):
            ready = threading.Barrier(T + 1, timeout=900)
            finished = threading.Barrier(T + 1, timeout=900)
            seen = [0] * T
            errors = []

            def worker(i):
                try:
                    sid = (s * T + i) % len(ctx)
                    n = int(ctx[sid])
                    g = wl.generator(431 + 900 + s * T + i)
                    nb = wl.ceil_div(n, 16)
                    table = torch.arange(nb, dtype=torch.int32).view(1, nb)
                    opool = oracle.Pool(nb, H_kv, d, dt)
                    k, v = wl.kv_source(n, H_kv, d, g) if quant else (wl.normal((n, H_kv, d), torch.bfloat16, g),
                                                                     wl.normal((n, H_kv, d), torch.bfloat16, g))
                    oracle.kv_append(opool, k, v, oracle.BF16, np.arange(n, dtype=np.int32))
                    del k, v
                    q = wl.normal((1, H_q, d), torch.bfloat16, g)
                    ready.wait()
                    oracle.paged_decode(opool, q, oracle.BF16, table, [n], np.float32(d ** -0.5), window=window)
                    seen[i] = min(n, window) if window else n
                    finished.wait()
                except Exception as e:
                    errors.append(repr(e))
                    ready.abort()
                    finished.abort()

            threads = [threading.Thread(target=worker, args=(i,), daemon=True) for i in range(T)]
            for t in threads:
                t.start()
            try:   # a failed worker aborts both barriers: report its own exception, not the barrier's
                ready.wait()
                t0 = time.perf_counter()
                finished.wait()
                dt_s = time.perf_counter() - t0
            except threading.BrokenBarrierError:
                dt_s = None
            for t in threads:
                t.join(timeout=60)
            if errors or dt_s is None:
                raise RuntimeError(errors[0] if errors else "a host thread did not reach the barrier")
            if s >= warmup:
                step_secs.append(dt_s)
                total_tok += sum(seen)
                total_kv += sum(seen) * 2 * H_kv * d * ELEM_BYTES[dt]
    finally:
        torch.set_num_threads(prev_threads)
    total_s = sum(step_secs)
    res = {"value": round(total_kv / total_s / 1e9, 4), "unit": "GB/s", "cores": T, "kind": "oracle",
           "seq_tokens_per_s_per_layer": round(total_tok / total_s),
           "sample": f"{steps} step(s) of {T} whole sequences of one layer of the {workload} workload, one per "
                     f"host thread, fp64 C oracle called concurrently ({total_tok} cached tokens, {total_s:.1f} s)"}
    return res, step_secs


def cpu_oracle_blocks(cfg, workload, budget_s, per_step=None, steps=None, warmup=0):
    """The oracle's block copy (numpy byte moves, every layer) on a bounded sample of pairs
    from a small pool of the same shape."""
    import oracle

    L, H_kv, d = cfg["layers"], cfg["H_kv"], cfg["d"]
    n_blocks, pairs = 64, per_step or 16
    rng = np.random.default_rng(431)
    pools = []
    for _ in range(L):
        pl = oracle.Pool(n_blocks, H_kv, d, oracle.BF16)
        pl.k[...] = rng.integers(0, 256, pl.k.shape, dtype=np.uint8)
        pl.v[...] = rng.integers(0, 256, pl.v.shape, dtype=np.uint8)
        pools.append(pl)
    per_block = L * 2 * H_kv * 16 * d * 2
    total_s, moved, step_secs, s = 0.0, 0, [], 0
    n_steps = (warmup + steps) if per_step else 10 ** 9
    while s < n_steps:
        perm = rng.permutation(n_blocks)
        t0 = time.perf_counter()
        oracle.copy_blocks(pools, perm[:pairs], perm[pairs:2 * pairs])
        dt = time.perf_counter() - t0
        if s >= warmup:
            total_s += dt
            moved += pairs * per_block
            step_secs.append(dt)
        s += 1
        if not per_step and total_s >= budget_s:
            break
    res = {"value": round(moved / total_s / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
           "seq_tokens_per_s_per_layer": round(moved / per_block * 16 / total_s),
           "sample": f"{len(step_secs)} x {pairs} block copies of the {workload} shape ({L} layers, numpy), "
                     f"single thread, {total_s:.1f} s"}
    return (res, step_secs) if per_step else res


def run_reference(args):
    """--impl reference: the CPU oracle on this host's cores, same workload, metric and unit;
    each step is a bounded sample: one wave of whole sequences of one layer, one per host
    thread (--ref-threads 1: --ref-seqs sequences on one thread)."""
    rank, _, world = dist_env()
    if rank != 0:
        return
    if args.ref_threads == 1 or WORKLOADS[args.workload]["kind"] == "blocks":
        cpu, secs = cpu_oracle(args.workload, per_step=max(1, args.ref_seqs), steps=args.steps, warmup=args.warmup)
    else:
        cpu, secs = cpu_oracle_waves(args.workload, steps=args.steps, warmup=args.warmup,
                                     max_threads=args.ref_threads if args.ref_threads > 0 else 64)
    res = {"metric": METRIC, "value": cpu["value"], "unit": "GB/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(1e3 * statistics.mean(secs), 2), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None,
           "dtype": "u8" if WORKLOADS[args.workload]["kind"] == "blocks" else "f64", "data": "synthetic",
           "impl": "reference",
           "config": {"workload": args.workload, "description": WORKLOADS[args.workload]["desc"]},
           "seq_tokens_per_s_per_layer": cpu["seq_tokens_per_s_per_layer"],
           "cpu_baseline": cpu,
           "e2e": {"value": cpu["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="gqa70b", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--pool-fraction", type=float, default=0.4,
                    help="fraction of free HBM used for distinct per-layer pools")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-seqs", type=int, default=2,
                    help="--impl reference with --ref-threads 1: whole sequences per step")
    ap.add_argument("--ref-threads", type=int, default=0,
                    help="--impl reference: host threads calling the oracle concurrently, one sequence "
                         "each per step (0: every usable core, at most 64; 1: one thread)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=0,
                    help="blocks: layers of the pool (default 80); fewer for counter captures on a small pool")
    ap.add_argument("--partition", type=int, default=0,
                    help="split-K partition size in tokens (0: chosen by the library)")
    ap.add_argument("--decode-form", default="cascade", choices=["cascade", "plain"],
                    help="prefix_chunk: decode the shared-prefix batch in the cascade form or plainly")
    ap.add_argument("--graph", type=int, default=1, choices=[0, 1],
                    help="1: time the device-resident steps as replays of one CUDA-graph-captured step")
    ap.add_argument("--batch", type=int, default=0,
                    help="decode workloads: sequences per call instead of the workload's own batch (small "
                         "cases for profiler captures; the JSON line is then not the named workload)")
    ap.add_argument("--engine", type=int, default=0, choices=[0, 1, 2, 3],
                    help="decode engine: 0/1 tensor cores, 2 CUDA-core packed FMA, 3 CUDA-core FMA")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
