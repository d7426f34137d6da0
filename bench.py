"""Benchmark: paged GQA decode over a paged KV cache on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload gqa70b|llama8b|prefix_chunk|quant_int8|...]
    python bench.py --impl reference ...      # the CPU oracle on this host's cores

A step is one pass of the hot path over one batch: for every layer, kv_append of each
sequence's new token followed by paged_decode_attn over the whole cached context.
Default workload: the 70B-class GQA decode -- 80 layers, 64 query heads, 8 KV heads,
head dim 128, bf16 K/V, 170 sequences with contexts ~ N(3000, 400) clipped to
[1024, 4096], block tables permuted over a pool of 170 x 256 blocks per layer.

Prints ONE JSON line (rank 0).  `value` is KV GB/s (algorithmic K/V bytes read by the
decode calls of all ranks / the max-over-ranks device time of the K timed steps).
With --gpus N > 1 (torchrun), every rank runs an independent replica: the path has no
data exchange, so there is no collective beyond the timing barrier.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_431_b200 import workloads as wl  # noqa: E402

METRIC = "paged GQA decode: KV HBM GB/s (% of ~8 TB/s peak); seq-tokens/s per layer"
PROFILES = os.path.join(ROOT, "profiles")


# ------------------------------------------------------------------ utils --

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join(ROOT, "gpurun_out", f"clocks_rank{gpu_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
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
        sm, mx, reasons = [], 0.0, set()
        for line in open(self.path):
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


def kernel_traffic(kernel_key: str, src_files):
    """DRAM bytes per launch from a committed ncu summary, only if the kernel sources are
    unchanged since the capture (their hash is stored with the figure)."""
    path = os.path.join(PROFILES, "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel_key)
    except Exception:
        return None
    if not rec:
        return None
    h = hashlib.sha256()
    for s in src_files:
        with open(os.path.join(ROOT, s), "rb") as f:
            h.update(f.read())
    if rec.get("src_sha256") != h.hexdigest():
        return None
    return rec.get("bytes_per_launch")


def source_hash(src_files):
    h = hashlib.sha256()
    for s in src_files:
        with open(os.path.join(ROOT, s), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


DECODE_SRCS = ["paged_kv_cache_431_b200/csrc/decode.cu", "paged_kv_cache_431_b200/csrc/common.cuh"]


# -------------------------------------------------------------- workloads --

WORKLOADS = {
    "gqa70b": dict(layers=80, B=170, H_q=64, H_kv=8, d=128, dtype=wl.BF16, width=256,
                   desc="70B-class GQA decode: 80 layers, H_q 64, H_kv 8, d 128, bf16, B 170, "
                        "ctx ~ N(3000, 400) clipped to [1024, 4096], pool 170 x 256 blocks per layer"),
    "llama8b": dict(layers=1, B=64, H_q=32, H_kv=8, d=128, dtype=wl.BF16, width=256,
                    desc="Llama-3-8B-shaped decode, 1 layer: H_q 32, H_kv 8, d 128, bf16, B 64, "
                         "ctx ~ U[512, 4096], pool for 64 x 4096 tokens"),
}


def make_lens(name, gen, B):
    if name == "gqa70b":
        return wl.gqa70b_lens(gen, B)
    if name == "llama8b":
        return wl.llama8b_lens(gen, B)
    raise ValueError(name)


def algorithmic_bytes(ctx_lens, B, H_q, H_kv, d, elem_bytes):
    """Bytes a decode call must move: every cached K and V element once, plus q, out,
    the used block-table entries and the context lengths."""
    sum_ctx = int(ctx_lens.sum())
    kv = sum_ctx * 2 * H_kv * d * elem_bytes
    blocks = int(sum(wl.ceil_div(int(n), 16) for n in ctx_lens))
    other = B * H_q * d * elem_bytes + B * H_q * d * 4 + blocks * 4 + B * 4
    return kv, kv + other


# ------------------------------------------------------------- GPU arm --

def run_gpu(args):
    from paged_kv_cache_431_b200 import pkv

    rank, local_rank, world = dist_env()
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local_rank if world > 1 else 0)
    torch.cuda.set_device(dev)
    cfg = WORKLOADS[args.workload]
    L, B, H_q, H_kv, d, dt = cfg["layers"], cfg["B"], cfg["H_q"], cfg["H_kv"], cfg["d"], cfg["dtype"]
    tdt = wl.TORCH_DTYPE[dt]
    elem = 2

    gen = wl.generator(431 + 3 + rank)
    ctx = make_lens(args.workload, gen, B)
    N = B * cfg["width"]
    paging = wl.allocate(ctx, N, cfg["width"], gen)
    per_layer_pool = 2 * N * H_kv * 16 * d * elem
    free, _ = torch.cuda.mem_get_info(dev)
    L_phys = max(1, min(L, int(args.pool_fraction * free // per_layer_pool)))
    gd = wl.generator(431 + 100 + rank, dev)
    k_pool = torch.empty(L_phys, N, H_kv, 16, d, dtype=tdt, device=dev)
    v_pool = torch.empty_like(k_pool)
    for l in range(L_phys):
        k_pool[l] = wl.normal((N, H_kv, 16, d), tdt, gd, dev)
        v_pool[l] = wl.normal((N, H_kv, 16, d), tdt, gd, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    pool = pkv.KVPool(k_pool, v_pool, dt, d, device_status=status)

    tables = paging.tables.to(dev)
    ctx_d = ctx.to(dev)
    max_ctx = int(ctx.max())
    slots = wl.slots_for(paging.tables, range(B), (ctx - 1).long()).to(dev)   # each step's new token
    q = wl.normal((L, B, H_q, d), tdt, gd, dev)
    k_new = wl.normal((L, B, H_kv, d), tdt, gd, dev)
    v_new = wl.normal((L, B, H_kv, d), tdt, gd, dev)
    out = torch.empty(L, B, H_q, d, dtype=torch.float32, device=dev)
    ws_bytes = pkv.paged_decode_workspace_bytes(pool, B, H_q, max_ctx)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        for l in range(L):
            lp = l % L_phys
            pkv.kv_append(pool, lp, k_new[l], v_new[l], slots)
            if ev is not None:
                ev[l][0].record(stream)
            pkv.paged_decode_attn(pool, lp, q[l], tables, ctx_d, d ** -0.5, max_ctx, out=out[l], workspace=ws)
            if ev is not None:
                ev[l][1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if pkv.read_device_status(pool):
        raise RuntimeError("device status set during warm-up")

    kv_bytes, alg_bytes = algorithmic_bytes(ctx, B, H_q, H_kv, d, elem)
    call_events = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in range(L)]
                   for _ in range(args.steps)]
    clocks = ClockSampler(dev.index)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for s in range(args.steps):
        step(call_events[s])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    elapsed_ms = t0.elapsed_time(t1)
    call_ms = [e0.elapsed_time(e1) for st in call_events for (e0, e1) in st]
    if world > 1:
        t = torch.tensor([elapsed_ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        elapsed_ms = float(t.item())
    if pkv.read_device_status(pool):
        raise RuntimeError("device status set during timing")

    ms_per_step = elapsed_ms / args.steps
    total_kv = kv_bytes * L * args.steps * world
    value = total_kv / (elapsed_ms * 1e-3) / 1e9
    seq_tokens_per_s_layer = int(ctx.sum()) * L * args.steps * world / (elapsed_ms * 1e-3) / L
    peak, peak_kind = measured_peaks()
    avg_call_s = statistics.mean(call_ms) * 1e-3
    achieved = alg_bytes / avg_call_s / 1e9
    traffic = kernel_traffic(f"decode_mma16_{args.workload}", DECODE_SRCS)
    launches_per_layer = 2 + (1 if ws_bytes > 0 else 0)

    e2e = run_e2e(args, pool, L, L_phys, B, H_q, H_kv, d, tdt, paging, ctx, max_ctx, kv_bytes, world, dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(pool, paging, ctx, H_q, H_kv, d, dt, q[0], budget_s=args.cpu_seconds)

    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "description": cfg["desc"], "layers": L, "batch": B,
                   "q_heads": H_q, "kv_heads": H_kv, "head_dim": d, "sum_ctx": int(ctx.sum()),
                   "physical_layer_pools": L_phys, "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2: each decode call reads {kv_bytes / 1e9:.2f} GB of K/V",
                   "partition_tokens": "auto"},
        "seq_tokens_per_s_per_layer": round(seq_tokens_per_s_layer),
        "pct_of_8tbs_nominal": round(100 * value / world / 8000.0, 1),
        "roofline": {"bound": "hbm", "kernel": "paged_decode_attn (main + split-K merge)",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)",
                     "traffic": traffic, "algorithmic_bytes_per_launch": alg_bytes,
                     "avg_launch_us": round(avg_call_s * 1e6, 2)},
        "e2e": e2e,
        "gpu_launches": args.steps * L * launches_per_layer,
        "clocks": clk,
    }
    if cpu is not None:
        res["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def run_e2e(args, pool, L, L_phys, B, H_q, H_kv, d, tdt, paging, ctx, max_ctx, kv_bytes, world, dev):
    """The same step through the C-ABI with host buffers: every step copies each layer's
    q and new K/V (and the block tables, context lengths and slots) from pinned host
    memory and reads every layer's attention output back.  Copies run on two copy
    streams overlapped with the kernels of neighbouring layers."""
    from paged_kv_cache_431_b200 import pkv

    g = wl.generator(999)
    hq = wl.normal((L, B, H_q, d), tdt, g).pin_memory()
    hk = wl.normal((L, B, H_kv, d), tdt, g).pin_memory()
    hv = wl.normal((L, B, H_kv, d), tdt, g).pin_memory()
    htab = paging.tables.clone().pin_memory()
    hctx = ctx.clone().pin_memory()
    hslots = wl.slots_for(paging.tables, range(B), (ctx - 1).long()).pin_memory()
    hout = torch.empty(L, B, H_q, d, dtype=torch.float32).pin_memory()
    dq, dk, dv = (torch.empty(t.shape, dtype=t.dtype, device=dev) for t in (hq, hk, hv))
    dtab, dctx, dslots = (torch.empty(t.shape, dtype=t.dtype, device=dev) for t in (htab, hctx, hslots))
    dout = torch.empty(hout.shape, dtype=torch.float32, device=dev)
    ws = torch.empty(max(pkv.paged_decode_workspace_bytes(pool, B, H_q, max_ctx), 16), dtype=torch.uint8, device=dev)
    comp = torch.cuda.current_stream(dev)
    h2d = torch.cuda.Stream(dev)
    d2h = torch.cuda.Stream(dev)

    def step():
        start = torch.cuda.Event()
        start.record(comp)
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
            comp.wait_event(ready[l])
            pkv.kv_append(pool, l % L_phys, dk[l], dv[l], dslots)
            pkv.paged_decode_attn(pool, l % L_phys, dq[l], dtab, dctx, d ** -0.5, max_ctx, out=dout[l], workspace=ws)
            e = torch.cuda.Event()
            e.record(comp)
            done.append(e)
        with torch.cuda.stream(d2h):
            for l in range(L):
                d2h.wait_event(done[l])
                hout[l].copy_(dout[l], non_blocking=True)
        fin = torch.cuda.Event()
        fin.record(d2h)
        comp.wait_event(fin)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(comp)
    for _ in range(args.steps):
        step()
    t1.record(comp)
    torch.cuda.synchronize(dev)
    ms = t0.elapsed_time(t1)
    if world > 1:
        t = torch.tensor([ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    h2d_bytes = sum(t.numel() * t.element_size() for t in (hq, hk, hv, htab, hctx, hslots))
    d2h_bytes = hout.numel() * hout.element_size()
    value = kv_bytes * L * args.steps * world / (ms * 1e-3) / 1e9
    return {"value": round(value, 1), "unit": "GB/s", "ms_per_step": round(ms / args.steps, 4),
            "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes}


# ------------------------------------------------------ CPU oracle timing --

def oracle_decode_sample(k_host, v_host, dt, tables, ctx, q_host, seq_ids, H_q, d):
    """Run the oracle over the given sequences of one layer; returns (seconds, kv bytes)."""
    import oracle
    blocks, sub_t, sub_c = wl.compact_subset(tables, ctx, seq_ids)
    idx = torch.as_tensor(blocks, dtype=torch.long)
    kraw = k_host[idx].contiguous().view(torch.int16).numpy().view(np.uint8)
    vraw = v_host[idx].contiguous().view(torch.int16).numpy().view(np.uint8)
    opool = oracle.Pool(len(blocks), k_host.shape[1], d, dt, kraw, vraw)
    qs = q_host[seq_ids]
    t0 = time.perf_counter()
    oracle.paged_decode(opool, qs, dt, sub_t, sub_c, np.float32(d ** -0.5))
    sec = time.perf_counter() - t0
    kv = int(sub_c.sum()) * 2 * k_host.shape[1] * d * 2
    return sec, kv


def cpu_baseline(pool, paging, ctx, H_q, H_kv, d, dt, q_layer, budget_s=15.0):
    """The oracle as it stands (single-threaded C, fp64) on a bounded sample of one layer:
    whole sequences in order until about `budget_s` seconds of CPU work."""
    k_host = pool.k_data[0].cpu()
    v_host = pool.v_data[0].cpu()
    qh = q_layer.cpu()
    total_s, total_kv, total_tok, seqs = 0.0, 0, 0, 0
    for b in range(len(ctx)):
        sec, kv = oracle_decode_sample(k_host, v_host, dt, paging.tables, ctx, qh, [b], H_q, d)
        total_s += sec
        total_kv += kv
        total_tok += int(ctx[b])
        seqs += 1
        if total_s >= budget_s:
            break
    return {"value": round(total_kv / total_s / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "seq_tokens_per_s_per_layer": round(total_tok / total_s),
            "sample": f"{seqs} of {len(ctx)} sequences of one layer ({total_tok} cached tokens), "
                      f"fp64 C oracle, single thread, {total_s:.1f} s"}


def run_reference(args):
    """--impl reference: the CPU oracle on this host, same workload, metric and unit.
    Each step is a bounded sample: a few whole sequences of one layer."""
    rank, _, world = dist_env()
    if rank != 0:
        return
    import oracle
    cfg = WORKLOADS[args.workload]
    B, H_q, H_kv, d, dt = cfg["B"], cfg["H_q"], cfg["H_kv"], cfg["d"], cfg["dtype"]
    tdt = wl.TORCH_DTYPE[dt]
    oracle.build()
    gen = wl.generator(431 + 3)
    ctx = make_lens(args.workload, gen, B)
    N = B * cfg["width"]
    paging = wl.allocate(ctx, N, cfg["width"], gen)
    per_step = max(1, args.ref_seqs)
    need = sorted(set(range(min(B, per_step * (args.steps + args.warmup)))))
    # only the blocks the sampled sequences reference are materialised on the host
    gh = wl.generator(431 + 200)
    k_host = torch.zeros(N, H_kv, 16, d, dtype=tdt)
    v_host = torch.zeros_like(k_host)
    for b in need:
        nb = wl.ceil_div(int(ctx[b]), 16)
        blk = paging.tables[b, :nb].long()
        k_host[blk] = wl.normal((nb, H_kv, 16, d), tdt, gh)
        v_host[blk] = wl.normal((nb, H_kv, 16, d), tdt, gh)
    q = wl.normal((B, H_q, d), tdt, gh)
    secs, kvs, toks = [], 0, 0
    for s in range(args.warmup + args.steps):
        ids = [(s * per_step + i) % B for i in range(per_step)]
        sec, kv = oracle_decode_sample(k_host, v_host, dt, paging.tables, ctx, q, ids, H_q, d)
        if s >= args.warmup:
            secs.append(sec)
            kvs += kv
            toks += int(ctx[ids].sum())
    total = sum(secs)
    value = kvs / total / 1e9
    sample = (f"{per_step} whole sequence(s) of one layer per step ({args.workload}), fp64 C oracle, "
              f"single thread")
    res = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 2), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
           "config": {"workload": args.workload, "description": cfg["desc"]},
           "seq_tokens_per_s_per_layer": round(toks / total),
           "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
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
    ap.add_argument("--ref-seqs", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
