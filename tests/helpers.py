"""Shared test plumbing: moving seeded inputs between the CUDA path and the oracle.

Nothing here computes attention or quantization; it only copies the same input bytes to
both sides and, for full-size workloads, gives the oracle a compact copy of just the
blocks a sampled subset of sequences references (block ids renumbered).
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle
from paged_kv_cache_431_b200 import workloads as wl
from paged_kv_cache_431_b200.workloads import compact_subset  # noqa: F401

TOL = 2e-3   # max |GPU - oracle| for fp32 attention outputs


def oracle_pool_from_tensors(k_pool, v_pool, dtype, k_scale=None, v_scale=None) -> oracle.Pool:
    """Oracle pool holding the bytes of one layer's [N, H_kv, 16, row] pool tensors."""
    N, H, _, _ = k_pool.shape
    d = k_pool.shape[-1] if dtype in (oracle.F16, oracle.BF16) else (
        k_pool.shape[-1] * (2 if dtype == oracle.INT4 else 1))

    def raw(t):
        t = t.detach().contiguous().cpu()
        if t.dtype in (torch.float16, torch.bfloat16):
            return t.view(torch.int16).numpy().view(np.uint8)
        return t.numpy().view(np.uint8)
    ks = None if k_scale is None else k_scale.detach().cpu().numpy()
    vs = None if v_scale is None else v_scale.detach().cpu().numpy()
    return oracle.Pool(N, H, d, dtype, raw(k_pool), raw(v_pool), ks, vs)


def oracle_subset_pool(k_pool, v_pool, dtype, blocks, k_scale=None, v_scale=None) -> oracle.Pool:
    idx = torch.as_tensor(blocks, dtype=torch.long, device=k_pool.device)
    ks = None if k_scale is None else k_scale[idx]
    vs = None if v_scale is None else v_scale[idx]
    return oracle_pool_from_tensors(k_pool[idx], v_pool[idx], dtype, ks, vs)


def max_abs_diff(gpu_out: torch.Tensor, ref: np.ndarray) -> float:
    g = gpu_out.detach().cpu().double().numpy()
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.isfinite(g).all(), "non-finite GPU output"
    return float(np.abs(g - ref).max()) if g.size else 0.0


def host_threads(cap: int = 64) -> int:
    """Host cores this process may run on (at most `cap`)."""
    n = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    return max(1, min(n, cap))


def oracle_decode_threaded(opool, q, q_dtype, tables, ctx_lens, scale, window: int = 0) -> np.ndarray:
    """oracle.paged_decode with the sequences split over host threads.  Each sequence is
    computed on its own in the oracle, so the result is the one a single call gives; the
    C oracle runs without the GIL (ctypes releases it)."""
    B = q.shape[0]
    tables = torch.as_tensor(tables)
    ctx_lens = torch.as_tensor(ctx_lens)
    n = min(host_threads(), max(1, B))
    bounds = [B * i // n for i in range(n + 1)]

    def part(i):
        a, b = bounds[i], bounds[i + 1]
        if a == b:
            return np.zeros((0,) + tuple(q.shape[1:]), np.float64)
        return oracle.paged_decode(opool, q[a:b], q_dtype, tables[a:b], ctx_lens[a:b], scale, window=window)

    with ThreadPoolExecutor(n) as ex:
        return np.concatenate(list(ex.map(part, range(n))))


def oracle_chunk_threaded(opool, q, q_dtype, block_table, ctx_before: int, scale, rows) -> np.ndarray:
    """oracle.paged_prefill_chunk for the listed chunk rows, over host threads.  Row i of a
    chunk after ctx_before positions is row 0 of a one-row chunk after ctx_before + i
    positions (the same keys, the same causal bound), so each row is its own oracle call."""
    rows = list(rows)

    def one(i):
        return oracle.paged_prefill_chunk(opool, q[i:i + 1], q_dtype, block_table, ctx_before + i, scale)[0]

    with ThreadPoolExecutor(host_threads()) as ex:
        return np.stack(list(ex.map(one, rows)))
