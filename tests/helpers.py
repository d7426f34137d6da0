"""Shared test plumbing: moving seeded inputs between the CUDA path and the oracle.

Nothing here computes attention or quantization; it only copies the same input bytes to
both sides and, for full-size workloads, gives the oracle a compact copy of just the
blocks a sampled subset of sequences references (block ids renumbered).
"""
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
