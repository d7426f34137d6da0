"""The bounded-wait path of every attention kernel, made to run without faulting anything.

pkv_test_withhold_copy makes each kernel arm the barrier of one K/V tile without issuing
the copy, and bounds its waits at 1e5 SM cycles (~50 us).  The wait then runs out, the CTA
records PKV_DEV_TIMEOUT, waits (bounded) for the copies it did issue and for its tensor-core
work, and returns.  The host reads the status (PKV_ERR_TIMEOUT) and the same call, with the
hook off, then matches the oracle on the same pool: the context is still usable.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_431_b200 import pkv
from paged_kv_cache_431_b200 import workloads as wl
from tests.helpers import TOL, max_abs_diff, oracle_pool_from_tensors

pytestmark = pytest.mark.gpu
DEV = "cuda"
WAIT = 100_000          # SM cycles


def expect_timeout(pool):
    rc, bits = pkv.get_device_status(pool)
    assert rc == -7 and bits & pkv.DEV_TIMEOUT, (rc, bits)


def decode_case(H_q, H_kv, dtype, seed, lens=(100, 300, 17, 500)):
    g = wl.generator(seed)
    N = sum(wl.ceil_div(n, 16) for n in lens) + 4
    if dtype in (wl.BF16, wl.F16):
        wk = wl.decode_workload("timeout", list(lens), H_q, H_kv, 128, dtype, N, 40, seed)
        pool = pkv.KVPool(wk.k_pool.to(DEV).unsqueeze(0), wk.v_pool.to(DEV).unsqueeze(0), dtype, 128,
                          device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
        ref = oracle.paged_decode(oracle_pool_from_tensors(wk.k_pool, wk.v_pool, dtype), wk.q, dtype,
                                  wk.paging.tables, wk.paging.ctx_lens, np.float32(wk.scale))
        return pool, wk.q.to(DEV), wk.paging.tables.to(DEV), wk.paging.ctx_lens.to(DEV), ref
    paging = wl.allocate(list(lens), N, 40, g)
    pool = pkv.KVPool.allocate(1, N, H_kv, 128, dtype)
    seq = torch.cat([torch.full((n,), b) for b, n in enumerate(lens)])
    pos = torch.cat([torch.arange(n) for n in lens])
    k, v = wl.kv_source(len(seq), H_kv, 128, g)
    pkv.kv_append(pool, 0, k.to(DEV), v.to(DEV), wl.slots_for(paging.tables, seq, pos).to(DEV))
    q = wl.normal((len(lens), H_q, 128), torch.bfloat16, g)
    torch.cuda.synchronize()
    opool = oracle.Pool(N, H_kv, 128, dtype, pool.k_data[0].cpu().numpy(), pool.v_data[0].cpu().numpy(),
                        pool.k_scale[0].cpu().numpy(), pool.v_scale[0].cpu().numpy())
    ref = oracle.paged_decode(opool, q, oracle.BF16, paging.tables, paging.ctx_lens, np.float32(128 ** -0.5))
    return pool, q.to(DEV), paging.tables.to(DEV), paging.ctx_lens.to(DEV), ref


DECODES = {
    # name: (H_q, H_kv, pool dtype, engine, partition tokens)
    "bf16_g8": (32, 4, wl.BF16, pkv.ENGINE_MMA, 64),
    "bf16_g32_shared_ring": (64, 2, wl.BF16, pkv.ENGINE_MMA, 128),
    "int8": (32, 4, wl.INT8, pkv.ENGINE_MMA, 64),
    "fp8": (32, 4, wl.FP8, pkv.ENGINE_MMA, 64),
    "int4": (32, 4, wl.INT4, pkv.ENGINE_MMA, 64),
    "cuda_cores": (32, 4, wl.BF16, pkv.ENGINE_FMA2, 64),
    "tcgen05_g64": (64, 1, wl.BF16, pkv.ENGINE_AUTO, 256),
    "tcgen05_fp8": (32, 4, wl.FP8, pkv.ENGINE_AUTO, 256),
}


@pytest.mark.parametrize("name", list(DECODES))
def test_decode_gives_up_and_recovers(name):
    H_q, H_kv, dtype, engine, part = DECODES[name]
    pool, q, tables, ctx, ref = decode_case(H_q, H_kv, dtype, 2100 + list(DECODES).index(name))
    args = (pool, 0, q, tables, ctx, 128 ** -0.5, 500)
    pkv.test_withhold_copy(1, WAIT)
    try:
        pkv.paged_decode_attn(*args, engine=engine, partition_tokens=part)
        torch.cuda.synchronize()
    finally:
        pkv.test_withhold_copy(-1)
    expect_timeout(pool)
    out = pkv.paged_decode_attn(*args, engine=engine, partition_tokens=part)
    torch.cuda.synchronize()
    assert pkv.get_device_status(pool) == (0, 0)
    assert max_abs_diff(out, ref) <= TOL


def chunk_case(P0, C, H_q, H_kv, seed):
    g = wl.generator(seed)
    n = P0 + C
    W = wl.ceil_div(n, 16) + 1
    paging = wl.allocate([n], W + 3, W, g)
    k = wl.normal((W + 3, H_kv, 16, 128), torch.bfloat16, g)
    v = wl.normal((W + 3, H_kv, 16, 128), torch.bfloat16, g)
    q = wl.normal((C, H_q, 128), torch.bfloat16, g)
    pool = pkv.KVPool(k.to(DEV).unsqueeze(0), v.to(DEV).unsqueeze(0), wl.BF16, 128,
                      device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
    return pool, paging, k, v, q


@pytest.mark.parametrize("window", [0, 150], ids=["tensor_memory_form", "warp_level_window_form"])
def test_prefill_chunk_gives_up_and_recovers(window):
    P0, C, H_q, H_kv = 300, 200, 32, 4
    pool, paging, k, v, q = chunk_case(P0, C, H_q, H_kv, 2200 + window)
    table = paging.tables[0].to(DEV)
    call = lambda: pkv.paged_prefill_chunk_attn(pool, 0, q.to(DEV), table, P0, 128 ** -0.5,  # noqa: E731
                                                 sliding_window=window)
    pkv.test_withhold_copy(1, WAIT)
    try:
        call()
        torch.cuda.synchronize()
    finally:
        pkv.test_withhold_copy(-1)
    expect_timeout(pool)
    out = call()
    torch.cuda.synchronize()
    assert pkv.get_device_status(pool) == (0, 0)
    ref = oracle.paged_prefill_chunk(oracle_pool_from_tensors(k, v, wl.BF16), q, wl.BF16, paging.tables[0], P0,
                                     np.float32(128 ** -0.5), window=window)
    assert max_abs_diff(out, ref) <= TOL


def test_cascade_decode_gives_up_and_recovers():
    """Both passes of the shared-prefix decode (the tensor-core prefix pass and the suffix
    partitions) take the hook; afterwards the merged result matches the oracle."""
    g = wl.generator(2300)
    H_q, H_kv, d, prefix = 32, 4, 128, 512
    lens = [prefix + n for n in (1, 40, 200, 333)]
    N = prefix // 16 + sum(wl.ceil_div(n - prefix, 16) + 1 for n in lens) + 4
    paging = wl.allocate(lens, N, 64, g, shared_prefix_blocks=prefix // 16)
    k = wl.normal((N, H_kv, 16, d), torch.bfloat16, g)
    v = wl.normal((N, H_kv, 16, d), torch.bfloat16, g)
    q = wl.normal((len(lens), H_q, d), torch.bfloat16, g)
    pool = pkv.KVPool(k.to(DEV).unsqueeze(0), v.to(DEV).unsqueeze(0), wl.BF16, d,
                      device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
    call = lambda: pkv.paged_decode_attn_cascade(pool, 0, q.to(DEV), paging.tables.to(DEV),  # noqa: E731
                                                 paging.ctx_lens.to(DEV), d ** -0.5, max(lens), prefix)
    pkv.test_withhold_copy(1, WAIT)
    try:
        call()
        torch.cuda.synchronize()
    finally:
        pkv.test_withhold_copy(-1)
    expect_timeout(pool)
    out = call()
    torch.cuda.synchronize()
    assert pkv.get_device_status(pool) == (0, 0)
    ref = oracle.paged_decode(oracle_pool_from_tensors(k, v, wl.BF16), q, wl.BF16, paging.tables, paging.ctx_lens,
                              np.float32(d ** -0.5))
    assert max_abs_diff(out, ref) <= TOL
