"""GPU parity for sliding-window attention (decode and chunked prefill) and for query-head
groups wider than 16 (MQA-like G = 20 .. 64), against the oracle.

Blocks that lie wholly before a sequence's window are poisoned with NaN: the kernels must
not read them (a read shows up as a non-finite output)."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_431_b200 import pkv
from paged_kv_cache_431_b200 import workloads as wl
from tests.helpers import TOL, max_abs_diff, oracle_pool_from_tensors
from tests.test_gpu_quant import oracle_copy

pytestmark = pytest.mark.gpu
DEV = "cuda"


def poison_before_window_(pool_t, tables, lens, window):
    for b, n in enumerate(lens):
        lo = max(0, n - window)
        for j in range(lo // 16):
            pool_t[int(tables[b, j])] = float("nan")


def decode_case(lens, H_q, H_kv, d, dtype, seed, window):
    W = max(wl.ceil_div(n, 16) for n in lens) + 1
    N = sum(wl.ceil_div(n, 16) for n in lens) + 5
    wk = wl.decode_workload("win", lens, H_q, H_kv, d, dtype, N, W, seed)
    if window:
        poison_before_window_(wk.k_pool, wk.paging.tables, lens, window)
        poison_before_window_(wk.v_pool, wk.paging.tables, lens, window)
    return wk


@pytest.mark.parametrize("window", [1, 16, 17, 100, 300])
@pytest.mark.parametrize("shape", [(32, 8, 128, wl.BF16), (8, 2, 64, wl.F16), (16, 4, 128, wl.F16)],
                         ids=["G4-bf16", "G4-d64-f16", "G4-f16"])
def test_decode_window(shape, window):
    H_q, H_kv, d, dtype = shape
    g = wl.generator(900 + window)
    lens = [0, 1, 15, 16, 17, window, window + 1, window + 15, window + 16] + \
        torch.randint(1, 700, (5,), generator=g).tolist()
    wk = decode_case(lens, H_q, H_kv, d, dtype, 910 + window, window)
    k = wk.k_pool.to(DEV).unsqueeze(0)
    v = wk.v_pool.to(DEV).unsqueeze(0)
    pool = pkv.KVPool(k, v, dtype, d, device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
    opool = oracle_pool_from_tensors(wk.k_pool, wk.v_pool, dtype)
    ref = oracle.paged_decode(opool, wk.q, dtype, wk.paging.tables, wk.paging.ctx_lens, np.float32(wk.scale),
                              window=window)
    engines = [1] + ([2, 3] if d == 128 and H_q // H_kv in (4, 8) else [])
    for engine in engines:
        for part in (0, 64):
            out = pkv.paged_decode_attn(pool, 0, wk.q.to(DEV), wk.paging.tables.to(DEV),
                                        wk.paging.ctx_lens.to(DEV), wk.scale, max(lens), engine=engine,
                                        partition_tokens=part, sliding_window=window)
            torch.cuda.synchronize()
            assert pkv.read_device_status(pool) == 0
            assert max_abs_diff(out, ref) <= TOL, (engine, part)


@pytest.mark.parametrize("dt", [pkv.INT8, pkv.FP8E4M3, pkv.INT4], ids=["int8", "fp8", "int4"])
def test_quantized_decode_window(dt):
    g = wl.generator(950 + dt)
    H_q, H_kv, d, window = 32, 4, 128, 200
    lens = [1, 40, 199, 200, 201, 350, 1000]
    W = max(wl.ceil_div(n, 16) for n in lens)
    N = sum(wl.ceil_div(n, 16) for n in lens) + 3
    paging = wl.allocate(lens, N, W, g)
    pool = pkv.KVPool.allocate(1, N, H_kv, d, dt)
    seq = torch.cat([torch.full((n,), b) for b, n in enumerate(lens)])
    pos = torch.cat([torch.arange(n) for n in lens])
    slots = wl.slots_for(paging.tables, seq, pos)
    k, v = wl.kv_source(len(seq), H_kv, d, g)
    pkv.kv_append(pool, 0, k.to(DEV), v.to(DEV), slots.to(DEV))
    q = wl.normal((len(lens), H_q, d), torch.bfloat16, g)
    cl = torch.tensor(lens, dtype=torch.int32)
    out = pkv.paged_decode_attn(pool, 0, q.to(DEV), paging.tables.to(DEV), cl.to(DEV), d ** -0.5, max(lens),
                                sliding_window=window)
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    ref = oracle.paged_decode(oracle_copy(pool), q, oracle.BF16, paging.tables, cl, np.float32(d ** -0.5),
                              window=window)
    assert max_abs_diff(out, ref) <= TOL


@pytest.mark.parametrize("shape", [(64, 1, wl.BF16), (40, 2, wl.F16), (32, 1, wl.BF16), (128, 2, wl.BF16)],
                         ids=["MQA-G64", "G20", "G32", "G64x2"])
@pytest.mark.parametrize("window", [0, 50])
def test_decode_wide_groups(shape, window):
    """G > 16: the group's query heads are split over CTAs of 16 heads that read the same K/V."""
    H_q, H_kv, dtype = shape
    g = wl.generator(970 + H_q)
    lens = [0, 5, 16, 77, 300] + torch.randint(1, 1500, (4,), generator=g).tolist()
    wk = decode_case(lens, H_q, H_kv, 128, dtype, 980 + H_q + window, window)
    pool = pkv.KVPool(wk.k_pool.to(DEV).unsqueeze(0), wk.v_pool.to(DEV).unsqueeze(0), dtype, 128,
                      device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
    out = pkv.paged_decode_attn(pool, 0, wk.q.to(DEV), wk.paging.tables.to(DEV), wk.paging.ctx_lens.to(DEV),
                                wk.scale, max(lens), sliding_window=window)
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    opool = oracle_pool_from_tensors(wk.k_pool, wk.v_pool, dtype)
    ref = oracle.paged_decode(opool, wk.q, dtype, wk.paging.tables, wk.paging.ctx_lens, np.float32(wk.scale),
                              window=window)
    assert max_abs_diff(out, ref) <= TOL


def test_quantized_mqa():
    g = wl.generator(990)
    H_q, H_kv, d = 64, 1, 128
    lens = [3, 33, 500, 129]
    W = max(wl.ceil_div(n, 16) for n in lens)
    N = sum(wl.ceil_div(n, 16) for n in lens) + 2
    paging = wl.allocate(lens, N, W, g)
    pool = pkv.KVPool.allocate(1, N, H_kv, d, pkv.INT8)
    seq = torch.cat([torch.full((n,), b) for b, n in enumerate(lens)])
    pos = torch.cat([torch.arange(n) for n in lens])
    k, v = wl.kv_source(len(seq), H_kv, d, g)
    pkv.kv_append(pool, 0, k.to(DEV), v.to(DEV), wl.slots_for(paging.tables, seq, pos).to(DEV))
    q = wl.normal((len(lens), H_q, d), torch.bfloat16, g)
    cl = torch.tensor(lens, dtype=torch.int32)
    out = pkv.paged_decode_attn(pool, 0, q.to(DEV), paging.tables.to(DEV), cl.to(DEV), d ** -0.5, max(lens))
    torch.cuda.synchronize()
    ref = oracle.paged_decode(oracle_copy(pool), q, oracle.BF16, paging.tables, cl, np.float32(d ** -0.5))
    assert max_abs_diff(out, ref) <= TOL


PREFILL = [
    # (P0, C, H_q, H_kv, d, dtype, window)
    (0, 100, 8, 2, 64, wl.F16, 1),
    (40, 77, 16, 2, 128, wl.BF16, 16),
    (300, 129, 64, 8, 128, wl.BF16, 100),
    (1000, 64, 8, 8, 128, wl.BF16, 129),
    (123, 70, 12, 4, 128, wl.F16, 4096),      # window longer than every row: plain causal
]


@pytest.mark.parametrize("case", range(len(PREFILL)))
def test_prefill_window(case):
    P0, C, H_q, H_kv, d, dtype, window = PREFILL[case]
    g = wl.generator(1000 + case)
    n = P0 + C
    W = wl.ceil_div(n, 16) + 1
    N = W + 4
    paging = wl.allocate([n], N, W, g)
    tdt = wl.TORCH_DTYPE[dtype]
    k = wl.normal((N, H_kv, 16, d), tdt, g)
    v = wl.normal((N, H_kv, 16, d), tdt, g)
    wl.poison_pool_(k, paging)
    wl.poison_pool_(v, paging)
    # blocks no row's window reaches
    first_lo = max(0, P0 + 1 - window)
    for j in range(first_lo // 16):
        k[int(paging.tables[0, j])] = float("nan")
        v[int(paging.tables[0, j])] = float("nan")
    q = wl.normal((C, H_q, d), tdt, g)
    pool = pkv.KVPool(k.to(DEV).unsqueeze(0), v.to(DEV).unsqueeze(0), dtype, d,
                      device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
    out = pkv.paged_prefill_chunk_attn(pool, 0, q.to(DEV), paging.tables[0].to(DEV), P0, d ** -0.5,
                                       sliding_window=window)
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    ref = oracle.paged_prefill_chunk(oracle_pool_from_tensors(k, v, dtype), q, dtype, paging.tables[0], P0,
                                     np.float32(d ** -0.5), window=window)
    assert max_abs_diff(out, ref) <= TOL


def test_cascade_refuses_a_window():
    pool = pkv.KVPool.allocate(1, 64, 2, 128, pkv.BF16)
    q = torch.zeros(4, 16, 128, dtype=torch.bfloat16, device=DEV)
    tables = torch.zeros(4, 8, dtype=torch.int32, device=DEV)
    cl = torch.full((4,), 64, dtype=torch.int32, device=DEV)
    with pytest.raises(pkv.PkvError) as e:
        pkv.paged_decode_attn_cascade(pool, 0, q, tables, cl, 0.1, 64, 32, sliding_window=32)
    assert e.value.status == -9
