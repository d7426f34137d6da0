"""GPU parity: paged_prefill_chunk_attn against the CPU oracle, and chunk rows against
decode (row i of a chunk is the decode of length ctx_before + i + 1)."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_431_b200 import pkv
from paged_kv_cache_431_b200 import workloads as wl
from tests.helpers import TOL, max_abs_diff, oracle_chunk_threaded, oracle_pool_from_tensors

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    # (P0, C, H_q, H_kv, d, dtype)
    (0, 1, 8, 2, 64, wl.F16),
    (0, 37, 8, 2, 64, wl.F16),
    (5, 16, 8, 8, 128, wl.BF16),       # MHA
    (16, 33, 16, 2, 128, wl.BF16),     # G = 8
    (40, 100, 32, 2, 128, wl.BF16),    # G = 16
    (123, 70, 12, 4, 128, wl.F16),     # G = 3
    (300, 129, 64, 8, 128, wl.BF16),   # 70B head shape
    (77, 200, 16, 4, 128, wl.F16),     # G = 4, fp16
    (0, 300, 4, 4, 128, wl.BF16),      # MHA from an empty context: rows with 1..300 keys
]


def chunk_case(P0, C, H_q, H_kv, d, dtype, seed):
    g = wl.generator(seed)
    n = P0 + C
    W = wl.ceil_div(n, 16) + 2
    N = W + 5
    paging = wl.allocate([n], N, W, g)
    tdt = wl.TORCH_DTYPE[dtype]
    k = wl.normal((N, H_kv, 16, d), tdt, g)
    v = wl.normal((N, H_kv, 16, d), tdt, g)
    wl.poison_pool_(k, paging)
    wl.poison_pool_(v, paging)
    q = wl.normal((C, H_q, d), tdt, g)
    return paging, k, v, q


@pytest.mark.parametrize("case", range(len(CASES)))
def test_chunk_parity(case):
    P0, C, H_q, H_kv, d, dtype = CASES[case]
    paging, k, v, q = chunk_case(P0, C, H_q, H_kv, d, dtype, 700 + case)
    pool = pkv.KVPool(k.to(DEV).unsqueeze(0), v.to(DEV).unsqueeze(0), dtype, d,
                      device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
    table = paging.tables[0].to(DEV)
    scale = d ** -0.5
    out = pkv.paged_prefill_chunk_attn(pool, 0, q.to(DEV), table, P0, scale)
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    ref = oracle.paged_prefill_chunk(oracle_pool_from_tensors(k, v, dtype), q, dtype, paging.tables[0], P0,
                                     np.float32(scale))
    assert max_abs_diff(out, ref) <= TOL
    # row i equals the decode of length P0 + i + 1 (GPU against GPU)
    rows = sorted({0, C // 2, C - 1})
    dq = q[rows].to(DEV)
    tables = paging.tables[0].repeat(len(rows), 1).to(DEV)
    ctx = torch.tensor([P0 + i + 1 for i in rows], dtype=torch.int32, device=DEV)
    dec = pkv.paged_decode_attn(pool, 0, dq, tables, ctx, scale, P0 + C)
    assert (dec - out[rows]).abs().max().item() <= TOL


def test_prefix_plus_chunk_config():
    """One layer of the 70B shape: a 4,000-token shared prefix (250 blocks) and a 512-token
    chunk appended after it, then the chunk attends to prefix + itself; every row checked."""
    g = wl.generator(435)
    H_q, H_kv, d, P0, C = 64, 8, 128, 4000, 512
    N = 250 + 32 + 64
    paging = wl.allocate([P0 + C], N, wl.ceil_div(P0 + C, 16), g, shared_prefix_blocks=250)
    gd = wl.generator(436, DEV)
    k_pool = wl.normal((N, H_kv, 16, d), torch.bfloat16, gd, DEV)
    v_pool = wl.normal((N, H_kv, 16, d), torch.bfloat16, gd, DEV)
    k_new = wl.normal((C, H_kv, d), torch.bfloat16, gd, DEV)
    v_new = wl.normal((C, H_kv, d), torch.bfloat16, gd, DEV)
    q = wl.normal((C, H_q, d), torch.bfloat16, gd, DEV)
    pool = pkv.KVPool(k_pool.unsqueeze(0), v_pool.unsqueeze(0), wl.BF16, d,
                      device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
    slots = wl.slots_for(paging.tables, [0] * C, torch.arange(P0, P0 + C))
    opool = oracle_pool_from_tensors(k_pool, v_pool, wl.BF16)
    pkv.kv_append(pool, 0, k_new, v_new, slots.to(DEV))
    out = pkv.paged_prefill_chunk_attn(pool, 0, q, paging.tables[0].to(DEV), P0, d ** -0.5)
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    oracle.kv_append(opool, k_new.cpu(), v_new.cpu(), wl.BF16, slots.numpy())
    # every row of the chunk (all 32 query tiles of the kernel), the oracle on all host cores
    ref = oracle_chunk_threaded(opool, q.cpu(), wl.BF16, paging.tables[0], P0, np.float32(d ** -0.5), range(C))
    assert max_abs_diff(out, ref) <= TOL
    # and the first rows through the oracle's own multi-row chunk form
    ref = oracle.paged_prefill_chunk(opool, q[:3].cpu(), wl.BF16, paging.tables[0], P0, np.float32(d ** -0.5))
    assert max_abs_diff(out[:3], ref) <= TOL


@pytest.mark.parametrize("scale", [0.0, -0.05], ids=["zero", "negative"])
def test_chunk_parity_nonpositive_scale(scale):
    """A softmax scale <= 0 (the C-ABI takes any float): scale 0 gives uniform weights over
    each row's keys, a negative scale favours the keys least aligned with q; causal masking
    must still exclude the later keys."""
    P0, C, H_q, H_kv, d = 60, 140, 16, 2, 128
    paging, k, v, q = chunk_case(P0, C, H_q, H_kv, d, wl.BF16, 790)
    pool = pkv.KVPool(k.to(DEV).unsqueeze(0), v.to(DEV).unsqueeze(0), wl.BF16, d,
                      device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
    out = pkv.paged_prefill_chunk_attn(pool, 0, q.to(DEV), paging.tables[0].to(DEV), P0, scale)
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    ref = oracle.paged_prefill_chunk(oracle_pool_from_tensors(k, v, wl.BF16), q, wl.BF16, paging.tables[0], P0,
                                     np.float32(scale))
    assert max_abs_diff(out, ref) <= TOL
