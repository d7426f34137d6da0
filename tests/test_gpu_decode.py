"""GPU parity: paged_decode_attn and 16-bit kv_append against the CPU oracle.

Same seeded input bytes on both sides; fp32 outputs within max |diff| <= 2e-3, slot
writes bit-exact.  Pools are poisoned with NaN outside every sequence's context, so a
read outside the block table or past a sequence's end shows up as a non-finite output.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_431_b200 import pkv
from paged_kv_cache_431_b200 import workloads as wl
from tests.helpers import TOL, compact_subset, max_abs_diff, oracle_pool_from_tensors, oracle_subset_pool

pytestmark = pytest.mark.gpu
DEV = "cuda"


def gpu_pool_from(wk: wl.DecodeWorkload) -> pkv.KVPool:
    k = wk.k_pool.to(DEV).unsqueeze(0).contiguous()
    v = wk.v_pool.to(DEV).unsqueeze(0).contiguous()
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    return pkv.KVPool(k, v, wk.dtype, wk.d, device_status=st)


def run_decode(wk, pool, **kw):
    q = wk.q.to(DEV)
    tables = wk.paging.tables.to(DEV)
    ctx = wk.paging.ctx_lens.to(DEV)
    out = pkv.paged_decode_attn(pool, 0, q, tables, ctx, wk.scale, int(wk.paging.ctx_lens.max()), **kw)
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    return out


def oracle_decode(wk):
    opool = oracle_pool_from_tensors(wk.k_pool, wk.v_pool, wk.dtype)
    return oracle.paged_decode(opool, wk.q, wk.dtype, wk.paging.tables, wk.paging.ctx_lens, np.float32(wk.scale))


def test_tiny_config():
    """4 sequences {17, 33, 40, 64}, G = 4, head dim 64, fp16, scale 1/8."""
    wk = wl.tiny_decode(device="cpu")
    assert wk.scale == 0.125
    pool = gpu_pool_from(wk)
    ref = oracle_decode(wk)
    for engine, part in ((1, 0), (1, 64)):
        out = run_decode(wk, pool, engine=engine, partition_tokens=part)
        assert max_abs_diff(out, ref) <= TOL


def test_block_table_figure_fixture(golden):
    """The pages' block-table figure: A = 41 tokens in blocks [7, 3, 12], B = 16 tokens in [9]."""
    fig = golden("block_table_example.json")
    A, B = fig["sequences"]["A"], fig["sequences"]["B"]
    g = wl.generator(133)
    N, H_kv, H_q, d = 13, 2, 8, 64
    k = wl.normal((N, H_kv, 16, d), torch.float16, g)
    v = wl.normal((N, H_kv, 16, d), torch.float16, g)
    k[0] = float("nan")                       # the figure's free block
    v[0] = float("nan")
    k[12, :, 9:] = float("nan")               # A's partly filled block: 9 of 16 used
    v[12, :, 9:] = float("nan")
    tables = torch.tensor([A["table"], B["table"] + [-1, -1]], dtype=torch.int32)
    ctx = torch.tensor([A["tokens"], B["tokens"]], dtype=torch.int32)
    q = wl.normal((2, H_q, d), torch.float16, g)
    paging = wl.Paging(N, ctx, tables, torch.zeros(N, dtype=torch.bool))
    wk = wl.DecodeWorkload("figure", H_q, H_kv, d, wl.F16, 0.125, paging, q, k, v)
    out = run_decode(wk, gpu_pool_from(wk))
    assert max_abs_diff(out, oracle_decode(wk)) <= TOL


CASES = [
    # (H_q, H_kv, d, dtype, partition_tokens)
    (8, 8, 64, wl.F16, 0),      # MHA (G = 1)
    (8, 1, 128, wl.BF16, 0),    # MQA (H_kv = 1, G = 8)
    (16, 4, 128, wl.BF16, 64),  # G = 4, split into 64-token partitions
    (32, 4, 128, wl.F16, 128),  # G = 8
    (32, 2, 64, wl.BF16, 64),   # G = 16: two head tiles
    (12, 4, 128, wl.BF16, 0),   # G = 3, not a power of two
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_random_small_cases(case):
    H_q, H_kv, d, dtype, part = CASES[case]
    g = wl.generator(500 + case)
    lens = [0, 1, 15, 16, 17, 31, 32, 33] + torch.randint(1, 201, (6,), generator=g).tolist()
    W = 16
    N = sum(wl.ceil_div(n, 16) for n in lens) + 7
    wk = wl.decode_workload(f"rand{case}", lens, H_q, H_kv, d, dtype, N, W, 600 + case)
    pool = gpu_pool_from(wk)
    out = run_decode(wk, pool, partition_tokens=part)
    assert max_abs_diff(out, oracle_decode(wk)) <= TOL
    assert torch.all(out[0] == 0)              # empty context -> zero row


def test_split_k_matches_single_partition():
    """The split-K merge reproduces the single-pass result for every partition size."""
    g = wl.generator(77)
    lens = torch.randint(1, 1200, (9,), generator=g).tolist() + [1024, 1025]
    N = sum(wl.ceil_div(n, 16) for n in lens) + 3
    wk = wl.decode_workload("split", lens, 32, 8, 128, wl.BF16, N, 80, 78)
    pool = gpu_pool_from(wk)
    ref = oracle_decode(wk)
    outs = [run_decode(wk, pool, partition_tokens=p) for p in (64, 256, 512, 2048)]
    for o in outs:
        assert max_abs_diff(o, ref) <= TOL
    assert (outs[0] - outs[-1]).abs().max().item() < 1e-4


def test_prefix_sharing_equals_private_copies():
    """Sequences sharing physical prefix blocks give what private copies give."""
    g = wl.generator(91)
    H_q, H_kv, d = 16, 2, 128
    lens = [100, 130, 77, 260]
    pre_blocks = 4                                     # 64 shared tokens
    N = 64
    shared = wl.allocate(lens, N, 20, g, shared_prefix_blocks=pre_blocks)
    k = wl.normal((N, H_kv, 16, d), torch.bfloat16, g)
    v = wl.normal((N, H_kv, 16, d), torch.bfloat16, g)
    q = wl.normal((len(lens), H_q, d), torch.bfloat16, g)
    # private copies: give every sequence its own copy of the prefix blocks
    priv_tables = shared.tables.clone()
    k2, v2 = k.clone(), v.clone()
    free = [b for b in range(N) if not bool(shared.used[b])]
    for b in range(1, len(lens)):
        for j in range(pre_blocks):
            nb = free.pop()
            k2[nb], v2[nb] = k[int(shared.tables[b, j])], v[int(shared.tables[b, j])]
            priv_tables[b, j] = nb
    outs = []
    for kk, vv, tb in ((k, v, shared.tables), (k2, v2, priv_tables)):
        paging = wl.Paging(N, shared.ctx_lens, tb, shared.used)
        wk = wl.DecodeWorkload("prefix", H_q, H_kv, d, wl.BF16, d ** -0.5, paging, q, kk, vv)
        outs.append(run_decode(wk, gpu_pool_from(wk)))
    assert torch.equal(outs[0], outs[1])


def test_append16_is_a_bit_exact_slot_copy():
    g = wl.generator(5)
    N, H_kv, d, T = 40, 4, 128, 300
    for dtype in (wl.BF16, wl.F16):
        pool = pkv.KVPool.allocate(2, N, H_kv, d, dtype)
        pool.k_data.fill_(float("nan"))
        k = wl.normal((T, H_kv, d), wl.TORCH_DTYPE[dtype], g).to(DEV)
        v = wl.normal((T, H_kv, d), wl.TORCH_DTYPE[dtype], g).to(DEV)
        slots = torch.randperm(N * 16, generator=g)[:T].to(torch.int32)
        slots[::7] = -1                                  # padding tokens
        opool = oracle_pool_from_tensors(pool.k_data[1], pool.v_data[1], dtype)   # bytes before the call
        pkv.kv_append(pool, 1, k, v, slots.to(DEV))
        torch.cuda.synchronize()
        assert pkv.read_device_status(pool) == 0
        oracle.kv_append(opool, k.cpu(), v.cpu(), dtype, slots.numpy())
        got = oracle_pool_from_tensors(pool.k_data[1], pool.v_data[1], dtype)
        assert np.array_equal(got.k, opool.k) and np.array_equal(got.v, opool.v)
        assert torch.isnan(pool.k_data[0]).all()        # layer 0 untouched


def test_bad_block_id_is_reported_not_faulted():
    wk = wl.tiny_decode(device="cpu")
    pool = gpu_pool_from(wk)
    tables = wk.paging.tables.clone()
    tables[1, 0] = 10 ** 6
    out = pkv.paged_decode_attn(pool, 0, wk.q.to(DEV), tables.to(DEV), wk.paging.ctx_lens.to(DEV), wk.scale, 64)
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) & pkv.DEV_BAD_BLOCK
    assert pkv.read_device_status(pool) == 0             # reading clears it
    ctx = wk.paging.ctx_lens.clone()
    ctx[2] = 1000                                        # longer than the table covers
    pkv.paged_decode_attn(pool, 0, wk.q.to(DEV), wk.paging.tables.to(DEV), ctx.to(DEV), wk.scale, 64)
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) & pkv.DEV_BAD_LENGTH


def _sampled_parity(wk_gpu_pool, k_pool, v_pool, dtype, q, tables, ctx, out, scale, seq_ids):
    blocks, sub_t, sub_c = compact_subset(tables, ctx, seq_ids)
    opool = oracle_subset_pool(k_pool, v_pool, dtype, blocks)
    ref = oracle.paged_decode(opool, q[seq_ids].cpu(), dtype, sub_t, sub_c, np.float32(scale))
    return max_abs_diff(out[seq_ids], ref)


def test_llama8b_config_with_append():
    """Llama-3-8B-shaped decode: B 64, H_q 32, H_kv 8, d 128, bf16, contexts U[512, 4096],
    pool for 64 x 4096 tokens; each sequence's new token is appended first."""
    g = wl.generator(433)
    B, H_q, H_kv, d = 64, 32, 8, 128
    ctx = wl.llama8b_lens(g, B)
    N = B * 4096 // 16
    paging = wl.allocate(ctx, N, 256, g)
    gd = wl.generator(434, DEV)
    k_pool = wl.normal((N, H_kv, 16, d), torch.bfloat16, gd, DEV)
    v_pool = wl.normal((N, H_kv, 16, d), torch.bfloat16, gd, DEV)
    q = wl.normal((B, H_q, d), torch.bfloat16, gd, DEV)
    k_new = wl.normal((B, H_kv, d), torch.bfloat16, gd, DEV)
    v_new = wl.normal((B, H_kv, d), torch.bfloat16, gd, DEV)
    slots = wl.slots_for(paging.tables, range(B), (ctx - 1).long())
    pool = pkv.KVPool(k_pool.unsqueeze(0), v_pool.unsqueeze(0), wl.BF16, d,
                      device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
    k_before = k_pool.clone()
    pkv.kv_append(pool, 0, k_new, v_new, slots.to(DEV))
    out = pkv.paged_decode_attn(pool, 0, q, paging.tables.to(DEV), ctx.to(DEV), d ** -0.5, int(ctx.max()))
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    # the append wrote exactly the new rows
    written = torch.zeros(N * 16, dtype=torch.bool)
    written[slots.long()] = True
    kv = pool.k_data[0].view(N, H_kv, 16, d).permute(0, 2, 1, 3).reshape(N * 16, H_kv, d)
    kb = k_before.view(N, H_kv, 16, d).permute(0, 2, 1, 3).reshape(N * 16, H_kv, d)
    assert torch.equal(kv[slots.long().to(DEV)].view(torch.int16), k_new.view(torch.int16))
    assert torch.equal(kv[~written.to(DEV)].view(torch.int16), kb[~written.to(DEV)].view(torch.int16))
    seq_ids = torch.randperm(B, generator=g)[:6].tolist()
    assert _sampled_parity(pool, pool.k_data[0], pool.v_data[0], wl.BF16, q, paging.tables, ctx, out,
                           d ** -0.5, seq_ids) <= TOL


def test_gqa70b_config_one_layer():
    """70B-class GQA layer: B 170, H_q 64, H_kv 8, d 128, bf16, contexts N(3000, 400)
    clipped to [1024, 4096], a permuted pool of 170 x 256 blocks; 8 sequences sampled."""
    g = wl.generator(434)
    B, H_q, H_kv, d = 170, 64, 8, 128
    ctx = wl.gqa70b_lens(g, B)
    N = B * 256
    paging = wl.allocate(ctx, N, 256, g)
    gd = wl.generator(435, DEV)
    k_pool = wl.normal((N, H_kv, 16, d), torch.bfloat16, gd, DEV)
    v_pool = wl.normal((N, H_kv, 16, d), torch.bfloat16, gd, DEV)
    q = wl.normal((B, H_q, d), torch.bfloat16, gd, DEV)
    pool = pkv.KVPool(k_pool.unsqueeze(0), v_pool.unsqueeze(0), wl.BF16, d,
                      device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
    out = pkv.paged_decode_attn(pool, 0, q, paging.tables.to(DEV), ctx.to(DEV), d ** -0.5, int(ctx.max()))
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    seq_ids = torch.randperm(B, generator=g)[:8].tolist()
    assert _sampled_parity(pool, k_pool, v_pool, wl.BF16, q, paging.tables, ctx, out, d ** -0.5, seq_ids) <= TOL


@pytest.mark.parametrize("engine", [pkv.ENGINE_FMA2, pkv.ENGINE_FMA], ids=["fma2", "fma"])
@pytest.mark.parametrize("G,dtype", [(8, wl.BF16), (4, wl.F16)])
def test_cuda_core_engines(engine, G, dtype):
    """The CUDA-core (FP32 FMA) decode engines against the oracle, with split-K."""
    g = wl.generator(1200 + G + engine)
    H_kv = 4
    lens = [1, 15, 16, 17, 100, 777, 1500] + torch.randint(1, 600, (3,), generator=g).tolist()
    N = sum(wl.ceil_div(n, 16) for n in lens) + 3
    wk = wl.decode_workload("fma", lens, H_kv * G, H_kv, 128, dtype, N, 100, 1300 + G)
    pool = gpu_pool_from(wk)
    ref = oracle_decode(wk)
    for part in (0, 256):
        out = run_decode(wk, pool, engine=engine, partition_tokens=part)
        assert max_abs_diff(out, ref) <= TOL


def test_workspace_reuse_across_shapes():
    """One workspace, never cleared by the caller, serves a series of split-K calls of
    different shapes in stream order (each call writes every partial it reads)."""
    g = wl.generator(1400)
    H_q, H_kv, d = 32, 8, 128
    cases = []
    for i, B in enumerate((7, 20, 3)):
        lens = torch.randint(200, 2000, (B,), generator=g).tolist()
        N = sum(wl.ceil_div(n, 16) for n in lens) + 2
        cases.append(wl.decode_workload(f"reuse{i}", lens, H_q, H_kv, d, wl.BF16, N, 130, 1410 + i))
    need = max(pkv.paged_decode_workspace_bytes(gpu_pool_from(wk), wk.B, H_q, 2000, partition_tokens=128)
               for wk in cases)
    ws = torch.full((need,), 0x5A, dtype=torch.uint8, device=DEV)   # stale contents
    for rep in range(2):
        for wk in cases:
            pool = gpu_pool_from(wk)
            out = pkv.paged_decode_attn(pool, 0, wk.q.to(DEV), wk.paging.tables.to(DEV), wk.paging.ctx_lens.to(DEV),
                                        wk.scale, 2000, workspace=ws, partition_tokens=128)
            torch.cuda.synchronize()
            assert pkv.read_device_status(pool) == 0
            assert max_abs_diff(out, oracle_decode(wk)) <= TOL
