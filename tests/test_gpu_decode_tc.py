"""GPU parity of the tcgen05 decode for wide query groups (G = 64: two sequences per 128-row
tile, G = 128: one), which paged_decode_attn uses by default for 16-bit pools with head dim
128; the warp-level mma.sync form (engine 1) computes the same attention on the same inputs.
Slots outside every context hold NaN, so a read past a sequence's end shows up."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_431_b200 import pkv
from paged_kv_cache_431_b200 import workloads as wl
from tests.helpers import TOL, compact_subset, max_abs_diff, oracle_decode_threaded, oracle_pool_from_tensors

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    # (H_q, H_kv, dtype, partition tokens, context lengths)
    (64, 1, wl.BF16, 0, [1, 31, 32, 33, 64, 65, 700, 2000, 4100]),       # MQA, odd batch
    (64, 1, wl.F16, 128, [0, 16, 17, 128, 129, 255, 600, 1000]),         # empty context, split-K
    (128, 2, wl.BF16, 64, [5, 63, 64, 65, 300, 1111]),                   # G = 64 with two KV heads
    (128, 1, wl.BF16, 0, [1, 64, 65, 500, 3000]),                        # G = 128: one sequence per tile
    (256, 2, wl.F16, 256, [7, 100, 1000, 2049]),                         # G = 128, two KV heads
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_wide_group_decode_matches_oracle_and_warp_level_form(case):
    H_q, H_kv, dtype, part, lens = CASES[case]
    N = sum(wl.ceil_div(n, 16) for n in lens) + 5
    wk = wl.decode_workload(f"tc{case}", lens, H_q, H_kv, 128, dtype, N, wl.ceil_div(max(lens), 16) + 1,
                            1500 + case)
    pool = pkv.KVPool(wk.k_pool.to(DEV).unsqueeze(0), wk.v_pool.to(DEV).unsqueeze(0), dtype, 128,
                      device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
    args = (pool, 0, wk.q.to(DEV), wk.paging.tables.to(DEV), wk.paging.ctx_lens.to(DEV), wk.scale, max(lens))
    out = pkv.paged_decode_attn(*args, partition_tokens=part)
    warp_level = pkv.paged_decode_attn(*args, partition_tokens=part, engine=pkv.ENGINE_MMA)
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    ref = oracle_decode_threaded(oracle_pool_from_tensors(wk.k_pool, wk.v_pool, dtype), wk.q, dtype,
                                 wk.paging.tables, wk.paging.ctx_lens, np.float32(wk.scale))
    assert max_abs_diff(out, ref) <= TOL
    assert max_abs_diff(warp_level, ref) <= TOL
    for b, n in enumerate(lens):
        if n == 0:
            assert torch.all(out[b] == 0)


def test_mqa_workload_shape():
    """The benchmark's MQA decode: B 256, H_q 64, H_kv 1, d 128, bf16, contexts N(3000, 400)
    clipped to [1024, 4096], a permuted pool of 256 x 256 blocks; 8 sequences sampled."""
    g = wl.generator(1600)
    B, H_q, H_kv, d = 256, 64, 1, 128
    ctx = wl.gqa70b_lens(g, B)
    N = B * 256
    paging = wl.allocate(ctx, N, 256, g)
    gd = wl.generator(1601, DEV)
    k_pool = wl.normal((N, H_kv, 16, d), torch.bfloat16, gd, DEV)
    v_pool = wl.normal((N, H_kv, 16, d), torch.bfloat16, gd, DEV)
    q = wl.normal((B, H_q, d), torch.bfloat16, gd, DEV)
    pool = pkv.KVPool(k_pool.unsqueeze(0), v_pool.unsqueeze(0), wl.BF16, d,
                      device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
    out = pkv.paged_decode_attn(pool, 0, q, paging.tables.to(DEV), ctx.to(DEV), d ** -0.5, int(ctx.max()))
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    seq_ids = torch.randperm(B, generator=g)[:8].tolist()
    blocks, sub_t, sub_c = compact_subset(paging.tables, ctx, seq_ids)
    idx = torch.as_tensor(blocks, dtype=torch.long, device=DEV)
    opool = oracle_pool_from_tensors(k_pool[idx], v_pool[idx], wl.BF16)
    ref = oracle_decode_threaded(opool, q[seq_ids].cpu(), wl.BF16, sub_t, sub_c, np.float32(d ** -0.5))
    assert max_abs_diff(out[seq_ids], ref) <= TOL
