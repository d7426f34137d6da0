"""GPU parity at the full sizes of the benchmark workloads, element by element.

The 70B-class decode step runs as the benchmark runs it: 80 layers, each a kv_append of
every sequence's new token and a paged_decode_attn over its whole context, on distinct
full-size layer pools (170 x 256 blocks, H_kv 8, d 128, bf16) that the layers cycle over.
Two whole layers (every sequence, every head) and 8 seeded sequences in all 80 layers are
compared with the oracle, which runs on all host cores (each sequence on its own).
"""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_431_b200 import pkv
from paged_kv_cache_431_b200 import workloads as wl
from tests.helpers import (TOL, compact_subset, host_threads, max_abs_diff, oracle_decode_threaded,
                           oracle_pool_from_tensors, oracle_subset_pool)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_gqa70b_80_layer_step():
    """70B-class GQA decode step: L 80, B 170, H_q 64, H_kv 8, d 128, bf16, contexts
    N(3000, 400) clipped to [1024, 4096] (the new token included), a permuted pool of
    170 x 256 blocks per layer.  Layer l uses physical pool l mod 8; slots outside every
    context hold NaN."""
    L, L_phys, B, H_q, H_kv, d = 80, 8, 170, 64, 8, 128
    g = wl.generator(434)
    ctx = wl.gqa70b_lens(g, B)
    N = B * 256
    paging = wl.allocate(ctx, N, 256, g)
    gd = wl.generator(435, DEV)
    k_pool = torch.empty(L_phys, N, H_kv, 16, d, dtype=torch.bfloat16, device=DEV)
    v_pool = torch.empty_like(k_pool)
    for lp in range(L_phys):
        k_pool[lp] = wl.normal((N, H_kv, 16, d), torch.bfloat16, gd, DEV)
        v_pool[lp] = wl.normal((N, H_kv, 16, d), torch.bfloat16, gd, DEV)
        wl.poison_pool_(k_pool[lp], paging)
        wl.poison_pool_(v_pool[lp], paging)
    pool = pkv.KVPool(k_pool, v_pool, wl.BF16, d, device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
    q = wl.normal((L, B, H_q, d), torch.bfloat16, gd, DEV)
    k_new = wl.normal((L, B, H_kv, d), torch.bfloat16, gd, DEV)
    v_new = wl.normal((L, B, H_kv, d), torch.bfloat16, gd, DEV)
    slots = wl.slots_for(paging.tables, range(B), (ctx - 1).long())
    tables, ctx_d, slots_d = paging.tables.to(DEV), ctx.to(DEV), slots.to(DEV)
    max_ctx = int(ctx.max())
    ws = torch.empty(max(pkv.paged_decode_workspace_bytes(pool, B, H_q, max_ctx), 16), dtype=torch.uint8, device=DEV)
    out = torch.empty(L, B, H_q, d, dtype=torch.float32, device=DEV)
    for layer in range(L):
        lp = layer % L_phys
        pkv.kv_append(pool, lp, k_new[layer], v_new[layer], slots_d)
        pkv.paged_decode_attn(pool, lp, q[layer], tables, ctx_d, d ** -0.5, max_ctx, out=out[layer], workspace=ws)
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    assert torch.isfinite(out).all()
    scale = np.float32(d ** -0.5)

    # the pools now hold the last layer's new token of each pool; layer l's view of pool
    # l mod 8 is that with its own new token written at each sequence's slot ctx - 1
    def layer_pool(layer, ids, blocks=None):
        lp = layer % L_phys
        if blocks is None:
            op = oracle_pool_from_tensors(k_pool[lp], v_pool[lp], wl.BF16)
            sl = slots[ids].numpy()
        else:
            op = oracle_subset_pool(k_pool[lp], v_pool[lp], wl.BF16, blocks)
            at = {blk: i for i, blk in enumerate(blocks)}
            sl = np.array([at[int(s) // 16] * 16 + int(s) % 16 for s in slots[ids]], np.int32)
        oracle.kv_append(op, k_new[layer, ids].cpu(), v_new[layer, ids].cpu(), wl.BF16, sl)
        return op

    # two whole layers: every sequence and head
    for layer in (0, L - 1):
        ref = oracle_decode_threaded(layer_pool(layer, list(range(B))), q[layer].cpu(), wl.BF16, paging.tables,
                                     ctx, scale)
        assert max_abs_diff(out[layer], ref) <= TOL, f"layer {layer}"

    # 8 seeded sequences in every layer
    seq_ids = torch.randperm(B, generator=g)[:8].tolist()
    blocks, sub_t, sub_c = compact_subset(paging.tables, ctx, seq_ids)

    def check(layer):
        ref = oracle.paged_decode(layer_pool(layer, seq_ids, blocks), q[layer, seq_ids].cpu(), wl.BF16, sub_t, sub_c,
                                  scale)
        return max_abs_diff(out[layer, seq_ids], ref)

    with ThreadPoolExecutor(host_threads()) as ex:
        worst = list(ex.map(check, range(L)))
    assert max(worst) <= TOL, f"layer {int(np.argmax(worst))}: {max(worst)}"
