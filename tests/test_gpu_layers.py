"""Pools whose layers live in separate allocations (kv_pool_create_layers) behave exactly like
a dense pool holding the same bytes: every call gives bit-identical results, and the
attention matches the oracle."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_431_b200 import pkv
from paged_kv_cache_431_b200 import workloads as wl
from tests.helpers import TOL, max_abs_diff, oracle_pool_from_tensors

pytestmark = pytest.mark.gpu
DEV = "cuda"


def twin_pools(L, N, H_kv, d, dtype, g):
    """A dense pool and a per-layer pool (each layer its own allocation, in reverse order of
    allocation) with the same random contents."""
    dense = pkv.KVPool.allocate(L, N, H_kv, d, dtype)
    if dtype in (wl.BF16, wl.F16):
        dense.k_data.copy_(wl.normal(dense.k_data.shape, wl.TORCH_DTYPE[dtype], g))
        dense.v_data.copy_(wl.normal(dense.v_data.shape, wl.TORCH_DTYPE[dtype], g))
    layers = {}
    for name in ("k_data", "v_data", "k_scale", "v_scale"):
        t = getattr(dense, name)
        if t is not None:
            layers[name] = [torch.empty_like(t[l]) for l in reversed(range(L))][::-1]
            for l in range(L):
                layers[name][l].copy_(t[l])
    split = pkv.KVPool.from_layers(layers["k_data"], layers["v_data"], dtype, d, layers.get("k_scale"),
                                   layers.get("v_scale"), device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
    return dense, split


def same_bytes(dense, split):
    for name in ("k_data", "v_data", "k_scale", "v_scale"):
        t = getattr(dense, name)
        if t is None:
            continue
        for l in range(dense.num_layers):
            a, b = t[l], getattr(split, name)[l]
            assert torch.equal(a.view(torch.uint8) if a.dtype != torch.float32 else a.view(torch.int32),
                               b.view(torch.uint8) if b.dtype != torch.float32 else b.view(torch.int32)), (name, l)


@pytest.mark.parametrize("dtype", [wl.BF16, wl.INT8, wl.INT4], ids=["bf16", "int8", "int4"])
def test_split_layers_match_a_dense_pool(dtype):
    g = wl.generator(2500 + dtype)
    L, H_q, H_kv, d = 3, 16, 4, 128
    lens = [40, 257, 1000, 16]
    N = sum(wl.ceil_div(n, 16) for n in lens) + 70
    paging = wl.allocate(lens, N, 70, g)
    dense, split = twin_pools(L, N, H_kv, d, dtype, g)
    seq = torch.cat([torch.full((n,), b) for b, n in enumerate(lens)])
    pos = torch.cat([torch.arange(n) for n in lens])
    slots = wl.slots_for(paging.tables, seq, pos).to(DEV)
    src = torch.bfloat16 if dtype not in (wl.BF16, wl.F16) else wl.TORCH_DTYPE[dtype]
    for layer in range(L):                    # every layer gets its own tokens
        k = wl.normal((len(seq), H_kv, d), src, g).to(DEV)
        v = wl.normal((len(seq), H_kv, d), src, g).to(DEV)
        pkv.kv_append(dense, layer, k, v, slots)
        pkv.kv_append(split, layer, k, v, slots)
    torch.cuda.synchronize()
    same_bytes(dense, split)
    q = wl.normal((len(lens), H_q, d), src, g).to(DEV)
    tables, ctx = paging.tables.to(DEV), paging.ctx_lens.to(DEV)
    for layer in range(L):
        a = pkv.paged_decode_attn(dense, layer, q, tables, ctx, d ** -0.5, max(lens))
        b = pkv.paged_decode_attn(split, layer, q, tables, ctx, d ** -0.5, max(lens))
        torch.cuda.synchronize()
        assert torch.equal(a, b), layer
    assert pkv.read_device_status(split) == 0
    if dtype == wl.BF16:
        ref = oracle.paged_decode(oracle_pool_from_tensors(split.k_data[1].cpu(), split.v_data[1].cpu(), dtype),
                                  q.cpu(), dtype, paging.tables, paging.ctx_lens, np.float32(d ** -0.5))
        out = pkv.paged_decode_attn(split, 1, q, tables, ctx, d ** -0.5, max(lens))
        assert max_abs_diff(out, ref) <= TOL
        # the prefill chunk on layer 2: positions 700 .. 999 of sequence 2
        P0 = 700
        a = pkv.paged_prefill_chunk_attn(dense, 2, q[:1].repeat(300, 1, 1), tables[2], P0, d ** -0.5)
        b = pkv.paged_prefill_chunk_attn(split, 2, q[:1].repeat(300, 1, 1), tables[2], P0, d ** -0.5)
        torch.cuda.synchronize()
        assert torch.equal(a, b)

    # whole-block moves touch every layer through its own base pointer
    perm = torch.randperm(N, generator=g).to(torch.int32)
    src_b, dst_b = perm[:9].to(DEV), perm[9:18].to(DEV)
    for pool in (dense, split):
        pkv.kv_copy_blocks(pool, src_b, dst_b)
    torch.cuda.synchronize()
    same_bytes(dense, split)
    per = pkv.kv_swap_bytes_per_block(split)
    hosts = [torch.empty(5, per, dtype=torch.uint8).pin_memory() for _ in range(2)]
    ids = perm[20:25].to(DEV)
    for pool, h in zip((dense, split), hosts):
        pkv.kv_swap_out(pool, ids, h)
    torch.cuda.synchronize()
    assert torch.equal(hosts[0], hosts[1])
    back = perm[30:35].to(DEV)
    for pool, h in zip((dense, split), hosts):
        pkv.kv_swap_in(pool, back, h)
    torch.cuda.synchronize()
    same_bytes(dense, split)
