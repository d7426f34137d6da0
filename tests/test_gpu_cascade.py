"""GPU parity for the shared-prefix (cascade) decode: paged_decode_attn_cascade against
the oracle's plain decode over each sequence's whole context (the cascade form must reach
the same attention), and against the GPU's own paged_decode_attn."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_431_b200 import pkv
from paged_kv_cache_431_b200 import workloads as wl
from tests.helpers import TOL, max_abs_diff, oracle_pool_from_tensors, oracle_subset_pool

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    # (B, prefix tokens, suffix lengths (low, high), H_q, H_kv, dtype, partition_tokens)
    (20, 48, (0, 100), 16, 2, wl.BF16, 0),       # G = 8, ragged query tile, empty suffixes
    (7, 16, (1, 40), 8, 2, wl.F16, 0),           # one prefix block, G = 4
    (33, 256, (0, 700), 32, 2, wl.BF16, 128),    # G = 16, suffixes over several partitions
    (5, 128, (3, 3), 4, 4, wl.BF16, 0),          # MHA (G = 1)
    (40, 4000, (0, 60), 64, 8, wl.BF16, 0),      # the 70B head shape, 4,000-token prompt
]


def cascade_case(B, prefix, suffix, H_q, H_kv, dtype, seed):
    g = wl.generator(seed)
    suf = torch.randint(suffix[0], suffix[1] + 1, (B,), generator=g)
    lens = (prefix + suf).to(torch.int32)
    pblocks = prefix // 16
    W = wl.ceil_div(int(lens.max()), 16) + 1
    N = pblocks + sum(wl.ceil_div(int(s) + 16, 16) for s in suf) + 8
    paging = wl.allocate(lens.tolist(), N, W, g, shared_prefix_blocks=pblocks)
    tdt = wl.TORCH_DTYPE[dtype]
    k = wl.normal((N, H_kv, 16, 128), tdt, g)
    v = wl.normal((N, H_kv, 16, 128), tdt, g)
    wl.poison_pool_(k, paging)
    wl.poison_pool_(v, paging)
    q = wl.normal((B, H_q, 128), tdt, g)
    return paging, lens, k, v, q


@pytest.mark.parametrize("case", range(len(CASES)))
def test_cascade_parity(case):
    B, prefix, suffix, H_q, H_kv, dtype, part = CASES[case]
    paging, lens, k, v, q = cascade_case(B, prefix, suffix, H_q, H_kv, dtype, 800 + case)
    pool = pkv.KVPool(k.to(DEV).unsqueeze(0), v.to(DEV).unsqueeze(0), dtype, 128,
                      device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
    tables, cl = paging.tables.to(DEV), lens.to(DEV)
    scale = 128 ** -0.5
    maxc = int(lens.max())
    out = pkv.paged_decode_attn_cascade(pool, 0, q.to(DEV), tables, cl, scale, maxc, prefix,
                                        partition_tokens=part)
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    plain = pkv.paged_decode_attn(pool, 0, q.to(DEV), tables, cl, scale, maxc)
    assert (out - plain).abs().max().item() <= TOL
    if prefix * B <= 40000:
        ref = oracle.paged_decode(oracle_pool_from_tensors(k, v, dtype), q, dtype, paging.tables, lens,
                                  np.float32(scale))
        assert max_abs_diff(out, ref) <= TOL
    else:   # sampled sequences, each against the oracle on a compact copy of its blocks
        for b in (0, B // 2, B - 1):
            blocks, t, c = wl.compact_subset(paging.tables, lens, [b])
            opool = oracle_subset_pool(k, v, dtype, blocks)
            ref = oracle.paged_decode(opool, q[[b]], dtype, t, c, np.float32(scale))
            assert max_abs_diff(out[[b]], ref) <= TOL


def test_cascade_prefix_chunk_shape():
    """The decode half of the prefix + chunk workload: 256 sequences share a 4,000-token
    prompt (250 blocks), then a private 200-token query and U{0..300} decoded tokens."""
    g = wl.generator(820)
    B, H_q, H_kv, prefix = 256, 64, 8, 4000
    lens = (prefix + 200 + torch.randint(0, 301, (B,), generator=g)).to(torch.int32)
    W = wl.ceil_div(int(lens.max()), 16)
    N = 250 + sum(wl.ceil_div(int(n) - prefix + 16, 16) for n in lens) + 8
    paging = wl.allocate(lens.tolist(), N, W, g, shared_prefix_blocks=250)
    gd = wl.generator(821, DEV)
    k = wl.normal((N, H_kv, 16, 128), torch.bfloat16, gd, DEV)
    v = wl.normal((N, H_kv, 16, 128), torch.bfloat16, gd, DEV)
    q = wl.normal((B, H_q, 128), torch.bfloat16, gd, DEV)
    pool = pkv.KVPool(k.unsqueeze(0), v.unsqueeze(0), wl.BF16, 128,
                      device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
    tables, cl = paging.tables.to(DEV), lens.to(DEV)
    out = pkv.paged_decode_attn_cascade(pool, 0, q, tables, cl, 128 ** -0.5, int(lens.max()), prefix)
    plain = pkv.paged_decode_attn(pool, 0, q, tables, cl, 128 ** -0.5, int(lens.max()))
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    assert (out - plain).abs().max().item() <= TOL
    for b in (0, 77, 255):
        blocks, t, c = wl.compact_subset(paging.tables, lens, [b])
        opool = oracle_subset_pool(k, v, wl.BF16, blocks)
        ref = oracle.paged_decode(opool, q[[b]].cpu(), wl.BF16, t, c, np.float32(128 ** -0.5))
        assert max_abs_diff(out[[b]], ref) <= TOL


def test_cascade_reports_a_table_without_the_prefix():
    B, prefix = 6, 64
    paging, lens, k, v, q = cascade_case(B, prefix, (5, 20), 16, 2, wl.BF16, 830)
    tables = paging.tables.clone()
    tables[3, 1] = tables[3, wl.ceil_div(int(lens[3]), 16) - 1]   # row 3 leaves the shared prefix
    pool = pkv.KVPool(k.to(DEV).unsqueeze(0), v.to(DEV).unsqueeze(0), wl.BF16, 128,
                      device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
    pkv.paged_decode_attn_cascade(pool, 0, q.to(DEV), tables.to(DEV), lens.to(DEV), 0.1, int(lens.max()), prefix)
    assert pkv.read_device_status(pool) & pkv.DEV_BAD_PREFIX
    short = lens.clone()
    short[2] = prefix - 16
    pkv.paged_decode_attn_cascade(pool, 0, q.to(DEV), paging.tables.to(DEV), short.to(DEV), 0.1, int(lens.max()),
                                  prefix)
    assert pkv.read_device_status(pool) & pkv.DEV_BAD_LENGTH


def test_cascade_validates_on_the_host():
    pool = pkv.KVPool.allocate(1, 64, 2, 128, pkv.BF16)
    q = torch.zeros(4, 16, 128, dtype=torch.bfloat16, device=DEV)
    tables = torch.zeros(4, 8, dtype=torch.int32, device=DEV)
    cl = torch.full((4,), 64, dtype=torch.int32, device=DEV)
    for bad_prefix, status in ((24, -4), (256, -4), (-16, -2)):
        with pytest.raises(pkv.PkvError) as e:
            pkv.paged_decode_attn_cascade(pool, 0, q, tables, cl, 0.1, 64, bad_prefix)
        assert e.value.status == status
    # d = 64 is served by paged_decode_attn only
    pool64 = pkv.KVPool.allocate(1, 64, 2, 64, pkv.BF16)
    with pytest.raises(pkv.PkvError) as e:
        pkv.paged_decode_attn_cascade(pool64, 0, q[..., :64].contiguous(), tables, cl, 0.1, 64, 32)
    assert e.value.status == -9
