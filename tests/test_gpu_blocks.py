"""GPU parity for whole-block moves: kv_copy_blocks (copy-on-write at divergence) and
kv_swap_out / kv_swap_in (preemption to host memory), bit-exact against the oracle's
byte moves, for every storage dtype, over several layers."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_431_b200 import pkv
from paged_kv_cache_431_b200 import workloads as wl
from tests.helpers import TOL, max_abs_diff, oracle_pool_from_tensors

pytestmark = pytest.mark.gpu
DEV = "cuda"
DTYPES = [pkv.BF16, pkv.F16, pkv.INT8, pkv.INT4, pkv.FP8E4M3]
NAMES = {pkv.BF16: "bf16", pkv.F16: "f16", pkv.INT8: "int8", pkv.INT4: "int4", pkv.FP8E4M3: "fp8"}


def filled_pool(L, N, H, d, dt, seed):
    g = wl.generator(seed)
    pool = pkv.KVPool.allocate(L, N, H, d, dt)
    if dt in (pkv.F16, pkv.BF16):
        pool.k_data.copy_(wl.normal(pool.k_data.shape, pool.k_data.dtype, g))
        pool.v_data.copy_(wl.normal(pool.v_data.shape, pool.v_data.dtype, g))
    else:
        for t in (pool.k_data, pool.v_data):
            c = torch.randint(0, 256, t.shape, generator=g, dtype=torch.int32).to(torch.uint8)
            if dt == pkv.FP8E4M3:
                c[(c & 0x7F) == 0x7F] = 0x7E
            t.copy_(c)
        pool.k_scale.copy_(torch.rand(pool.k_scale.shape, generator=g) * 0.05)
        pool.v_scale.copy_(torch.rand(pool.v_scale.shape, generator=g) * 0.05)
    return pool


def oracle_layers(pool):
    ks = [None] * pool.num_layers if pool.k_scale is None else list(pool.k_scale)
    vs = [None] * pool.num_layers if pool.v_scale is None else list(pool.v_scale)
    return [oracle_pool_from_tensors(pool.k_data[l], pool.v_data[l], pool.kv_dtype, ks[l], vs[l])
            for l in range(pool.num_layers)]


def assert_pools_equal(pool, opools):
    got = oracle_layers(pool)
    for l, (a, b) in enumerate(zip(got, opools)):
        assert np.array_equal(a.k, b.k), f"layer {l}: K bytes differ"
        assert np.array_equal(a.v, b.v), f"layer {l}: V bytes differ"
        assert np.array_equal(a.k_scale.view(np.uint32), b.k_scale.view(np.uint32)), f"layer {l}: K scales differ"
        assert np.array_equal(a.v_scale.view(np.uint32), b.v_scale.view(np.uint32)), f"layer {l}: V scales differ"


@pytest.mark.parametrize("shape", [(3, 40, 4, 64), (2, 64, 8, 128)], ids=["L3-H4-d64", "L2-H8-d128"])
@pytest.mark.parametrize("dt", DTYPES, ids=lambda x: NAMES[x])
def test_copy_blocks_bit_exact(dt, shape):
    L, N, H, d = shape
    pool = filled_pool(L, N, H, d, dt, 7100 + dt)
    opools = oracle_layers(pool)
    perm = torch.randperm(N, generator=wl.generator(7200 + dt)).tolist()
    src, dst = perm[:N // 3], perm[N // 3: 2 * (N // 3)]
    pkv.kv_copy_blocks(pool, torch.tensor(src, dtype=torch.int32, device=DEV),
                       torch.tensor(dst, dtype=torch.int32, device=DEV))
    assert pkv.read_device_status(pool) == 0
    oracle.copy_blocks(opools, src, dst)
    assert_pools_equal(pool, opools)


@pytest.mark.parametrize("dt", DTYPES, ids=lambda x: NAMES[x])
def test_swap_out_and_in_bit_exact(dt):
    L, N, H, d = 3, 48, 4, 128
    pool = filled_pool(L, N, H, d, dt, 7300 + dt)
    opools = oracle_layers(pool)
    perm = torch.randperm(N, generator=wl.generator(7400 + dt)).tolist()
    out_ids, in_ids = perm[:13], perm[13:26]
    per = pkv.kv_swap_bytes_per_block(pool)
    host = torch.full((len(out_ids), per), 0xA5, dtype=torch.uint8).pin_memory()
    pkv.kv_swap_out(pool, torch.tensor(out_ids, dtype=torch.int32, device=DEV), host)
    torch.cuda.synchronize()
    image = oracle.swap_image(opools, out_ids)
    assert image.shape == (len(out_ids), per)
    assert np.array_equal(host.numpy(), image), "swapped-out bytes differ from the oracle's image"
    # bring the image back into other blocks
    pkv.kv_swap_in(pool, torch.tensor(in_ids, dtype=torch.int32, device=DEV), host)
    assert pkv.read_device_status(pool) == 0
    oracle.swap_restore(opools, in_ids, image)
    assert_pools_equal(pool, opools)


def test_decode_reads_a_copied_sequence_like_the_original():
    """A sequence whose blocks were all copied to new ids decodes to the same output through
    its new table (bit-identical on the GPU) and matches the oracle."""
    B, H_q, H_kv, d, N = 6, 16, 2, 128, 200
    lens = [17, 40, 255, 1, 96, 130]
    g = wl.generator(7500)
    paging = wl.allocate(lens, N // 2, 16, g)
    pool = pkv.KVPool.allocate(1, N, H_kv, d, pkv.BF16)
    pool.k_data.copy_(wl.normal(pool.k_data.shape, torch.bfloat16, g))
    pool.v_data.copy_(wl.normal(pool.v_data.shape, torch.bfloat16, g))
    tables = paging.tables.clone()
    used = sorted({int(b) for row, n in zip(tables.tolist(), lens) for b in row[:(n + 15) // 16]})
    fresh = list(range(N // 2, N // 2 + len(used)))
    remap = dict(zip(used, fresh))
    new_tables = tables.clone()
    for b, n in enumerate(lens):
        for j in range((n + 15) // 16):
            new_tables[b, j] = remap[int(tables[b, j])]
    pkv.kv_copy_blocks(pool, torch.tensor(used, dtype=torch.int32, device=DEV),
                       torch.tensor(fresh, dtype=torch.int32, device=DEV))
    q = wl.normal((B, H_q, d), torch.bfloat16, g)
    cl = torch.tensor(lens, dtype=torch.int32)
    scale = 1.0 / np.sqrt(d)
    a = pkv.paged_decode_attn(pool, 0, q.to(DEV), tables.to(DEV), cl.to(DEV), scale, max(lens))
    b = pkv.paged_decode_attn(pool, 0, q.to(DEV), new_tables.to(DEV), cl.to(DEV), scale, max(lens))
    assert pkv.read_device_status(pool) == 0
    assert torch.equal(a, b)
    opool = oracle_layers(pool)[0]
    ref = oracle.paged_decode(opool, q, oracle.BF16, new_tables.numpy(), cl.numpy(), scale)
    assert max_abs_diff(b, ref) < TOL


def test_bad_block_id_is_reported_and_skipped():
    pool = filled_pool(2, 16, 2, 64, pkv.BF16, 7600)
    opools = oracle_layers(pool)
    src = torch.tensor([1, 99, 3], dtype=torch.int32, device=DEV)
    dst = torch.tensor([5, 6, -1], dtype=torch.int32, device=DEV)
    pkv.kv_copy_blocks(pool, src, dst)
    assert pkv.read_device_status(pool) & pkv.DEV_BAD_BLOCK
    oracle.copy_blocks(opools, [1], [5])
    assert_pools_equal(pool, opools)
    host = torch.zeros((2, pkv.kv_swap_bytes_per_block(pool)), dtype=torch.uint8).pin_memory()
    pkv.kv_swap_out(pool, torch.tensor([2, 16], dtype=torch.int32, device=DEV), host)
    assert pkv.read_device_status(pool) & pkv.DEV_BAD_BLOCK
    assert np.array_equal(host.numpy()[0], oracle.swap_image(opools, [2])[0])
    assert not host.numpy()[1].any()


def test_block_manager_drives_append_copy_swap_and_decode():
    """The host block manager plans slots, copy-on-write pairs and swaps; the kernels carry
    them out; every sequence then decodes like attention over its own contiguous K/V
    (the oracle, laid out in fresh blocks in order)."""
    H_q, H_kv, d, N = 8, 2, 128, 96
    g = wl.generator(7700)
    pool = pkv.KVPool.allocate(1, N, H_kv, d, pkv.BF16)
    bm = pkv.BlockManager(N)
    rows = {}          # token prefix -> (k, v) rows [H_kv, d] bf16: K/V depend on the whole prefix
    seqs = {}          # seq id -> token list
    kv_ws = None

    def kv_for(prefix):
        if prefix not in rows:
            rows[prefix] = (wl.normal((H_kv, d), torch.bfloat16, g), wl.normal((H_kv, d), torch.bfloat16, g))
        return rows[prefix]

    def append(sid, new):
        toks = seqs[sid]
        start = len(toks)
        slots, cow = bm.append_slots(sid, len(new), new)
        if cow:
            pkv.kv_copy_blocks(pool, torch.tensor([cow[0]], dtype=torch.int32, device=DEV),
                               torch.tensor([cow[1]], dtype=torch.int32, device=DEV))
        toks.extend(new)
        k = torch.stack([kv_for(tuple(toks[:start + i + 1]))[0] for i in range(len(new))])
        v = torch.stack([kv_for(tuple(toks[:start + i + 1]))[1] for i in range(len(new))])
        pkv.kv_append(pool, 0, k.to(DEV), v.to(DEV), torch.tensor(slots, dtype=torch.int32, device=DEV))

    prompt = [int(x) for x in torch.randint(0, 1000, (37,), generator=g)]
    assert bm.add_sequence(0, prompt) == 0
    seqs[0] = []
    append(0, prompt)
    for child in (1, 2):                       # beams sharing the prompt's partial block
        bm.fork(0, child)
        seqs[child] = list(seqs[0])
    for sid in (0, 1, 2):
        append(sid, [1000 + sid, 7])
    assert bm.stats()["cow_copies"] == 2
    other = prompt[:32] + [5, 6, 7]            # shares two full blocks through the prefix cache
    cached = bm.add_sequence(3, other)
    assert cached == 32
    seqs[3] = list(other[:cached])
    append(3, other[cached:])
    # preempt seq 2: copy its blocks out, let seq 3 grow into the freed pool, bring it back
    out_blocks = bm.swap_out(2)
    host = torch.zeros((len(out_blocks), pkv.kv_swap_bytes_per_block(pool)), dtype=torch.uint8).pin_memory()
    pkv.kv_swap_out(pool, torch.tensor(out_blocks, dtype=torch.int32, device=DEV), host)
    append(3, [int(x) for x in torch.randint(0, 1000, (40,), generator=g)])
    in_blocks = bm.swap_in(2, len(out_blocks))
    pkv.kv_swap_in(pool, torch.tensor(in_blocks, dtype=torch.int32, device=DEV), host)
    append(2, [11, 12, 13])
    bm.check()
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0

    ids = sorted(seqs)
    lens = [len(seqs[s]) for s in ids]
    W = max(-(-n // 16) for n in lens)
    tables = torch.full((len(ids), W), -1, dtype=torch.int32)
    for r, s in enumerate(ids):
        t, n = bm.block_table(s)
        assert n == lens[r]
        tables[r, :len(t)] = torch.tensor(t, dtype=torch.int32)
    q = wl.normal((len(ids), H_q, d), torch.bfloat16, g)
    cl = torch.tensor(lens, dtype=torch.int32)
    out = pkv.paged_decode_attn(pool, 0, q.to(DEV), tables.to(DEV), cl.to(DEV), 1.0 / np.sqrt(d), max(lens))
    # oracle: each sequence's K/V written in order into its own fresh blocks
    nblk = sum(-(-n // 16) for n in lens)
    opool = oracle.Pool(nblk, H_kv, d, oracle.BF16)
    otables = np.full((len(ids), W), -1, np.int32)
    at = 0
    for r, s in enumerate(ids):
        nb = -(-lens[r] // 16)
        otables[r, :nb] = np.arange(at, at + nb)
        k = torch.stack([rows[tuple(seqs[s][:p + 1])][0] for p in range(lens[r])])
        v = torch.stack([rows[tuple(seqs[s][:p + 1])][1] for p in range(lens[r])])
        slots = np.array([otables[r, p // 16] * 16 + p % 16 for p in range(lens[r])], np.int32)
        oracle.kv_append(opool, k, v, oracle.BF16, slots)
        at += nb
    ref = oracle.paged_decode(opool, q, oracle.BF16, otables, cl.numpy(), 1.0 / np.sqrt(d))
    assert max_abs_diff(out, ref) < TOL
