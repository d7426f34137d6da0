"""GPU parity for quantized pools (int8, fp8 e4m3, int4): kv_append codes and scales
bit-exact against the oracle's own quantization of the same bf16 source, and
paged_decode_attn within 2e-3 of the oracle's fp64 attention over its dequantized values."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_431_b200 import pkv
from paged_kv_cache_431_b200 import workloads as wl
from tests.helpers import TOL, max_abs_diff, oracle_decode_threaded

pytestmark = pytest.mark.gpu
DEV = "cuda"
QDTYPES = [pkv.INT8, pkv.FP8E4M3, pkv.INT4]
NAMES = {pkv.INT8: "int8", pkv.FP8E4M3: "fp8", pkv.INT4: "int4"}


def oracle_copy(pool: pkv.KVPool, layer: int = 0) -> oracle.Pool:
    k = pool.k_data[layer].cpu().numpy()
    v = pool.v_data[layer].cpu().numpy()
    return oracle.Pool(pool.num_blocks, pool.num_kv_heads, pool.head_dim, pool.kv_dtype, k, v,
                       pool.k_scale[layer].cpu().numpy(), pool.v_scale[layer].cpu().numpy())


def assert_same_pool(pool: pkv.KVPool, opool: oracle.Pool, layer: int = 0, blocks=None):
    got = oracle_copy(pool, layer)
    sel = slice(None) if blocks is None else np.asarray(blocks)
    assert np.array_equal(got.k_scale[sel].view(np.uint32), opool.k_scale[sel].view(np.uint32)), "K scales differ"
    assert np.array_equal(got.v_scale[sel].view(np.uint32), opool.v_scale[sel].view(np.uint32)), "V scales differ"
    assert np.array_equal(got.k[sel], opool.k[sel]), "K codes differ"
    assert np.array_equal(got.v[sel], opool.v[sel]), "V codes differ"


def random_initial_state(pool: pkv.KVPool, g):
    """Stale codes and scales, as left by earlier sequences (no NaN fp8 codes)."""
    k = torch.randint(0, 256, pool.k_data.shape, generator=g, dtype=torch.int32).to(torch.uint8)
    v = torch.randint(0, 256, pool.v_data.shape, generator=g, dtype=torch.int32).to(torch.uint8)
    if pool.kv_dtype == pkv.FP8E4M3:
        k[(k & 0x7F) == 0x7F] = 0x7E
        v[(v & 0x7F) == 0x7F] = 0x7E
    pool.k_data.copy_(k)
    pool.v_data.copy_(v)
    pool.k_scale.copy_(torch.rand(pool.k_scale.shape, generator=g) * 0.05)
    pool.v_scale.copy_(torch.rand(pool.v_scale.shape, generator=g) * 0.05)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dt", QDTYPES, ids=lambda x: NAMES[x])
def test_append_codes_bit_exact(dt, d):
    """Bulk fill, decode-style single-token appends (growing scales, requantization) and
    multi-token appends into partly filled blocks, with padding slots."""
    g = wl.generator(900 + dt * 10 + d)
    N, H_kv = 24, 2
    pool = pkv.KVPool.allocate(1, N, H_kv, d, dt)
    random_initial_state(pool, g)
    opool = oracle_copy(pool)
    lens = [5, 16, 33, 47, 20]
    paging = wl.allocate(lens, N, 6, g, extra_tokens=[20] * len(lens))

    def both(k, v, slots):
        pkv.kv_append(pool, 0, k.to(DEV), v.to(DEV), slots.to(DEV))
        torch.cuda.synchronize()
        assert pkv.read_device_status(pool) == 0
        oracle.kv_append(opool, k, v, oracle.BF16, slots.numpy())
        assert_same_pool(pool, opool)

    # 1. prompt fill: every sequence's first tokens in one call (fresh blocks)
    seq = torch.cat([torch.full((n,), b) for b, n in enumerate(lens)])
    pos = torch.cat([torch.arange(n) for n in lens])
    slots = wl.slots_for(paging.tables, seq, pos)
    k, v = wl.kv_source(len(seq), H_kv, d, g)
    both(k, v, slots)
    # 2. decode steps: one token per sequence per call, magnitudes growing so scales grow
    for step in range(6):
        slots = wl.slots_for(paging.tables, range(len(lens)), torch.tensor(lens) + step)
        k, v = wl.kv_source(len(lens), H_kv, d, g)
        gain = torch.tensor([1.0, 4.0, 0.5, 16.0, 2.0])[step % 5].to(torch.bfloat16)
        both(k * gain, v * gain, slots)
    # 3. a multi-token append into partly filled blocks, with padding tokens
    seq = torch.tensor([0, 0, 0, 2, 2, 4, 4, 4, 4])
    pos = torch.tensor([11, 12, 13, 39, 40, 26, 27, 28, 29])
    slots = wl.slots_for(paging.tables, seq, pos)
    slots[4] = -1
    k, v = wl.kv_source(len(seq), H_kv, d, g)
    both(k * 3, v * 3, slots)


def test_fp8_conversion_at_ties_and_extremes():
    """A block whose amax is 448 has scale exactly 1, so its codes are the e4m3 encoding of
    the bf16 values themselves: midpoints between neighbouring codes (ties to even),
    subnormals, saturation edges."""
    vals = oracle.e4m3_decode(np.arange(0, 127, dtype=np.uint8))
    mids = (vals[:-1] + vals[1:]) / 2
    x = np.concatenate([vals, mids, -vals, -mids, [448.0] * 2])
    x = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16)
    assert np.all(x.float().numpy() == np.concatenate([vals, mids, -vals, -mids, [448.0] * 2]))
    d = 64
    per_block = 16 * d
    nblk = (x.numel() + per_block - 1) // per_block
    src = torch.zeros(nblk * per_block, dtype=torch.bfloat16)
    src[:x.numel()] = x
    src = src.view(nblk, 16, d)
    src[:, 0, 0] = 448.0                       # amax 448 in every block -> scale 1
    src = src.reshape(nblk * 16, 1, d)
    pool = pkv.KVPool.allocate(1, nblk, 1, d, pkv.FP8E4M3)
    slots = torch.arange(nblk * 16, dtype=torch.int32)
    pkv.kv_append(pool, 0, src.to(DEV), src.to(DEV), slots.to(DEV))
    torch.cuda.synchronize()
    assert torch.all(pool.k_scale.cpu() == 1.0)
    want = oracle.e4m3_encode(src.float().numpy().reshape(-1))
    assert np.array_equal(pool.k_data.cpu().numpy().reshape(-1), want)


DECODE_CASES = [
    # (H_q, H_kv, d, partition_tokens)
    (8, 2, 64, 0),
    (8, 8, 128, 64),      # MHA
    (32, 4, 128, 0),      # G = 8
    (32, 2, 128, 128),    # G = 16
    (12, 4, 64, 64),      # G = 3
    (32, 4, 128, 128),    # G = 8, split-K over one-tile partitions
    (16, 2, 128, 256),    # G = 8, two tiles per partition
]


@pytest.mark.parametrize("case", range(len(DECODE_CASES)))
@pytest.mark.parametrize("dt", QDTYPES, ids=lambda x: NAMES[x])
def test_quantized_decode_parity(dt, case):
    H_q, H_kv, d, part = DECODE_CASES[case]
    g = wl.generator(950 + case + 10 * dt)
    lens = [0, 1, 15, 16, 17, 33] + torch.randint(1, 300, (5,), generator=g).tolist()
    N = sum(wl.ceil_div(n, 16) for n in lens) + 4
    W = 20
    paging = wl.allocate(lens, N, W, g)
    pool = pkv.KVPool.allocate(1, N, H_kv, d, dt)
    random_initial_state(pool, g)
    opool = oracle_copy(pool)
    seq = torch.cat([torch.full((n,), b) for b, n in enumerate(lens)])
    pos = torch.cat([torch.arange(n) for n in lens])
    slots = wl.slots_for(paging.tables, seq, pos)
    out_ch = wl.outlier_channels(g, H_kv, d)
    k, v = wl.kv_source(len(seq), H_kv, d, g, outliers=out_ch)
    pkv.kv_append(pool, 0, k.to(DEV), v.to(DEV), slots.to(DEV))
    oracle.kv_append(opool, k, v, oracle.BF16, slots.numpy())
    q = wl.normal((len(lens), H_q, d), torch.bfloat16, g)
    out = pkv.paged_decode_attn(pool, 0, q.to(DEV), paging.tables.to(DEV), paging.ctx_lens.to(DEV), d ** -0.5,
                                max(lens), partition_tokens=part)
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    assert_same_pool(pool, opool)
    ref = oracle.paged_decode(opool, q, oracle.BF16, paging.tables, paging.ctx_lens, np.float32(d ** -0.5))
    assert max_abs_diff(out, ref) <= TOL
    assert torch.all(out[0] == 0)


@pytest.mark.parametrize("H_q", [64, 32])
@pytest.mark.parametrize("dt", QDTYPES, ids=lambda x: NAMES[x])
def test_quantized_decode_fp16_query(dt, H_q):
    """q in fp16 instead of bf16 (both are accepted for quantized pools): 8 query heads per KV
    head (for fp8 the tcgen05 kernel, which reads q itself) and 4 (the warp-level kernel), with
    split-K partitions, against the oracle given the same fp16 q."""
    H_kv, d = 8, 128
    g = wl.generator(1300 + dt + H_q)
    lens = [1, 17, 200] + torch.randint(300, 900, (3,), generator=g).tolist()
    N = sum(wl.ceil_div(n, 16) for n in lens) + 2
    paging = wl.allocate(lens, N, 64, g)
    pool = pkv.KVPool.allocate(1, N, H_kv, d, dt)
    opool = oracle_copy(pool)
    seq = torch.cat([torch.full((n,), b) for b, n in enumerate(lens)])
    pos = torch.cat([torch.arange(n) for n in lens])
    slots = wl.slots_for(paging.tables, seq, pos)
    k, v = wl.kv_source(len(seq), H_kv, d, g)
    pkv.kv_append(pool, 0, k.to(DEV), v.to(DEV), slots.to(DEV))
    oracle.kv_append(opool, k, v, oracle.BF16, slots.numpy())
    q = wl.normal((len(lens), H_q, d), torch.float16, g)
    out = pkv.paged_decode_attn(pool, 0, q.to(DEV), paging.tables.to(DEV), paging.ctx_lens.to(DEV), d ** -0.5,
                                max(lens), partition_tokens=256)
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    ref = oracle.paged_decode(opool, q, oracle.F16, paging.tables, paging.ctx_lens, np.float32(d ** -0.5))
    assert max_abs_diff(out, ref) <= TOL


@pytest.mark.parametrize("dt", QDTYPES, ids=lambda x: NAMES[x])
def test_quantized_long_context_config(dt):
    """Quantized long-context decode, 1 layer: B 16, H_q 64, H_kv 8, d 128, contexts
    U[32768, 131072], bf16 N(0, 1) source with 1% outlier channels x8, bulk-filled by
    kv_append; the oracle checks the codes and the outputs of 4 sampled sequences (the
    shortest and 3 seeded others)."""
    g = wl.generator(436)
    B, H_q, H_kv, d = 16, 64, 8, 128
    ctx = wl.quant_long_lens(g, B)
    W = 8192
    N = B * W
    paging = wl.allocate(ctx, N, W, g)
    out_ch = wl.outlier_channels(g, H_kv, d)
    pool = pkv.KVPool.allocate(1, N, H_kv, d, dt)
    shortest = int(torch.argmin(ctx))
    sampled = [shortest] + [b for b in torch.randperm(B, generator=g).tolist() if b != shortest][:3]
    gd = wl.generator(437, DEV)
    host_src = {}
    for b in range(B):
        n = int(ctx[b])
        k, v = wl.kv_source(n, H_kv, d, gd, DEV, outliers=out_ch)
        slots = wl.slots_for(paging.tables, [b] * n, torch.arange(n)).to(DEV)
        pkv.kv_append(pool, 0, k, v, slots)
        if b in sampled:
            host_src[b] = (k.cpu(), v.cpu())
        del k, v
    q = wl.normal((B, H_q, d), torch.bfloat16, gd, DEV)
    out = pkv.paged_decode_attn(pool, 0, q, paging.tables.to(DEV), ctx.to(DEV), d ** -0.5, int(ctx.max()))
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    blocks, sub_t, sub_c = wl.compact_subset(paging.tables, ctx, sampled)
    opool = oracle.Pool(len(blocks), H_kv, d, dt)
    for i, b in enumerate(sampled):
        n = int(ctx[b])
        slots = wl.slots_for(sub_t, [i] * n, torch.arange(n)).numpy()
        oracle.kv_append(opool, host_src[b][0], host_src[b][1], oracle.BF16, slots)
    idx = torch.as_tensor(blocks, dtype=torch.long, device=DEV)
    assert np.array_equal(pool.k_data[0][idx].cpu().numpy().reshape(opool.k.shape), opool.k)
    assert np.array_equal(pool.v_data[0][idx].cpu().numpy().reshape(opool.v.shape), opool.v)
    assert np.array_equal(pool.k_scale[0][idx].cpu().numpy(), opool.k_scale)
    ref = oracle_decode_threaded(opool, q[sampled].cpu(), oracle.BF16, sub_t, sub_c, np.float32(d ** -0.5))
    assert max_abs_diff(out[sampled], ref) <= TOL


# q magnitudes: every quantized kernel pre-scales q by a power of two chosen per CTA from its
# largest |q| before converting it to fp16 (all-zero q takes the largest shift).
Q_MAGNITUDES = {
    "zero": lambda q: q * 0,                 # every score 0: out = mean of the dequantized V
    "tiny": lambda q: q * 1e-3,              # q near the bottom of fp16's normal range
    "large": lambda q: q * 4,                # peaked softmax
    "mixed": lambda q: q * torch.where(torch.arange(q.shape[1]) % 4 == 0, 4.0, 0.01)[None, :, None],
}


@pytest.mark.parametrize("mag", list(Q_MAGNITUDES))
@pytest.mark.parametrize("dt", QDTYPES, ids=lambda x: NAMES[x])
def test_quantized_decode_query_magnitudes(dt, mag):
    H_q, H_kv, d = 32, 4, 128
    g = wl.generator(1200 + 10 * dt + list(Q_MAGNITUDES).index(mag))
    lens = [1, 16, 40] + torch.randint(100, 400, (3,), generator=g).tolist()
    N = sum(wl.ceil_div(n, 16) for n in lens) + 2
    paging = wl.allocate(lens, N, 32, g)
    pool = pkv.KVPool.allocate(1, N, H_kv, d, dt)
    seq = torch.cat([torch.full((n,), b) for b, n in enumerate(lens)])
    pos = torch.cat([torch.arange(n) for n in lens])
    slots = wl.slots_for(paging.tables, seq, pos)
    k, v = wl.kv_source(len(seq), H_kv, d, g, outliers=wl.outlier_channels(g, H_kv, d))
    pkv.kv_append(pool, 0, k.to(DEV), v.to(DEV), slots.to(DEV))
    opool = oracle_copy(pool)
    q = Q_MAGNITUDES[mag](wl.normal((len(lens), H_q, d), torch.float32, g)).to(torch.bfloat16)
    out = pkv.paged_decode_attn(pool, 0, q.to(DEV), paging.tables.to(DEV), paging.ctx_lens.to(DEV), d ** -0.5,
                                max(lens))
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    ref = oracle.paged_decode(opool, q, oracle.BF16, paging.tables, paging.ctx_lens, np.float32(d ** -0.5))
    assert max_abs_diff(out, ref) <= TOL
    if mag == "zero":   # closed form: uniform weights, out = mean of each sequence's V rows
        vdq = opool.dequant("v")
        G = H_q // H_kv
        for b, n in enumerate(lens):
            t = np.arange(n)
            rows = vdq[paging.tables[b].numpy()[t // 16], :, t % 16, :]      # [n, H_kv, d]
            want = np.repeat(rows.mean(axis=0), G, axis=0)                     # [H_q, d]
            assert np.abs(out[b].cpu().double().numpy() - want).max() <= TOL


# q shapes that stress the score arithmetic of the quantized kernels at long contexts:
#   same_sign -- every q_d > 0: the integer-code kernels add offset * sum(q) to the raw
#                scores and take it off again; with one sign that share is ~20x the score;
#   constant  -- q_d = 0.75 for every d and head: the same offset share, and every head
#                of a group computes the same scores;
#   huge      -- max |q| = 1e5 (bf16 holds it, fp16 does not): q of head h is the bf16 K
#                source of one token t_b of the sequence, scaled up; without outlier channels
#                q . k_t is ~128 x the scale and any other key's ~N(0, 128) x the scale, so the
#                softmax is one-hot at t_b by thousands of log2 units (no near-tie for
#                rounding to flip) and the output is that token's dequantized V row;
#   small     -- |q| ~ 1e-6 (below fp16's normal range): near-uniform weights.
Q_STRESS = ("same_sign", "constant", "huge", "small")


def stress_q(mag, q, k_src, lens, G):
    """q [B, H_q, d] fp32 N(0, 1) -> the stressing form; k_src [sum(lens), H_kv, d] bf16."""
    if mag == "same_sign":
        return q.abs()
    if mag == "constant":
        return torch.full_like(q, 0.75)
    if mag == "small":
        return q * 1e-6
    starts = np.cumsum([0] + list(lens[:-1]))
    for b, n in enumerate(lens):
        t = (n * 2) // 3                                   # the token each head aligns with
        q[b] = k_src[starts[b] + t].float().repeat_interleave(G, dim=0)
    return q * (1e5 / q.abs().max())


@pytest.mark.parametrize("mag", Q_STRESS)
@pytest.mark.parametrize("dt", QDTYPES, ids=lambda x: NAMES[x])
def test_quantized_decode_query_stress_long_context(dt, mag):
    """The 70B head shape (H_q 64, H_kv 8, d 128) at contexts of 1,000-4,100 tokens (split-K
    partitions of 1,024 / 2,048 tokens, plus one short sequence), with the stressing q
    shapes above, against the oracle at 2e-3."""
    H_q, H_kv, d = 64, 8, 128
    g = wl.generator(1300 + 10 * dt + Q_STRESS.index(mag))
    lens = [1000, 1777, 3000, 4100, 33]
    N = sum(wl.ceil_div(n, 16) for n in lens) + 3
    paging = wl.allocate(lens, N, 260, g)
    pool = pkv.KVPool.allocate(1, N, H_kv, d, dt)
    seq = torch.cat([torch.full((n,), b) for b, n in enumerate(lens)])
    pos = torch.cat([torch.arange(n) for n in lens])
    slots = wl.slots_for(paging.tables, seq, pos)
    out_ch = wl.outlier_channels(g, H_kv, d)
    k, v = wl.kv_source(len(seq), H_kv, d, g, outliers=None if mag == "huge" else out_ch)
    pkv.kv_append(pool, 0, k.to(DEV), v.to(DEV), slots.to(DEV))
    opool = oracle_copy(pool)
    q = stress_q(mag, wl.normal((len(lens), H_q, d), torch.float32, g), k, lens, H_q // H_kv).to(torch.bfloat16)
    if mag == "huge":
        assert q.float().abs().max().item() > 65504.0      # outside fp16's range
    out = pkv.paged_decode_attn(pool, 0, q.to(DEV), paging.tables.to(DEV), paging.ctx_lens.to(DEV), d ** -0.5,
                                max(lens))
    torch.cuda.synchronize()
    assert pkv.read_device_status(pool) == 0
    ref = oracle_decode_threaded(opool, q, oracle.BF16, paging.tables, paging.ctx_lens, np.float32(d ** -0.5))
    assert max_abs_diff(out, ref) <= TOL
    if mag == "huge":   # one-hot: the aligned token's dequantized V row (oracle side, fp64)
        vdq = opool.dequant("v")
        for b, n in enumerate(lens):
            t = (n * 2) // 3
            row = np.repeat(vdq[int(paging.tables[b, t // 16]), :, t % 16, :], H_q // H_kv, axis=0)
            assert np.abs(ref[b] - row).max() <= 1e-9
