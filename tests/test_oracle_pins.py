"""Pins for the CPU oracle: it is checked against what the pages and the mathematics fix,
never against itself.  Each test names the fact it pins.

- worked numbers printed on the pages (tests/golden/*.json, each with its citation);
- closed forms (one token, equal keys, constant values, two tokens);
- special cases that reduce to a library routine (contiguous softmax attention via
  scipy.special.softmax; fp8 e4m3 rounding via torch's float8_e4m3fn conversion);
- invariants (block placement, prefix sharing, one partly filled block per sequence,
  token order within an append, code round trips, chunk row == decode).
"""
import math

import numpy as np
import pytest
import torch
from scipy.special import softmax

import oracle
from paged_kv_cache_431_b200 import workloads as wl

BS = 16


def f16_bits(a):
    return np.asarray(a, np.float16).view(np.uint16)


def bf16_bits(a):
    return oracle.as_u16(torch.as_tensor(np.asarray(a, np.float32)).to(torch.bfloat16))


def library_attention(q, K, V, scale):
    """softmax(scale * K q) V for one query row over contiguous K, V (library softmax)."""
    if K.shape[0] == 0:
        return np.zeros(V.shape[1])
    return softmax(scale * (K @ q)) @ V


def build_pool_from_logical(seqs_K, seqs_V, tables, N, H_kv, d, dtype=oracle.F16, fill=np.nan):
    """Place each sequence's logical K/V rows [n, H_kv, d] into a pool following its table,
    writing element by element; every other slot holds ``fill``."""
    np_dt = np.float16
    kp = np.full((N, H_kv, BS, d), fill, np_dt)
    vp = np.full((N, H_kv, BS, d), fill, np_dt)
    for K, V, table in zip(seqs_K, seqs_V, tables):
        for t in range(K.shape[0]):
            blk = table[t // BS]
            kp[blk, :, t % BS, :] = K[t]
            vp[blk, :, t % BS, :] = V[t]
    return oracle.Pool(N, H_kv, d, dtype, kp.view(np.uint16), vp.view(np.uint16))


def random_logical(rng, n, H_kv, d):
    K = rng.standard_normal((n, H_kv, d)).astype(np.float16)
    V = rng.standard_normal((n, H_kv, d)).astype(np.float16)
    return K, V


# ------------------------------------------------------------ worked numbers --

def test_bytes_per_token_worked_values(golden):
    g = golden("kv_sizes.json")
    m = g["model_70b"]
    for row in g["bytes_per_token"]:
        assert oracle.kv_bytes_per_token(m["layers"], row["kv_heads"], m["head_dim"], m["bytes"]) == row["bytes"]
    assert 2621440 == int(2.5 * 2 ** 20) and 327680 == 320 * 1024 and 40960 == 40 * 1024


def test_per_sequence_cache_at_8k(golden):
    g = golden("kv_sizes.json")
    m, s = g["model_70b"], g["per_sequence_8k"]
    for scheme, kvh in (("MHA", 64), ("GQA", 8), ("MQA", 1)):
        got = oracle.kv_cache_bytes(m["layers"], kvh, m["head_dim"], m["bytes"], s["tokens"], 1)
        assert got == s["gib"][scheme] * 2 ** 30
    # the printed "0.3 GiB" for MQA is 0.3125 rounded
    assert round(s["gib"]["MQA"], 1) == 0.3


def test_sizing_example_and_its_rounding(golden):
    g = golden("kv_sizes.json")
    m, s = g["model_70b"], g["sizing_example"]
    per_seq = oracle.kv_cache_bytes(m["layers"], 8, m["head_dim"], m["bytes"], s["tokens"], 1)
    assert per_seq == s["exact_mib"] * 2 ** 20
    # the page's 0.94 "GiB" is MiB / 1000; exact value is 0.9155 GiB
    assert round(per_seq / 2 ** 20 / 1000, 2) == s["printed_gib"]
    assert abs(per_seq / 2 ** 30 - 0.9155) < 1e-4
    assert round(s["free_gb"] / s["printed_gib"], -1) == s["printed_seqs_per_node"]


def test_capacity_examples(golden):
    g = golden("kv_sizes.json")["capacity_8x80"]
    per_token = oracle.kv_bytes_per_token(80, 8, 128, 2)
    n4k = g["kv_room_gb"] * 1e9 / oracle.kv_cache_bytes(80, 8, 128, 2, 4096, 1)
    n128k = g["kv_room_gb"] * 1e9 / oracle.kv_cache_bytes(80, 8, 128, 2, 131072, 1)
    assert per_token == 327680
    assert abs(n4k - g["seqs_4k_printed"]) / g["seqs_4k_printed"] < 0.02      # 335.3 ~ "about 340"
    assert round(n128k) == g["seqs_128k_printed"]                             # 10.5 ~ "~10"


def test_reservation_waste_and_prefix_savings(golden):
    r = golden("kv_sizes.json")["reservation_waste"]
    assert round(100 * (1 - r["average"] / r["max_seq_len"])) == r["printed_percent"]
    p = golden("kv_sizes.json")["prefix_savings"]
    assert round(100 * (1 - p["query"] / (p["prefix"] + p["query"]))) == p["printed_percent"]


# ------------------------------------------------------- block-table figure --

def test_block_table_figure(golden):
    fig = golden("block_table_example.json")
    A, B = fig["sequences"]["A"], fig["sequences"]["B"]
    assert oracle.blocks_for_tokens(A["tokens"]) == len(A["table"])
    assert oracle.blocks_for_tokens(B["tokens"]) == len(B["table"])
    part = fig["only_partial_block"]
    assert oracle.waste_slots(A["tokens"]) == part["empty"] and BS - part["empty"] == part["filled"]
    assert oracle.waste_slots(B["tokens"]) == 0

    rng = np.random.default_rng(7)
    H_kv, H_q, d, N = 2, 4, 16, 13
    KA, VA = random_logical(rng, A["tokens"], H_kv, d)
    KB, VB = random_logical(rng, B["tokens"], H_kv, d)
    pool = build_pool_from_logical([KA, KB], [VA, VB], [A["table"], B["table"]], N, H_kv, d)
    # the figure's placement literally: A's tokens 32..40 sit in block 12, offsets 0..8
    assert np.array_equal(pool.k.view(np.float16)[12, :, :9, :].reshape(-1), KA[32:41].transpose(1, 0, 2).reshape(-1))
    tables = np.full((2, 3), -1, np.int32)
    tables[0, :3] = A["table"]
    tables[1, :1] = B["table"]
    q = rng.standard_normal((2, H_q, d)).astype(np.float16)
    out = oracle.paged_decode(pool, f16_bits(q), oracle.F16, tables, [A["tokens"], B["tokens"]], 0.25)
    G = H_q // H_kv
    for b, (K, V) in enumerate(((KA, VA), (KB, VB))):
        for h in range(H_q):
            ref = library_attention(q[b, h].astype(np.float64), K[:, h // G].astype(np.float64),
                                    V[:, h // G].astype(np.float64), 0.25)
            assert np.allclose(out[b, h], ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------- attention vs library routine --

@pytest.mark.parametrize("seed", range(6))
def test_decode_equals_contiguous_attention(seed):
    """Paged gather + softmax == library softmax attention on the logical sequence,
    for random lengths (including 0, 1 and block boundaries) and GQA groupings."""
    rng = np.random.default_rng(seed)
    H_kv = [1, 2, 2, 4, 1, 3][seed]
    G = [1, 1, 4, 2, 8, 2][seed]
    H_q, d = H_kv * G, [8, 16, 32, 8, 16, 24][seed]
    lens = [0, 1, 15, 16, 17, 31, 32, 33, int(rng.integers(1, 120))]
    W = max(oracle.blocks_for_tokens(n) for n in lens)
    N = sum(oracle.blocks_for_tokens(n) for n in lens) + 5
    perm = rng.permutation(N)
    tables, cur = np.full((len(lens), W), -1, np.int32), 0
    Ks, Vs = [], []
    for b, n in enumerate(lens):
        nb = oracle.blocks_for_tokens(n)
        tables[b, :nb] = perm[cur:cur + nb]
        cur += nb
        K, V = random_logical(rng, n, H_kv, d)
        Ks.append(K)
        Vs.append(V)
    pool = build_pool_from_logical(Ks, Vs, tables, N, H_kv, d)
    q = rng.standard_normal((len(lens), H_q, d)).astype(np.float16)
    scale = 1.0 / math.sqrt(d)
    out = oracle.paged_decode(pool, f16_bits(q), oracle.F16, tables, lens, np.float32(scale))
    for b in range(len(lens)):
        for h in range(H_q):
            g = h // G   # contiguous query-head groups share one KV head
            ref = library_attention(q[b, h].astype(np.float64), Ks[b][:, g].astype(np.float64),
                                    Vs[b][:, g].astype(np.float64), float(np.float32(scale)))
            assert np.allclose(out[b, h], ref, rtol=1e-11, atol=1e-12), (b, h)
    assert np.isfinite(out).all()   # NaN-filled slots outside every context are never read


def test_gqa_group_mapping_is_contiguous():
    """Query head h reads KV head h // G: with H_kv = 2, G = 4, heads 0-3 see KV head 0."""
    rng = np.random.default_rng(11)
    H_kv, G, d, n = 2, 4, 8, 20
    K, V = random_logical(rng, n, H_kv, d)
    V[:, 0, :] = 1.0    # KV head 0 values are all 1, KV head 1 values all -1
    V[:, 1, :] = -1.0
    pool = build_pool_from_logical([K], [V], [[0, 1]], 2, H_kv, d)
    q = rng.standard_normal((1, H_kv * G, d)).astype(np.float16)
    out = oracle.paged_decode(pool, f16_bits(q), oracle.F16, [[0, 1]], [n], 0.3)
    assert np.all(out[0, :4] == 1.0) and np.all(out[0, 4:] == -1.0)


# --------------------------------------------------------------- closed forms --

def test_closed_forms():
    rng = np.random.default_rng(3)
    H_kv, H_q, d = 1, 2, 16
    # one token: out == v0 exactly
    K, V = random_logical(rng, 1, H_kv, d)
    pool = build_pool_from_logical([K], [V], [[4]], 6, H_kv, d)
    q = rng.standard_normal((1, H_q, d)).astype(np.float16)
    out = oracle.paged_decode(pool, f16_bits(q), oracle.F16, [[4]], [1], 0.25)
    assert np.array_equal(out[0, 0], V[0, 0].astype(np.float64)) and np.array_equal(out[0, 1], out[0, 0])
    # identical keys: uniform weights, out == mean(V)
    n = 37
    K, V = random_logical(rng, n, H_kv, d)
    K[:] = K[0]
    pool = build_pool_from_logical([K], [V], [[2, 0, 5]], 6, H_kv, d)
    out = oracle.paged_decode(pool, f16_bits(q), oracle.F16, [[2, 0, 5]], [n], 0.25)
    assert np.allclose(out[0, 0], V[:, 0].astype(np.float64).mean(0), rtol=0, atol=1e-13)
    # constant values: out == that constant for any keys
    K, V = random_logical(rng, n, H_kv, d)
    V[:] = np.float16(0.375)
    pool = build_pool_from_logical([K], [V], [[1, 3, 4]], 6, H_kv, d)
    out = oracle.paged_decode(pool, f16_bits(q), oracle.F16, [[1, 3, 4]], [n], 0.25)
    assert np.allclose(out, 0.375, rtol=0, atol=1e-14)
    # two tokens: out = sigma(s0 - s1) v0 + sigma(s1 - s0) v1 (logistic closed form)
    K, V = random_logical(rng, 2, H_kv, d)
    pool = build_pool_from_logical([K], [V], [[3]], 6, H_kv, d)
    out = oracle.paged_decode(pool, f16_bits(q), oracle.F16, [[3]], [2], 0.25)
    qq, kk, vv = q[0, 0].astype(np.float64), K[:, 0].astype(np.float64), V[:, 0].astype(np.float64)
    s0, s1 = 0.25 * kk[0] @ qq, 0.25 * kk[1] @ qq
    w0 = 1.0 / (1.0 + math.exp(s1 - s0))
    assert np.allclose(out[0, 0], w0 * vv[0] + (1.0 - w0) * vv[1], rtol=0, atol=1e-13)
    # one dominant key: softmax picks the maximum score, not the minimum
    K, V = random_logical(rng, 5, H_kv, d)
    K[:] = 0
    K[3, 0, :] = np.sign(q[0, 0]) * 4
    pool = build_pool_from_logical([K], [V], [[0]], 6, H_kv, d)
    out = oracle.paged_decode(pool, f16_bits(q), oracle.F16, [[0]], [5], 4.0)
    assert np.allclose(out[0, 0], V[3, 0].astype(np.float64), atol=1e-6)
    # empty context gives zeros
    out = oracle.paged_decode(pool, f16_bits(q), oracle.F16, [[0]], [0], 1.0)
    assert np.all(out == 0.0)


# ------------------------------------------------------------------- invariants --

def test_placement_invariance_and_prefix_sharing():
    """Any physical placement gives the same output bit for bit; sequences sharing
    prefix blocks give the same output as sequences holding private copies."""
    rng = np.random.default_rng(5)
    H_kv, H_q, d, n_pre, B = 2, 4, 16, 48, 3
    Kp, Vp = random_logical(rng, n_pre, H_kv, d)
    sufs = [random_logical(rng, int(m), H_kv, d) for m in (5, 16, 23)]
    Ks = [np.concatenate([Kp, s[0]]) for s in sufs]
    Vs = [np.concatenate([Vp, s[1]]) for s in sufs]
    lens = [k.shape[0] for k in Ks]
    W = max(oracle.blocks_for_tokens(n) for n in lens)
    q = rng.standard_normal((B, H_q, d)).astype(np.float16)
    outs = []
    for trial in range(3):
        N = 40
        perm = rng.permutation(N)
        tables, cur = np.full((B, W), -1, np.int32), 0
        for b, n in enumerate(lens):
            nb = oracle.blocks_for_tokens(n)
            tables[b, :nb] = perm[cur:cur + nb]
            cur += nb
        pool = build_pool_from_logical(Ks, Vs, tables, N, H_kv, d)
        outs.append(oracle.paged_decode(pool, f16_bits(q), oracle.F16, tables, lens, 0.25))
    # shared: the 3 prefix blocks are the same physical blocks in every table
    shared = np.full((B, W), -1, np.int32)
    shared[:, :3] = [30, 31, 32]
    nxt = 0
    for b, n in enumerate(lens):
        for j in range(3, oracle.blocks_for_tokens(n)):
            shared[b, j] = nxt
            nxt += 1
    pool = build_pool_from_logical(Ks, Vs, shared, 40, H_kv, d)
    outs.append(oracle.paged_decode(pool, f16_bits(q), oracle.F16, shared, lens, 0.25))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_one_partial_block_per_sequence():
    """Waste is at most one partly filled block per sequence: the seeded allocator in the
    input generator gives ceil(n/16) blocks and leaves fewer than 16 slots empty."""
    g = wl.generator(99)
    lens = list(range(0, 70)) + [4095, 4096, 4097]
    paging = wl.allocate(lens, 2000, 257, g)
    for b, n in enumerate(lens):
        nb = int((paging.tables[b] >= 0).sum())
        assert nb == oracle.blocks_for_tokens(n)
        assert 0 <= oracle.waste_slots(n) < BS
        assert nb * BS - n == oracle.waste_slots(n)
    used = paging.tables[paging.tables >= 0]
    assert used.unique().numel() == used.numel()     # no block handed out twice


def test_prefill_chunk_rows_equal_decode_and_causal_library():
    rng = np.random.default_rng(9)
    H_kv, G, d, P0, C = 2, 2, 16, 21, 13
    H_q = H_kv * G
    K, V = random_logical(rng, P0 + C, H_kv, d)
    table = [5, 1, 7]
    pool = build_pool_from_logical([K], [V], [table], 9, H_kv, d)
    q = rng.standard_normal((C, H_q, d)).astype(np.float16)
    out = oracle.paged_prefill_chunk(pool, f16_bits(q), oracle.F16, table, P0, 0.25)
    for i in range(C):
        dec = oracle.paged_decode(pool, f16_bits(q[i:i + 1]), oracle.F16, [table], [P0 + i + 1], 0.25)
        assert np.array_equal(out[i], dec[0])
        for h in range(H_q):
            ref = library_attention(q[i, h].astype(np.float64), K[:P0 + i + 1, h // G].astype(np.float64),
                                    V[:P0 + i + 1, h // G].astype(np.float64), 0.25)
            assert np.allclose(out[i, h], ref, rtol=1e-11, atol=1e-12)


# ------------------------------------------------------------ sliding window --

@pytest.mark.parametrize("window", [1, 5, 16, 17, 40])
def test_sliding_window_equals_library_attention_over_the_last_positions(window):
    """A window of w ("The KV cache" on the continuous-batching page: sliding-window
    attention layers) sees positions n-w .. n-1 of a decode of length n and
    p-w+1 .. p for chunk row at position p: library softmax attention over exactly those
    rows of the logical sequence.  w = 1 returns the last V row exactly."""
    rng = np.random.default_rng(100 + window)
    H_kv, G, d = 2, 2, 16
    H_q = H_kv * G
    lens = [0, 1, 3, 16, 17, 33, 64]
    W = max(oracle.blocks_for_tokens(n) for n in lens)
    N = sum(oracle.blocks_for_tokens(n) for n in lens) + 3
    perm = rng.permutation(N)
    tables, cur, Ks, Vs = np.full((len(lens), W), -1, np.int32), 0, [], []
    for b, n in enumerate(lens):
        nb = oracle.blocks_for_tokens(n)
        tables[b, :nb] = perm[cur:cur + nb]
        cur += nb
        K, V = random_logical(rng, n, H_kv, d)
        Ks.append(K)
        Vs.append(V)
    pool = build_pool_from_logical(Ks, Vs, tables, N, H_kv, d)
    q = rng.standard_normal((len(lens), H_q, d)).astype(np.float16)
    out = oracle.paged_decode(pool, f16_bits(q), oracle.F16, tables, lens, 0.25, window=window)
    for b, n in enumerate(lens):
        lo = max(0, n - window)
        for h in range(H_q):
            if n == 0:
                assert not out[b, h].any()
                continue
            ref = library_attention(q[b, h].astype(np.float64), Ks[b][lo:, h // G].astype(np.float64),
                                    Vs[b][lo:, h // G].astype(np.float64), 0.25)
            assert np.allclose(out[b, h], ref, rtol=1e-11, atol=1e-12), (b, h)
            if window == 1:
                assert np.array_equal(out[b, h], Vs[b][n - 1, h // G].astype(np.float64))
    # a window at least as long as every context is no window at all
    full = oracle.paged_decode(pool, f16_bits(q), oracle.F16, tables, lens, 0.25)
    wide = oracle.paged_decode(pool, f16_bits(q), oracle.F16, tables, lens, 0.25, window=64)
    assert np.array_equal(full, wide)
    # chunk rows: row i at position P0 + i sees max(0, P0 + i + 1 - w) .. P0 + i
    P0, C = 20, 13
    K, V = random_logical(rng, P0 + C, H_kv, d)
    table = [4, 0, 2]
    cpool = build_pool_from_logical([K], [V], [table], 6, H_kv, d)
    qc = rng.standard_normal((C, H_q, d)).astype(np.float16)
    cout = oracle.paged_prefill_chunk(cpool, f16_bits(qc), oracle.F16, table, P0, 0.25, window=window)
    for i in range(C):
        lo = max(0, P0 + i + 1 - window)
        for h in range(H_q):
            ref = library_attention(qc[i, h].astype(np.float64), K[lo:P0 + i + 1, h // G].astype(np.float64),
                                    V[lo:P0 + i + 1, h // G].astype(np.float64), 0.25)
            assert np.allclose(cout[i, h], ref, rtol=1e-11, atol=1e-12)


# ------------------------------------------------------------------ 16-bit append --

def test_append_16bit_is_a_slot_copy():
    rng = np.random.default_rng(4)
    N, H_kv, d, T = 6, 2, 8, 20
    pool = oracle.Pool(N, H_kv, d, oracle.BF16)
    before = pool.copy()
    k = bf16_bits(rng.standard_normal((T, H_kv, d)))
    v = bf16_bits(rng.standard_normal((T, H_kv, d)))
    slots = rng.permutation(N * BS)[:T].astype(np.int32)
    slots[3] = -1     # padding token: skipped
    oracle.kv_append(pool, k, v, oracle.BF16, slots)
    kk = pool.k.view(np.uint16).reshape(N, H_kv, BS, d)
    written = np.zeros((N, BS), bool)
    for i, s in enumerate(slots):
        if s < 0:
            continue
        written[s // BS, s % BS] = True
        assert np.array_equal(kk[s // BS, :, s % BS], k[i])
    untouched = ~written
    assert np.array_equal(kk.transpose(0, 2, 1, 3)[untouched], before.k.view(np.uint16).reshape(N, H_kv, BS, d)
                          .transpose(0, 2, 1, 3)[untouched])


# ----------------------------------------------------------------- quantization --

def test_quant_golden_codes(golden):
    g = golden("quant_codes.json")
    for dtype, key in ((oracle.INT8, "int8_block"), (oracle.INT4, "int4_block")):
        blk = g[key]
        d = len(blk["values"])
        pool = oracle.Pool(1, 1, d, dtype)
        x = bf16_bits(np.array(blk["values"]).reshape(1, 1, d))
        oracle.kv_append(pool, x, x, oracle.BF16, [0])
        assert pool.k_scale[0, 0] == np.float32(blk["scale"])
        deq = pool.dequant("k")[0, 0, 0]
        assert np.array_equal(deq / blk["scale"], np.array(blk["codes"], np.float64))
        if dtype == oracle.INT4:   # element 2j in the low nibble, 2j+1 in the high nibble
            c = [(x_ & 0xF) for x_ in blk["codes"]]
            packed = [c[2 * j] | (c[2 * j + 1] << 4) for j in range(d // 2)]
            assert list(pool.k[0, 0, 0]) == packed
        else:
            assert list(pool.k[0, 0, 0].view(np.int8)) == blk["codes"]


def test_e4m3_golden_and_exhaustive(golden):
    for row in golden("quant_codes.json")["e4m3"]:
        assert oracle.e4m3_encode(np.float32(row["x"])) == row["code"], row
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    finite = ~np.isnan(vals)
    assert finite.sum() == 254 and np.isnan(vals[0x7F]) and np.isnan(vals[0xFF])
    assert np.array_equal(oracle.e4m3_encode(vals[finite].astype(np.float32)), codes[finite])
    assert vals[finite].max() == 448.0 and vals[1] == 2.0 ** -9 and vals[8] == 2.0 ** -6


def test_e4m3_matches_library_conversion():
    """In range, round-to-nearest-even e4m3 agrees with torch's float8_e4m3fn conversion;
    torch does not saturate, so only |x| < 464 is compared."""
    g = torch.Generator().manual_seed(17)
    x = torch.cat([torch.randn(200000, generator=g) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)])
    mids = torch.tensor(oracle.e4m3_decode(np.arange(0, 126, dtype=np.uint8)), dtype=torch.float32)
    x = torch.cat([x, (mids[:-1] + mids[1:]) / 2, -(mids[:-1] + mids[1:]) / 2])   # exact ties
    x = x[x.abs() < 464]
    ours = oracle.e4m3_encode(x.numpy())
    lib = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, lib)


@pytest.mark.parametrize("dtype", [oracle.INT8, oracle.INT4, oracle.FP8])
def test_quant_fresh_block_properties(dtype):
    """Fresh blocks: s = amax / Q; max |code| == Q; |x - c s| <= s/2 (int); round trip of
    dequantized values with the stored scale returns the codes; token order is irrelevant."""
    rng = np.random.default_rng(dtype)
    N, H_kv, d = 8, 2, 32
    Q = {oracle.INT8: 127, oracle.INT4: 7, oracle.FP8: 448}[dtype]
    T = N * BS
    src = rng.standard_normal((T, H_kv, d)) * rng.uniform(0.01, 10, size=(T, 1, 1))
    src[BS:2 * BS] = 0.0           # an all-zero block: scale 0, codes 0
    xk = bf16_bits(src)
    slots = np.arange(T, dtype=np.int32)
    pool = oracle.Pool(N, H_kv, d, dtype)
    oracle.kv_append(pool, xk, xk, oracle.BF16, slots)
    x = oracle.bf16_decode(xk).reshape(N, BS, H_kv, d).transpose(0, 2, 1, 3)
    deq = pool.dequant("k")
    for blk in range(N):
        for g in range(H_kv):
            s = float(pool.k_scale[blk, g])
            amax = np.abs(x[blk, g]).max()
            assert s == float(np.float32(amax) / np.float32(Q))
            if s == 0:
                assert np.all(deq[blk, g] == 0)
                continue
            codes = deq[blk, g] / s
            if dtype == oracle.FP8:
                assert np.abs(codes).max() == Q
                rt = oracle.e4m3_encode((deq[blk, g] / s).astype(np.float32))
                assert np.array_equal(oracle.e4m3_decode(rt), codes)
            else:
                assert np.all(codes == np.round(codes)) and np.abs(codes).max() == Q
                # half a code step, plus the fp32 rounding of the quotient x / s (<= Q 2^-24 steps)
                assert np.all(np.abs(x[blk, g] - deq[blk, g]) <= s * (0.5 + Q * 2.0 ** -23))
                # re-quantizing the dequantized values with the stored scale returns the codes
                again = oracle.Pool(1, 1, d, dtype)
                again.k_scale[:] = s
                y = (codes * s).astype(np.float32)
                assert np.all(np.rint(y / np.float32(s)) == codes)
    # a permutation of the call's tokens gives the same bytes
    perm = rng.permutation(T)
    pool2 = oracle.Pool(N, H_kv, d, dtype)
    oracle.kv_append(pool2, xk[perm], xk[perm], oracle.BF16, slots[perm])
    assert np.array_equal(pool.k, pool2.k) and np.array_equal(pool.k_scale, pool2.k_scale)


@pytest.mark.parametrize("dtype", [oracle.INT8, oracle.INT4, oracle.FP8])
def test_quant_incremental_appends(dtype):
    """Decode-style appends one token at a time: the block scale never shrinks, equals the
    running amax / Q, and every cached value stays within the accumulated rounding of
    its re-quantizations (k re-quantizations -> error <= (k+1) s / 2 for int codes)."""
    rng = np.random.default_rng(100 + dtype)
    H_kv, d = 1, 16
    Q = {oracle.INT8: 127, oracle.INT4: 7, oracle.FP8: 448}[dtype]
    src = rng.standard_normal((BS, H_kv, d)) * np.linspace(0.5, 3.0, BS)[:, None, None]
    xk = bf16_bits(src)
    x = oracle.bf16_decode(xk)
    pool = oracle.Pool(2, H_kv, d, dtype)
    grows = 0
    prev = 0.0
    for t in range(BS):
        oracle.kv_append(pool, xk[t:t + 1], xk[t:t + 1], oracle.BF16, [BS + t])   # block 1
        s = float(pool.k_scale[1, 0])
        assert s >= prev
        assert s == max(prev, float(np.float32(np.abs(x[t]).max()) / np.float32(Q)))
        if prev > 0 and s > prev:
            grows += 1
        prev = s
        deq = pool.dequant("k")[1, 0, :t + 1]
        if dtype != oracle.FP8:
            assert np.all(np.abs(deq - x[:t + 1, 0]) <= (grows + 1) * s * (0.5 + Q * 2.0 ** -23))
        else:
            assert np.all(np.abs(deq - x[:t + 1, 0]) <= (grows + 1) * np.abs(x[:t + 1, 0]).max() / 8)
    assert grows > 0


def test_quantized_decode_attends_to_dequantized_values():
    """Attention over a quantized pool equals library attention over the pool's
    dequantized values (the oracle computes on code * scale in fp64)."""
    rng = np.random.default_rng(21)
    for dtype in (oracle.INT8, oracle.INT4, oracle.FP8):
        N, H_kv, d, n = 4, 1, 16, 50
        src = rng.standard_normal((n, H_kv, d))
        xk, xv = bf16_bits(src), bf16_bits(rng.standard_normal((n, H_kv, d)))
        pool = oracle.Pool(N, H_kv, d, dtype)
        table = [2, 0, 3, 1]
        slots = np.array([table[t // BS] * BS + t % BS for t in range(n)], np.int32)
        oracle.kv_append(pool, xk, xv, oracle.BF16, slots)
        dk, dv = pool.dequant("k"), pool.dequant("v")
        Kl = np.stack([dk[table[t // BS], 0, t % BS] for t in range(n)])
        Vl = np.stack([dv[table[t // BS], 0, t % BS] for t in range(n)])
        q = bf16_bits(rng.standard_normal((1, 2, d)))
        out = oracle.paged_decode(pool, q, oracle.BF16, [table], [n], 0.25)
        qd = oracle.bf16_decode(q)
        for h in range(2):
            assert np.allclose(out[0, h], library_attention(qd[0, h], Kl, Vl, 0.25), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("dtype", [oracle.INT8, oracle.INT4, oracle.FP8])
def test_quant_block_reuse_starts_fresh(dtype):
    """A block freed by a finished sequence and handed to a new one starts afresh when the
    new sequence writes its offset 0: the old (larger) scale is not kept."""
    rng = np.random.default_rng(300 + dtype)
    d = 16
    Q = {oracle.INT8: 127, oracle.INT4: 7, oracle.FP8: 448}[dtype]
    big = bf16_bits(rng.standard_normal((BS, 1, d)) * 50)
    small = bf16_bits(rng.standard_normal((3, 1, d)) * 0.1)
    pool = oracle.Pool(1, 1, d, dtype)
    oracle.kv_append(pool, big, big, oracle.BF16, np.arange(BS, dtype=np.int32))
    oracle.kv_append(pool, small, small, oracle.BF16, np.arange(3, dtype=np.int32))
    amax = np.abs(oracle.bf16_decode(small)).max()
    assert pool.k_scale[0, 0] == np.float32(amax) / np.float32(Q)
    # ...but a write that does not start the block keeps (and may only grow) the scale
    oracle.kv_append(pool, small[:1], small[:1], oracle.BF16, np.array([3], np.int32))
    assert pool.k_scale[0, 0] >= np.float32(amax) / np.float32(Q)


def _random_layers(L, N, H, d, dtype, seed):
    rng = np.random.default_rng(seed)
    pools = []
    for _ in range(L):
        p = oracle.Pool(N, H, d, dtype)
        p.k[...] = rng.integers(0, 256, p.k.shape, dtype=np.uint8)
        p.v[...] = rng.integers(0, 256, p.v.shape, dtype=np.uint8)
        if dtype == oracle.FP8:
            p.k[(p.k & 0x7F) == 0x7F] = 0x7E
            p.v[(p.v & 0x7F) == 0x7F] = 0x7E
        p.k_scale[...] = rng.random(p.k_scale.shape, dtype=np.float32) * 0.05
        p.v_scale[...] = rng.random(p.v_scale.shape, dtype=np.float32) * 0.05
        pools.append(p)
    return pools


@pytest.mark.parametrize("dtype", [oracle.F16, oracle.INT8, oracle.INT4, oracle.FP8])
def test_copied_block_reads_like_its_source(dtype):
    """Copy-on-write ("Paged attention" on the continuous-batching page): after copying a
    sequence's blocks to fresh ids, attention through the new table equals attention
    through the old one in every layer, and blocks outside the pairs are untouched."""
    L, N, H, d = 2, 24, 2, 64
    pools = _random_layers(L, N, H, d, dtype, 11 + dtype)
    if dtype == oracle.F16:   # finite halves only
        for p in pools:
            p.k[...] = (np.random.default_rng(1).standard_normal(p.k.shape[:-1] + (d,)).astype(np.float16)
                        .view(np.uint8))
            p.v[...] = (np.random.default_rng(2).standard_normal(p.v.shape[:-1] + (d,)).astype(np.float16)
                        .view(np.uint8))
    before = [p.copy() for p in pools]
    old, new = [3, 17, 5], [20, 1, 9]
    oracle.copy_blocks(pools, old, new)
    q = f16_bits(np.random.default_rng(3).standard_normal((1, 4, d)))
    for l, p in enumerate(pools):
        a = oracle.paged_decode(p, q, oracle.F16, np.array([old]), np.array([40]), 0.125)
        b = oracle.paged_decode(p, q, oracle.F16, np.array([new]), np.array([40]), 0.125)
        np.testing.assert_array_equal(a, b)
        keep = [i for i in range(N) if i not in new]
        assert np.array_equal(p.k[keep], before[l].k[keep]) and np.array_equal(p.v[keep], before[l].v[keep])
        assert np.array_equal(p.k_scale[keep], before[l].k_scale[keep])


@pytest.mark.parametrize("dtype,row", [(oracle.BF16, 128), (oracle.INT8, 64), (oracle.INT4, 32), (oracle.FP8, 64)])
def test_swap_image_size_and_round_trip(dtype, row):
    """Swapping ("The scheduler, and preemption" on the GQA page): a block's host image is
    all of its layers' K and V tiles (and scales), L * 2 * H * 16 * row_bytes (+ L * 2 * H * 4)
    bytes; restoring the image into other blocks reproduces the pool contents there."""
    L, N, H, d = 3, 20, 2, 64
    pools = _random_layers(L, N, H, d, dtype, 40 + dtype)
    quant = dtype in (oracle.INT8, oracle.INT4, oracle.FP8)
    img = oracle.swap_image(pools, [4, 11])
    assert img.shape == (2, L * 2 * H * 16 * row + (L * 2 * H * 4 if quant else 0))
    # the first tile in the image is layer 0's K tile of head 0 of block 4
    assert np.array_equal(img[0, :16 * row], pools[0].k[4, 0].reshape(-1))
    target = [p.copy() for p in pools]
    oracle.swap_restore(target, [0, 19], img)
    for p, t in zip(pools, target):
        for s, dd in ((4, 0), (11, 19)):
            assert np.array_equal(t.k[dd], p.k[s]) and np.array_equal(t.v[dd], p.v[s])
            if quant:
                assert np.array_equal(t.k_scale[dd], p.k_scale[s]) and np.array_equal(t.v_scale[dd], p.v_scale[s])
    assert oracle.swap_image(pools, []).shape == (0, img.shape[1])
