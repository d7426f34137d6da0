"""CPU checks of the C-ABI boundary: the library loads without a GPU, exports every
entry point include/pkv.h declares, sizes pools by the memory equation, and rejects bad
arguments on the host (no CUDA call is reached by these cases)."""
import ctypes
import os
import re

import pytest

import oracle
from paged_kv_cache_431_b200 import pkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"^PKV_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, re.M)
    return names


def test_header_declares_the_entry_points():
    names = set(declared_functions())
    for n in ("kv_pool_create", "kv_append", "paged_decode_attn", "paged_prefill_chunk_attn", "kv_copy_blocks",
              "kv_swap_out", "kv_swap_in", "pkv_bm_create", "pkv_bm_append_slots", "pkv_bm_check"):
        assert n in names
    assert len(names) >= 30


def test_library_exports_every_declared_symbol():
    L = pkv.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
    assert L.pkv_version() >= 100
    assert pkv.strerror(0) == "ok" and "workspace" in pkv.strerror(-5)


@pytest.mark.parametrize("dtype,nbytes", [(pkv.BF16, 2), (pkv.F16, 2), (pkv.INT8, 1), (pkv.FP8E4M3, 1)])
def test_pool_bytes_follow_the_memory_equation(dtype, nbytes):
    """K + V pool bytes for N blocks == the oracle's cache size for N * 16 tokens."""
    for (L, N, H, d) in ((80, 43520, 8, 128), (1, 64, 2, 64), (1, 131072, 8, 128)):
        kb, sb = pkv.pkv_pool_bytes(L, N, H, d, dtype)
        assert 2 * kb == oracle.kv_cache_bytes(L, H, d, nbytes, N * 16, 1)
        assert sb == (L * N * H * 4 if dtype in pkv.QUANTIZED else 0)


def test_int4_pool_bytes_are_half_of_int8():
    kb8, _ = pkv.pkv_pool_bytes(1, 1000, 8, 128, pkv.INT8)
    kb4, _ = pkv.pkv_pool_bytes(1, 1000, 8, 128, pkv.INT4)
    assert kb4 * 2 == kb8


def _desc(**kw):
    base = dict(num_layers=1, num_blocks=64, block_size=16, num_kv_heads=2, head_dim=64, kv_dtype=pkv.F16,
                k_data=0x10000, v_data=0x20000, k_scale=None, v_scale=None, device_status=None)
    base.update(kw)
    return pkv._PoolDesc(*[base[f] for f, _ in pkv._PoolDesc._fields_])


def _create(**kw):
    h = ctypes.c_void_p()
    rc = pkv.lib().kv_pool_create(ctypes.byref(_desc(**kw)), ctypes.byref(h))
    return rc, h


def test_pool_create_validation():
    L = pkv.lib()
    rc, h = _create()
    assert rc == 0 and h.value
    assert L.kv_pool_destroy(h) == 0
    assert L.kv_pool_destroy(None) == 0
    assert L.kv_pool_create(None, ctypes.byref(ctypes.c_void_p())) == -1
    assert _create(block_size=8)[0] == -2
    assert _create(head_dim=96)[0] == -9
    assert _create(kv_dtype=7)[0] == -3
    assert _create(k_data=None)[0] == -1
    assert _create(k_data=0x10008)[0] == -2              # not 16-byte aligned
    assert _create(kv_dtype=pkv.INT8)[0] == -1           # quantized without scales
    assert _create(kv_dtype=pkv.INT8, k_scale=0x30000, v_scale=0x40000)[0] == 0
    assert _create(num_blocks=0)[0] == -2


def test_decode_and_append_argument_checks():
    L = pkv.lib()
    rc, h = _create(num_kv_heads=2, head_dim=64)
    assert rc == 0
    P = ctypes.c_void_p
    fake = P(0x50000)
    try:
        # H_q not a multiple of H_kv
        assert L.paged_decode_attn(h, 0, fake, pkv.F16, fake, 4, fake, 4, 3, 64, 0.1, fake, None, 0, None, None) == -4
        # a negative sliding window
        bad = pkv._DecodeOpts(0, 0, -1)
        assert L.paged_decode_attn(h, 0, fake, pkv.F16, fake, 4, fake, 4, 8, 64, 0.1, fake, None, 0,
                                   ctypes.byref(bad), None) == -2
        assert L.paged_decode_workspace_bytes(h, 4, 8, 64, ctypes.byref(bad)) == 0
        # a window shrinks the split-K grid: 100,000 tokens with a 256-token window need no more
        # partials than 271 tokens do
        win = pkv._DecodeOpts(0, 0, 256)
        assert L.paged_decode_workspace_bytes(h, 4, 8, 100000, ctypes.byref(win)) == \
            L.paged_decode_workspace_bytes(h, 4, 8, 271, None)
        # q dtype must match a 16-bit pool
        assert L.paged_decode_attn(h, 0, fake, pkv.BF16, fake, 4, fake, 4, 8, 64, 0.1, fake, None, 0, None, None) == -3
        # bad layer
        assert L.paged_decode_attn(h, 1, fake, pkv.F16, fake, 4, fake, 4, 8, 64, 0.1, fake, None, 0, None, None) == -2
        # a split-K grid needs a workspace
        assert L.paged_decode_attn(h, 0, fake, pkv.F16, fake, 4, fake, 4, 8, 100000, 0.1, fake, None, 0, None,
                                   None) == -5
        # empty batch is a no-op
        assert L.paged_decode_attn(h, 0, None, pkv.F16, None, 4, None, 0, 8, 0, 0.1, None, None, 0, None, None) == 0
        # append: source dtype must equal a 16-bit pool's dtype; zero tokens is a no-op
        assert L.kv_append(h, 0, fake, fake, pkv.BF16, fake, 3, None, 0, None) == -3
        assert L.kv_append(h, 0, None, None, pkv.F16, None, 0, None, 0, None) == 0
        # prefill: table too narrow for the chunk
        assert L.paged_prefill_chunk_attn(h, 0, fake, pkv.F16, fake, 2, 20, 20, 8, 0.1, fake, None, 0, None) == -4
        assert L.paged_decode_workspace_bytes(h, 4, 8, 64, None) == 0          # one partition
        assert L.paged_decode_workspace_bytes(h, 4, 8, 4096, None) > 0
    finally:
        L.kv_pool_destroy(h)


def test_quantized_append_needs_bf16_source_and_workspace():
    L = pkv.lib()
    rc, h = _create(kv_dtype=pkv.INT8, k_scale=0x30000, v_scale=0x40000)
    fake = ctypes.c_void_p(0x50000)
    try:
        need = L.kv_append_workspace_bytes(h, 10)
        assert need == (2 * 64 * 2 + 64) * 4
        assert L.kv_append(h, 0, fake, fake, pkv.F16, fake, 10, fake, need, None) == -3
        assert L.kv_append(h, 0, fake, fake, pkv.BF16, fake, 10, None, 0, None) == -5
        assert L.kv_append(h, 0, fake, fake, pkv.BF16, fake, 10, fake, need - 4, None) == -5
    finally:
        L.kv_pool_destroy(h)


@pytest.mark.parametrize("dtype,row", [(pkv.BF16, 256), (pkv.INT8, 128), (pkv.INT4, 64), (pkv.FP8E4M3, 128)])
def test_swap_slot_size_is_one_block_of_every_layer(dtype, row):
    """A swapped block holds, for each layer, K and V of every KV head (16 rows each) and,
    quantized, one fp32 scale per (K/V, head)."""
    L = pkv.lib()
    quant = dtype in pkv.QUANTIZED
    rc, h = _create(num_layers=3, num_kv_heads=8, head_dim=128, kv_dtype=dtype,
                    k_scale=0x30000 if quant else None, v_scale=0x40000 if quant else None)
    assert rc == 0
    try:
        assert L.kv_swap_bytes_per_block(h) == 3 * 2 * 8 * 16 * row + (3 * 2 * 8 * 4 if quant else 0)
    finally:
        L.kv_pool_destroy(h)
    assert L.kv_swap_bytes_per_block(None) == 0


def test_block_moves_validate_on_the_host():
    L = pkv.lib()
    rc, h = _create()
    fake = ctypes.c_void_p(0x50000)
    try:
        assert L.kv_copy_blocks(None, fake, fake, 1, None) == -1
        assert L.kv_copy_blocks(h, fake, fake, -1, None) == -2
        assert L.kv_copy_blocks(h, None, None, 0, None) == 0
        assert L.kv_copy_blocks(h, None, fake, 2, None) == -1
        assert L.kv_swap_out(h, fake, -1, fake, None) == -2
        assert L.kv_swap_out(h, None, 0, None, None) == 0
        assert L.kv_swap_in(h, fake, 1, None, None) == -1
        # pageable (not page-locked) or misaligned host memory is refused
        buf = ctypes.create_string_buffer(1 << 16)
        assert L.kv_swap_out(h, fake, 1, ctypes.cast(buf, ctypes.c_void_p), None) == -2
        assert L.kv_swap_in(h, fake, 1, ctypes.c_void_p(ctypes.addressof(buf) + 8), None) == -2
    finally:
        L.kv_pool_destroy(h)


def _decode_ws(h, B, H_q, ctx, opts=None):
    return pkv.lib().paged_decode_workspace_bytes(h, B, H_q, ctx, ctypes.byref(opts) if opts is not None else None)


def _ws_expected(B, H_q, H_kv, parts, d=128):
    """fp32 partials o[d] + (m, l) per (sequence, query head, partition); nothing for one
    partition (H_kv does not enter: the partials are per query head)."""
    if parts <= 1:
        return 0
    return B * H_q * parts * (d + 2) * 4


@pytest.mark.parametrize("dtype,P", [(pkv.BF16, 512), (pkv.F16, 512), (pkv.INT8, 768), (pkv.INT4, 1536)])
def test_decode_workspace_follows_the_partition_policy(dtype, P):
    """Split-K partitions of ~256 KiB of K + V for 16-bit pools and ~192 KiB for quantized ones (512 /
    768 / 1536 tokens at d = 128) when the batch fills the GPU; the workspace is fp32 o[d] + (m, l)
    per (sequence, query head, partition).  (fp8 pools with 8 query heads per KV head run on the
    tcgen05 kernel and its own rule: test_decode_workspace_of_the_keys_on_m_engines.)"""
    kw = dict(num_kv_heads=8, head_dim=128, kv_dtype=dtype)
    if dtype in pkv.QUANTIZED:
        kw.update(k_scale=0x30000, v_scale=0x40000)
    rc, h = _create(**kw)
    assert rc == 0
    try:
        B, H_q, ctx = 170, 64, 8192
        assert _decode_ws(h, B, H_q, ctx) == _ws_expected(B, H_q, 8, -(-ctx // P))
        # a context of one default partition: with only B * H_kv CTAs the grid cannot fill the GPU, so
        # partitions are halved (to 128 or 192 tokens at least) and the partials come back
        short = _decode_ws(h, B, H_q, P) - _ws_expected(B, H_q, 8, 2) + B * H_q * 2 * (128 + 2) * 4
        parts, rem = divmod(short, B * H_q * (128 + 2) * 4)
        assert rem == 0 and 2 <= parts <= P // 128 and parts & (parts - 1) == 0
        assert _decode_ws(h, B, H_q, 128) == 0                         # one partition: no partials
    finally:
        pkv.lib().kv_pool_destroy(h)


def test_decode_workspace_small_batches_and_explicit_partitions():
    rc, h = _create(num_kv_heads=8, head_dim=128, kv_dtype=pkv.BF16)
    assert rc == 0
    try:
        # 2 sequences cannot fill 148 SMs with 512-token partitions: they shrink to the 128-token floor
        assert _decode_ws(h, 2, 64, 8192) == _ws_expected(2, 64, 8, 64)
        # an explicit partition size is taken as given (a multiple of 16 in [64, 4096])
        assert _decode_ws(h, 3, 16, 1000, pkv._DecodeOpts(0, 64, 0)) == _ws_expected(3, 16, 8, 16)
        assert _decode_ws(h, 3, 16, 1000, pkv._DecodeOpts(0, 4096, 0)) == 0
        for bad in (100, 48, 8192):
            assert _decode_ws(h, 3, 16, 1000, pkv._DecodeOpts(0, bad, 0)) == 0
        # the workspace scales with the batch
        assert _decode_ws(h, 340, 64, 8192) == 2 * _decode_ws(h, 170, 64, 8192)
        # wide groups: still per query head
        assert _decode_ws(h, 3, 8 * 40, 1000, pkv._DecodeOpts(0, 64, 0)) == _ws_expected(3, 320, 8, 16)
    finally:
        pkv.lib().kv_pool_destroy(h)


def test_decode_workspace_of_the_keys_on_m_engines():
    """64 query heads per KV head (16-bit pools, d = 128, engine auto) run on the keys-on-M tcgen05
    kernel, one CTA per SM: as few partitions per sequence as fill 148 SMs, each at most 4096
    tokens in whole 128-key tiles; engine 1, other group sizes and explicit sizes keep the general
    rule.  fp8 pools with 8 query heads per KV head: the same rule with two CTAs per SM."""
    rc, h = _create(num_kv_heads=1, head_dim=128, kv_dtype=pkv.BF16)
    assert rc == 0
    try:
        assert _decode_ws(h, 256, 64, 4096) == 0                              # one 4096-token partition
        assert _decode_ws(h, 256, 64, 8000) == _ws_expected(256, 64, 1, 2)    # two of 4096 tokens
        assert _decode_ws(h, 4, 64, 4096) == _ws_expected(4, 64, 1, 32)       # 4 sequences: 37 wanted, 128-token floor
        assert _decode_ws(h, 100, 64, 1000) == _ws_expected(100, 64, 1, 2)    # 2 x 512 tokens fill 148 SMs
        assert _decode_ws(h, 256, 64, 4096, pkv._DecodeOpts(1, 0, 0)) == _ws_expected(256, 64, 1, 8)   # engine 1: 512
        assert _decode_ws(h, 256, 64, 4096, pkv._DecodeOpts(0, 1024, 0)) == _ws_expected(256, 64, 1, 4)
        assert _decode_ws(h, 256, 128, 4096) == _ws_expected(256, 128, 1, 8)  # G = 128: the general rule
    finally:
        pkv.lib().kv_pool_destroy(h)
    rc, h = _create(num_kv_heads=8, head_dim=128, kv_dtype=pkv.FP8E4M3, k_scale=0x30000, v_scale=0x40000)
    assert rc == 0
    try:
        assert _decode_ws(h, 170, 64, 8192) == _ws_expected(170, 64, 8, 2)    # 2 x 4096 tokens
        assert _decode_ws(h, 16, 64, 131072) == _ws_expected(16, 64, 8, 32)   # the long-context layer
        assert _decode_ws(h, 4, 64, 4096) == _ws_expected(4, 64, 8, 8)        # 10 parts wanted, 410 -> 512 tokens: 8
        assert _decode_ws(h, 16, 64, 131072, pkv._DecodeOpts(1, 0, 0)) == _ws_expected(16, 64, 8, 171)   # engine 1: 768
        assert _decode_ws(h, 16, 32, 131072) == _ws_expected(16, 32, 8, 171)  # G = 4: the general rule
    finally:
        pkv.lib().kv_pool_destroy(h)


def test_wait_hook_arguments_are_checked_on_the_host():
    """pkv_test_withhold_copy only stores process-wide settings; out-of-range bounds are
    rejected and tile < 0 restores the defaults (no CUDA call)."""
    L = pkv.lib()
    assert L.pkv_test_withhold_copy(0, 0) == -2
    assert L.pkv_test_withhold_copy(0, 3_000_000_000) == -2
    assert L.pkv_test_withhold_copy(1, 100_000) == 0
    assert L.pkv_test_withhold_copy(-1, 0) == 0


def test_get_device_status_is_read_device_status():
    """Both names validate the same way before touching the device."""
    L = pkv.lib()
    st = ctypes.c_int32(5)
    assert L.pkv_get_device_status(None, None, ctypes.byref(st)) == -1
    assert L.pkv_read_device_status(None, None, ctypes.byref(st)) == -1


def test_per_layer_pool_create_validation():
    """kv_pool_create_layers checks every layer's pointers on the host (no CUDA call): NULL
    arrays or entries, misaligned bases, missing scales of a quantized pool, too many layers."""
    L = pkv.lib()
    P = ctypes.c_void_p

    def arr(vals):
        return (P * len(vals))(*vals)

    def create(desc, k, v, ks=None, vs=None):
        h = ctypes.c_void_p()
        rc = L.kv_pool_create_layers(ctypes.byref(desc), k, v, ks, vs, ctypes.byref(h))
        if rc == 0:
            assert h.value and L.kv_pool_destroy(h) == 0
        return rc

    d3 = _desc(num_layers=3, k_data=None, v_data=None)
    k = arr([0x100000, 0x900000, 0x500000])          # any order, any spacing
    v = arr([0x200000, 0x300000, 0x700000])
    assert create(d3, k, v) == 0
    assert create(d3, None, v) == -1
    assert create(d3, k, arr([0x200000, None, 0x700000])) == -1
    assert create(d3, k, arr([0x200000, 0x300008, 0x700000])) == -2      # not 16-byte aligned
    q3 = _desc(num_layers=3, kv_dtype=pkv.INT8, k_data=None, v_data=None)
    assert create(q3, k, v) == -1                                        # quantized without scales
    s = arr([0x1000, 0x2000, 0x3000])
    assert create(q3, k, v, s, arr([0x4000, 0x5000, 0x6000])) == 0
    assert create(q3, k, v, s, arr([0x4000, 0x5002, 0x6000])) == -2     # scales not 4-byte aligned
    big = _desc(num_layers=pkv.MAX_LAYERS + 1, k_data=None, v_data=None)
    many = arr([0x100000] * (pkv.MAX_LAYERS + 1))
    assert create(big, many, many) == -2
    assert _create(num_layers=pkv.MAX_LAYERS + 1)[0] == -2
