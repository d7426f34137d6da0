"""paged_decode_attn_noalloc: the decode entry point for callers that cannot allocate device
memory (its split-K partials live in the library's fixed 32 MiB device buffer).

Checked through the C-ABI against the regular entry point on two calls in a row, with
different inputs, so the second call also shows that what the first left in the shared
buffer does not leak into its result.  Kept in its own file, collected last."""
import pytest
import torch

from paged_kv_cache_431_b200 import pkv
from paged_kv_cache_431_b200 import workloads as wl
from tests.helpers import TOL

pytestmark = pytest.mark.gpu
DEV = "cuda"


def decode_inputs(seed, B, H_q, H_kv, d, kv_dtype=wl.BF16):
    g = wl.generator(seed)
    ctx = wl.llama8b_lens(g, B)
    N = B * 4096 // 16
    paging = wl.allocate(ctx, N, 256, g)
    gd = wl.generator(seed + 1, DEV)
    if kv_dtype == wl.BF16:
        k = wl.normal((1, N, H_kv, 16, d), torch.bfloat16, gd, DEV)
        v = wl.normal((1, N, H_kv, 16, d), torch.bfloat16, gd, DEV)
        pool = pkv.KVPool(k, v, wl.BF16, d, device_status=torch.zeros(1, dtype=torch.int32, device=DEV))
    else:   # a quantized pool filled through kv_append
        pool = pkv.KVPool.allocate(1, N, H_kv, d, kv_dtype)
        for b in range(B):
            n = int(ctx[b])
            k, v = wl.kv_source(n, H_kv, d, gd, DEV)
            pkv.kv_append(pool, 0, k, v, wl.slots_for(paging.tables, [b] * n, torch.arange(n)).to(DEV))
    q = wl.normal((B, H_q, d), torch.bfloat16, gd, DEV)
    return pool, q, paging.tables.to(DEV), ctx.to(DEV), int(ctx.max())


CASES = {
    # name: (pool dtype, sliding window, query heads (8 KV heads), batches of the two calls)
    "bf16": (wl.BF16, 0, 32, (64, 24)),
    "int8": (wl.INT8, 0, 32, (64, 24)),
    "bf16_window": (wl.BF16, 1000, 32, (64, 24)),
    "fp8_g8": (wl.FP8, 0, 64, (24, 8)),   # 8 query heads per KV head: the tcgen05 fp8 kernel
}


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_regular_decode_on_two_calls(name):
    kv_dtype, window, H_q, batches = CASES[name]
    for seed, B in zip((801, 802), batches):
        pool, q, tables, ctx, max_ctx = decode_inputs(seed, B, H_q, 8, 128, kv_dtype)
        need = pkv.paged_decode_workspace_bytes(pool, B, H_q, max_ctx, sliding_window=window)
        assert 0 < need <= pkv.NOALLOC_SCRATCH_BYTES          # the split-K path is exercised
        ref = pkv.paged_decode_attn(pool, 0, q, tables, ctx, 128 ** -0.5, max_ctx, sliding_window=window)
        out = pkv.paged_decode_attn_noalloc(pool, 0, q, tables, ctx, 128 ** -0.5, max_ctx, sliding_window=window)
        torch.cuda.synchronize()
        assert pkv.read_device_status(pool) == 0
        assert torch.isfinite(out).all()
        assert (out - ref).abs().max().item() <= TOL


def test_noalloc_rejects_requests_beyond_its_buffer():
    pool, q, tables, ctx, _ = decode_inputs(803, 8, 32, 8, 128)
    huge_ctx = 1 << 20                   # partials for 2048 partitions: far beyond 32 MiB
    assert pkv.paged_decode_workspace_bytes(pool, 8, 32, huge_ctx) > pkv.NOALLOC_SCRATCH_BYTES
    with pytest.raises(pkv.PkvError) as e:
        pkv.paged_decode_attn_noalloc(pool, 0, q, tables, ctx, 128 ** -0.5, huge_ctx)
    assert e.value.status == -5
