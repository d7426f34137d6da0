"""Seeded synthetic inputs for paged KV-cache attention.

Shared by the tests, the benchmark and the oracle-side checks, so that both the CUDA
path and the CPU oracle see the same bytes.  It holds random number generation and
the shapes of the workloads only -- no attention, quantization or dequantization.
The one piece of indexing it does is the caller's own allocation: choosing physical
blocks for each sequence (a seeded permutation of the pool) and listing the slots
(block * 16 + offset) that new tokens are written to, as a serving engine's block
manager would before calling ``kv_append``.

Workload shapes follow the pages' examples:
  - a 70B-class GQA model: 80 layers, 64 query heads, 8 KV heads, head dim 128
    ("KV cache, GQA, paging and continuous batching", section "Mechanics");
  - contexts around 3,000 tokens ("A worked example: sizing a deployment");
  - a 4,000-token shared system prompt with 200-token queries (section "Prefix caching");
  - 512-2,048-token prefill chunks ("KV cache, continuous batching and paged attention",
    section "Scheduling prefill and decode");
  - 8-bit / 4-bit / fp8 KV storage (inference guide a2-inf-2, "KV-cache quantization").
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

BLOCK = 16

# pool storage dtypes, numbered as in the C-ABI
F16, BF16, INT8, INT4, FP8 = 0, 1, 2, 3, 4
TORCH_DTYPE = {F16: torch.float16, BF16: torch.bfloat16}


def generator(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal(shape, dtype, gen: torch.Generator, device="cpu") -> torch.Tensor:
    """N(0, 1) values, drawn in fp32 and rounded once to ``dtype`` (round to nearest even)."""
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(dtype)


def row_bytes(dtype: int, d: int) -> int:
    return {F16: 2 * d, BF16: 2 * d, INT8: d, FP8: d, INT4: d // 2}[dtype]


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


@dataclass
class Paging:
    """Physical placement of a batch of sequences in a pool of ``num_blocks`` blocks.

    ``tables[b, j]`` is the physical block of logical block j of sequence b; unused
    entries are -1 (never read by a correct kernel).
    """
    num_blocks: int
    ctx_lens: torch.Tensor          # int32 [B]
    tables: torch.Tensor            # int32 [B, W]
    used: torch.Tensor              # bool [num_blocks]: referenced by some table


def allocate(ctx_lens, num_blocks: int, width: int, gen: torch.Generator,
             shared_prefix_blocks: int = 0, extra_tokens=None) -> Paging:
    """Give each sequence ceil(len / 16) blocks drawn without replacement from a seeded
    permutation of the pool.  With ``shared_prefix_blocks`` > 0 the first that many
    logical blocks of every sequence map to the same physical blocks (a shared prefix).
    ``extra_tokens[b]`` reserves room for tokens beyond ``ctx_lens[b]``."""
    ctx = torch.as_tensor(ctx_lens, dtype=torch.int32).cpu()
    B = ctx.shape[0]
    extra = torch.zeros(B, dtype=torch.int32) if extra_tokens is None else torch.as_tensor(extra_tokens,
                                                                                           dtype=torch.int32)
    perm = torch.randperm(num_blocks, generator=gen).to(torch.int32)
    tables = torch.full((B, width), -1, dtype=torch.int32)
    cursor = 0
    prefix = perm[:shared_prefix_blocks]
    cursor += shared_prefix_blocks
    for b in range(B):
        nb = ceil_div(int(ctx[b]) + int(extra[b]), BLOCK)
        if nb > width:
            raise ValueError("block table too narrow")
        npre = min(shared_prefix_blocks, nb)
        tables[b, :npre] = prefix[:npre]
        own = nb - npre
        if cursor + own > num_blocks:
            raise ValueError("pool too small")
        tables[b, npre:nb] = perm[cursor:cursor + own]
        cursor += own
    used = torch.zeros(num_blocks, dtype=torch.bool)
    valid = tables[tables >= 0].long()
    used[valid] = True
    return Paging(num_blocks, ctx, tables, used)


def slots_for(tables: torch.Tensor, seq_ids, positions) -> torch.Tensor:
    """Slots (physical block * 16 + offset) of logical ``positions`` of sequences ``seq_ids``."""
    seq_ids = torch.as_tensor(seq_ids, dtype=torch.long)
    positions = torch.as_tensor(positions, dtype=torch.long)
    blk = tables[seq_ids, positions // BLOCK].long()
    return (blk * BLOCK + positions % BLOCK).to(torch.int32)


def poison_pool_(pool: torch.Tensor, paging: Paging, poison: float = float("nan")) -> None:
    """Fill every slot that no sequence's context covers with ``poison``.

    pool is [N, H_kv, 16, d] of a 16-bit float dtype.  A kernel that reads outside
    the block table, or past a sequence's length, then sees NaN."""
    pool[~paging.used.to(pool.device)] = poison
    for b in range(paging.ctx_lens.shape[0]):
        n = int(paging.ctx_lens[b])
        if n % BLOCK:
            last = int(paging.tables[b, n // BLOCK])
            pool[last, :, n % BLOCK:] = poison


# ------------------------------------------------------------ workloads --

@dataclass
class DecodeWorkload:
    """One layer's decode batch over a 16-bit pool."""
    name: str
    H_q: int
    H_kv: int
    d: int
    dtype: int
    scale: float
    paging: Paging
    q: torch.Tensor                 # [B, H_q, d]
    k_pool: torch.Tensor            # [N, H_kv, 16, d]
    v_pool: torch.Tensor
    extra: dict = field(default_factory=dict)

    @property
    def B(self):
        return self.q.shape[0]

    @property
    def W(self):
        return self.paging.tables.shape[1]


def decode_workload(name: str, ctx_lens, H_q: int, H_kv: int, d: int, dtype: int, num_blocks: int,
                    width: int, seed: int, device="cpu", poison: bool = True,
                    shared_prefix_blocks: int = 0) -> DecodeWorkload:
    """A decode batch with K/V drawn i.i.d. N(0, 1) over the whole pool and placed by a
    seeded permutation.  Slots outside every sequence's context are poisoned with NaN."""
    gen_host = generator(seed)
    paging = allocate(ctx_lens, num_blocks, width, gen_host, shared_prefix_blocks)
    tdt = TORCH_DTYPE[dtype]
    gen = generator(seed + 1, device)
    B = paging.ctx_lens.shape[0]
    q = normal((B, H_q, d), tdt, gen, device)
    k_pool = normal((num_blocks, H_kv, BLOCK, d), tdt, gen, device)
    v_pool = normal((num_blocks, H_kv, BLOCK, d), tdt, gen, device)
    if poison:
        poison_pool_(k_pool, paging)
        poison_pool_(v_pool, paging)
    return DecodeWorkload(name, H_q, H_kv, d, dtype, 1.0 / (d ** 0.5), paging, q, k_pool, v_pool)


def tiny_decode(seed: int = 432, device="cpu") -> DecodeWorkload:
    """Tiny paged decode: 4 sequences of {17, 33, 40, 64} tokens in a 64-block pool,
    H_q 8, H_kv 2, head dim 64, fp16, softmax scale 1/sqrt(64)."""
    return decode_workload("tiny", [17, 33, 40, 64], 8, 2, 64, F16, 64, 4, seed, device)


def llama8b_lens(gen: torch.Generator, B: int = 64):
    return torch.randint(512, 4097, (B,), generator=gen, dtype=torch.int32)


def gqa70b_lens(gen: torch.Generator, B: int = 170):
    x = torch.randn(B, generator=gen, dtype=torch.float64) * 400.0 + 3000.0
    return x.round().clamp(1024, 4096).to(torch.int32)


def quant_long_lens(gen: torch.Generator, B: int = 16):
    return torch.randint(32768, 131073, (B,), generator=gen, dtype=torch.int32)


def outlier_channels(gen: torch.Generator, H_kv: int, d: int, frac: float = 0.01) -> torch.Tensor:
    """A seeded set of round(frac * H_kv * d) (head, dim) channels, as a flat index list."""
    n = int(round(frac * H_kv * d))
    return torch.randperm(H_kv * d, generator=gen)[:n]


def kv_source(T: int, H_kv: int, d: int, gen: torch.Generator, device="cpu",
              outliers: torch.Tensor | None = None, outlier_gain: float = 8.0):
    """bf16 K and V source rows [T, H_kv, d], N(0, 1), with the listed (head, dim)
    channels multiplied by ``outlier_gain`` (a power of two, so exact in bf16)."""
    k = normal((T, H_kv, d), torch.bfloat16, gen, device)
    v = normal((T, H_kv, d), torch.bfloat16, gen, device)
    if outliers is not None and outliers.numel():
        idx = outliers.to(device)
        k.view(T, H_kv * d)[:, idx] *= outlier_gain
        v.view(T, H_kv * d)[:, idx] *= outlier_gain
    return k, v


def compact_subset(tables: torch.Tensor, ctx_lens: torch.Tensor, seq_ids):
    """For sequences `seq_ids`: the physical blocks they reference (sorted) and their
    tables renumbered into that list."""
    seq_ids = list(seq_ids)
    sub_t = tables[seq_ids].clone()
    sub_c = ctx_lens[seq_ids].clone()
    used = []
    for r, b in enumerate(seq_ids):
        nb = ceil_div(int(ctx_lens[b]), BLOCK)
        used.extend(int(x) for x in tables[b, :nb])
    uniq = sorted(set(used))
    remap = {blk: i for i, blk in enumerate(uniq)}
    for r, b in enumerate(seq_ids):
        nb = ceil_div(int(ctx_lens[b]), BLOCK)
        for j in range(nb):
            sub_t[r, j] = remap[int(tables[b, j])]
    return uniq, sub_t, sub_c
