"""CPU tests of the host block manager in libpkv (pkv_bm_*): no GPU is involved.

What is pinned, and where it comes from:
- the block-table figure of "KV cache, GQA, paging and continuous batching" (section
  "PagedAttention"): 41 tokens take three blocks, the last one partly filled;
- the prefix-caching worked example of the same page (section "Prefix caching"): with a
  4,000-token system prompt and a 200-token query, a second request prefills only its
  200 tokens (about 95% of the prefill eliminated);
- at most one partly filled block per sequence ("KV cache, continuous batching and paged
  attention", section "Paged attention");
- a randomized run of adds, appends, forks, frees and swaps checked after every step
  against a content model: every slot a sequence's table reaches must hold exactly the
  K/V that sequence's own token prefix would produce (so prefix-cache hits, copy-on-write
  and swaps are all checked), and pkv_bm_check's invariants must hold.
"""
import random

import pytest

from paged_kv_cache_431_b200 import pkv

BS = 16


def test_block_table_figure():
    bm = pkv.BlockManager(16, enable_prefix_cache=False)
    assert bm.add_sequence(0, list(range(41))) == 0
    slots, cow = bm.append_slots(0, 41, list(range(41)))
    table, n = bm.block_table(0)
    assert cow is None and n == 41 and len(table) == 3
    # token t lives at block table[t // 16], offset t % 16
    assert slots == [table[t // BS] * BS + t % BS for t in range(41)]
    # the only waste is the 7 empty slots of the last block
    assert len(table) * BS - n == 7
    assert bm.free_blocks() == 13
    bm.check()


def test_prefix_caching_worked_example():
    """4,000-token shared system prompt + 200-token query: the second request finds 250
    cached blocks and prefills 200 tokens instead of 4,200."""
    rng = random.Random(5)
    system = [rng.randrange(32000) for _ in range(4000)]
    bm = pkv.BlockManager(2000)
    first = system + [rng.randrange(32000) for _ in range(200)]
    assert bm.add_sequence(1, first) == 0
    bm.append_slots(1, len(first), first)
    second = system + [rng.randrange(32000) for _ in range(200)]
    cached = bm.add_sequence(2, second)
    assert cached == 4000
    prefill = len(second) - cached
    assert prefill == 200
    assert round(1 - prefill / len(second), 3) == 0.952   # "~95% of prefill work eliminated"
    t1, _ = bm.block_table(1)
    t2, n2 = bm.block_table(2)
    assert n2 == 4000 and t2 == t1[:250]
    assert all(bm.refcount(b) == 2 for b in t2)
    bm.append_slots(2, prefill, second[4000:])
    st = bm.stats()
    assert st["prefix_hits"] == 250 and st["shared_blocks"] == 250
    bm.check()


def test_a_fully_cached_prompt_still_computes_its_last_token():
    bm = pkv.BlockManager(64)
    p = list(range(64))
    bm.add_sequence(1, p)
    bm.append_slots(1, 64, p)
    assert bm.add_sequence(2, p) == 48          # 3 of 4 blocks: the last token is left to compute
    assert bm.add_sequence(3, p[:49]) == 48
    assert bm.add_sequence(4, p[:48]) == 32
    bm.check()


def test_different_earlier_tokens_never_match():
    """The key of a block covers its whole prefix: equal second blocks after different
    first blocks are different cache entries."""
    bm = pkv.BlockManager(64)
    a = list(range(16)) + list(range(100, 116)) + [7]
    b = list(range(1, 17)) + list(range(100, 116)) + [7]
    bm.add_sequence(1, a)
    bm.append_slots(1, len(a), a)
    assert bm.add_sequence(2, b) == 0
    c = list(range(16)) + list(range(100, 116)) + [9, 9]
    assert bm.add_sequence(3, c) == 32
    # b's own blocks enter the cache; a prompt starting like b then reaching a's second
    # block's tokens must take b's second block, not a's
    bm.append_slots(2, len(b), b)
    ta, _ = bm.block_table(1)
    tb, _ = bm.block_table(2)
    assert bm.add_sequence(4, b[:32] + [1, 2]) == 32
    t4, _ = bm.block_table(4)
    assert t4 == tb[:2] and t4[1] != ta[1]
    bm.check()


def test_fork_then_diverge_copies_the_shared_partial_block_once():
    bm = pkv.BlockManager(32, enable_prefix_cache=False)
    bm.add_sequence(1, list(range(20)))
    bm.append_slots(1, 20, list(range(20)))
    bm.fork(1, 2)
    t1, _ = bm.block_table(1)
    assert [bm.refcount(b) for b in t1] == [2, 2]
    slots, cow = bm.append_slots(2, 1, [99])
    assert cow is not None and cow[0] == t1[1]
    t2, n2 = bm.block_table(2)
    assert t2[0] == t1[0] and t2[1] == cow[1] and n2 == 21
    assert slots == [cow[1] * BS + 4]
    assert bm.refcount(t1[1]) == 1 and bm.refcount(cow[1]) == 1
    # the parent now owns its partial block alone: no second copy
    slots1, cow1 = bm.append_slots(1, 1, [98])
    assert cow1 is None and slots1 == [t1[1] * BS + 4]
    # appends that start a new block never copy
    bm.fork(2, 3)
    bm.append_slots(2, 11, list(range(11)))          # fills block 1 of seq 2 ... copy happens here
    assert bm.stats()["cow_copies"] == 2
    bm.check()


def test_out_of_blocks_changes_nothing_and_eviction_reclaims_cache():
    bm = pkv.BlockManager(4)
    bm.add_sequence(1, list(range(40)))
    bm.append_slots(1, 40, list(range(40)))          # 3 blocks, 2 full and cached
    bm.add_sequence(2, None, 0)
    assert bm.blocks_needed(2, 17) == 2
    with pytest.raises(pkv.PkvError) as e:
        bm.append_slots(2, 17)
    assert e.value.status == pkv.ERR_NO_BLOCKS
    assert bm.block_table(2) == ([], 0) and bm.free_blocks() == 1
    bm.free_sequence(1)                               # 2 keyed blocks stay cached, 1 goes free
    st = bm.stats()
    assert st["cached_blocks"] == 2 and st["free_blocks"] == 2 and bm.free_blocks() == 4
    bm.append_slots(2, 48)                            # needs 3: one free + evicts...
    assert bm.stats()["evictions"] >= 1
    bm.check()
    # a freed-and-reused block can no longer be found under its old key
    assert bm.add_sequence(3, list(range(40))) <= 16
    bm.check()


def test_swap_out_and_in_keep_length_and_release_blocks():
    bm = pkv.BlockManager(16, enable_prefix_cache=False)
    bm.add_sequence(1, None, 0)
    bm.append_slots(1, 35)
    t, _ = bm.block_table(1)
    out = bm.swap_out(1)
    assert out == t and bm.free_blocks() == 16
    assert bm.block_table(1) == ([], 35)
    with pytest.raises(pkv.PkvError):
        bm.append_slots(1, 1)
    back = bm.swap_in(1, len(out))
    assert len(back) == 3 and bm.block_table(1) == (back, 35)
    slots, _ = bm.append_slots(1, 1)
    assert slots == [back[2] * BS + 3]
    bm.check()


class ContentModel:
    """What each physical slot holds: the token prefix whose K/V was written there."""

    def __init__(self):
        self.slot = {}
        self.host = {}

    def write(self, slots, tokens, start_pos):
        for i, s in enumerate(slots):
            self.slot[s] = tuple(tokens[:start_pos + i + 1])

    def copy_block(self, src, dst):
        for o in range(BS):
            if src * BS + o in self.slot:
                self.slot[dst * BS + o] = self.slot[src * BS + o]
            else:
                self.slot.pop(dst * BS + o, None)

    def verify(self, bm, seqs):
        for sid, toks in seqs.items():
            table, n = bm.block_table(sid)
            if not table and n:
                continue  # swapped out
            assert n == len(toks)
            assert len(table) == -(-n // BS)              # one partly filled block at most
            for p in range(n):
                assert self.slot.get(table[p // BS] * BS + p % BS) == tuple(toks[:p + 1]), (sid, p)


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_randomized_operations_keep_every_sequence_intact(seed):
    rng = random.Random(seed)
    bm = pkv.BlockManager(160)
    model = ContentModel()
    prefixes = [[rng.randrange(50) for _ in range(rng.choice([16, 40, 64]))] for _ in range(3)]
    seqs, swapped, next_id = {}, {}, 0

    def append(sid, new):
        toks = seqs[sid]
        need = bm.blocks_needed(sid, len(new))
        if need > bm.free_blocks():
            with pytest.raises(pkv.PkvError):
                bm.append_slots(sid, len(new), new)
            return False
        start = len(toks)
        slots, cow = bm.append_slots(sid, len(new), new)
        if cow:
            model.copy_block(*cow)
        toks.extend(new)
        model.write(slots, toks, start)
        return True

    for step in range(600):
        op = rng.random()
        live = [s for s in seqs if s not in swapped]
        if op < 0.25 or not live:
            prompt = list(rng.choice(prefixes)) + [rng.randrange(50) for _ in range(rng.randrange(1, 30))]
            sid, next_id = next_id, next_id + 1
            cached = bm.add_sequence(sid, prompt)
            assert cached % BS == 0 and cached < len(prompt)
            seqs[sid] = list(prompt[:cached])
            if not append(sid, prompt[cached:]):
                bm.free_sequence(sid)
                del seqs[sid]
        elif op < 0.6:
            sid = rng.choice(live)
            append(sid, [rng.randrange(50) for _ in range(rng.choice([1, 1, 1, 5, 17]))])
        elif op < 0.7:
            sid = rng.choice(live)
            child, next_id = next_id, next_id + 1
            bm.fork(sid, child)
            seqs[child] = list(seqs[sid])
        elif op < 0.85:
            sid = rng.choice(list(seqs))
            bm.free_sequence(sid)
            del seqs[sid]
            swapped.pop(sid, None)
        elif op < 0.93:
            sid = rng.choice(live)
            blocks = bm.swap_out(sid)
            swapped[sid] = [[model.slot.get(b * BS + o) for o in range(BS)] for b in blocks]
        elif swapped:
            sid = rng.choice(list(swapped))
            img = swapped[sid]
            if len(img) <= bm.free_blocks():
                blocks = bm.swap_in(sid, len(img))
                for b, row in zip(blocks, img):
                    for o, v in enumerate(row):
                        if v is None:
                            model.slot.pop(b * BS + o, None)
                        else:
                            model.slot[b * BS + o] = v
                del swapped[sid]
        bm.check()
        model.verify(bm, {s: t for s, t in seqs.items() if s not in swapped})
    st = bm.stats()
    assert st["prefix_hits"] > 0 and st["cow_copies"] > 0
