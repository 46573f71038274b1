"""Pins of the block-manager oracle (``oracle.KvManager``) against what the
pages state, independent of the oracle's own bookkeeping.

The strongest pin is a content simulation: a host pool holds token ids instead
of K/V vectors; every reported slot is written with its token, every reported
copy pair copies a block, and then each sequence read back through its block
table must equal the token list the test tracks on its own ("vLLM 基本原理",
PagedAttention: the block table maps each logical block to the physical block
that holds it)."""
from __future__ import annotations

import copy
import random

import pytest

from oracle import KvManager, KvManagerError, NoBlocks


class Sim:
    """A manager plus a token-id pool and the expected token list per sequence."""

    def __init__(self, num_blocks, bs, prefix_caching, num_host_blocks=0):
        self.m = KvManager(num_blocks, bs, prefix_caching, num_host_blocks)
        self.bs = bs
        self.pool = [[None] * bs for _ in range(num_blocks)]
        self.host = [[None] * bs for _ in range(num_host_blocks)]
        self.swapped = set()
        self.expect = {}

    def _write(self, slots, tokens):
        for s, t in zip(slots, tokens):
            if s >= 0:
                self.pool[s // self.bs][s % self.bs] = t

    def _copy(self, pairs):
        for src, dst in pairs:
            self.pool[dst] = list(self.pool[src])

    def add(self, sid, tokens):
        slots, cached = self.m.add_sequence(sid, tokens)
        assert all(s == -1 for s in slots[:cached]) and all(s >= 0 for s in slots[cached:])
        self._write(slots, tokens)
        self.expect[sid] = list(tokens)
        return cached

    def append(self, sid, tokens):
        slots, pairs = self.m.append_tokens(sid, tokens)
        self._copy(pairs)
        self._write(slots, tokens)
        self.expect[sid] += list(tokens)
        return slots, pairs

    def step(self, sids, tokens):
        slots, pairs = self.m.decode_step(sids, tokens)
        self._copy(pairs)
        self._write(slots, tokens)
        for sid, t in zip(sids, tokens):
            self.expect[sid].append(t)
        return slots, pairs

    def fork(self, p, c):
        self.m.fork(p, c)
        self.expect[c] = list(self.expect[p])

    def share_prefix(self, src, dst, n):
        self.m.share_prefix(src, dst, n)
        self.expect[dst] = self.expect[src][:min(len(self.expect[src]), n * self.bs)]

    def share_blocks(self, src, dst, idx):
        self.m.share_blocks(src, dst, idx)
        for i in idx:
            for t in range(i * self.bs, min((i + 1) * self.bs, len(self.expect[dst]),
                                            len(self.expect[src]))):
                self.expect[dst][t] = self.expect[src][t]

    def free(self, sid):
        self.m.free_sequence(sid)
        del self.expect[sid]
        self.swapped.discard(sid)

    def swap_out(self, sid):
        pairs = self.m.swap_out(sid)
        for d, h in pairs:
            self.host[h] = list(self.pool[d])
        self.swapped.add(sid)
        return pairs

    def swap_in(self, sid):
        pairs = self.m.swap_in(sid)
        for h, d in pairs:
            self.pool[d] = list(self.host[h])
        self.swapped.discard(sid)
        return pairs

    def check(self):
        m, bs = self.m, self.bs
        refs = [0] * m.num_blocks
        for sid, toks in self.expect.items():
            table = m.block_table(sid)
            assert m.context_len(sid) == len(toks)
            # on-demand allocation: only the last block may be partly used
            assert len(table) == -(-len(toks) // bs)
            src = self.host if sid in self.swapped else self.pool
            got = [src[table[t // bs]][t % bs] for t in range(len(toks))]
            assert got == toks, (sid, got, toks)
            if sid not in self.swapped:
                for b in table:
                    refs[b] += 1
        assert refs == [m.ref_count(b) for b in range(m.num_blocks)]
        unref = {b for b in range(m.num_blocks) if refs[b] == 0}
        assert m.num_free_blocks() == len(unref)


def test_on_demand_allocation_uses_every_block_but_the_last():
    sim = Sim(64, 16, False)
    for sid, n in enumerate([1, 15, 16, 17, 33, 48]):
        sim.add(sid, list(range(n)))
    used = 64 - sim.m.num_free_blocks()
    assert used == sum(-(-n // 16) for n in [1, 15, 16, 17, 33, 48])
    for step in range(40):
        sim.append(step % 6, [step])
    sim.check()
    assert 64 - sim.m.num_free_blocks() == sum(-(-len(t) // 16) for t in sim.expect.values())


def test_outputs_of_one_prompt_share_its_blocks_and_the_first_writers_copy():
    # "vLLM 基本原理", memory sharing: 3 outputs of one prompt point at the same
    # prompt blocks; "当大模型推理遇上内存瓶颈" 3.3: only the first writer copies.
    sim = Sim(32, 16, False)
    prompt = list(range(56))  # 3 full blocks + 8 tokens
    sim.add(0, prompt)
    for c in (1, 2, 3):
        sim.fork(0, c)
    assert 32 - sim.m.num_free_blocks() == 4
    last = sim.m.block_table(0)[-1]
    assert sim.m.ref_count(last) == 4
    copies = []
    for sid in (1, 2, 3, 0):
        slots, pairs = sim.append(sid, [1000 + sid])
        copies.append(pairs)
    # the first three writers copy the shared partial block, the last writes in place
    assert [len(p) for p in copies] == [1, 1, 1, 0]
    assert all(p[0][0] == last for p in copies[:3])
    assert sim.m.block_table(0)[-1] == last and sim.m.ref_count(last) == 1
    assert 32 - sim.m.num_free_blocks() == 4 + 3
    # the full prompt blocks stay shared by all four
    for b in sim.m.block_table(0)[:3]:
        assert sim.m.ref_count(b) == 4
    sim.check()


def test_full_block_tail_needs_no_copy():
    sim = Sim(16, 16, False)
    sim.add(0, list(range(32)))
    sim.fork(0, 1)
    _, pairs = sim.append(1, [7])
    assert pairs == []            # the shared blocks are full: a fresh block, no copy
    assert 16 - sim.m.num_free_blocks() == 3
    sim.check()


def test_share_prefix_and_share_blocks():
    sim = Sim(32, 4, False)
    sim.add(0, list(range(10)))          # blocks: 4 + 4 + 2
    sim.share_prefix(0, 1, 2)            # first two blocks, 8 tokens
    assert sim.m.context_len(1) == 8
    assert sim.m.block_table(1) == sim.m.block_table(0)[:2]
    sim.share_prefix(0, 2, 3)            # all three blocks: length capped at 10
    assert sim.m.context_len(2) == 10
    sim.add(3, [50 + i for i in range(12)])
    sim.share_blocks(0, 3, [1])          # sparse sharing of a full block
    t0, t3 = sim.m.block_table(0), sim.m.block_table(3)
    assert t3[1] == t0[1] and t3[0] != t0[0] and t3[2] != t0[2]
    with pytest.raises(KvManagerError):
        sim.share_blocks(0, 3, [2])      # block 2 of sequence 0 is not full
    sim.check()
    sim.append(2, [99])                  # 2's last block is shared and partial: copy
    sim.check()


def test_prefix_cache_reuses_whole_blocks_from_position_zero():
    # "vLLM 定位与核心机制详解" 六.3: identical tokens from the first one, whole
    # blocks only; a partial tail is never reused.
    sim = Sim(64, 16, True)
    a = list(range(40))
    assert sim.add(0, a) == 0
    assert sim.add(1, a[:40]) == 32           # two full blocks hit, the 8-token tail does not
    assert sim.m.block_table(1)[:2] == sim.m.block_table(0)[:2]
    assert sim.m.block_table(1)[2] != sim.m.block_table(0)[2]
    assert sim.add(2, [999] + a[1:40]) == 0   # differs at position 0
    assert sim.add(3, [7] * 8 + a[:32]) == 0  # the same tokens at another offset
    assert sim.add(4, a[:16] + [5] * 20) == 16
    sim.check()


def test_prefix_cache_survives_free_and_blocks_filled_by_decode_are_cached():
    sim = Sim(64, 16, True)
    a = list(range(20))
    sim.add(0, a)
    sim.append(0, list(range(20, 32)))        # fills block 1 during decode
    full = sim.m.block_table(0)[:2]
    sim.free(0)
    assert sim.m.num_free_blocks() == 64      # cached blocks count as free
    assert sim.add(1, list(range(40))) == 32  # ... and are found again
    assert sim.m.block_table(1)[:2] == full
    sim.check()


def test_eviction_takes_the_longest_unreferenced_and_its_extensions():
    sim = Sim(6, 4, True)
    sim.add(0, [1, 1, 1, 1, 2, 2, 2, 2])      # blocks for prefixes P1, P1P2
    sim.add(1, [3, 3, 3, 3])                  # prefix Q
    sim.free(0)                               # released tail first: P1P2 then P1
    sim.free(1)
    # 6 blocks: 3 cached and unreferenced, 3 never used
    sim.add(2, list(range(100, 112)))         # takes the 3 never-used blocks
    assert sim.add(3, [3, 3, 3, 3]) == 4      # Q still cached
    sim.free(3)
    sim.add(4, [9, 9, 9, 9])                  # evicts the oldest: P1P2
    assert sim.add(5, [1, 1, 1, 1, 2, 2, 2, 2]) == 4   # P1 hits, P1P2 was evicted
    sim.check()


def test_evicting_a_block_drops_the_prefixes_through_it():
    sim = Sim(5, 4, True)
    sim.add(0, [1] * 4)                       # block 0: P1
    sim.add(1, [1] * 4 + [2] * 4)             # P1 hits; block 1: P1P2
    sim.add(2, [5] * 8)                       # blocks 2, 3
    sim.share_blocks(1, 2, [1])               # seq 2 now holds block 1 (P1P2); block 3 unreferenced
    sim.free(0)
    sim.free(1)                               # block 0 (P1) unreferenced; block 1 still held by seq 2
    sim.add(3, [6] * 4)                       # block 4 (never used)
    sim.add(4, [7] * 4)                       # evicts block 3 (oldest unreferenced)
    sim.add(5, [8] * 4)                       # evicts block 0 (P1): P1P2 loses its entry too
    sim.free(3)
    sim.free(2)
    assert 1 in sim.m.free                    # block 1: unreferenced, no longer cached
    assert sim.add(6, [1] * 4 + [2] * 4) == 0
    sim.check()


def test_operations_are_all_or_nothing():
    m = KvManager(4, 4, True)
    m.add_sequence(0, list(range(12)))        # 3 blocks
    before = copy.deepcopy(m.__dict__)
    with pytest.raises(NoBlocks):
        m.add_sequence(1, list(range(100, 108)))  # needs 2, 1 free
    assert m.__dict__ == before
    m.append_tokens(0, [1, 2, 3, 4])          # the last free block
    before = copy.deepcopy(m.__dict__)
    with pytest.raises(NoBlocks):
        m.append_tokens(0, [5])
    assert m.__dict__ == before
    with pytest.raises(KvManagerError):
        m.append_tokens(9, [1])
    with pytest.raises(KvManagerError):
        m.fork(0, 0)


def random_ops(seed, n_ops, num_blocks, bs, prefix_caching):
    """A seeded stream of operations on a small pool, with prompts built from a
    few shared templates so that prefixes repeat."""
    rng = random.Random(seed)
    templates = [[rng.randrange(4) for _ in range(rng.randrange(1, 5 * bs))] for _ in range(4)]
    live, next_id, ops, outs = [], 0, [], []
    for _ in range(n_ops):
        r = rng.random()
        if r < 0.25 or not live:
            t = list(rng.choice(templates))[:rng.randrange(1, 5 * bs)]
            t += [rng.randrange(4) for _ in range(rng.randrange(0, 2 * bs))]
            if not t:
                t = [0]
            ops.append(("add", next_id, t))
            live.append(next_id)
            next_id += 1
        elif r < 0.6:
            ops.append(("append", rng.choice(live),
                        [rng.randrange(4) for _ in range(rng.choice([1, 1, 1, 3, bs + 1]))]))
        elif r < 0.66:
            ids = rng.sample(live, rng.randrange(1, len(live) + 1))
            if rng.random() < 0.1:
                ids.append(ids[0])            # a duplicate: rejected
            ops.append(("step", ids, [rng.randrange(4) for _ in ids]))
        elif r < 0.7:
            ops.append(("fork", rng.choice(live), next_id))
            live.append(next_id)
            next_id += 1
        elif r < 0.75:
            ops.append(("share_prefix", rng.choice(live), next_id, rng.randrange(0, 4)))
            live.append(next_id)
            next_id += 1
        elif r < 0.8 and len(live) > 1:
            a, b = rng.sample(live, 2)
            ops.append(("share_blocks", a, b, sorted(rng.sample(range(3), rng.randrange(1, 3)))))
        elif r < 0.83:
            sid = rng.choice(live)
            ops.append(("swap_out", sid))
            outs.append(sid)
        elif r < 0.86:
            ops.append(("swap_in", outs.pop(rng.randrange(len(outs))) if outs else rng.choice(live)))
        else:
            sid = rng.choice(live)
            live.remove(sid)
            ops.append(("free", sid))
    return ops


def apply_op(target, op):
    """Apply one op to a Sim; returns its result or the exception class."""
    kind = op[0]
    try:
        if kind == "add":
            return target.add(op[1], op[2])
        if kind == "append":
            return target.append(op[1], op[2])
        if kind == "step":
            return target.step(op[1], op[2])
        if kind == "fork":
            return target.fork(op[1], op[2])
        if kind == "share_prefix":
            return target.share_prefix(op[1], op[2], op[3])
        if kind == "share_blocks":
            return target.share_blocks(op[1], op[2], op[3])
        if kind == "swap_out":
            return target.swap_out(op[1])
        if kind == "swap_in":
            return target.swap_in(op[1])
        return target.free(op[1])
    except (NoBlocks, KvManagerError) as e:
        return type(e)


@pytest.mark.parametrize("prefix_caching", [False, True])
@pytest.mark.parametrize("seed", range(6))
def test_random_streams_keep_every_sequence_readable(seed, prefix_caching):
    sim = Sim(24, 4, prefix_caching, num_host_blocks=10)
    for op in random_ops(seed, 400, 24, 4, prefix_caching):
        res = apply_op(sim, op)
        if res in (NoBlocks, KvManagerError):
            # failed ops leave no trace: drop any id the stream thought it created
            if op[0] in ("add", "fork", "share_prefix"):
                new = op[1] if op[0] == "add" else op[2]
                sim.expect.pop(new, None)
        sim.check()


def test_swap_out_and_in_move_a_sequence_through_host_blocks():
    # "当大模型推理遇上内存瓶颈" 5.1 / 7.3: KV blocks move to a CPU swap space and back
    sim = Sim(8, 4, False, num_host_blocks=4)
    sim.add(0, list(range(10)))               # 3 blocks
    sim.add(1, list(range(20, 25)))           # 2 blocks
    pairs = sim.swap_out(0)
    assert [d for d, _ in pairs] == [0, 1, 2] and [h for _, h in pairs] == [0, 1, 2]
    assert sim.m.num_free_blocks() == 6 and sim.m.num_free_host_blocks() == 1
    sim.check()
    with pytest.raises(KvManagerError):
        sim.append(0, [1])                    # swapped out: nothing but swap in / free
    sim.add(2, list(range(40, 52)))           # reuses the freed device blocks
    back = sim.swap_in(0)
    assert [h for h, _ in back] == [0, 1, 2] and sim.m.num_free_host_blocks() == 4
    sim.append(0, [7, 8])
    sim.check()
    sim.fork(1, 3)
    with pytest.raises(KvManagerError):
        sim.swap_out(1)                       # shares its blocks with 3
    sim.swap_out(2)                           # 3 of the 4 host blocks
    with pytest.raises(NoBlocks):
        sim.swap_out(0)                       # 3 more blocks, 1 host block left
    sim.check()
