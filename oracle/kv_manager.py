"""Plain Python model of the host KV-cache block manager (TEST INFRASTRUCTURE ONLY).

What the library's C++ manager (``pa_kvm_*``) must do, written as directly as
the pages state it, with Python dicts and lists and no attention to speed.

Sources, by page title and section:

* "vLLM 基本原理", section "PagedAttention": a sequence's KV cache is cut into
  fixed-size logical blocks mapped by a block table to physical blocks drawn
  from a pool; a new physical block is requested only when the current one is
  full, so every block but a sequence's last is completely used (on-demand
  allocation); several outputs of one prompt point at the same physical
  prompt blocks and get private blocks only for their own new tokens (memory
  sharing).
* "当大模型推理遇上内存瓶颈", section 2.2 (each physical block carries a
  reference count that drives copy-on-write) and section 2.3 (sharing modes:
  a whole sequence, the first n blocks of one -- ``share_prefix`` -- or
  chosen logical blocks -- ``share_blocks``); section 3.3 (with reference
  counting only the first writer of a shared block copies it).
* "vLLM 定位与核心机制详解", section 六.1 (a finished sequence's blocks are freed
  at once for other requests) and section 六.3 (prefix caching: each full block
  is identified by its content, and a new request reuses cached blocks when
  its tokens are identical from position 0; only whole blocks, never a
  partial tail).

Readings taken where the pages are silent or leave a choice:

* Allocation order: the lowest-numbered free physical block first.
* A block freed with ``ref_count`` 0 that holds a cached full block stays
  reusable ("evictable") until an allocation finds no never-cached free block;
  then the one that became unreferenced longest ago is evicted.  Evicting a
  block also drops every cached block whose prefix runs through it (their
  whole prefix is no longer cached); unreferenced ones among them become
  plain free blocks.
* A cached block's identity is the full token sequence from position 0 to its
  last token.  Prefix-cache hits form a contiguous run from block 0 and stop
  at the first miss.  A full block is registered when it becomes full (at
  allocation for a prompt, when its last slot is reserved during decode) if
  the prefix before it is cached (or it is block 0); if its own prefix is
  already cached by another block, the new block stays unregistered.  The caller runs each step's prefill before the next step's
  lookups.
* Prompt tokens found in the cache get slot -1 (nothing to write: the block is
  shared), the others their slot ``block * block_size + offset``.
* Appending to a sequence whose last block is partly filled and shared
  (``ref_count`` > 1) first copies that block: a fresh block is allocated, the
  pair (shared, fresh) is reported for the caller's ``copy_blocks``, the
  shared block's count drops by one and the table points at the fresh block.
  The last holder (count 1) writes in place.
* ``share_prefix(src, dst, n)``: ``dst`` is a new sequence holding the first
  ``n`` blocks of ``src`` (counts raised), length ``min(len(src), n * bs)``.
* ``share_blocks(src, dst, idx)``: for each logical index ``i`` in ``idx`` (a
  full block of ``src`` and within ``dst``'s table), ``dst``'s block ``i``
  becomes ``src``'s block ``i``;
  the block ``dst`` held there loses a reference, and ``dst``'s tokens in that
  block's positions become ``src``'s.
* Swapping ("当大模型推理遇上内存瓶颈" 5.1 CPU swap space, 7.3 cold blocks to
  slower storage): a sequence that holds every one of its blocks alone can be
  swapped out -- each block gets the lowest free host block, the device blocks
  are released (last first; cached ones stay cached) and the table lists host
  blocks; swapping in takes fresh device blocks (registering nothing in the
  prefix cache).  A swapped-out sequence can only be swapped in or freed.
* Every operation is all-or-nothing: when the pool cannot supply the blocks it
  needs, it raises ``NoBlocks`` and changes nothing.
"""
from __future__ import annotations

from collections import OrderedDict


class NoBlocks(RuntimeError):
    """The pool has too few free blocks for the operation."""


class KvManagerError(ValueError):
    """An unknown or duplicate sequence id, or an out-of-range argument."""


class KvManager:
    def __init__(self, num_blocks: int, block_size: int, prefix_caching: bool,
                 num_host_blocks: int = 0):
        if num_blocks <= 0 or block_size <= 0 or num_host_blocks < 0:
            raise KvManagerError("bad sizes")
        self.host_free = set(range(num_host_blocks))  # host swap-space blocks
        self.num_blocks = num_blocks
        self.bs = block_size
        self.prefix_caching = bool(prefix_caching)
        self.ref = [0] * num_blocks
        self.free = set(range(num_blocks))          # never-cached free blocks
        self.evictable = OrderedDict()              # cached, unreferenced: oldest first
        self.cache = {}                             # prefix tuple -> block
        self.prefix_of = {}                         # block -> prefix tuple (cached blocks)
        self.seqs = {}                              # id -> {"table", "len", "tokens"}

    # ------------------------------------------------------------------ pool
    def num_free_blocks(self) -> int:
        return len(self.free) + len(self.evictable)

    def _uncache(self, b):
        """Drop block b's cache entry and every entry whose prefix runs through it."""
        p = self.prefix_of.pop(b)
        del self.cache[p]
        for q in [q for q in self.cache if len(q) > len(p) and q[:len(p)] == p]:
            c = self.cache.pop(q)
            del self.prefix_of[c]
            if c in self.evictable:
                del self.evictable[c]
                self.free.add(c)

    def _alloc(self) -> int:
        if self.free:
            b = min(self.free)
            self.free.remove(b)
        elif self.evictable:
            b = next(iter(self.evictable))
            del self.evictable[b]
            self._uncache(b)
        else:
            raise NoBlocks("pool exhausted")
        self.ref[b] = 1
        return b

    def _release(self, b):
        self.ref[b] -= 1
        assert self.ref[b] >= 0
        if self.ref[b] == 0:
            if b in self.prefix_of:
                self.evictable[b] = None
            else:
                self.free.add(b)

    def _retain(self, b):
        if self.ref[b] == 0:
            del self.evictable[b]   # a reused cached block leaves the evictable set
        self.ref[b] += 1

    def _register(self, b, prefix):
        # only a block whose whole prefix is cached can ever be found (lookups
        # start at position 0), so only such a block is registered
        if not self.prefix_caching or prefix in self.cache:
            return
        if len(prefix) > self.bs and prefix[:-self.bs] not in self.cache:
            return
        self.cache[prefix] = b
        self.prefix_of[b] = prefix

    def _need(self, n):
        if n > self.num_free_blocks():
            raise NoBlocks(f"need {n} blocks, {self.num_free_blocks()} free")

    def _seq(self, sid, resident=True):
        if sid not in self.seqs:
            raise KvManagerError(f"unknown sequence {sid}")
        s = self.seqs[sid]
        if resident and s.get("swapped"):
            raise KvManagerError(f"sequence {sid} is swapped out")
        return s

    # ------------------------------------------------------------- sequences
    def add_sequence(self, sid, tokens):
        """A new sequence with prompt ``tokens``.  Returns (slots, cached_tokens)."""
        if sid in self.seqs:
            raise KvManagerError(f"duplicate sequence {sid}")
        tokens = [int(t) for t in tokens]
        n = len(tokens)
        nblk = -(-n // self.bs)
        hits = []
        if self.prefix_caching:
            for i in range(n // self.bs):
                b = self.cache.get(tuple(tokens[:(i + 1) * self.bs]))
                if b is None:
                    break
                hits.append(b)
        # blocks that must come from the pool: the misses, counted before any change
        revived = sum(1 for b in hits if self.ref[b] == 0)
        if nblk - len(hits) > self.num_free_blocks() - revived:
            raise NoBlocks("pool exhausted")
        table = []
        for b in hits:
            self._retain(b)
            table.append(b)
        for i in range(len(hits), nblk):
            b = self._alloc()
            table.append(b)
            if (i + 1) * self.bs <= n:
                self._register(b, tuple(tokens[:(i + 1) * self.bs]))
        cached = len(hits) * self.bs
        slots = [-1 if t < cached else table[t // self.bs] * self.bs + t % self.bs
                 for t in range(n)]
        self.seqs[sid] = {"table": table, "len": n, "tokens": tokens}
        return slots, cached

    def append_tokens(self, sid, tokens):
        """Reserve slots for ``tokens`` at the end of the sequence.
        Returns (slots, copy_pairs)."""
        s = self._seq(sid)
        tokens = [int(t) for t in tokens]
        n = len(tokens)
        L = s["len"]
        # blocks needed: copy of a shared partial last block, then fresh blocks
        cow = n > 0 and L % self.bs != 0 and self.ref[s["table"][-1]] > 1
        new_blocks = -(-(L + n) // self.bs) - -(-L // self.bs)
        self._need(new_blocks + (1 if cow else 0))
        pairs = []
        if cow:
            old = s["table"][-1]
            fresh = self._alloc()
            self._release(old)
            s["table"][-1] = fresh
            pairs.append((old, fresh))
        slots = []
        for t in tokens:
            if L % self.bs == 0:
                s["table"].append(self._alloc())
            slots.append(s["table"][L // self.bs] * self.bs + L % self.bs)
            s["tokens"].append(t)
            L += 1
            if L % self.bs == 0:
                self._register(s["table"][L // self.bs - 1], tuple(s["tokens"][:L]))
        s["len"] = L
        return slots, pairs

    def decode_step(self, sids, tokens):
        """One new token for each of ``sids`` (in order), all or nothing.
        Returns (slots, copy_pairs)."""
        if len(set(sids)) != len(sids):
            raise KvManagerError("a sequence listed twice")
        need, drops = 0, {}
        for sid in sids:
            st = self._seq(sid)
            L = st["len"]
            if L % self.bs == 0:
                need += 1
            else:
                b = st["table"][-1]
                if self.ref[b] - drops.get(b, 0) > 1:   # shared: a copy
                    need += 1
                    drops[b] = drops.get(b, 0) + 1
        self._need(need)
        slots, pairs = [], []
        for sid, t in zip(sids, tokens):
            sl, pr = self.append_tokens(sid, [t])
            slots += sl
            pairs += pr
        return slots, pairs

    def fork(self, parent, child):
        """Whole-sequence sharing: ``child`` holds every block of ``parent``."""
        p = self._seq(parent)
        if child in self.seqs:
            raise KvManagerError(f"duplicate sequence {child}")
        for b in p["table"]:
            self._retain(b)
        self.seqs[child] = {"table": list(p["table"]), "len": p["len"], "tokens": list(p["tokens"])}

    def share_prefix(self, src, dst, n_blocks):
        s = self._seq(src)
        if dst in self.seqs:
            raise KvManagerError(f"duplicate sequence {dst}")
        if n_blocks < 0 or n_blocks > len(s["table"]):
            raise KvManagerError("prefix longer than the source")
        L = min(s["len"], n_blocks * self.bs)
        for b in s["table"][:n_blocks]:
            self._retain(b)
        self.seqs[dst] = {"table": list(s["table"][:n_blocks]), "len": L,
                          "tokens": list(s["tokens"][:L])}

    def share_blocks(self, src, dst, idx):
        s, d = self._seq(src), self._seq(dst)
        idx = [int(i) for i in idx]
        for i in idx:
            if i < 0 or (i + 1) * self.bs > s["len"] or i >= len(d["table"]):
                raise KvManagerError("logical block out of range or not full in the source")
        for i in idx:
            b = s["table"][i]
            self._retain(b)
            self._release(d["table"][i])
            d["table"][i] = b
            # dst now sees src's tokens in that block's positions
            for t in range(i * self.bs, min((i + 1) * self.bs, d["len"], s["len"])):
                d["tokens"][t] = s["tokens"][t]

    def free_sequence(self, sid):
        s = self._seq(sid, resident=False)
        if s.get("swapped"):
            self.host_free.update(s["table"])
        else:
            # the last blocks first, so a released prompt's early blocks stay cached longest
            for b in reversed(s["table"]):
                self._release(b)
        del self.seqs[sid]

    # ---------------------------------------------------------------- swapping
    def swap_out(self, sid):
        """Move a sequence's blocks to host blocks ("当大模型推理遇上内存瓶颈" 5.1,
        7.3).  Only a sequence that holds all its blocks alone can move.
        Returns the (device, host) pairs to copy."""
        s = self._seq(sid)
        if any(self.ref[b] != 1 for b in s["table"]):
            raise KvManagerError("a shared block cannot be swapped out")
        if len(s["table"]) > len(self.host_free):
            raise NoBlocks("host swap space exhausted")
        host = []
        for _ in s["table"]:
            h = min(self.host_free)
            self.host_free.remove(h)
            host.append(h)
        pairs = list(zip(s["table"], host))
        for b in reversed(s["table"]):
            self._release(b)
        s["table"] = host
        s["swapped"] = True
        return pairs

    def swap_in(self, sid):
        """Bring a swapped-out sequence back into fresh device blocks.  Returns
        the (host, device) pairs to copy."""
        s = self._seq(sid, resident=False)
        if not s.get("swapped"):
            raise KvManagerError(f"sequence {sid} is not swapped out")
        self._need(len(s["table"]))
        dev = [self._alloc() for _ in s["table"]]
        pairs = list(zip(s["table"], dev))
        self.host_free.update(s["table"])
        s["table"] = dev
        s["swapped"] = False
        return pairs

    def num_free_host_blocks(self) -> int:
        return len(self.host_free)

    # ----------------------------------------------------------------- views
    def block_table(self, sid):
        return list(self._seq(sid, resident=False)["table"])

    def context_len(self, sid):
        return self._seq(sid, resident=False)["len"]

    def ref_count(self, b):
        return self.ref[b]
